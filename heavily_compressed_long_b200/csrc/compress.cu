// compress.cu -- softmax-gated pooling compressor (CSA overlapped window, HCA plain window).
//
// [Tripbot §3.1] Every m tokens of KV become one entry by softmax-gated pooling with a
// learned position bias; [CSDN §1.1 工程细节] CSA entry i also pools the previous window's
// last m tokens (C^b) with its own m tokens (C^a), 2m slots in all; [Tripbot §3.2] HCA pools
// m' = 128 tokens per entry without overlap.  Per channel c of entry i, with slot j holding
// token t_j (slots outside [0, L) dropped):
//     out[i, c] = sum_j softmax_j(gate[t_j, c] + bias[j]) * kv[t_j, c]
//
// HBM-streaming kernels: each thread owns 8 channels (one 16-byte load of kv and of gate per
// token row, coalesced along d) and keeps an online (max, sum, weighted sum) softmax in fp32
// (pool.cuh).  Small spans give each entry to one group of d/8 threads; long spans (HCA) split
// the slots over the 128 threads of a block and merge the partial softmaxes in shared memory.
//
// Optional RMSNorm epilogue [Tripbot §5: queries and compressed KV entries are RMS-normalised,
// so attention needs no extra QK normalisation]: with gamma given, every pooled entry c is
// written as c / sqrt(mean_ch(c^2) + eps) * gamma, in fp32 before the output rounding (so
// before any later quantisation of the cache).
#include <cuda_bf16.h>

#include <algorithm>

#include "hcl_common.cuh"
#include "hcl_internal.h"
#include "pool.cuh"

namespace hcl {
namespace {

__device__ __forceinline__ void store8(void* out, int out_fmt, size_t off, const float* v) {
  if (out_fmt == HCL_FP32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 pk;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
    for (int c = 0; c < 4; c++) h[c] = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + off) = pk;
  }
}

// One group of G = d/8 threads per entry; SPAN > 0: compile-time span, else `span`.
template <int SPAN>
__global__ void compress_small_kernel(const __nv_bfloat16* __restrict__ kv,
                                      const __nv_bfloat16* __restrict__ gate,
                                      const float* __restrict__ bias, int B, int L, int d,
                                      int m, int span, int first_off, int e0, int e1, void* out,
                                      int out_fmt, int out_cap, const float* __restrict__ gamma,
                                      float eps) {
  const int G = d >> 3;
  const long long n_ent = (long long)(e1 - e0) * B;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long item = gt / G;
  const int chunk = int(gt % G);
  if (item >= n_ent) return;  // whole groups only (G divides the block)
  const int b = int(item / (e1 - e0));
  const int i = e0 + int(item % (e1 - e0));
  const long long first = (long long)m * i + first_off;
  const __nv_bfloat16* kvb = kv + (size_t)b * L * d;
  const __nv_bfloat16* gb = gate + (size_t)b * L * d;
  auto row = [&](int j, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
    const long long t = first + j;
    if (t < 0 || t >= L) return false;
    kp = kvb + (size_t)t * d;
    gp = gb + (size_t)t * d;
    return true;
  };
  float v[8];
  if (SPAN > 0) pool8_span<(SPAN > 0 ? SPAN : 1)>(row, bias, chunk, v);
  else pool8_any(row, bias, span, chunk, v);
  if (gamma != nullptr) rmsnorm8_group(v, G, d, chunk, gamma, eps);
  store8(out, out_fmt, ((size_t)b * out_cap + i) * d + chunk * 8, v);
}

// One block of 128 threads per entry (pool_long_block).
__global__ void __launch_bounds__(128) compress_long_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int B, int L, int d, int m, int span, int e0, int e1,
    void* out, int out_fmt, int out_cap, const float* __restrict__ gamma, float eps) {
  extern __shared__ float sm[];  // [streams][3][d], then 4 floats for the RMSNorm reduction
  const int b = blockIdx.x / (e1 - e0);
  const int i = e0 + blockIdx.x % (e1 - e0);
  const long long first = (long long)m * i;
  const __nv_bfloat16* kvb = kv + (size_t)b * L * d;
  const __nv_bfloat16* gb = gate + (size_t)b * L * d;
  auto row = [&](int j, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
    const long long t = first + j;
    if (t < 0 || t >= L) return false;
    kp = kvb + (size_t)t * d;
    gp = gb + (size_t)t * d;
    return true;
  };
  float vals[8];
  pool_long_block(row, bias, span, d, sm, gamma, eps, vals);
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = threadIdx.x + u * 128;
    if (c >= d) continue;
    const size_t o = ((size_t)b * out_cap + i) * d + c;
    if (out_fmt == HCL_FP32) static_cast<float*>(out)[o] = vals[u];
    else static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(vals[u]);
  }
}

// ---- staged compressors: token rows brought into shared memory by bulk async copies -------
// A tile of entries of one sequence needs a contiguous range of token rows; one thread issues
// two bulk copies (kv rows, gate rows) completing on the stage's mbarrier, two stages ring so
// that the next tile streams in while the current one is pooled.  The per-slot arithmetic is
// Online8's (pool.cuh), in the same slot order as the batch and append paths.

constexpr int CS_THREADS = 256;
constexpr int CS_E = 16;           // CSA entries per tile
constexpr int CS_BLOCKS_PER_SM = 3;

struct StageRange {
  int b, e0, e1, tf, tl;           // sequence, entries [e0, e1), token rows [tf, tl)
};

__device__ __forceinline__ StageRange csa_tile(int t, int tiles_per_seq, int e0, int e1, int m,
                                               int L) {
  StageRange r;
  r.b = t / tiles_per_seq;
  r.e0 = e0 + (t % tiles_per_seq) * CS_E;
  r.e1 = min(e1, r.e0 + CS_E);
  r.tf = max(0, m * r.e0 - m);
  r.tl = min(L, m * r.e1);
  return r;
}

// CSA (span 2m, overlapped): tile = CS_E consecutive entries, rows [m(e0-1), m*e1).
__global__ void __launch_bounds__(CS_THREADS) csa_compress_staged_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int L, int d, int m, int e0, int e1, void* out, int out_fmt,
    int out_cap, const float* __restrict__ gamma, float eps, int tiles_per_seq, int n_tiles,
    int stage_rows, long long limit) {
  extern __shared__ __align__(128) uint8_t smc[];
  __shared__ uint64_t full[2];
  const int tid = threadIdx.x;
  const int G = d >> 3;
  const size_t row_b = (size_t)d * 2;
  auto st_kv = [&](int s) { return smc + (size_t)s * 2 * stage_rows * row_b; };
  auto st_g = [&](int s) { return smc + (size_t)s * 2 * stage_rows * row_b + stage_rows * row_b; };
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int t, int s) {
    const StageRange r = csa_tile(t, tiles_per_seq, e0, e1, m, L);
    const uint32_t bytes = uint32_t((r.tl - r.tf) * row_b);
    mbar_arrive_expect_tx(&full[s], 2 * bytes);
    bulk_load(st_kv(s), kv + ((size_t)r.b * L + r.tf) * d, bytes, &full[s]);
    bulk_load(st_g(s), gate + ((size_t)r.b * L + r.tf) * d, bytes, &full[s]);
  };
  if (tid == 0) {
    if ((int)blockIdx.x < n_tiles) issue(blockIdx.x, 0);
    if ((int)(blockIdx.x + gridDim.x) < n_tiles) issue(blockIdx.x + gridDim.x, 1);
  }
  int it = 0;
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, it++) {
    const int s = it & 1;
    const bool ok = mbar_wait(&full[s], (it >> 1) & 1, limit, nullptr);
    if (__syncthreads_or(!ok)) break;                 // uniform: a timed-out copy ends the block
    const StageRange r = csa_tile(t, tiles_per_seq, e0, e1, m, L);
    const __nv_bfloat16* skv = reinterpret_cast<const __nv_bfloat16*>(st_kv(s));
    const __nv_bfloat16* sg = reinterpret_cast<const __nv_bfloat16*>(st_g(s));
    const int items = (r.e1 - r.e0) * G;
    for (int item0 = 0; item0 < items; item0 += CS_THREADS) {
      const int item = item0 + tid;
      if (item < items) {                              // whole groups of G threads
        const int i = r.e0 + item / G, chunk = item % G;
        Online8 o;
        o.init();
        for (int j = 0; j < 2 * m; j++) {
          const long long u = (long long)m * (i - 1) + j;
          if (u < 0 || u >= L) continue;
          const size_t off = (size_t)(u - r.tf) * d;
          const uint4 xv = *(reinterpret_cast<const uint4*>(skv + off) + chunk);
          const uint4 gv = *(reinterpret_cast<const uint4*>(sg + off) + chunk);
          o.add(xv, gv, __ldg(bias + j));
        }
        float v[8];
        o.result(v);
        if (gamma != nullptr) rmsnorm8_group(v, G, d, chunk, gamma, eps);
        store8(out, out_fmt, ((size_t)r.b * out_cap + i) * d + chunk * 8, v);
      }
    }
    __syncthreads();                                   // stage s fully read
    if (tid == 0 && t + 2 * (int)gridDim.x < n_tiles) issue(t + 2 * gridDim.x, s);
  }
  // copies still in flight (only after a timeout) land before the block exits
  if (tid == 0) {
    for (int q = 0; q < 2; q++) {
      const int t = blockIdx.x + (it + q) * gridDim.x;
      if (t < n_tiles) mbar_wait(&full[(it + q) & 1], ((it + q) >> 1) & 1, limit, nullptr);
    }
  }
}

// HCA (span mh, no overlap): tile = one entry, rows [mh*i, mh*i + mh); 128 threads as in
// pool_long_block (d/8 channel chunks x 128/(d/8) slot streams, merged in shared memory).
__global__ void __launch_bounds__(128) hca_compress_staged_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int L, int d, int mh, int e0, int e1, void* out, int out_fmt,
    int out_cap, const float* __restrict__ gamma, float eps, int n_tiles, long long limit) {
  extern __shared__ __align__(128) uint8_t smh[];
  __shared__ uint64_t full[2];
  const int tid = threadIdx.x;
  const int G = d >> 3, streams = 128 / G, chunk = tid % G, stream = tid / G;
  const size_t row_b = (size_t)d * 2;
  const int ne = e1 - e0;
  float* part = reinterpret_cast<float*>(smh + (size_t)4 * mh * row_b);   // [streams][3][d] + 4
  auto st_kv = [&](int s) { return smh + (size_t)s * 2 * mh * row_b; };
  auto st_g = [&](int s) { return smh + (size_t)s * 2 * mh * row_b + mh * row_b; };
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int t, int s) {
    const int b = t / ne, i = e0 + t % ne;
    const int tf = mh * i, tl = min(L, mh * i + mh);
    const uint32_t bytes = uint32_t((tl - tf) * row_b);
    mbar_arrive_expect_tx(&full[s], 2 * bytes);
    bulk_load(st_kv(s), kv + ((size_t)b * L + tf) * d, bytes, &full[s]);
    bulk_load(st_g(s), gate + ((size_t)b * L + tf) * d, bytes, &full[s]);
  };
  if (tid == 0) {
    if ((int)blockIdx.x < n_tiles) issue(blockIdx.x, 0);
    if ((int)(blockIdx.x + gridDim.x) < n_tiles) issue(blockIdx.x + gridDim.x, 1);
  }
  int it = 0;
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, it++) {
    const int s = it & 1;
    const bool ok = mbar_wait(&full[s], (it >> 1) & 1, limit, nullptr);
    if (__syncthreads_or(!ok)) break;
    const int b = t / ne, i = e0 + t % ne;
    const int nrow = min(L, mh * i + mh) - mh * i;
    const __nv_bfloat16* skv = reinterpret_cast<const __nv_bfloat16*>(st_kv(s));
    const __nv_bfloat16* sg = reinterpret_cast<const __nv_bfloat16*>(st_g(s));
    Online8 o;
    o.init();
    if (stream < streams) {
      for (int j = stream; j < mh; j += streams) {
        if (j >= nrow) continue;                        // token past the end of the sequence
        const uint4 xv = *(reinterpret_cast<const uint4*>(skv + (size_t)j * d) + chunk);
        const uint4 gv = *(reinterpret_cast<const uint4*>(sg + (size_t)j * d) + chunk);
        o.add(xv, gv, __ldg(bias + j));
      }
      float* base = part + (size_t)stream * 3 * d;
#pragma unroll
      for (int c = 0; c < 8; c++) {
        base[chunk * 8 + c] = o.mx[c];
        base[d + chunk * 8 + c] = o.sum[c];
        base[2 * d + chunk * 8 + c] = o.acc[c];
      }
    }
    __syncthreads();                                   // stage s read; partials complete
    if (tid == 0 && t + 2 * (int)gridDim.x < n_tiles) issue(t + 2 * gridDim.x, s);
    float vals[8];
    merge_streams_block(part, streams, d, gamma, eps, vals);
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const int c = tid + u * 128;
      if (c >= d) continue;
      const size_t o2 = ((size_t)b * out_cap + i) * d + c;
      if (out_fmt == HCL_FP32) static_cast<float*>(out)[o2] = vals[u];
      else static_cast<__nv_bfloat16*>(out)[o2] = __float2bfloat16_rn(vals[u]);
    }
    __syncthreads();                                   // partials consumed
  }
  if (tid == 0) {
    for (int q = 0; q < 2; q++) {
      const int t = blockIdx.x + (it + q) * gridDim.x;
      if (t < n_tiles) mbar_wait(&full[(it + q) & 1], ((it + q) >> 1) & 1, limit, nullptr);
    }
  }
}

}  // namespace

hcl_status_t launch_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                             int d, int m, int overlap, int e0, int e1, void* out, int out_fmt,
                             int out_cap, const float* gamma, float eps, cudaStream_t st) {
  if (e1 <= e0 || B == 0) return HCL_OK;
  {
    // an error left by an earlier runtime call would otherwise be reported as this launch's
    const cudaError_t stale = cudaGetLastError();
    if (stale != cudaSuccess)
      return fail(HCL_ERR_CUDA, "compress: error pending before the launch: %s",
                  cudaGetErrorString(stale));
  }
  const int span = overlap ? 2 * m : m;
  const int G = d / 8;
  auto kvp = static_cast<const __nv_bfloat16*>(kv);
  auto gp = static_cast<const __nv_bfloat16*>(gate);
  const bool g_ok = G <= 32 && (G & (G - 1)) == 0;     // channel groups aligned in a warp
  if (overlap && g_ok && m <= 8) {
    // staged CSA path
    const int tiles_per_seq = (e1 - e0 + CS_E - 1) / CS_E;
    const int n_tiles = tiles_per_seq * B;
    const int stage_rows = CS_E * m + m;
    const int smem = 2 * 2 * stage_rows * d * 2;
    hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(csa_compress_staged_kernel),
                                      smem, false);
    if (e != HCL_OK) return e;
    const int grid = std::min(n_tiles, CS_BLOCKS_PER_SM * num_sms());
    csa_compress_staged_kernel<<<grid, CS_THREADS, smem, st>>>(
        kvp, gp, bias, L, d, m, e0, e1, out, out_fmt, out_cap, gamma, eps, tiles_per_seq, n_tiles,
        stage_rows, wait_limit_cycles());
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess)
      return fail(HCL_ERR_CUDA, "staged CSA compress launch (grid %d, %d threads, %d B shared): %s",
                  grid, CS_THREADS, smem, cudaGetErrorString(le));
    return HCL_OK;
  }
  if (!overlap && 128 % G == 0 && (size_t)4 * m * d * 2 + ((size_t)(128 / G) * 3 * d + 4) * 4 <= 200 * 1024) {
    // staged HCA path
    const int n_tiles = (e1 - e0) * B;
    const int smem = (int)((size_t)4 * m * d * 2 + ((size_t)(128 / G) * 3 * d + 4) * 4);
    hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(hca_compress_staged_kernel),
                                      smem, false);
    if (e != HCL_OK) return e;
    int per_sm = (228 * 1024) / (smem + 1024);
    per_sm = std::max(1, std::min(per_sm, 16));
    const int grid = std::min(n_tiles, per_sm * num_sms());
    hca_compress_staged_kernel<<<grid, 128, smem, st>>>(kvp, gp, bias, L, d, m, e0, e1, out,
                                                        out_fmt, out_cap, gamma, eps, n_tiles,
                                                        wait_limit_cycles());
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess)
      return fail(HCL_ERR_CUDA, "staged HCA compress launch (grid %d, 128 threads, %d B shared): %s",
                  grid, smem, cudaGetErrorString(le));
    return HCL_OK;
  }
  if (span <= 16 || 128 % G != 0) {
    const long long threads = (long long)(e1 - e0) * B * G;
    // whole groups per block: a multiple of G threads (G <= 128)
    const int blk = (256 / G) * G;
    const long long grid = (threads + blk - 1) / blk;
    const int first_off = overlap ? -m : 0;
    compress_small_kernel<0><<<(unsigned)grid, blk, 0, st>>>(kvp, gp, bias, B, L, d, m, span,
                                                              first_off, e0, e1, out, out_fmt,
                                                              out_cap, gamma, eps);
  } else {
    const int streams = 128 / G;
    const size_t smem = ((size_t)streams * 3 * d + 4) * sizeof(float);
    const long long grid = (long long)(e1 - e0) * B;
    compress_long_kernel<<<(unsigned)grid, 128, smem, st>>>(kvp, gp, bias, B, L, d, m, span, e0,
                                                            e1, out, out_fmt, out_cap, gamma, eps);
  }
  return check_launch("compress");
}

}  // namespace hcl
