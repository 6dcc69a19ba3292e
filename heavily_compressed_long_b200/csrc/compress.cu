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
// token row, coalesced along d), issues the loads of 8 slots before any arithmetic and pools
// them in two branch-free passes in fp32 (pool.cuh).  CSA (and any d/8 that does not divide
// 256) gives each entry to one group of d/8 threads; HCA splits an entry's slots into 256/(d/8)
// streams, one per group of a 256-thread block, merged in shared memory.
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

// One group of G = d/8 threads per entry (all `span` slots as one run, blocks of 8 slots;
// ONE: span <= 8).
template <bool ONE>
__global__ void __launch_bounds__(128, ONE ? 5 : 1) compress_entry_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int B, int L, int d, int m, int span, int first_off, int e0,
    int e1, void* out, int out_fmt, int out_cap, const float* __restrict__ gamma, float eps) {
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
  pool8_any<true, ONE>(row, bias, span, chunk, v);
  if (gamma != nullptr) rmsnorm8_group(v, G, d, chunk, gamma, eps);
  store8(out, out_fmt, ((size_t)b * out_cap + i) * d + chunk * 8, v);
}

// CSA with m = 4 (span 8) and d/8 = 2^lgG: one group of d/8 threads per entry, a grid row per
// sequence (no index division), the bias (times log2 e) in shared memory, and entries whose 8
// slots all lie in [0, L) loaded without per-slot checks.  Same arithmetic as pool8_any.
__global__ void __launch_bounds__(128, 5) compress_span8_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int L, int d, int lgG, int m, int first_off, int e0, int e1,
    void* out, int out_fmt, int out_cap, const float* __restrict__ gamma, float eps) {
  __shared__ float bls[8];
  if (threadIdx.x < 8) bls[threadIdx.x] = __ldg(bias + threadIdx.x) * kPoolLog2e;
  __syncthreads();
  const int b = blockIdx.y;
  const int item = blockIdx.x * 128 + threadIdx.x;
  const int i = e0 + (item >> lgG), chunk = item & ((1 << lgG) - 1);
  if (i >= e1) return;  // whole groups only (the group size divides 128)
  const long long t0 = (long long)m * i + first_off;
  const size_t rs = (size_t)d >> 3;                      // row stride in 16-byte vectors
  const uint4* kvb = reinterpret_cast<const uint4*>(kv + (size_t)b * L * d) + chunk;
  const uint4* gb = reinterpret_cast<const uint4*>(gate + (size_t)b * L * d) + chunk;
  uint4 xv[8], gv[8];
  float bl[8];
  if (t0 >= 0 && t0 + 8 <= L) {
    const uint4* kp = kvb + (size_t)t0 * rs;
    const uint4* gp = gb + (size_t)t0 * rs;
#pragma unroll
    for (int j = 0; j < 8; j++) {
      xv[j] = __ldg(kp + j * rs);
      gv[j] = __ldg(gp + j * rs);
      bl[j] = bls[j];
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const long long t = t0 + j;
      xv[j] = make_uint4(0, 0, 0, 0);
      gv[j] = make_uint4(0, 0, 0, 0);
      bl[j] = -INFINITY;
      if (t >= 0 && t < L) {
        xv[j] = __ldg(kvb + (size_t)t * rs);
        gv[j] = __ldg(gb + (size_t)t * rs);
        bl[j] = bls[j];
      }
    }
  }
  Pool8 P;
  P.init();
  P.block<true>(xv, gv, bl);
  float v[8];
  P.result(v);
  if (gamma != nullptr) rmsnorm8_group(v, 1 << lgG, d, chunk, gamma, eps);
  store8(out, out_fmt, ((size_t)b * out_cap + i) * d + chunk * 8, v);
}

// One block of 256 threads per entry: thread t pools channel chunk t % G of slot stream t / G
// (pool_streams / pool_stream_len), the block's first 128 threads merge the streams.  ONE:
// streams of at most 8 slots.
template <bool ONE>
__global__ void __launch_bounds__(256, 2) compress_streams_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int L, int d, int m, int e0, int e1, void* out,
    int out_fmt, int out_cap, const float* __restrict__ gamma, float eps) {
  __shared__ __align__(16) float part[3 * 2048];   // [NS][3][d]: NS * d = 2048 for every d
  __shared__ float red[4];
  const int G = d >> 3;
  const int b = blockIdx.x / (e1 - e0);
  const int i = e0 + blockIdx.x % (e1 - e0);
  const long long first = (long long)m * i;
  const __nv_bfloat16* kvb = kv + (size_t)b * L * d;
  const __nv_bfloat16* gb = gate + (size_t)b * L * d;
  auto row = [&](int j, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
    const long long t = first + j;
    if (t >= L) return false;
    kp = kvb + (size_t)t * d;
    gp = gb + (size_t)t * d;
    return true;
  };
  pool_stream_partial<true, ONE>(row, bias, m, d, threadIdx.x / G, threadIdx.x % G, part);
  __syncthreads();
  float vals[8];
  pool_merge_streams(part, d, red, gamma, eps, vals);
  if (threadIdx.x >= 128) return;
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = threadIdx.x + u * 128;
    if (c >= d) continue;
    const size_t o = ((size_t)b * out_cap + i) * d + c;
    if (out_fmt == HCL_FP32) static_cast<float*>(out)[o] = vals[u];
    else static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(vals[u]);
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
  if (!overlap && 256 % G == 0) {
    const unsigned grid = (unsigned)((long long)(e1 - e0) * B);
    if (pool_stream_len(m, d) <= 8)
      compress_streams_kernel<true><<<grid, 256, 0, st>>>(kvp, gp, bias, L, d, m, e0, e1, out,
                                                          out_fmt, out_cap, gamma, eps);
    else
      compress_streams_kernel<false><<<grid, 256, 0, st>>>(kvp, gp, bias, L, d, m, e0, e1, out,
                                                           out_fmt, out_cap, gamma, eps);
  } else if (overlap && m == 4 && (G & (G - 1)) == 0 && B <= 65535) {
    int lg = 0;
    while ((1 << lg) < G) lg++;
    const dim3 grid((unsigned)(((long long)(e1 - e0) * G + 127) / 128), (unsigned)B);
    compress_span8_kernel<<<grid, 128, 0, st>>>(kvp, gp, bias, L, d, lg, m, -m, e0, e1, out,
                                                out_fmt, out_cap, gamma, eps);
  } else {
    const long long threads = (long long)(e1 - e0) * B * G;
    const int blk = (128 / G) * G;                     // whole groups per block (G <= 128)
    const long long grid = (threads + blk - 1) / blk;
    if (span <= 8)
      compress_entry_kernel<true><<<(unsigned)grid, blk, 0, st>>>(
          kvp, gp, bias, B, L, d, m, span, overlap ? -m : 0, e0, e1, out, out_fmt, out_cap, gamma,
          eps);
    else
      compress_entry_kernel<false><<<(unsigned)grid, blk, 0, st>>>(
          kvp, gp, bias, B, L, d, m, span, overlap ? -m : 0, e0, e1, out, out_fmt, out_cap, gamma,
          eps);
  }
  return check_launch("compress");
}

}  // namespace hcl
