// compress.cu -- softmax-gated pooling compressor (CSA overlapped window, HCA plain window).
//
// [Tripbot §3.1] Every m tokens of KV become one entry by softmax-gated pooling with a
// learned position bias; [CSDN §1.1 工程细节] CSA entry i also pools the previous window's
// last m tokens (C^b) with its own m tokens (C^a), 2m slots in all; [Tripbot §3.2] HCA pools
// m' = 128 tokens per entry without overlap.  Per channel c of entry i, with slot j holding
// token t_j (slots outside [0, L) dropped):
//     out[i, c] = sum_j softmax_j(gate[t_j, c] + bias[j]) * kv[t_j, c]
//
// HBM-streaming kernel: each thread owns 8 channels (one 16-byte load of kv and of gate per
// token row, coalesced along d) and keeps an online (max, sum, weighted sum) softmax in fp32.
// Small spans (CSA: 2m <= 16) give each entry to one group of d/8 threads; long spans (HCA)
// split the slots over the 128 threads of a block and merge the partial softmaxes in shared
// memory.
#include <cuda_bf16.h>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace hcl {
namespace {

struct Online8 {
  float mx[8], sum[8], acc[8];
  __device__ void init() {
#pragma unroll
    for (int c = 0; c < 8; c++) { mx[c] = -INFINITY; sum[c] = 0.f; acc[c] = 0.f; }
  }
  __device__ void add(const uint4& xv, const uint4& gv, float b) {
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&xv);
    const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(&gv);
#pragma unroll
    for (int c = 0; c < 8; c++) {
      float z = bf2f(g[c]) + b;
      float xc = bf2f(x[c]);
      if (z > mx[c]) {
        float r = __expf(mx[c] - z);  // exp(-inf) = 0 on the first slot
        sum[c] = sum[c] * r + 1.f;
        acc[c] = acc[c] * r + xc;
        mx[c] = z;
      } else {
        float e = __expf(z - mx[c]);
        sum[c] += e;
        acc[c] += e * xc;
      }
    }
  }
};

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

// One group of G = d/8 threads per entry.
__global__ void compress_small_kernel(const __nv_bfloat16* __restrict__ kv,
                                      const __nv_bfloat16* __restrict__ gate,
                                      const float* __restrict__ bias, int B, int L, int d,
                                      int m, int span, int first_off, int e0, int e1, void* out,
                                      int out_fmt, int out_cap) {
  const int G = d >> 3;
  const long long n_ent = (long long)(e1 - e0) * B;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long item = gt / G;
  const int chunk = int(gt % G);
  if (item >= n_ent) return;
  const int b = int(item / (e1 - e0));
  const int i = e0 + int(item % (e1 - e0));
  const long long first = (long long)m * i + first_off;
  Online8 s;
  s.init();
  for (int j = 0; j < span; j++) {
    long long t = first + j;
    if (t < 0 || t >= L) continue;
    size_t off = ((size_t)b * L + t) * d + chunk * 8;
    uint4 xv = __ldg(reinterpret_cast<const uint4*>(kv + off));
    uint4 gv = __ldg(reinterpret_cast<const uint4*>(gate + off));
    s.add(xv, gv, __ldg(bias + j));
  }
  float v[8];
#pragma unroll
  for (int c = 0; c < 8; c++) v[c] = s.sum[c] > 0.f ? s.acc[c] / s.sum[c] : 0.f;
  store8(out, out_fmt, ((size_t)b * out_cap + i) * d + chunk * 8, v);
}

// One block of 128 threads per entry; the span is split over 128/G slot streams.
__global__ void __launch_bounds__(128) compress_long_kernel(
    const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ gate,
    const float* __restrict__ bias, int B, int L, int d, int m, int span, int e0, int e1,
    void* out, int out_fmt, int out_cap) {
  extern __shared__ float sm[];  // [streams][3][d]
  const int G = d >> 3;
  const int streams = 128 / G;
  const int chunk = threadIdx.x % G;
  const int stream = threadIdx.x / G;
  const int b = blockIdx.x / (e1 - e0);
  const int i = e0 + blockIdx.x % (e1 - e0);
  const long long first = (long long)m * i;
  Online8 s;
  s.init();
  if (stream < streams) {
    for (int j = stream; j < span; j += streams) {
      long long t = first + j;
      if (t < 0 || t >= L) continue;
      size_t off = ((size_t)b * L + t) * d + chunk * 8;
      uint4 xv = __ldg(reinterpret_cast<const uint4*>(kv + off));
      uint4 gv = __ldg(reinterpret_cast<const uint4*>(gate + off));
      s.add(xv, gv, __ldg(bias + j));
    }
    float* base = sm + (size_t)stream * 3 * d;
#pragma unroll
    for (int c = 0; c < 8; c++) {
      base[chunk * 8 + c] = s.mx[c];
      base[d + chunk * 8 + c] = s.sum[c];
      base[2 * d + chunk * 8 + c] = s.acc[c];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float M = -INFINITY;
    for (int q = 0; q < streams; q++) M = fmaxf(M, sm[(size_t)q * 3 * d + c]);
    float S = 0.f, A = 0.f;
    if (M > -INFINITY) {
      for (int q = 0; q < streams; q++) {
        const float* base = sm + (size_t)q * 3 * d;
        if (base[c] == -INFINITY) continue;
        float r = __expf(base[c] - M);
        S += base[d + c] * r;
        A += base[2 * d + c] * r;
      }
    }
    float v = S > 0.f ? A / S : 0.f;
    size_t o = ((size_t)b * out_cap + i) * d + c;
    if (out_fmt == HCL_FP32) static_cast<float*>(out)[o] = v;
    else static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(v);
  }
}

}  // namespace

hcl_status_t launch_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                             int d, int m, int overlap, int e0, int e1, void* out, int out_fmt,
                             int out_cap, cudaStream_t st) {
  if (e1 <= e0 || B == 0) return HCL_OK;
  const int span = overlap ? 2 * m : m;
  const int G = d / 8;
  auto kvp = static_cast<const __nv_bfloat16*>(kv);
  auto gp = static_cast<const __nv_bfloat16*>(gate);
  if (span <= 16 || 128 % G != 0) {
    long long threads = (long long)(e1 - e0) * B * G;
    int blk = 256;
    long long grid = (threads + blk - 1) / blk;
    compress_small_kernel<<<(unsigned)grid, blk, 0, st>>>(kvp, gp, bias, B, L, d, m, span,
                                                          overlap ? -m : 0, e0, e1, out, out_fmt,
                                                          out_cap);
  } else {
    const int streams = 128 / G;
    size_t smem = (size_t)streams * 3 * d * sizeof(float);
    long long grid = (long long)(e1 - e0) * B;
    compress_long_kernel<<<(unsigned)grid, 128, smem, st>>>(kvp, gp, bias, B, L, d, m, span, e0,
                                                            e1, out, out_fmt, out_cap);
  }
  return check_launch("compress");
}

}  // namespace hcl
