// pool.cuh -- softmax-gated pooling of token rows into one compressed entry, shared by the
// batch compressors (compress.cu) and the decode-time cache append (cache.cu), so that an
// entry appended during decode is bit for bit the entry the batch compressor writes.
//
// [Tripbot §3.1] every m tokens of KV become one entry by softmax-gated pooling with a learned
// position bias; [CSDN §1.1 工程细节] a CSA entry also pools the previous window's last m tokens;
// [Tripbot §3.2] an HCA entry pools m' = 128 tokens.  Per channel c, over the present slots j:
//     entry[c] = sum_j softmax_j(gate[t_j, c] + bias[j]) * kv[t_j, c]
// computed as an online (running max, sum, weighted sum) softmax in fp32, slot by slot.
// [Tripbot §5] the optional RMSNorm of the entry: entry / sqrt(mean_c(entry^2) + eps) * gamma.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hcl {

struct Online8 {
  float mx[8], sum[8], acc[8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int c = 0; c < 8; c++) { mx[c] = -INFINITY; sum[c] = 0.f; acc[c] = 0.f; }
  }
  // one slot: 8 channels of kv and gate (16-byte vectors) with the slot's position bias
  __device__ __forceinline__ void add(const uint4& xv, const uint4& gv, float b) {
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&xv);
    const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(&gv);
#pragma unroll
    for (int c = 0; c < 8; c++) {
      const float z = __bfloat162float(g[c]) + b;
      const float xc = __bfloat162float(x[c]);
      if (z > mx[c]) {
        const float r = __expf(mx[c] - z);  // exp(-inf) = 0 on the first slot
        sum[c] = sum[c] * r + 1.f;
        acc[c] = acc[c] * r + xc;
        mx[c] = z;
      } else {
        const float e = __expf(z - mx[c]);
        sum[c] += e;
        acc[c] += e * xc;
      }
    }
  }
  __device__ __forceinline__ void result(float (&v)[8]) const {
#pragma unroll
    for (int c = 0; c < 8; c++) v[c] = sum[c] > 0.f ? acc[c] / sum[c] : 0.f;
  }
};

// 16-byte row loads: through the read-only (non-coherent) path, or -- for rows the calling
// kernel itself may have written (the decode-time append) -- through the coherent L1/L2 path.
template <bool NC>
__device__ __forceinline__ uint4 ld_row16(const __nv_bfloat16* p, int chunk) {
  const uint4* q = reinterpret_cast<const uint4*>(p) + chunk;
  if (NC) return __ldg(q);
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(q)
               : "memory");
  return v;
}

// Channels [8*chunk, 8*chunk + 8) of one entry over SPAN slots (a compile-time span, fully
// unrolled so that all 2*SPAN 16-byte loads are in flight before the arithmetic).
// row(j, kvp, gp) returns false for an absent slot, else the slot's kv and gate row pointers.
template <int SPAN, bool NC = true, class RowFn>
__device__ __forceinline__ void pool8_span(RowFn row, const float* __restrict__ bias, int chunk,
                                           float (&v)[8]) {
  uint4 xv[SPAN], gv[SPAN];
  bool ok[SPAN];
#pragma unroll
  for (int j = 0; j < SPAN; j++) {
    const __nv_bfloat16* kp;
    const __nv_bfloat16* gp;
    ok[j] = row(j, kp, gp);
    if (ok[j]) {
      xv[j] = ld_row16<NC>(kp, chunk);
      gv[j] = ld_row16<NC>(gp, chunk);
    }
  }
  Online8 s;
  s.init();
#pragma unroll
  for (int j = 0; j < SPAN; j++)
    if (ok[j]) s.add(xv[j], gv[j], __ldg(bias + j));
  s.result(v);
}

// The same for a span known only at run time (slot by slot).
template <bool NC = true, class RowFn>
__device__ __forceinline__ void pool8_any(RowFn row, const float* __restrict__ bias, int span,
                                          int chunk, float (&v)[8]) {
  Online8 s;
  s.init();
  for (int j = 0; j < span; j++) {
    const __nv_bfloat16* kp;
    const __nv_bfloat16* gp;
    if (!row(j, kp, gp)) continue;
    const uint4 xv = ld_row16<NC>(kp, chunk);
    const uint4 gv = ld_row16<NC>(gp, chunk);
    s.add(xv, gv, __ldg(bias + j));
  }
  s.result(v);
}

// RMSNorm of an entry held by a group of G = d/8 threads (8 channels each; G a power of two
// <= 32, aligned within the warp, all its lanes active): sums of squares added by shuffles.
__device__ __forceinline__ void rmsnorm8_group(float (&v)[8], int G, int d, int chunk,
                                               const float* __restrict__ gamma, float eps) {
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 8; c++) ss = fmaf(v[c], v[c], ss);
  const int lane = threadIdx.x & 31;
  const unsigned gmask = G >= 32 ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
  for (int o = G >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
  const float r = 1.f / sqrtf(ss / float(d) + eps);
#pragma unroll
  for (int c = 0; c < 8; c++) v[c] = v[c] * r * __ldg(gamma + chunk * 8 + c);
}

// The second half of a long-span pooling (see pool_long_block): thread t of a block of 128
// merges, for channels c = t + 128u (c < d), the S stream partials (max, sum, weighted sum)
// that sm holds ([S][3][d] floats, then 4 floats of scratch) into the entry value vals[u],
// RMS-normalised with gamma when given.  All 128 threads must call it.
__device__ __forceinline__ void merge_streams_block(float* sm, int streams, int d,
                                                    const float* __restrict__ gamma, float eps,
                                                    float (&vals)[8]) {
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = threadIdx.x + u * 128;
    vals[u] = 0.f;
    if (c >= d) continue;
    float M = -INFINITY;
    for (int q = 0; q < streams; q++) M = fmaxf(M, sm[(size_t)q * 3 * d + c]);
    float S = 0.f, A = 0.f;
    if (M > -INFINITY) {
      for (int q = 0; q < streams; q++) {
        const float* base = sm + (size_t)q * 3 * d;
        if (base[c] == -INFINITY) continue;
        const float r = __expf(base[c] - M);
        S += base[d + c] * r;
        A += base[2 * d + c] * r;
      }
    }
    vals[u] = S > 0.f ? A / S : 0.f;
    ss = fmaf(vals[u], vals[u], ss);
  }
  if (gamma != nullptr) {
    float* red = sm + (size_t)streams * 3 * d;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    const float rn = 1.f / sqrtf((red[0] + red[1] + red[2] + red[3]) / float(d) + eps);
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const int c = threadIdx.x + u * 128;
      if (c < d) vals[u] = vals[u] * rn * __ldg(gamma + c);
    }
  }
}

// Long spans (HCA): one entry per block of 128 threads.  Thread t works on channel chunk
// t % G (G = d/8) of slot stream t / G; stream s takes slots s, s + S, s + 2S, ... (S = 128/G
// streams); the streams' partial softmaxes are merged
// through shared memory `sm` ([S][3][d] floats, then 4 floats).  On return thread t holds, for
// channels c = t + 128u (u < MAXV, c < d), the entry in vals[u] -- RMS-normalised with gamma.
// All 128 threads must call it.
template <bool NC = true, class RowFn>
__device__ __forceinline__ void pool_long_block(RowFn row, const float* __restrict__ bias,
                                                int span, int d, float* sm,
                                                const float* __restrict__ gamma, float eps,
                                                float (&vals)[8]) {
  const int G = d >> 3;
  const int streams = 128 / G;
  const int chunk = threadIdx.x % G;
  const int stream = threadIdx.x / G;
  Online8 s;
  s.init();
  if (stream < streams) {
    for (int j = stream; j < span; j += streams) {
      const __nv_bfloat16* kp;
      const __nv_bfloat16* gp;
      if (!row(j, kp, gp)) continue;
      const uint4 xv = ld_row16<NC>(kp, chunk);
      const uint4 gv = ld_row16<NC>(gp, chunk);
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
  merge_streams_block(sm, streams, d, gamma, eps, vals);
}

}  // namespace hcl
