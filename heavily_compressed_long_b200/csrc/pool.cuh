// pool.cuh -- softmax-gated pooling of token rows into one compressed entry, shared by the
// batch compressors (compress.cu) and the decode-time cache append (cache.cu), so that an
// entry appended during decode is bit for bit the entry the batch compressor writes.
//
// [Tripbot §3.1] every m tokens of KV become one entry by softmax-gated pooling with a learned
// position bias; [CSDN §1.1 工程细节] a CSA entry also pools the previous window's last m tokens;
// [Tripbot §3.2] an HCA entry pools m' = 128 tokens.  Per channel c, over the present slots j:
//     entry[c] = sum_j softmax_j(gate[t_j, c] + bias[j]) * kv[t_j, c]
//
// Arithmetic (fp32, base 2: z_j = gate * log2(e) + bias_j * log2(e), weights 2^(z_j - max)):
//   * a block of up to 8 slots is taken in two passes over registers -- the block's maximum,
//     then the weights, their sum and the weighted sum of kv -- with no data-dependent branch
//     (an absent slot has z = -inf and weight 0), two channels per paired-fp32 instruction;
//   * consecutive blocks of one run of slots combine as a blocked online softmax: the running
//     (max, sum, weighted sum) is rescaled once per block by 2^(old max - new max);
//   * long spans split their slots into NS streams of K consecutive slots (pool_streams); the
//     streams' partial (max, sum, weighted sum) are merged in stream order.
// [Tripbot §5] the optional RMSNorm of the entry: entry / sqrt(mean_c(entry^2) + eps) * gamma.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hcl_common.cuh"

namespace hcl {

constexpr float kPoolLog2e = 1.4426950408889634f;

__device__ __forceinline__ float pool_ex2(float x) { return ex2_ftz(x); }

// channels 2w, 2w+1 of a 16-byte row of 8 bf16, widened exactly to an fp32 pair
__device__ __forceinline__ unsigned long long bf16_pair(const uint4& v, int w) {
  const uint32_t u = w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
  return f2_make(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Running softmax state of 8 channels.
struct Pool8 {
  float M[8], S[8], A[8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int c = 0; c < 8; c++) { M[c] = -INFINITY; S[c] = 0.f; A[c] = 0.f; }
  }
  // One block of 8 slots: kv / gate rows (zero for an absent slot), bl[j] = bias_j * log2(e)
  // (-inf for an absent slot, so its z is -inf and its weight 0).  FIRST: the state is still the
  // initial one.  Channels go in pairs through the paired-fp32 instructions.
  template <bool FIRST>
  __device__ __forceinline__ void block(const uint4 (&xv)[8], const uint4 (&gv)[8],
                                        const float (&bl)[8]) {
    const unsigned long long l2e = f2_make(kPoolLog2e, kPoolLog2e);
#pragma unroll
    for (int w = 0; w < 4; w++) {
      unsigned long long z[8];
      float m0 = FIRST ? -INFINITY : M[2 * w], m1 = FIRST ? -INFINITY : M[2 * w + 1];
#pragma unroll
      for (int j = 0; j < 8; j++) z[j] = f2_fma(bf16_pair(gv[j], w), l2e, f2_make(bl[j], bl[j]));
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        m0 = fmax3(m0, f2_lo(z[j]), f2_lo(z[j + 1]));
        m1 = fmax3(m1, f2_hi(z[j]), f2_hi(z[j + 1]));
      }
      const float r0 = m0 == -INFINITY ? 0.f : m0, r1 = m1 == -INFINITY ? 0.f : m1;
      const unsigned long long neg = f2_make(-r0, -r1);
      unsigned long long s2 = 0ull, a2 = 0ull;   // +0.0f in both halves
      if (!FIRST) {
        // 0 while nothing was present
        const unsigned long long r = f2_make(pool_ex2(M[2 * w] - r0), pool_ex2(M[2 * w + 1] - r1));
        s2 = f2_mul(f2_make(S[2 * w], S[2 * w + 1]), r);
        a2 = f2_mul(f2_make(A[2 * w], A[2 * w + 1]), r);
      }
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const unsigned long long t = f2_add(z[j], neg);
        const unsigned long long e = f2_make(pool_ex2(f2_lo(t)), pool_ex2(f2_hi(t)));
        s2 = f2_add(s2, e);
        a2 = f2_fma(e, bf16_pair(xv[j], w), a2);
      }
      M[2 * w] = m0;
      M[2 * w + 1] = m1;
      S[2 * w] = f2_lo(s2);
      S[2 * w + 1] = f2_hi(s2);
      A[2 * w] = f2_lo(a2);
      A[2 * w + 1] = f2_hi(a2);
    }
  }
  __device__ __forceinline__ void result(float (&v)[8]) const {
#pragma unroll
    for (int c = 0; c < 8; c++) v[c] = S[c] > 0.f ? __fdividef(A[c], S[c]) : 0.f;
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

// Slots j0 .. j0+7 (those < jend) of channel chunk `chunk` into registers, all loads issued
// before any use.  row(j, kvp, gp) returns false for an absent slot, else its row pointers.
template <bool NC, class RowFn>
__device__ __forceinline__ void load_block8(RowFn row, const float* __restrict__ bias, int j0,
                                            int jend, int chunk, uint4 (&xv)[8], uint4 (&gv)[8],
                                            float (&bl)[8]) {
#pragma unroll
  for (int j = 0; j < 8; j++) {
    const int jj = j0 + j;
    const __nv_bfloat16* kp = nullptr;
    const __nv_bfloat16* gp = nullptr;
    const bool ok = jj < jend && row(jj, kp, gp);
    xv[j] = make_uint4(0, 0, 0, 0);
    gv[j] = make_uint4(0, 0, 0, 0);
    bl[j] = -INFINITY;
    if (ok) {
      xv[j] = ld_row16<NC>(kp, chunk);
      gv[j] = ld_row16<NC>(gp, chunk);
      bl[j] = __ldg(bias + jj) * kPoolLog2e;
    }
  }
}

// Slots [j0, j1) in blocks of 8 into a fresh state P.  ONE: the caller knows j1 - j0 <= 8
// (the same arithmetic without the loop).
template <bool NC, bool ONE = false, class RowFn>
__device__ __forceinline__ void pool_run(RowFn row, const float* __restrict__ bias, int j0,
                                         int j1, int chunk, Pool8& P) {
  uint4 xv[8], gv[8];
  float bl[8];
  P.init();
  load_block8<NC>(row, bias, j0, j1, chunk, xv, gv, bl);
  P.block<true>(xv, gv, bl);
  if (ONE) return;
  for (int jb = j0 + 8; jb < j1; jb += 8) {
    load_block8<NC>(row, bias, jb, j1, chunk, xv, gv, bl);
    P.block<false>(xv, gv, bl);
  }
}

// Channels [8*chunk, 8*chunk + 8) of one entry over all `span` slots, as one run.
template <bool NC = true, bool ONE = false, class RowFn>
__device__ __forceinline__ void pool8_any(RowFn row, const float* __restrict__ bias, int span,
                                          int chunk, float (&v)[8]) {
  Pool8 P;
  pool_run<NC, ONE>(row, bias, 0, span, chunk, P);
  P.result(v);
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

// ---- long spans: NS = 256 / (d/8) slot streams of K = ceil(span / NS) consecutive slots ------
__host__ __device__ constexpr int pool_streams(int d) { return 256 / (d / 8); }
__host__ __device__ constexpr int pool_stream_len(int span, int d) {
  return (span + pool_streams(d) - 1) / pool_streams(d);
}

// A stream's partial state into part ([NS][3][d] floats, 16-byte aligned), as 16-byte stores.
__device__ __forceinline__ void pool_store_partial(const Pool8& P, float* part, int d, int s,
                                                   int chunk) {
  float4* base = reinterpret_cast<float4*>(part + (size_t)s * 3 * d + chunk * 8);
  const int q = d / 4;                                    // float4s per [d] row
  base[0] = make_float4(P.M[0], P.M[1], P.M[2], P.M[3]);
  base[1] = make_float4(P.M[4], P.M[5], P.M[6], P.M[7]);
  base[q] = make_float4(P.S[0], P.S[1], P.S[2], P.S[3]);
  base[q + 1] = make_float4(P.S[4], P.S[5], P.S[6], P.S[7]);
  base[2 * q] = make_float4(P.A[0], P.A[1], P.A[2], P.A[3]);
  base[2 * q + 1] = make_float4(P.A[4], P.A[5], P.A[6], P.A[7]);
}

// Stream s's partial (max, sum, weighted sum) of channel chunk `chunk`, stored into
// part ([NS][3][d] floats).
template <bool NC, bool ONE = false, class RowFn>
__device__ __forceinline__ void pool_stream_partial(RowFn row, const float* __restrict__ bias,
                                                    int span, int d, int s, int chunk,
                                                    float* part) {
  const int K = pool_stream_len(span, d);
  const int j0 = s * K, j1 = min(span, j0 + K);
  Pool8 P;
  pool_run<NC, ONE>(row, bias, j0, j1, chunk, P);
  pool_store_partial(P, part, d, s, chunk);
}

// Merge of the NS stream partials in `part` (complete and visible to the block) by the block's
// first 128 threads: thread t < 128 returns, for channels c = t + 128u (u < 8, c < d), the
// entry in vals[u], RMS-normalised with gamma when given (red: 4 floats of shared scratch).
// Every thread of the block must call it.
__device__ __forceinline__ void pool_merge_streams(const float* part, int d, float* red,
                                                   const float* __restrict__ gamma, float eps,
                                                   float (&vals)[8]) {
  const int NS = pool_streams(d);
  const int t = threadIdx.x;
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = t + u * 128;
    vals[u] = 0.f;
    if (t >= 128 || c >= d) continue;
    float M = -INFINITY;
    for (int q = 0; q < NS; q++) M = fmaxf(M, part[(size_t)q * 3 * d + c]);
    const float mr = M == -INFINITY ? 0.f : M;
    float S = 0.f, A = 0.f;
    for (int q = 0; q < NS; q++) {
      const float* base = part + (size_t)q * 3 * d;
      const float w = pool_ex2(base[c] - mr);
      S = fmaf(base[d + c], w, S);
      A = fmaf(base[2 * d + c], w, A);
    }
    vals[u] = S > 0.f ? __fdividef(A, S) : 0.f;
    ss = fmaf(vals[u], vals[u], ss);
  }
  if (gamma != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (t < 128 && (t & 31) == 0) red[t >> 5] = ss;
    __syncthreads();
    const float rn = 1.f / sqrtf((red[0] + red[1] + red[2] + red[3]) / float(d) + eps);
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const int c = t + u * 128;
      if (t < 128 && c < d) vals[u] = vals[u] * rn * __ldg(gamma + c);
    }
  }
}

}  // namespace hcl
