// cache.cu -- decode-time maintenance of the heterogeneous KV cache.
//
// [Yanbaoke §5 KV cache management; Austery's talk notes, infrastructure section] the hybrid
// attention keeps a heterogeneous cache per layer: a raw sliding window of recent tokens, and
// compressed entries (CSA: one per m tokens with its lightning-indexer key; HCA: one per m'
// tokens).  During decode every sequence appends one token per step:
//   - its KV row goes into the raw window store at slot t mod cap (split rows quantised on
//     write exactly as hcl_quant_kv_fp8 does);
//   - its KV and gate rows go into the staging rings (slot t mod stage_cap) that keep the token
//     rows the compressors still need (the last 2m for CSA, m' for HCA);
//   - when t completes CSA entry i = t / m ((t + 1) % m == 0), the entry is pooled from the
//     staged rows by the batch compressor's own arithmetic (pool.cuh), optionally
//     RMS-normalised [Tripbot §5], rounded to bf16 and written at slot i mod cap (split rows
//     quantised as above), and the entry's index key is written (MXFP4 quantised exactly as
//     hcl_quant_mxfp4 does, or bf16);
//   - when t completes HCA entry i = t / m' the same for the HCA store.
// One block of 128 threads per sequence: warp 0 stages and writes the raw row, warp 1 pools the
// CSA entry (16 threads x 8 channels), warp 2 writes the index key, and all four warps pool
// the HCA entry.
#include <cuda_bf16.h>

#include "hcl_common.cuh"
#include "hcl_internal.h"
#include "mxfp4.cuh"
#include "pool.cuh"

namespace hcl {
namespace {

constexpr int AP_THREADS = 128;
constexpr int AP_D = 128;

struct AppendParams {
  const __nv_bfloat16* kv_new;
  const __nv_bfloat16* gate_new;
  const __nv_bfloat16* kI_new;
  const int32_t* t_new;
  __nv_bfloat16* stage_kv;
  __nv_bfloat16* stage_gate;
  int stage_cap;
  hcl_kv_t raw, kvc, kvh;
  int has_csa, has_hca;
  const float* bias_csa;
  int m;
  const float* bias_hca;
  int mh;
  int kI_fmt;
  uint8_t* kI;
  uint8_t* kI_sf;
  int kI_cap;
  const float* gamma;
  float eps;
};

// One 128-dim row written by the 32 lanes of a warp: lanes 0..15 hold 8 bf16 channels each
// (lane l: channels 8l .. 8l+7); lanes 16..31 only take part in the shuffles.  bf16 stores
// copy the row; split stores quantise channels 0..63 to E4M3 with the row scale
// amax / 448 (1 when amax is 0) and copy channels 64..127 (the RoPE dims).
__device__ __forceinline__ void write_row_warp(const hcl_kv_t& st, long long slot, const uint4& v) {
  const int lane = threadIdx.x & 31;
  if (st.fmt == HCL_BF16) {
    if (lane < 16)
      reinterpret_cast<uint4*>(const_cast<void*>(st.data))[slot * (AP_D / 8) + lane] = v;
    return;
  }
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&v);
  float a = 0.f;
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; i++) a = fmaxf(a, fabsf(bf2f(x[i])));
  }
  for (int o = 1; o < 8; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  const float sc = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
  if (lane < 8) {
    uint16_t q[4];
#pragma unroll
    for (int i = 0; i < 4; i++)
      q[i] = cvt_e4m3x2(__fdiv_rn(bf2f(x[2 * i]), sc), __fdiv_rn(bf2f(x[2 * i + 1]), sc));
    uint8_t* nope = static_cast<uint8_t*>(const_cast<void*>(st.data));
    *reinterpret_cast<uint2*>(nope + slot * (AP_D / 2) + lane * 8) =
        make_uint2(uint32_t(q[0]) | (uint32_t(q[1]) << 16), uint32_t(q[2]) | (uint32_t(q[3]) << 16));
    if (lane == 0) const_cast<float*>(st.scale)[slot] = sc;
  } else if (lane < 16) {
    __nv_bfloat16* rope = static_cast<__nv_bfloat16*>(const_cast<void*>(st.rope));
    *reinterpret_cast<uint4*>(rope + slot * (AP_D / 2) + (lane - 8) * 8) = v;
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
  uint4 pk;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
  for (int c = 0; c < 4; c++) h[c] = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
  return pk;
}

__global__ void __launch_bounds__(AP_THREADS) cache_append_kernel(AppendParams p) {
  __shared__ __align__(16) float part[3 * 2048];   // stream partials [NS][3][d] (pool.cuh), NS * d = 2048
  __shared__ float red[4];
  __shared__ float amax2[2];
  pdl_enter();
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long t = p.t_new[b];
  if (t < 0) return;                       // uniform over the block
  const int S = p.stage_cap;
  const size_t rowe = AP_D;                // elements per row
  __nv_bfloat16* skv = p.stage_kv + (size_t)b * S * rowe;
  __nv_bfloat16* sg = p.stage_gate + (size_t)b * S * rowe;

  // ---- the new token: staging rings and the raw window store
  if (warp == 0) {
    const int l16 = lane & 15;
    const __nv_bfloat16* src = (lane < 16 ? p.kv_new : p.gate_new) + (size_t)b * rowe;
    const uint4 v = *(reinterpret_cast<const uint4*>(src) + l16);
    __nv_bfloat16* dst = (lane < 16 ? skv : sg) + (size_t)(t % S) * rowe;
    reinterpret_cast<uint4*>(dst)[l16] = v;
    write_row_warp(p.raw, (long long)b * p.raw.cap + t % p.raw.cap, v);
  }
  __syncthreads();   // the staged row of t is visible to the whole block

  // rows of token u (u <= t) from the staging rings; coherent loads (token t's row was
  // written above by this block)
  auto staged = [&](long long u, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
    if (u < 0) return false;
    kp = skv + (size_t)(u % S) * rowe;
    gp = sg + (size_t)(u % S) * rowe;
    return true;
  };

  // ---- CSA entry i = t / m completed by t: slots j = 0 .. 2m-1 hold tokens t + 1 - 2m + j
  if (p.has_csa && (t + 1) % p.m == 0) {
    const long long i = t / p.m;
    const int span = 2 * p.m;
    if (warp == 1) {
      float v[8];
      auto row = [&](int j, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
        return staged(t + 1 - span + j, kp, gp);
      };
      if (lane < 16) {
        pool8_any<false>(row, p.bias_csa, span, lane, v);
        if (p.gamma != nullptr) rmsnorm8_group(v, 16, AP_D, lane, p.gamma, p.eps);
      }
      uint4 pk = make_uint4(0, 0, 0, 0);
      if (lane < 16) pk = pack8_bf16(v);
      write_row_warp(p.kvc, (long long)b * p.kvc.cap + i % p.kvc.cap, pk);
    } else if (warp == 2 && p.kI != nullptr) {
      const long long slot = (long long)b * p.kI_cap + i % p.kI_cap;
      const uint4* src = reinterpret_cast<const uint4*>(p.kI_new + (size_t)b * 64);
      if (p.kI_fmt == HCL_MXFP4) {
        if (lane < 2) {                    // one MXFP4 block of 32 values per lane
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; u++) v[u] = src[lane * 4 + u];
          uint4 pk;
          const int code = mxfp4_encode32(v, pk);
          reinterpret_cast<uint4*>(p.kI + slot * 32)[lane] = pk;
          p.kI_sf[slot * 2 + lane] = uint8_t(code);
        }
      } else if (lane < 8) {
        reinterpret_cast<uint4*>(p.kI + slot * 128)[lane] = src[lane];
      }
    }
  }

  // ---- HCA entry i = t / mh completed by t: slots j = 0 .. mh-1 hold tokens t + 1 - mh + j
  if (p.has_hca && (t + 1) % p.mh == 0) {
    const long long i = t / p.mh;
    auto row = [&](int j, const __nv_bfloat16*& kp, const __nv_bfloat16*& gp) {
      return staged(t + 1 - p.mh + j, kp, gp);
    };
    // the batch compressor's 256 threads as 128: thread t takes streams t / 16 and t / 16 + 8
    constexpr int NS = pool_streams(AP_D), G = AP_D / 8;
    static_assert(NS * G == 2 * AP_THREADS, "two slot streams per thread");
    pool_stream_partial<false>(row, p.bias_hca, p.mh, AP_D, tid / G, tid % G, part);
    pool_stream_partial<false>(row, p.bias_hca, p.mh, AP_D, tid / G + NS / 2, tid % G, part);
    __syncthreads();
    float vals[8];
    pool_merge_streams(part, AP_D, red, p.gamma, p.eps, vals);
    // thread c holds channel c; round to bf16 as the batch compressor's bf16 output does
    const __nv_bfloat16 xb = __float2bfloat16_rn(vals[0]);
    const long long slot = (long long)b * p.kvh.cap + i % p.kvh.cap;
    if (p.kvh.fmt == HCL_BF16) {
      static_cast<__nv_bfloat16*>(const_cast<void*>(p.kvh.data))[slot * AP_D + tid] = xb;
    } else {
      // split row: amax over channels 0..63 (warps 0, 1), then E4M3 pairs of channels
      float a = tid < 64 ? fabsf(bf2f(xb)) : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0 && warp < 2) amax2[warp] = a;
      __syncthreads();
      const float am = fmaxf(amax2[0], amax2[1]);
      const float sc = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
      const float hi = __shfl_down_sync(0xffffffffu, bf2f(xb), 1);
      if (tid < 64) {
        if ((tid & 1) == 0) {
          const uint16_t q = cvt_e4m3x2(__fdiv_rn(bf2f(xb), sc), __fdiv_rn(hi, sc));
          uint8_t* nope = static_cast<uint8_t*>(const_cast<void*>(p.kvh.data));
          *reinterpret_cast<uint16_t*>(nope + slot * (AP_D / 2) + tid) = q;
        }
        if (tid == 0) const_cast<float*>(p.kvh.scale)[slot] = sc;
      } else {
        __nv_bfloat16* rope = static_cast<__nv_bfloat16*>(const_cast<void*>(p.kvh.rope));
        rope[slot * (AP_D / 2) + (tid - 64)] = xb;
      }
    }
  }
}

}  // namespace

hcl_status_t launch_cache_append(const CacheAppendArgs& a, cudaStream_t st) {
  if (a.B == 0) return HCL_OK;
  AppendParams p;
  p.kv_new = static_cast<const __nv_bfloat16*>(a.kv_new);
  p.gate_new = static_cast<const __nv_bfloat16*>(a.gate_new);
  p.kI_new = static_cast<const __nv_bfloat16*>(a.kI_new);
  p.t_new = a.t_new;
  p.stage_kv = static_cast<__nv_bfloat16*>(a.stage_kv);
  p.stage_gate = static_cast<__nv_bfloat16*>(a.stage_gate);
  p.stage_cap = a.stage_cap;
  p.raw = a.raw;
  p.has_csa = a.kvc != nullptr;
  p.has_hca = a.kvh != nullptr;
  if (a.kvc) p.kvc = *a.kvc; else p.kvc = hcl_kv_t{HCL_BF16, 1, nullptr, nullptr, nullptr};
  if (a.kvh) p.kvh = *a.kvh; else p.kvh = hcl_kv_t{HCL_BF16, 1, nullptr, nullptr, nullptr};
  p.bias_csa = a.bias_csa;
  p.m = a.m;
  p.bias_hca = a.bias_hca;
  p.mh = a.mh;
  p.kI_fmt = a.kI_fmt;
  p.kI = static_cast<uint8_t*>(a.kI);
  p.kI_sf = static_cast<uint8_t*>(a.kI_sf);
  p.kI_cap = a.kI_cap > 0 ? a.kI_cap : 1;
  p.gamma = a.gamma;
  p.eps = a.eps;
  return check_cuda(launch_pdl(cache_append_kernel, dim3((unsigned)a.B), dim3(AP_THREADS), 0, st,
                               1, p),
                    "cache append launch");
}

}  // namespace hcl
