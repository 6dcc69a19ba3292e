// attn_flash.cu -- prefill attention on tcgen05 tensor cores (HCA dense, CSA selected).
//
// [Tripbot §3.2; CSDN §1.2] HCA attends densely over every compressed entry visible to the
// query (entry i of ratio m' is visible at position p when m'(i+1) - 1 <= p) and [Tripbot §3.3]
// over the raw tokens of its sliding window, under one softmax (scale, optional sink); each
// row is both key and value of the one shared KV head.  [Tripbot §3.1 step 2] CSA attends
// over the query's own top-k entries plus the same window.
//
// HCA over bf16 rows runs on the warp-specialised two-tile kernel at the end of this file; the
// kernel described next serves FP8 split rows and CSA prefill.
//
// Design (B200): one block of 256 threads per query group: G = floor(128 / H) consecutive
// queries x H heads = up to 128 (query, head) rows = the UMMA M dimension = 128 TMEM lanes, two
// threads per row.  The group's KV list is the visible-entry prefix of its last query followed
// by the union of its queries' windows; it is processed in rounds of 64 rows.  A round's rows
// are gathered with cp.async into one of three KV buffers (4 threads per row, each resolving the
// row's store slot; split FP8 rows widened to bf16 with their scale), so the gather of round
// r + 1, issued right after round r's S, is in flight while round r runs S = Q K^T (N = 64)
// into TMEM, its softmax and
// O += P V (V read as the MN-major operand of the same SW128 tile; O accumulates in TMEM
// across all rounds).  The softmax runs in registers with each row's own causal mask (for
// query q: the list rows [0, visible entries of q) and the window rows of q -- two index
// intervals, turned into bit masks; full 32-column words skip the per-column selects), its
// probabilities taken against a reference maximum that is raised only when the row maximum
// grows by more than 2^8, and only then is O rescaled in TMEM (load, scale, store).  Paired
// fp32 instructions form the exponents and sums.  Two blocks fit per SM (about 113 KB of
// shared memory, 256 TMEM columns each), so one block's softmax overlaps the other's MMAs.
//
// CSA prefill (every query has its own selection) uses the same kernel with G = 128 / H
// queries per block (2 at H = 64): the KV list is the concatenation of the G queries' lists
// (selected entries, then window) and each row's mask keeps its own query's segment, so the
// MMAs do G times the useful work -- on the tensor pipe, which has the room, and used only for
// H >= 32.
#include <cuda_bf16.h>

#include <algorithm>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace hcl {
namespace {

constexpr int FA_THREADS = 256;
constexpr int FA_ROWS = 128;
constexpr int FA_D = 128;
constexpr int FA_CH = 64;        // list rows per round
constexpr float FA_LOG2E = 1.4426950408889634f;
constexpr float FA_LN2 = 0.6931471805599453f;

struct FaParams {
  int mode;                 // 1: HCA (shared visible prefix + window union); 0: CSA segments
  const __nv_bfloat16* q;   // [B, Tq, H, 128]
  int B, Tq, H, G, n_groups;
  const int32_t* idx;       // CSA: [B, Tq, k]
  int k;
  hcl_kv_t comp, raw;
  int Nh, mh, W;
  const int32_t* q_pos;
  float scale_log2;
  const float* sink;
  const float* q_gamma;
  float q_eps;
  __nv_bfloat16* out;
  float* lse;
  int32_t* status;
  long long limit;
};

constexpr int FA_NBUF = 3;       // KV buffers: round r + 1 gathers while r and r - 1 are read
struct FaOff {
  static constexpr uint32_t Q = 0;                          // 2 halves x 128 rows x 128 B
  static constexpr uint32_t KV = 32768;                     // FA_NBUF x (2 halves x 64 rows x 128 B)
  static constexpr uint32_t P = KV + FA_NBUF * 16384;       // 128 rows x 64 bf16
  static constexpr uint32_t STG = P + 16384;                // FA_NBUF x 64 rows x 64 B codes
  static constexpr uint32_t SCL = STG + FA_NBUF * 4096;     // FA_NBUF x 64 scales
  static constexpr uint32_t XCH = SCL + FA_NBUF * 256;      // 2 x 256 floats
  static constexpr uint32_t BAR = XCH + 2 * FA_THREADS * 4; // 2 mbarriers, TMEM base, row bits
  static constexpr uint32_t TOTAL = BAR + 64;
};
static_assert(2 * (FaOff::TOTAL + 2048) <= 233472, "two blocks per SM");

// Rescale O only when the running maximum grows by more than this (log2 units): until then the
// probabilities are taken against the stale maximum (values <= 2^8, exact in fp32 sums).
constexpr float FA_RESCALE_LOG2 = 8.f;

__device__ __forceinline__ uint32_t fa_pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t fa_e4m3x2(uint16_t codes, float scale) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
  const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h2));
  return fa_pack(f.x * scale, f.y * scale);
}

// Bits j (0..31) of the columns c0 + j inside [lo, hi).
__device__ __forceinline__ uint32_t range_bits(int c0, int lo, int hi) {
  const int a = max(lo - c0, 0), e = min(hi - c0, 32);
  if (a >= e) return 0u;
  const uint32_t upto = e >= 32 ? 0xFFFFFFFFu : ((1u << e) - 1u);
  const uint32_t from = a <= 0 ? 0xFFFFFFFFu : ~((1u << a) - 1u);
  return upto & from;
}

template <int KVFMT>
__global__ void __launch_bounds__(FA_THREADS, 2) hca_flash_kernel(FaParams p) {
  extern __shared__ __align__(1024) uint8_t fa_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fa_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (FA_ROWS - 1), hc = tid / FA_ROWS;
  const int grp = blockIdx.x % p.n_groups, b = blockIdx.x / p.n_groups;
  const int t0 = grp * p.G;
  const int gq = min(p.G, p.Tq - t0);
  float* xch = reinterpret_cast<float*>(sm + FaOff::XCH);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + FaOff::BAR);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + FaOff::BAR + 16);
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(sTmem, 256);
    tmem_relinquish();
  }
  pdl_enter();
  // this thread's (query, head) row and its visibility intervals
  const int qi = row / p.H, hh = row % p.H;
  const bool rv = qi < gq;
  const int my_p = rv ? p.q_pos[(size_t)b * p.Tq + t0 + qi] : -1;
  int pmin = 0x7fffffff, pmax = -1;
  for (int i = 0; i < gq; i++) {
    const int pp = p.q_pos[(size_t)b * p.Tq + t0 + i];
    pmin = min(pmin, pp);
    pmax = max(pmax, pp);
  }
  // HCA list: the visible-entry prefix [0, n_a) of the last query, then window tokens
  // raw_lo .. raw_lo + n_raw - 1; CSA list: G segments of k + W rows (query i's selection, then
  // its window)
  const int n_a = pmax < 0 ? 0 : min(p.Nh, (pmax + 1) / p.mh);
  const int raw_lo = pmin - p.W + 1;
  const int n_raw = (p.W > 0 && pmax >= 0) ? max(0, pmax - raw_lo + 1) : 0;
  const int seg = p.k + p.W;
  const int total = p.mode == 1 ? n_a + n_raw : gq * seg;
  // list rows visible to this row: HCA: entries [0, nv_e) and window rows [w_lo, w_hi);
  // CSA: its own segment [w_lo, w_hi) (invalid rows are masked by the round's row bits)
  int nv_e = 0, w_lo = 0, w_hi = 0;
  if (p.mode == 1) {
    nv_e = my_p < 0 ? 0 : min(n_a, (my_p + 1) / p.mh);
    if (rv && my_p >= 0 && p.W > 0) {
      const int u_lo = max(0, my_p - p.W + 1);
      w_lo = n_a + (u_lo - raw_lo);
      w_hi = n_a + (my_p - raw_lo) + 1;
    }
  } else if (rv) {
    w_lo = qi * seg;
    w_hi = w_lo + seg;
  }

  // Q rows (query qi, head hh) -> SW128 halves, optionally RMS-normalised
  {
    const uint4* src = reinterpret_cast<const uint4*>(
                           p.q + (((size_t)b * p.Tq + t0 + (rv ? qi : 0)) * p.H + hh) * FA_D) + hc * 8;
    uint4 qv[8];
#pragma unroll
    for (int i = 0; i < 8; i++) qv[i] = rv ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    if (p.q_gamma != nullptr) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          ss = fmaf(lo, lo, fmaf(hi, hi, ss));
        }
      }
      xch[tid] = ss;
      __syncthreads();
      const float rn = 1.f / sqrtf((xch[row] + xch[row + FA_ROWS]) / float(FA_D) + p.q_eps);
#pragma unroll
      for (int i = 0; i < 8; i++) {
        uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int dim = hc * 64 + i * 8 + 2 * j;
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          w4[j] = fa_pack(lo * rn * __ldg(p.q_gamma + dim), hi * rn * __ldg(p.q_gamma + dim + 1));
        }
        qv[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; i++)
      *reinterpret_cast<uint4*>(sm + FaOff::Q + hc * 16384 + row * 128 + ((i ^ (row & 7)) << 4)) = qv[i];
  }

  tc_fence_after();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const uint32_t ocol = FA_CH;                             // S: columns 0..63, O: 64..191
  const uint32_t trow = tbase + (uint32_t((warp & 3) * 32) << 16);
  uint8_t* rb8 = sm + FaOff::BAR + 24;                     // [FA_NBUF][8 bytes]: row validity
  const int nrounds = (total + FA_CH - 1) / FA_CH;

  // gather of list rows [r0, r0 + 64) into buffer `buf`: 4 threads per row, each resolving the
  // row's store slot and copying its share of the row's 16-byte pieces with cp.async (rows past
  // the list, or without a source: zeros); mode 0 also records which rows are valid
  auto gather = [&](int rd, int buf) {
    const int r0 = rd * FA_CH, nr = min(FA_CH, total - r0);
    const int jj = tid >> 2, qtr = tid & 3, e = r0 + jj;
    long long slot = -1;
    bool from_raw = false;
    if (jj < nr) {
      if (p.mode == 1) {
        if (e < n_a) {
          slot = (long long)b * p.comp.cap + (e % p.comp.cap);
        } else {
          const int tok = raw_lo + (e - n_a);
          if (tok >= 0) { slot = (long long)b * p.raw.cap + tok % p.raw.cap; from_raw = true; }
        }
      } else {
        const int sq = e / seg, se = e - sq * seg;
        if (se < p.k) {
          const int ent = p.idx[((size_t)b * p.Tq + t0 + sq) * p.k + se];
          if (ent >= 0 && ent < p.Nh) slot = (long long)b * p.comp.cap + (ent % p.comp.cap);
          else if (qtr == 0 && (ent >= p.Nh || ent < -1)) report(p.status, HCL_ERR_DEVICE_FAULT);
        } else {
          const int tok = p.q_pos[(size_t)b * p.Tq + t0 + sq] - p.W + 1 + (se - p.k);
          if (tok >= 0) { slot = (long long)b * p.raw.cap + tok % p.raw.cap; from_raw = true; }
        }
      }
    }
    if (p.mode == 0) {
      const uint32_t bal = __ballot_sync(0xffffffffu, slot >= 0);
      uint32_t byte = 0;
#pragma unroll
      for (int i = 0; i < 8; i++) byte |= ((bal >> (4 * i)) & 1u) << i;
      if ((tid & 31) == 0) rb8[buf * 8 + warp] = uint8_t(byte);   // rows 8 warp .. 8 warp + 7
    }
    const hcl_kv_t& st = from_raw ? p.raw : p.comp;
    uint8_t* kv = sm + FaOff::KV + buf * 16384;
    if (KVFMT == HCL_BF16) {
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int pc = qtr * 4 + i;
        uint8_t* dst = kv + (pc >> 3) * 8192 + jj * 128 + (((pc & 7) ^ (jj & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.data) + slot * 256 + pc * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    } else if (qtr < 2) {                                  // RoPE dims 64..127, as stored
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int pc = qtr * 4 + i;
        uint8_t* dst = kv + 8192 + jj * 128 + ((pc ^ (jj & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.rope) + slot * 128 + pc * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    } else if (qtr == 2) {                                 // E4M3 codes of dims 0..63
#pragma unroll
      for (int i = 0; i < 4; i++) {
        uint8_t* dst = sm + FaOff::STG + buf * 4096 + jj * 64 + i * 16;
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.data) + slot * 64 + i * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    } else {
      float* dst = reinterpret_cast<float*>(sm + FaOff::SCL + buf * 256) + jj;
      if (slot >= 0)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                     "l"(st.scale + slot)
                     : "memory");
      else *dst = 0.f;
    }
    cp_async_commit();
  };

  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  const float c2 = p.scale_log2;
  const unsigned long long c2x2 = f2_make(c2, c2);
  if (nrounds > 0) gather(0, 0);
  for (int rd = 0; rd < nrounds; rd++) {
    const int buf = rd % FA_NBUF, r0 = rd * FA_CH, nr = min(FA_CH, total - r0);
    cp_async_wait<0>();                                    // gather(rd), this thread's copies
    __syncthreads();
    if (KVFMT == HCL_FP8SPLIT) {
      // widen: 8 codes x scale -> one 16-byte bf16 piece of the first half
      for (int u = tid; u < FA_CH * 8; u += FA_THREADS) {
        const int jj = u >> 3, cc = u & 7;
        const uint2 codes = *reinterpret_cast<const uint2*>(sm + FaOff::STG + buf * 4096 + jj * 64 + cc * 8);
        const float sc = reinterpret_cast<const float*>(sm + FaOff::SCL + buf * 256)[jj];
        uint4 v;
        v.x = fa_e4m3x2(uint16_t(codes.x & 0xffff), sc);
        v.y = fa_e4m3x2(uint16_t(codes.x >> 16), sc);
        v.z = fa_e4m3x2(uint16_t(codes.y & 0xffff), sc);
        v.w = fa_e4m3x2(uint16_t(codes.y >> 16), sc);
        *reinterpret_cast<uint4*>(sm + FaOff::KV + buf * 16384 + jj * 128 + ((cc ^ (jj & 7)) << 4)) = v;
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    // S = Q K^T for the 64 rows of the round (M = 128, N = 64, K = 128 in 8 steps)
    if (tid == 0) {
      const uint32_t aq = smem_u32(sm + FaOff::Q);
      const uint32_t ak = smem_u32(sm + FaOff::KV + buf * 16384);
#pragma unroll
      for (int ks = 0; ks < 8; ks++) {
        const uint32_t h = ks >> 2, kk = ks & 3;
        umma_bf16(tbase, make_sdesc(aq + h * 16384 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  make_sdesc(ak + h * 8192 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  idesc_bf16(128, FA_CH), ks > 0 ? 1u : 0u);
      }
      umma_commit(bar_s);
    }
    __syncwarp();   // warp 0 reconverges before waiting (the issuing lane is not left behind)
    // the next round's rows go into the buffer the PV two rounds back read (finished: this
    // block saw the S after it complete), while this round's S and the previous PV run
    if (rd + 1 < nrounds) gather(rd + 1, (rd + 1) % FA_NBUF);
    // S completes after every earlier MMA of this thread: the previous PV has finished reading
    // P and its KV buffer and writing O
    ok = ok && mbar_wait(bar_s, rd & 1, p.limit, nullptr);
    tc_fence_after();
    // this thread's 32 columns of the round
    uint32_t sv[32];
    tmem_ld16(trow + hc * 32, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
    tmem_ld16(trow + hc * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
    uint32_t vb = 0u;
    if (rv) {
      const int c0 = r0 + hc * 32;
      vb = (range_bits(c0, 0, nv_e) | range_bits(c0, w_lo, w_hi)) & range_bits(c0, r0, r0 + nr);
      if (p.mode == 0) vb &= *reinterpret_cast<const uint32_t*>(rb8 + buf * 8 + hc * 4);
    }
    tmem_ld_wait();
    // row maximum of the raw scores (the scale is positive, so max(s) * scale = max(s * scale))
    float smax = -INFINITY;
    if (vb == 0xFFFFFFFFu) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) smax = fmax3(smax, __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; j++)
        if ((vb >> j) & 1u) smax = fmaxf(smax, __uint_as_float(sv[j]));
    }
    xch[tid] = smax == -INFINITY ? -INFINITY : smax * c2;
    __syncthreads();
    const float m_cand = fmaxf(m_run, fmaxf(xch[row], xch[row + FA_ROWS]));
    // the same decision in both threads of a row: a new reference maximum only when it grew by
    // more than FA_RESCALE_LOG2 (or is the first finite one)
    const bool grow = m_cand > m_run + FA_RESCALE_LOG2;
    const float m_new = grow ? m_cand : m_run;
    const float alpha = (grow && m_run > -INFINITY) ? ex2_ftz(m_run - m_new) : 1.f;
    const float muse = m_new == -INFINITY ? 0.f : m_new;
    const unsigned long long negm = f2_make(-muse, -muse);
    // probabilities 2^(s * scale - m) of the valid columns, bf16 into P, fp32 into the row sum
    uint8_t* prow = sm + FaOff::P + row * 128;
    unsigned long long lr = 0ull;
#pragma unroll
    for (int q4 = 0; q4 < 4; q4++) {
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int j = q4 * 8 + i;
        const unsigned long long t = f2_fma(f2_make(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2x2, negm);
        float p0 = ex2_ftz(f2_lo(t)), p1 = ex2_ftz(f2_hi(t));
        if (vb != 0xFFFFFFFFu) {
          p0 = ((vb >> j) & 1u) ? p0 : 0.f;
          p1 = ((vb >> (j + 1)) & 1u) ? p1 : 0.f;
        }
        lr = f2_add(lr, f2_make(p0, p1));
        pk[i >> 1] = fa_pack(p0, p1);
      }
      *reinterpret_cast<uint4*>(prow + (((hc * 4 + q4) ^ (row & 7)) << 4)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    // O rescaled in TMEM where the reference maximum moved (no PV in flight: the previous one
    // was waited for above); warp-uniform (TMEM loads and stores are warp-collective)
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int q4 = 0; q4 < 4; q4++) {
        uint32_t r16[16];
        tmem_ld16(trow + ocol + hc * 64 + q4 * 16, r16);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i++) r16[i] = __float_as_uint(__uint_as_float(r16[i]) * alpha);
        tmem_st16(trow + ocol + hc * 64 + q4 * 16, r16);
      }
      tmem_st_wait();
    }
    const float lsum = f2_lo(lr) + f2_hi(lr);
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // O += P V (M = 128, N = 128 dims, K = 64 rows in 4 steps; V is the MN-major view of the
    // same tile: 64-dim halves 8 KB apart, 8-row groups 1 KB apart)
    if (tid == 0) {
      const uint32_t ap = smem_u32(sm + FaOff::P);
      const uint32_t av = smem_u32(sm + FaOff::KV + buf * 16384);
#pragma unroll
      for (int ks = 0; ks < 4; ks++)
        umma_bf16(tbase + ocol, make_sdesc(ap + ks * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  make_sdesc(av + ks * 2048, 8192, 1024, SMEM_SWIZZLE_128B),
                  idesc_bf16(128, FA_D) | (1u << 16), (rd > 0 || ks > 0) ? 1u : 0u);
      umma_commit(bar_o);
    }
    __syncwarp();
  }
  if (nrounds > 0) ok = ok && mbar_wait(bar_o, (nrounds - 1) & 1, p.limit, nullptr);
  tc_fence_after();
  if (!ok) report(p.status, HCL_ERR_TIMEOUT);
  xch[FA_THREADS + tid] = l_run;
  __syncthreads();
  float l2 = xch[FA_THREADS + row] + xch[FA_THREADS + row + FA_ROWS];
  float m2 = m_run;
  float f = l2 > 0.f ? 1.f / l2 : 0.f;
  if (p.sink) {
    const float s2 = p.sink[hh] * FA_LOG2E;
    const float mm = fmaxf(m2, s2);
    const float fa = l2 > 0.f ? exp2f(m2 - mm) : 0.f;
    const float l3 = l2 * fa + exp2f(s2 - mm);
    f = l3 > 0.f ? fa / l3 : 0.f;
    l2 = l3;
    m2 = mm;
  }
  const bool have_o = nrounds > 0;   // else O was never written
  const size_t orow = ((size_t)b * p.Tq + t0 + qi) * p.H + hh;
#pragma unroll
  for (int q4 = 0; q4 < 4; q4++) {
    uint32_t r16[16];
    tmem_ld16(trow + ocol + hc * 64 + q4 * 16, r16);
    tmem_ld_wait();
    if (!have_o) {
#pragma unroll
      for (int i = 0; i < 16; i++) r16[i] = 0u;
    }
    if (rv) {
      __nv_bfloat16* dst = p.out + orow * FA_D + hc * 64 + q4 * 16;
#pragma unroll
      for (int i = 0; i < 16; i += 8)
        *reinterpret_cast<uint4*>(dst + i) = make_uint4(
            fa_pack(__uint_as_float(r16[i]) * f, __uint_as_float(r16[i + 1]) * f),
            fa_pack(__uint_as_float(r16[i + 2]) * f, __uint_as_float(r16[i + 3]) * f),
            fa_pack(__uint_as_float(r16[i + 4]) * f, __uint_as_float(r16[i + 5]) * f),
            fa_pack(__uint_as_float(r16[i + 6]) * f, __uint_as_float(r16[i + 7]) * f));
    }
  }
  if (rv && hc == 0 && p.lse) p.lse[orow] = l2 > 0.f ? (m2 + log2f(l2)) * FA_LN2 : -INFINITY;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

template <int KVFMT>
hcl_status_t launch_flash_t(const FaParams& p, cudaStream_t st) {
  auto kern = hca_flash_kernel<KVFMT>;
  const int smem = (int)FaOff::TOTAL + 1024;
  hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, false);
  if (e != HCL_OK) return e;
  return check_cuda(launch_pdl(kern, dim3((unsigned)((long long)p.B * p.n_groups)),
                               dim3(FA_THREADS), (size_t)smem, st, 1, p),
                    "hca flash attention launch");
}


// ---------------------------------------------------------------------------------------
// HCA prefill, warp-specialised: two query tiles per block share the KV rounds.
//
// Block = (sequence, pair of query groups): tile t in {0, 1} holds group 2 * pair + t (up to
// 128 (query, head) rows each).  The pair's KV list is the visible-entry prefix of its last
// query plus the union of its queries' windows, in rounds of 128 rows.  Warps 0..3 and 4..7
// are the softmax warpgroups of tiles 0 and 1 (one thread per row, no exchange between
// threads); warps 8 and 9 gather the rounds' rows with cp.async into a ring of three KV
// buffers (two rows per thread); one thread of warp 11 issues every MMA from descriptors built
// once.  S = Q K^T is an N = 128 MMA (full tensor rate; at N = 64 with both operands in shared
// memory it is bound by shared-memory bandwidth).  The softmax reads a round's 128 scores of
// its row from TMEM twice (row maximum, then exponentials) and writes P (bf16) over the first
// 64 columns of its S; PV reads P from TMEM as its A operand, so the MMAs' shared-memory
// traffic is Q, K and V only.  Issue order per round: PV_0(r), S_0(r+1), PV_1(r), S_1(r+1);
// S_t(r+1) waits until PV_t(r) has completed (it overwrites P_t), and while tile t's softmax
// runs the tensor pipe works on the other tile.
// TMEM: S_0 / P_0, S_1 / P_1 (128 columns each), O_0, O_1 (128 each) -- one block per SM.
//
//   kv_full[b]  (64 gather threads)   round rows landed in buffer b (copies done, proxy-fenced)
//   kv_empty[b] (MMA commit)          both tiles' PV of the buffer's round completed
//   s_full[t]   (MMA commit)          S_t of the round in TMEM (and PV_t of the previous round
//                                     completed: O_t stable)
//   p_full[t]   (128 softmax threads) P_t in TMEM (and O_t rescaled)
//   o_done[t]   (MMA commit)          PV_t of the round completed (P_t free, O_t stable)
// Every wait is bounded; a timeout sets the block's abort flag and HCL_ERR_TIMEOUT.

// D (+)= A B with A (M = 128 rows in the TMEM lanes, K packed two bf16 per column) read from
// tensor memory and B from shared memory.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr int WS_WARPS = 12;
constexpr int WS_GATHER = 64;   // warps 8, 9 (warp 10 idles: warps are allocated in fours)
constexpr int WS_THREADS = WS_WARPS * 32;
constexpr int WS_NBUF = 3;
constexpr int WS_CH = 128;          // list rows per round
constexpr uint32_t WS_OCOL = 256;   // TMEM: S_0, S_1 at 0, 128; O_0, O_1 at 256, 384
struct WsOff {
  static constexpr uint32_t Q = 0;                            // 2 tiles x 2 halves x 128 x 128 B
  static constexpr uint32_t KV = 65536;                       // 3 x (2 halves x 128 rows x 128 B)
  static constexpr uint32_t BAR = KV + WS_NBUF * 32768;       // mbarriers
  static constexpr int NBAR = 2 * WS_NBUF + 3 * 2 + 1;        // kv_full/empty, s/p/o x 2, drain
  static constexpr uint32_t MISC = BAR + NBAR * 8;            // TMEM base, abort flag
  static constexpr uint32_t TOTAL = MISC + 16;
};
static_assert(WsOff::TOTAL + 1024 <= 232448, "shared memory");

__global__ void __launch_bounds__(WS_THREADS, 1) hca_flash_ws_kernel(FaParams p) {
  extern __shared__ __align__(1024) uint8_t ws_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_pairs = (p.n_groups + 1) / 2;
  const int pair = blockIdx.x % n_pairs, b = blockIdx.x / n_pairs;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + WsOff::BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + WS_NBUF;
  uint64_t* s_full = bars + 2 * WS_NBUF;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = s_full + 4;
  uint64_t* drain = s_full + 6;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + WsOff::MISC);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sm + WsOff::MISC + 4);
  if (tid == 0) {
    for (int i = 0; i < WS_NBUF; i++) { mbar_init(&kv_full[i], WS_GATHER); mbar_init(&kv_empty[i], 1); }
    for (int t = 0; t < 2; t++) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    *sAbort = 0;
    fence_barrier_init();
  }
  if (warp == 11) {
    tmem_alloc(sTmem, 512);
    tmem_relinquish();
  }
  pdl_enter();

  // the pair's queries [q_lo, q_hi) and its KV list: visible-entry prefix [0, n_a) of the last
  // query, then window tokens raw_lo .. raw_lo + n_raw - 1
  const int q_lo = 2 * pair * p.G, q_hi = min(p.Tq, q_lo + 2 * p.G);
  int pmin = 0x7fffffff, pmax = -1;
  for (int i = q_lo; i < q_hi; i++) {
    const int pp = p.q_pos[(size_t)b * p.Tq + i];
    pmin = min(pmin, pp);
    pmax = max(pmax, pp);
  }
  const int n_a = pmax < 0 ? 0 : min(p.Nh, (pmax + 1) / p.mh);
  const int raw_lo = pmin - p.W + 1;
  const int n_raw = (p.W > 0 && pmax >= 0) ? max(0, pmax - raw_lo + 1) : 0;
  const int total = n_a + n_raw;
  const int nrounds = (total + WS_CH - 1) / WS_CH;

  // softmax threads: this thread's tile, row, query and visibility intervals
  const int t = (tid >> 7) & 1, row = tid & 127;
  const int t0 = q_lo + t * p.G, gq = max(0, min(p.G, p.Tq - t0));
  const int qi = row / p.H, hh = row % p.H;
  const bool rv = warp < 8 && qi < gq;
  int nv_e = 0, w_lo = 0, w_hi = 0;
  if (rv) {
    const int my_p = p.q_pos[(size_t)b * p.Tq + t0 + qi];
    nv_e = my_p < 0 ? 0 : min(n_a, (my_p + 1) / p.mh);
    if (my_p >= 0 && p.W > 0) {
      const int u_lo = max(0, my_p - p.W + 1);
      w_lo = n_a + (u_lo - raw_lo);
      w_hi = n_a + (my_p - raw_lo) + 1;
    }
  }
  if (warp < 8) {
    // Q row (query t0 + qi, head hh) -> tile t's SW128 halves, optionally RMS-normalised
    const uint4* src = reinterpret_cast<const uint4*>(
        p.q + (((size_t)b * p.Tq + t0 + (rv ? qi : 0)) * p.H + hh) * FA_D);
    uint4 qv[16];
#pragma unroll
    for (int i = 0; i < 16; i++) qv[i] = rv ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    if (p.q_gamma != nullptr) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          ss = fmaf(lo, lo, fmaf(hi, hi, ss));
        }
      }
      const float rn = 1.f / sqrtf(ss / float(FA_D) + p.q_eps);
#pragma unroll
      for (int i = 0; i < 16; i++) {
        uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int dim = i * 8 + 2 * j;
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          w4[j] = fa_pack(lo * rn * __ldg(p.q_gamma + dim), hi * rn * __ldg(p.q_gamma + dim + 1));
        }
        qv[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
    uint8_t* qt = sm + WsOff::Q + t * 32768;
#pragma unroll
    for (int i = 0; i < 16; i++)
      *reinterpret_cast<uint4*>(qt + (i >> 3) * 16384 + row * 128 + (((i & 7) ^ (row & 7)) << 4)) = qv[i];
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;

  if (warp == 8 || warp == 9) {
    // ---------------- gather: list rows jj and jj + 64 of each round, 16 pieces each ----------
    // a round is signalled as soon as its own copies have landed, so the MMA warp never waits
    // for the gather of a later round
    const int jj = tid - 256;
    for (int rd = 0; rd < nrounds; rd++) {
      const int buf = rd % WS_NBUF;
      if (rd >= WS_NBUF && !mbar_wait(&kv_empty[buf], ((rd / WS_NBUF) & 1) ^ 1, p.limit, sAbort)) {
        *sAbort = 1;
        report(p.status, HCL_ERR_TIMEOUT);
        break;
      }
#pragma unroll
      for (int hr = 0; hr < 2; hr++) {
        const int rr = jj + 64 * hr, e = rd * WS_CH + rr;
        long long slot = -1;
        bool from_raw = false;
        if (e < total) {
          if (e < n_a) {
            slot = (long long)b * p.comp.cap + (e < p.comp.cap ? e : e % p.comp.cap);
          } else {
            const int tok = raw_lo + (e - n_a);
            if (tok >= 0) {
              slot = (long long)b * p.raw.cap + (tok < p.raw.cap ? tok : tok % p.raw.cap);
              from_raw = true;
            }
          }
        }
        const uint8_t* srow = static_cast<const uint8_t*>(from_raw ? p.raw.data : p.comp.data) +
                              (slot < 0 ? 0 : slot) * 256;
        uint8_t* dst = sm + WsOff::KV + buf * 32768 + rr * 128;
#pragma unroll
        for (int i = 0; i < 16; i++) {
          uint8_t* d = dst + (i >> 3) * 16384 + (((i & 7) ^ (rr & 7)) << 4);
          if (slot >= 0) cp_async16(d, srow + i * 16);
          else *reinterpret_cast<uint4*>(d) = make_uint4(0, 0, 0, 0);
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[buf]);
    }
    cp_async_wait<0>();
  } else if (warp == 11) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nrounds > 0) {
      // descriptors built once; a k-step moves the start address field (16-byte units)
      const uint64_t dq = make_sdesc(smem_u32(sm + WsOff::Q), 16, 1024, SMEM_SWIZZLE_128B);
      const uint64_t dk = make_sdesc(smem_u32(sm + WsOff::KV), 16, 1024, SMEM_SWIZZLE_128B);
      const uint64_t dv = make_sdesc(smem_u32(sm + WsOff::KV), 16384, 1024, SMEM_SWIZZLE_128B);
      constexpr uint32_t idS = idesc_bf16(128, WS_CH), idPV = idesc_bf16(128, FA_D) | (1u << 16);
      auto issue_s = [&](int tt, int rd) {
        const uint64_t a0 = dq + uint64_t(tt * (32768 >> 4));
        const uint64_t b0 = dk + uint64_t((rd % WS_NBUF) * (32768 >> 4));
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
          const uint32_t off_a = (ks >> 2) * (16384 >> 4) + (ks & 3) * 2;
          const uint32_t off_b = (ks >> 2) * (16384 >> 4) + (ks & 3) * 2;
          umma_bf16(tbase + tt * WS_CH, a0 + off_a, b0 + off_b, idS, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[tt]);
      };
      auto issue_pv = [&](int tt, int rd) {
        const uint64_t b0 = dv + uint64_t((rd % WS_NBUF) * (32768 >> 4));
#pragma unroll
        for (int ks = 0; ks < 8; ks++)
          umma_bf16_ta(tbase + WS_OCOL + tt * FA_D, tbase + tt * WS_CH + ks * 8,
                       b0 + uint32_t(ks * (2048 >> 4)), idPV, (rd > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&o_done[tt]);
      };
      bool ok = mbar_wait(&kv_full[0], 0, p.limit, sAbort);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int rd = 0; ok && rd < nrounds; rd++) {
        for (int tt = 0; tt < 2 && ok; tt++) {
          ok = mbar_wait(&p_full[tt], rd & 1, p.limit, sAbort);
          if (!ok) break;
          tc_fence_after();
          issue_pv(tt, rd);
          if (tt == 1) umma_commit(&kv_empty[rd % WS_NBUF]);
          if (rd + 1 < nrounds) {
            // S_t(r + 1) overwrites P_t: PV_t(r) must have completed
            if (tt == 0) ok = mbar_wait(&kv_full[(rd + 1) % WS_NBUF], ((rd + 1) / WS_NBUF) & 1, p.limit, sAbort);
            ok = ok && mbar_wait(&o_done[tt], rd & 1, p.limit, sAbort);
            if (!ok) break;
            tc_fence_after();
            issue_s(tt, rd + 1);
          }
        }
      }
      if (!ok) {
        *sAbort = 1;
        report(p.status, HCL_ERR_TIMEOUT);
      }
      // every MMA issued has completed before TMEM may be freed
      umma_commit(drain);
      if (!mbar_wait(drain, 0, p.limit, nullptr)) report(p.status, HCL_ERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------- softmax of tile t: this thread's row ----------------
    const uint32_t lq = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lq + t * WS_CH;            // S_t; P_t over its first 64 columns
    const uint32_t tO = tbase + lq + WS_OCOL + t * FA_D;
    const float c2 = p.scale_log2;
    const unsigned long long c2x2 = f2_make(c2, c2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int rd = 0; rd < nrounds; rd++) {
      const int r0 = rd * WS_CH;
      ok = mbar_wait(&s_full[t], rd & 1, p.limit, sAbort);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t vb[4] = {0u, 0u, 0u, 0u};
      if (rv) {
#pragma unroll
        for (int w = 0; w < 4; w++) {
          const int c0 = r0 + 32 * w;
          vb[w] = range_bits(c0, 0, nv_e) | range_bits(c0, w_lo, w_hi);
        }
      }
      // row maximum of the raw scores over the valid columns (scale > 0)
      uint32_t sv[64];
      float smax = -INFINITY;
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
#pragma unroll
        for (int k = 0; k < 4; k++)
          tmem_ld16(tS + hf * 64 + 16 * k, *reinterpret_cast<uint32_t(*)[16]>(&sv[16 * k]));
        tmem_ld_wait();
#pragma unroll
        for (int w = 0; w < 2; w++) {
          const uint32_t bits = vb[2 * hf + w];
          if (bits == 0xFFFFFFFFu) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              smax = fmax3(smax, __uint_as_float(sv[32 * w + j]), __uint_as_float(sv[32 * w + j + 1]));
          } else if (bits != 0u) {
#pragma unroll
            for (int j = 0; j < 32; j++)
              if ((bits >> j) & 1u) smax = fmaxf(smax, __uint_as_float(sv[32 * w + j]));
          }
        }
      }
      const float m_cand = fmaxf(m_run, smax == -INFINITY ? -INFINITY : smax * c2);
      const bool grow = m_cand > m_run + FA_RESCALE_LOG2;
      const float m_new = grow ? m_cand : m_run;
      const float alpha = (grow && m_run > -INFINITY) ? ex2_ftz(m_run - m_new) : 1.f;
      const float muse = m_new == -INFINITY ? 0.f : m_new;
      const unsigned long long negm = f2_make(-muse, -muse);
      // O_t is stable: s_full of this round came after PV_t of the previous one completed
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int q8 = 0; q8 < 8; q8++) {
          uint32_t r16[16];
          tmem_ld16(tO + q8 * 16, r16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i++) r16[i] = __float_as_uint(__uint_as_float(r16[i]) * alpha);
          tmem_st16(tO + q8 * 16, r16);
        }
      }
      // probabilities, 64 columns per TMEM wait: P of columns 64c .. 64c + 63 (32 TMEM columns
      // of bf16 pairs) goes over S columns 32c .. 32c + 31, whose scores this thread has
      // already used (its own lane; the next load reads columns 64 .. 127)
      unsigned long long lr = 0ull;
#pragma unroll
      for (int c = 0; c < 2; c++) {
#pragma unroll
        for (int k = 0; k < 4; k++)
          tmem_ld16(tS + 64 * c + 16 * k, *reinterpret_cast<uint32_t(*)[16]>(&sv[16 * k]));
        tmem_ld_wait();
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const uint32_t bits = vb[2 * c + (j >> 5)];
          const unsigned long long x =
              f2_fma(f2_make(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2x2, negm);
          float p0 = ex2_ftz(f2_lo(x)), p1 = ex2_ftz(f2_hi(x));
          if (bits != 0xFFFFFFFFu) {
            p0 = ((bits >> (j & 31)) & 1u) ? p0 : 0.f;
            p1 = ((bits >> ((j + 1) & 31)) & 1u) ? p1 : 0.f;
          }
          lr = f2_add(lr, f2_make(p0, p1));
          pk[j >> 1] = fa_pack(p0, p1);
        }
        tmem_st16(tS + 32 * c, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
        tmem_st16(tS + 32 * c + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
      }
      l_run = l_run * alpha + (f2_lo(lr) + f2_hi(lr));
      m_run = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    if (ok && nrounds > 0) {
      ok = mbar_wait(&o_done[t], (nrounds - 1) & 1, p.limit, sAbort);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (!ok) {
      *sAbort = 1;
      report(p.status, HCL_ERR_TIMEOUT);
    }
    tc_fence_after();
    // epilogue: O / l (with the optional sink), bf16 rows, log-sum-exp
    float l2 = l_run, m2 = m_run;
    float f = l2 > 0.f ? 1.f / l2 : 0.f;
    if (p.sink) {
      const float s2 = p.sink[hh] * FA_LOG2E;
      const float mm = fmaxf(m2, s2);
      const float fa = l2 > 0.f ? exp2f(m2 - mm) : 0.f;
      const float l3 = l2 * fa + exp2f(s2 - mm);
      f = l3 > 0.f ? fa / l3 : 0.f;
      l2 = l3;
      m2 = mm;
    }
    const bool have_o = nrounds > 0 && ok;
    const size_t orow = ((size_t)b * p.Tq + t0 + qi) * p.H + hh;
#pragma unroll
    for (int q8 = 0; q8 < 8; q8++) {
      uint32_t r16[16];
      tmem_ld16(tO + q8 * 16, r16);
      tmem_ld_wait();
      if (!have_o) {
#pragma unroll
        for (int i = 0; i < 16; i++) r16[i] = 0u;
      }
      if (rv) {
        __nv_bfloat16* dst = p.out + orow * FA_D + q8 * 16;
#pragma unroll
        for (int i = 0; i < 16; i += 8)
          *reinterpret_cast<uint4*>(dst + i) = make_uint4(
              fa_pack(__uint_as_float(r16[i]) * f, __uint_as_float(r16[i + 1]) * f),
              fa_pack(__uint_as_float(r16[i + 2]) * f, __uint_as_float(r16[i + 3]) * f),
              fa_pack(__uint_as_float(r16[i + 4]) * f, __uint_as_float(r16[i + 5]) * f),
              fa_pack(__uint_as_float(r16[i + 6]) * f, __uint_as_float(r16[i + 7]) * f));
      }
    }
    if (rv && p.lse) p.lse[orow] = l2 > 0.f ? (m2 + log2f(l2)) * FA_LN2 : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

hcl_status_t launch_flash_ws(const FaParams& p, cudaStream_t st) {
  auto kern = hca_flash_ws_kernel;
  const int smem = (int)WsOff::TOTAL + 1024;
  hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, false);
  if (e != HCL_OK) return e;
  const long long n_pairs = (p.n_groups + 1) / 2;
  return check_cuda(launch_pdl(kern, dim3((unsigned)((long long)p.B * n_pairs)),
                               dim3(WS_THREADS), (size_t)smem, st, 1, p),
                    "hca flash attention (warp-specialised) launch");
}

}  // namespace

bool hca_flash_usable(const AttnArgs& a) {
  if (a.H > FA_ROWS || a.d != FA_D) return false;
  if (!(a.scale > 0.f)) return false;   // the row maximum is taken before scaling
  if (!(a.comp.fmt == HCL_BF16 || a.comp.fmt == HCL_FP8SPLIT)) return false;
  const int G = std::max(1, FA_ROWS / a.H);
  const int n_groups = (a.Tq + G - 1) / G;
  if (a.mode == 1) return n_groups >= 32;
  // CSA: the block's MMAs do G times the useful work; worth it while G <= 4
  return a.H >= 32 && n_groups >= 32 && a.k >= 1 && a.idx != nullptr;
}

hcl_status_t launch_hca_flash(const AttnArgs& a, cudaStream_t st) {
  FaParams p;
  p.mode = a.mode;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.B = a.B; p.Tq = a.Tq; p.H = a.H;
  p.G = std::min(std::max(1, FA_ROWS / a.H), a.Tq);
  p.n_groups = (a.Tq + p.G - 1) / p.G;
  p.idx = a.idx;
  p.k = a.mode == 0 ? a.k : 0;
  p.comp = a.comp; p.raw = a.raw;
  p.Nh = a.n_comp; p.mh = a.mode == 1 ? a.mh : 1; p.W = a.W;
  p.q_pos = a.q_pos;
  p.scale_log2 = a.scale * FA_LOG2E;
  p.sink = a.sink;
  p.q_gamma = a.q_gamma;
  p.q_eps = a.q_eps;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.status = a.status;
  p.limit = wait_limit_cycles();
  // HCA over bf16 rows: two query tiles per block, warp-specialised
  if (a.mode == 1 && a.comp.fmt == HCL_BF16 && a.raw.fmt == HCL_BF16) return launch_flash_ws(p, st);
  return a.comp.fmt == HCL_FP8SPLIT ? launch_flash_t<HCL_FP8SPLIT>(p, st) : launch_flash_t<HCL_BF16>(p, st);
}

}  // namespace hcl
