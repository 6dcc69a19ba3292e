// select_attn.cu -- the CSA decode step's selection and attention in one kernel.
//
// [Tripbot §3.1] After the lightning indexer scores every compressed entry, the query keeps the
// k best (ties to the lower entry index) and attends over them plus the raw sliding window
// under one softmax [Tripbot §3.3].  Here the indexer has also written, for every group of 16
// entries, the largest and second largest score (order-preserving 16-bit keys of the bf16
// scores) and the position of the largest.
//
// Design (B200): one thread-block cluster of S CTAs per sequence (S <= 16, a function of the
// entry count only, so a sequence's result does not depend on the batch); CTA c owns a
// contiguous range of G groups and a share of the window rows.
//   1. Before the indexer finishes (programmatic dependent launch), every CTA loads the
//      query heads (optionally RMS-normalised) and starts gathering its window rows.
//   2. L = the k-th largest group maximum, exactly, by a two-digit (8 + 8 bit) radix search:
//      every CTA pushes its per-digit counts into every CTA's shared memory (remote stores),
//      one cluster barrier per digit, and adds the copies locally.  L is a lower bound of the
//      k-th largest score (the maxima are scores of distinct entries).
//   3. Each CTA lists its candidates, the entries with key >= L (a group whose second largest
//      is below L gives its single candidate from the summary; the others' scores are read),
//      in index order, and pushes their keys (about k / S) to every CTA.  After one cluster
//      barrier every CTA holds all candidate keys and finds locally the exact k-th largest key
//      T, the ties to take and -- from the keys of the CTAs before it -- the output positions
//      of its own selected entries.  (Only remote stores cross CTAs: a remote load costs a
//      full round trip, a store is paid for at the barrier.)
//   4. Each CTA writes its part of the selected indices (ascending overall) and attends over
//      its own rows: S = Q K^T and O = P V on tcgen05 (heads = M = 128 TMEM lanes, rows in
//      chunks of 64, two chunks per round, online softmax across rounds in registers).
//   5. The S partial results merge by log-sum-exp: each CTA pushes its normalised partial rows
//      to the CTA owning each head (DSMEM), one cluster barrier, owners write the output.
// Candidate lists that do not fit (heavy ties) switch the whole cluster to an exact path that
// radix-selects over every visible score of the row.  Every wait is a hardware cluster barrier
// or a bounded mbarrier wait.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace cg = cooperative_groups;

namespace hcl {
namespace {

constexpr int SA_THREADS = 256;
constexpr int SA_WARPS = SA_THREADS / 32;
constexpr int SA_ROWS = 128;      // heads per CTA = UMMA M = TMEM lanes
constexpr int SA_D = 128;
constexpr int SA_CH = 64;         // KV rows per chunk (UMMA N of S = Q K^T)
constexpr int SA_RCH = 2;         // chunks per round
constexpr int SA_USE_S = 8;       // CTAs per sequence, at most (portable cluster size)
constexpr int SA_MAXS = SA_USE_S;
constexpr int SA_ALL_CAP = 4096;  // candidates of the whole cluster
constexpr int SA_CAPS = SA_ALL_CAP / SA_USE_S;   // candidates a CTA may list and push
constexpr int SA_CAND_CAP = SA_CAPS;
constexpr int SA_MAX_ROWS = 4096 + 256;  // a CTA's row list: selected entries + window share
constexpr float SA_LOG2E = 1.4426950408889634f;
constexpr float SA_LN2 = 0.6931471805599453f;
constexpr uint32_t RAW_FLAG = 0x80000000u;
constexpr uint32_t NO_ROW = 0xFFFFFFFFu;

struct SaParams {
  const uint16_t* scores;     // bf16 bits [B, Nc]
  const uint16_t* gmax;       // [B, NGP] order-preserving keys (0: no visible entry)
  const uint16_t* g2nd;
  const uint8_t* garg;
  int Nc, NGP, G, gpt;        // groups per CTA (G = 256 * gpt)
  const int32_t* q_pos;
  int m, k;
  int32_t* idx;               // [B, k]
  const __nv_bfloat16* q;     // [B, H, 128]
  int H;
  hcl_kv_t comp, raw;
  int W;
  float scale_log2;
  const float* sink;
  const float* q_gamma;
  float q_eps;
  __nv_bfloat16* out;
  float* lse;
  int32_t* status;
  long long limit;
};

struct SaOff {
  static constexpr uint32_t Q = 0;                        // 2 halves x 128 rows x 128 B
  static constexpr uint32_t KV = 32768;                   // SA_RCH x 16 KB (SW128 halves)
  static constexpr uint32_t P = KV + SA_RCH * 16384;      // SA_RCH x 16 KB
  static constexpr uint32_t STG = P + SA_RCH * 16384;     // E4M3 codes: SA_RCH x 64 x 64 B
  static constexpr uint32_t SCL = STG + SA_RCH * 4096;    // row scales
  static constexpr uint32_t ROWS = SCL + SA_RCH * 256;    // row list
  static constexpr uint32_t CAND = ROWS + SA_MAX_ROWS * 4;     // key << 16 | local entry
  static constexpr uint32_t ALLK = CAND + SA_CAND_CAP * 4;     // pushed keys [S][SA_CAPS] u16
  static constexpr uint32_t HA = ALLK + SA_ALL_CAP * 2;        // 256-bin digit counts (local)
  static constexpr uint32_t HB = HA + 1024;
  static constexpr uint32_t HC = HB + 1024;
  static constexpr uint32_t RA = HC + 1024;                    // pushed counts [S][256] u16
  static constexpr uint32_t RB = RA + SA_USE_S * 512;
  static constexpr uint32_t XCH = RB + SA_USE_S * 512;         // [2][256] floats
  static constexpr uint32_t META = XCH + 2048;                 // 64 u32 of scalars
  static constexpr uint32_t BAR = META + 256;                  // 2 mbarriers + TMEM address
  static constexpr uint32_t VIS = BAR + 32;                    // row visibility bits of a round
  static constexpr uint32_t RECV = VIS + 64;                   // merge: rpo x S x 128 floats
  static constexpr uint32_t RECV_BYTES = (SA_ROWS + SA_USE_S) * SA_D * 4;
  static constexpr uint32_t RLSE = RECV + RECV_BYTES;
  static constexpr uint32_t TOTAL = RLSE + (SA_ROWS + SA_USE_S) * 4;
};

// meta words
enum : int { M_NCAND = 0, M_OVF = 1, M_T = 2, M_ABOVE = 3, M_FOUND = 4, M_L = 5, M_NSEL = 6,
             M_CNTG = 7, M_CNTE = 8, M_TMP = 16,
             M_IN_CAND = 32,   // pushed by CTA r: [32 + 2r] candidates, [33 + 2r] overflow
             M_IN_CNT = 48 };  // pushed by CTA r: [48 + 2r] keys > T, [49 + 2r] keys == T

__device__ __forceinline__ uint32_t okey(uint16_t bits) {
  return uint32_t(bits ^ ((bits & 0x8000u) ? 0xFFFFu : 0x8000u));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t e4m3x2_bf16x2(uint16_t codes, float scale) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
  const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h2));
  return pack_bf16x2(f.x * scale, f.y * scale);
}

// Warp-aggregated increment of bin `bin` (valid lanes only); every lane of the warp calls it.
__device__ __forceinline__ void hist_inc(uint32_t* h, uint32_t bin, bool valid) {
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? bin : 0xFFFFFFFFu);
  if (valid && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
}

// Exclusive block scan (256 threads) of one value per thread; returns the block total.
__device__ __forceinline__ uint32_t scan256(uint32_t v, uint32_t* tmp, uint32_t& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    const uint32_t t = lane < SA_WARPS ? tmp[lane] : 0u;
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < SA_WARPS; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < SA_WARPS) tmp[lane] = s - t;
    if (lane == SA_WARPS - 1) tmp[SA_WARPS] = s;
  }
  __syncthreads();
  const uint32_t res = tmp[w] + x - v;
  total = tmp[SA_WARPS];
  __syncthreads();
  return res;
}

// Digit search over 256 per-digit counts cnt[0..255] (in smem): the largest digit d with
// target <= sum_{d' >= d} cnt[d'].  Warp 0 writes meta[M_T] = d, meta[M_ABOVE] = keys in
// digits above d, meta[M_FOUND] = 1 if found.  Caller synchronises.
__device__ __forceinline__ void find_digit(const uint32_t* cnt, uint32_t target, uint32_t* meta) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  // lane l covers digits 255 - 8l .. 248 - 8l (descending)
  uint32_t c[8], tot = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) { c[i] = cnt[255 - 8 * lane - i]; tot += c[i]; }
  uint32_t inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  const uint32_t before = inc - tot;
  const bool hit = before < target && target <= inc;
  if (hit) {
    uint32_t acc = before;
    int di = 7;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      if (acc + c[i] >= target) { di = i; break; }
      acc += c[i];
    }
    meta[M_T] = uint32_t(255 - 8 * lane - di);
    meta[M_ABOVE] = acc;
  }
  const unsigned any = __ballot_sync(0xffffffffu, hit);
  if (lane == 0) meta[M_FOUND] = any ? 1u : 0u;
}

// Every CTA of the cluster receives this CTA's count v (< 2^16) of digit threadIdx.x in slot
// [c][threadIdx.x] of its `recv` (remote stores, made visible by the next cluster barrier).
__device__ __forceinline__ void push16(cg::cluster_group& cl, uint16_t* recv, uint32_t v, int S,
                                       int c) {
#pragma unroll
  for (int r = 0; r < SA_MAXS; r++)
    if (r < S) cl.map_shared_rank(recv, r)[c * 256 + threadIdx.x] = uint16_t(v);
}

__device__ __forceinline__ uint32_t sum16(const uint16_t* recv, int S) {
  uint32_t s = 0;
#pragma unroll
  for (int r = 0; r < SA_MAXS; r++)
    if (r < S) s += recv[r * 256 + threadIdx.x];
  return s;
}

// Cluster-wide selection of the target-th largest 16-bit key among the keys the CTAs
// enumerate (for_each(f) calls f(key, valid) a uniform number of times per thread).  Two
// digits of 8 bits; each CTA counts its own keys (hA / hB) and pushes the counts to every CTA
// (rA / rB, [S][256] u16: per-CTA counts stay below 2^16), one cluster barrier per digit, then
// every CTA adds the S copies locally.  Returns found (false: fewer than target keys), T and
// the number of keys > T.  Two cluster barriers; a later call may push into rA / rB only after
// a barrier that follows this call's last local read of them.
template <class ForEach>
__device__ bool cluster_select16(cg::cluster_group& cl, ForEach for_each, uint32_t target,
                                 uint32_t* hA, uint32_t* hB, uint16_t* rA, uint16_t* rB,
                                 uint32_t* meta, uint32_t* tot, uint32_t& T, uint32_t& above) {
  const int tid = threadIdx.x;
  const int S = (int)cl.num_blocks(), c = (int)cl.block_rank();
  hA[tid] = 0u;
  hB[tid] = 0u;
  __syncthreads();
  for_each([&](uint32_t key, bool valid) { hist_inc(hA, key >> 8, valid); });
  __syncthreads();
  push16(cl, rA, hA[tid], S, c);
  cl.sync();
  tot[tid] = sum16(rA, S);
  __syncthreads();
  find_digit(tot, target, meta);
  __syncthreads();
  if (!meta[M_FOUND]) {
    cl.sync();   // keep the barrier count uniform
    return false;
  }
  const uint32_t hi = meta[M_T], ab_hi = meta[M_ABOVE];
  __syncthreads();
  for_each([&](uint32_t key, bool valid) { hist_inc(hB, key & 255u, valid && (key >> 8) == hi); });
  __syncthreads();
  push16(cl, rB, hB[tid], S, c);
  cl.sync();
  tot[tid] = sum16(rB, S);
  __syncthreads();
  find_digit(tot, target - ab_hi, meta);
  __syncthreads();
  T = (hi << 8) | meta[M_T];
  above = ab_hi + meta[M_ABOVE];
  __syncthreads();
  return true;
}

// The order-preserving keys of group g's 16 entries (0 for entries >= nvis).
__device__ __forceinline__ void group_keys(const uint16_t* sr, int g, int nvis, uint32_t (&kk)[16]) {
  const int e0 = 16 * g;
  if (e0 + 16 <= nvis && (reinterpret_cast<uintptr_t>(sr + e0) & 15) == 0) {
    const uint4 a = *reinterpret_cast<const uint4*>(sr + e0);
    const uint4 b = *reinterpret_cast<const uint4*>(sr + e0 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; i++) {
      kk[2 * i] = okey(uint16_t(w[i] & 0xFFFFu));
      kk[2 * i + 1] = okey(uint16_t(w[i] >> 16));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) kk[i] = e0 + i < nvis ? okey(sr[e0 + i]) : 0u;
  }
}

__global__ void __launch_bounds__(SA_THREADS, 1) select_attn_kernel(SaParams p) {
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(1024) uint8_t sa_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sa_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = (int)cl.num_blocks();
  const int c = (int)cl.block_rank();
  const int b = blockIdx.x / S;
  uint32_t* rows = reinterpret_cast<uint32_t*>(sm + SaOff::ROWS);
  uint32_t* cand = reinterpret_cast<uint32_t*>(sm + SaOff::CAND);
  uint16_t* allk = reinterpret_cast<uint16_t*>(sm + SaOff::ALLK);
  uint32_t* hA = reinterpret_cast<uint32_t*>(sm + SaOff::HA);
  uint32_t* hB = reinterpret_cast<uint32_t*>(sm + SaOff::HB);
  uint32_t* hC = reinterpret_cast<uint32_t*>(sm + SaOff::HC);
  uint16_t* rA = reinterpret_cast<uint16_t*>(sm + SaOff::RA);
  uint16_t* rB = reinterpret_cast<uint16_t*>(sm + SaOff::RB);
  float* xch = reinterpret_cast<float*>(sm + SaOff::XCH);
  uint32_t* meta = reinterpret_cast<uint32_t*>(sm + SaOff::META);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + SaOff::BAR);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + SaOff::BAR + 16);
  uint32_t* visw = reinterpret_cast<uint32_t*>(sm + SaOff::VIS);
  float* recv = reinterpret_cast<float*>(sm + SaOff::RECV);
  float* recv_lse = reinterpret_cast<float*>(sm + SaOff::RLSE);
  uint32_t* tmp = meta + M_TMP;

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(sTmem, 256);
    tmem_relinquish();
  }

  // ---- 1. before the indexer finishes: query heads and this CTA's window rows ----------
  const int row = tid & (SA_ROWS - 1), hc = tid / SA_ROWS;
  const int pos = p.q_pos[b];              // not written by the indexer
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.H + row) * SA_D) + hc * 8;
    uint4 qv[8];
#pragma unroll
    for (int i = 0; i < 8; i++) qv[i] = row < p.H ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    if (p.q_gamma != nullptr) {
      // RMSNorm of the head's query row [Tripbot §5] (two threads per row, fp32, back to bf16)
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
      const float rn = 1.f / sqrtf((xch[row] + xch[row + SA_ROWS]) / float(SA_D) + p.q_eps);
#pragma unroll
      for (int i = 0; i < 8; i++) {
        uint32_t w4[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int dim = hc * 64 + i * 8 + 2 * j;
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          w4[j] = pack_bf16x2(lo * rn * __ldg(p.q_gamma + dim), hi * rn * __ldg(p.q_gamma + dim + 1));
        }
        qv[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; i++)
      *reinterpret_cast<uint4*>(sm + SaOff::Q + hc * 16384 + row * 128 + ((i ^ (row & 7)) << 4)) = qv[i];
  }
  // window rows: tokens pos-W+1 .. pos; CTA c takes rows [c*nwc, (c+1)*nwc) of them
  const int nwc = (p.W + S - 1) / S;
  const int w_lo = min(p.W, c * nwc), nw = min(p.W, w_lo + nwc) - w_lo;
  for (int j = tid; j < nw; j += SA_THREADS) {
    const long long u = (long long)pos - p.W + 1 + w_lo + j;
    rows[j] = u >= 0 ? RAW_FLAG | uint32_t(u) : NO_ROW;
  }
  __syncthreads();

  // gather rows [r0, r0 + nr) of the list into chunk slots (rows r0.. -> KV row 0..)
  auto issue_gather = [&](int r0, int nr) {
    constexpr int PIECES_BF = 16, PIECES_8 = 13;
    const bool fp8 = p.comp.fmt == HCL_FP8SPLIT;
    const int pieces = fp8 ? PIECES_8 : PIECES_BF;
    for (int u = tid; u < nr * pieces; u += SA_THREADS) {
      const int jj = u / pieces, pc = u % pieces;
      const int ch = jj / SA_CH, r = jj % SA_CH;
      const uint32_t code = rows[r0 + jj];
      long long slot = -1;
      const hcl_kv_t* st = &p.comp;
      if (code != NO_ROW) {
        if (code & RAW_FLAG) {
          st = &p.raw;
          slot = (long long)b * p.raw.cap + (long long)(code & ~RAW_FLAG) % p.raw.cap;
        } else {
          slot = (long long)b * p.comp.cap + (long long)code % p.comp.cap;
        }
      }
      uint8_t* kv = sm + SaOff::KV + ch * 16384;
      if (!fp8) {
        uint8_t* dst = kv + (pc >> 3) * 8192 + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->data) + slot * 256 + pc * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      } else if (pc < 8) {
        uint8_t* dst = kv + 8192 + r * 128 + ((pc ^ (r & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->rope) + slot * 128 + pc * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      } else if (pc < 12) {
        uint8_t* dst = sm + SaOff::STG + (ch * SA_CH + r) * 64 + (pc - 8) * 16;
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->data) + slot * 64 + (pc - 8) * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      } else {
        float* dst = reinterpret_cast<float*>(sm + SaOff::SCL) + ch * SA_CH + r;
        if (slot >= 0)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                       "l"(st->scale + slot)
                       : "memory");
        else *dst = 0.f;
      }
    }
    cp_async_commit();
  };
  const int pre = min(nw, SA_RCH * SA_CH);   // window rows of the first round, gathered now
  if (pre > 0) issue_gather(0, pre);

  // ---- the indexer's scores and summaries are needed from here on ---------------------
  pdl_enter();
  const int nvis = pos < 0 ? 0 : min(p.Nc, (pos + 1) / p.m);
  const int k = p.k;
  const int ent_lo = 16 * c * p.G;                       // this CTA's first entry
  const uint16_t* sr = p.scores + (size_t)b * p.Nc;
  int32_t* idx_out = p.idx + (size_t)b * k;
  int nsel = 0;                                          // this CTA's selected entries

  if (nvis <= k) {
    // ---- every visible entry is selected; entries in this CTA's range, in order --------
    const int e0 = min(nvis, ent_lo), e1 = min(nvis, ent_lo + 16 * p.G);
    nsel = e1 - e0;
    for (int j = tid; j < nsel; j += SA_THREADS) {
      rows[nw + j] = uint32_t(e0 + j);
      idx_out[e0 + j] = e0 + j;
    }
    if (c == S - 1)
      for (int j = nvis + tid; j < k; j += SA_THREADS) idx_out[j] = -1;
  } else {
    const int ngv = (nvis + 15) / 16;                    // groups with a visible entry
    const int g0 = c * p.G + tid * p.gpt;                // this thread's first group
    // ---- 2. summaries and L ---------------------------------------------------------------
    uint32_t mx[16], m2[16], am[16];
    const size_t gb = (size_t)b * p.NGP;
#pragma unroll
    for (int i = 0; i < 16; i++) {
      mx[i] = 0u; m2[i] = 0u; am[i] = 0u;
      if (i < p.gpt && g0 + i < ngv) {
        mx[i] = p.gmax[gb + g0 + i];
        m2[i] = p.g2nd[gb + g0 + i];
        am[i] = p.garg[gb + g0 + i] & 15u;
      }
    }
    uint32_t L = 1u, ab = 0u;
    const bool haveL = cluster_select16(
        cl, [&](auto f) {
#pragma unroll
          for (int i = 0; i < 16; i++)
            if (i < p.gpt) f(mx[i], mx[i] != 0u);
        },
        (uint32_t)k, hA, hB, rA, rB, meta, hC, L, ab);
    if (!haveL || L == 0u) L = 1u;   // fewer than k groups: every visible entry is a candidate

    // ---- 3. candidates (key >= L) in index order -------------------------------------
    uint32_t nmine = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) {
      if (i >= p.gpt || mx[i] < L) continue;
      if (m2[i] < L) { nmine += 1; continue; }
      uint32_t kk[16];
      group_keys(sr, g0 + i, nvis, kk);
#pragma unroll
      for (int j = 0; j < 16; j++) nmine += kk[j] >= L;
    }
    uint32_t ncta;
    uint32_t off = scan256(nmine, tmp, ncta);
    const bool ovf_local = ncta > (uint32_t)SA_CAPS;
    if (!ovf_local) {
#pragma unroll
      for (int i = 0; i < 16; i++) {
        if (i >= p.gpt || mx[i] < L) continue;
        const uint32_t lg = uint32_t(g0 + i - c * p.G) * 16u;   // local entry of the group
        if (m2[i] < L) { cand[off++] = (mx[i] << 16) | (lg + am[i]); continue; }
        uint32_t kk[16];
        group_keys(sr, g0 + i, nvis, kk);
#pragma unroll
        for (int j = 0; j < 16; j++)
          if (kk[j] >= L) cand[off++] = (kk[j] << 16) | (lg + j);
      }
    }
    __syncthreads();
    // push this CTA's candidate count, overflow flag and keys to every CTA of the cluster
    if (tid < S) {
      uint32_t* dst = cl.map_shared_rank(meta, tid) + M_IN_CAND + 2 * c;
      dst[0] = ncta;
      dst[1] = ovf_local ? 1u : 0u;
    }
    if (!ovf_local) {
      for (uint32_t j = tid; j < ncta; j += SA_THREADS) {
        const uint16_t key = uint16_t(cand[j] >> 16);
#pragma unroll
        for (int r = 0; r < SA_MAXS; r++)
          if (r < S) cl.map_shared_rank(allk, r)[c * SA_CAPS + j] = key;
      }
    }
    cl.sync();
    uint32_t tot_c = 0, before_c = 0;
    bool ovf = false;
    for (int r = 0; r < S; r++) {
      const uint32_t n = meta[M_IN_CAND + 2 * r];
      ovf |= meta[M_IN_CAND + 2 * r + 1] != 0u;
      if (r < c) before_c += n;
      tot_c += n;
    }
    uint32_t T = 0u, above = 0u, gt_before = 0u, eq_before = 0u;
    const bool exact_path = !ovf;
    if (exact_path) {
      // ---- the exact k-th largest of the candidate keys (local two-digit search over the
      // pushed segments: CTA r's keys in allk[r * SA_CAPS, + n_r)) -----------------------
      constexpr int PER = SA_ALL_CAP / SA_THREADS;
      auto slot_key = [&](int it, uint32_t& key) {
        const int q2 = it * SA_THREADS + tid;
        const int r = q2 / SA_CAPS, j = q2 % SA_CAPS;
        const bool v = r < S && (uint32_t)j < meta[M_IN_CAND + 2 * min(r, S - 1)];
        key = v ? allk[q2] : 0u;
        return v;
      };
      hA[tid] = 0u;
      __syncthreads();
#pragma unroll 4
      for (int it = 0; it < PER; it++) {
        uint32_t key;
        const bool v = slot_key(it, key);
        hist_inc(hA, key >> 8, v);
      }
      __syncthreads();
      find_digit(hA, (uint32_t)k, meta);
      __syncthreads();
      const uint32_t hi = meta[M_T], ab_hi = meta[M_ABOVE];
      __syncthreads();
      hA[tid] = 0u;
      __syncthreads();
#pragma unroll 4
      for (int it = 0; it < PER; it++) {
        uint32_t key;
        const bool v = slot_key(it, key);
        hist_inc(hA, key & 255u, v && (key >> 8) == hi);
      }
      __syncthreads();
      find_digit(hA, (uint32_t)k - ab_hi, meta);
      __syncthreads();
      T = (hi << 8) | meta[M_T];
      above = ab_hi + meta[M_ABOVE];
      // keys > T and == T among the candidates of the CTAs before this one
      uint32_t g = 0, e = 0;
#pragma unroll 4
      for (int it = 0; it < PER; it++) {
        uint32_t key;
        const int q2 = it * SA_THREADS + tid;
        if (slot_key(it, key) && q2 / SA_CAPS < c) { g += key > T; e += key == T; }
      }
      uint32_t tg, te;
      scan256(g, tmp, tg);
      scan256(e, tmp, te);
      gt_before = tg;
      eq_before = te;
    } else {
      // ---- heavy ties or too many candidates: exact selection over every visible score --
      const bool ok = cluster_select16(
          cl, [&](auto f) {
            for (int i = 0; i < p.gpt; i++) {
              uint32_t kk[16];
              const bool any = g0 + i < ngv;
              if (any) group_keys(sr, g0 + i, nvis, kk);
#pragma unroll
              for (int j = 0; j < 16; j++) f(any ? kk[j] : 0u, any && kk[j] != 0u);
            }
          },
          (uint32_t)k, hA, hB, rA, rB, meta, hC, T, above);
      if (!ok) report(p.status, HCL_ERR_DEVICE_FAULT);   // cannot happen: nvis > k
      // this CTA's counts of > T and == T, pushed to every CTA, then those of the CTAs before
      uint32_t g = 0, e = 0;
      for (int i = 0; i < p.gpt; i++) {
        if (g0 + i >= ngv) break;
        uint32_t kk[16];
        group_keys(sr, g0 + i, nvis, kk);
#pragma unroll
        for (int j = 0; j < 16; j++) { g += kk[j] != 0u && kk[j] > T; e += kk[j] != 0u && kk[j] == T; }
      }
      uint32_t tg, te;
      scan256(g, tmp, tg);
      scan256(e, tmp, te);
      if (tid < S) {
        uint32_t* dst = cl.map_shared_rank(meta, tid) + M_IN_CNT + 2 * c;
        dst[0] = tg;
        dst[1] = te;
      }
      cl.sync();
      uint32_t gb2 = 0, eb2 = 0;
      for (int r = 0; r < c; r++) {
        gb2 += meta[M_IN_CNT + 2 * r];
        eb2 += meta[M_IN_CNT + 2 * r + 1];
      }
      gt_before = gb2;
      eq_before = eb2;
    }
    const uint32_t krem = (uint32_t)k - above;
    const uint32_t base_slot = gt_before + min(eq_before, krem);
    // ---- 4. emission: this CTA's selected entries, in index order ------------------------
    if (exact_path) {
      // own candidates: cand[0 .. ncta), thread t takes a contiguous segment
      const uint32_t per = (ncta + SA_THREADS - 1) / SA_THREADS;
      const uint32_t s0 = min(ncta, tid * per), s1 = min(ncta, s0 + per);
      uint32_t g = 0, e = 0;
      for (uint32_t j = s0; j < s1; j++) {
        const uint32_t key = cand[j] >> 16;
        g += key > T;
        e += key == T;
      }
      uint32_t gtot, etot;
      const uint32_t G0 = scan256(g, tmp, gtot);
      const uint32_t E0 = scan256(e, tmp, etot);
      const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, etot) : 0u;
      uint32_t gl = G0, el = E0;
      for (uint32_t j = s0; j < s1; j++) {
        const uint32_t key = cand[j] >> 16;
        const bool isg = key > T, ise = key == T;
        if (isg || (ise && el < eq_take)) {
          const uint32_t rank = gl + min(el, eq_take);     // among this CTA's selected
          const int ent = ent_lo + int(cand[j] & 0xFFFFu);
          if (base_slot + rank < (uint32_t)k) idx_out[base_slot + rank] = ent;
          else report(p.status, HCL_ERR_DEVICE_FAULT);
          rows[nw + rank] = uint32_t(ent);
        }
        gl += isg;
        el += ise;
      }
      nsel = int(gtot + eq_take);
    } else {
      uint32_t g = 0, e = 0;
      for (int i = 0; i < p.gpt; i++) {
        if (g0 + i >= ngv) break;
        uint32_t kk[16];
        group_keys(sr, g0 + i, nvis, kk);
#pragma unroll
        for (int j = 0; j < 16; j++) { g += kk[j] != 0u && kk[j] > T; e += kk[j] != 0u && kk[j] == T; }
      }
      uint32_t gtot, etot;
      const uint32_t G0 = scan256(g, tmp, gtot);
      const uint32_t E0 = scan256(e, tmp, etot);
      const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, etot) : 0u;
      uint32_t gl = G0, el = E0;
      for (int i = 0; i < p.gpt; i++) {
        if (g0 + i >= ngv) break;
        uint32_t kk[16];
        group_keys(sr, g0 + i, nvis, kk);
        for (int j = 0; j < 16; j++) {
          const bool isg = kk[j] != 0u && kk[j] > T, ise = kk[j] != 0u && kk[j] == T;
          if (isg || (ise && el < eq_take)) {
            const uint32_t rank = gl + min(el, eq_take);
            const int ent = 16 * (g0 + i) + j;
            if (base_slot + rank < (uint32_t)k) idx_out[base_slot + rank] = ent;
            else report(p.status, HCL_ERR_DEVICE_FAULT);
            if (nw + rank < (uint32_t)SA_MAX_ROWS) rows[nw + rank] = uint32_t(ent);
            else report(p.status, HCL_ERR_DEVICE_FAULT);
          }
          gl += isg;
          el += ise;
        }
      }
      nsel = int(gtot + eq_take);
    }
  }
  __syncthreads();

  // ---- 5. attention over rows [0, nrows): window share, then the selected entries ------
  const int nrows = min(nw + nsel, SA_MAX_ROWS);
  const int nrounds = (nrows + SA_RCH * SA_CH - 1) / (SA_RCH * SA_CH);
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const uint32_t ocol = SA_RCH * SA_CH;                  // O after the S columns
  const uint32_t trow = tbase + (uint32_t((warp & 3) * 32) << 16);
  float o_acc[64];
#pragma unroll
  for (int i = 0; i < 64; i++) o_acc[i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;                   // log2 domain; l: this thread's half
  bool ok = true;
  for (int rd = 0; rd < nrounds; rd++) {
    const int r0 = rd * SA_RCH * SA_CH;
    const int nr = min(SA_RCH * SA_CH, nrows - r0);
    const int nch = (nr + SA_CH - 1) / SA_CH;
    if (rd == 0) {
      if (nr > pre) {
        // selected rows of the first round (after the prefetched window rows): shift into
        // place by gathering rows pre.. nr-1 at KV rows pre..
        // (issue_gather places list row r0 + jj at KV row jj; gather the tail separately)
        const int t0 = pre;
        constexpr int dummy = 0;
        (void)dummy;
        // rows[t0 .. nr) -> KV rows t0 ..: temporarily offset the list base
        const bool fp8 = p.comp.fmt == HCL_FP8SPLIT;
        const int pieces = fp8 ? 13 : 16;
        for (int u = tid; u < (nr - t0) * pieces; u += SA_THREADS) {
          const int jj = t0 + u / pieces, pc = u % pieces;
          const int ch = jj / SA_CH, r = jj % SA_CH;
          const uint32_t code = rows[jj];
          long long slot = -1;
          const hcl_kv_t* st = &p.comp;
          if (code != NO_ROW) {
            if (code & RAW_FLAG) {
              st = &p.raw;
              slot = (long long)b * p.raw.cap + (long long)(code & ~RAW_FLAG) % p.raw.cap;
            } else {
              if ((long long)code >= p.Nc) { report(p.status, HCL_ERR_DEVICE_FAULT); }
              else slot = (long long)b * p.comp.cap + (long long)code % p.comp.cap;
            }
          }
          uint8_t* kv = sm + SaOff::KV + ch * 16384;
          if (!fp8) {
            uint8_t* dst = kv + (pc >> 3) * 8192 + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
            if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->data) + slot * 256 + pc * 16);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
          } else if (pc < 8) {
            uint8_t* dst = kv + 8192 + r * 128 + ((pc ^ (r & 7)) << 4);
            if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->rope) + slot * 128 + pc * 16);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
          } else if (pc < 12) {
            uint8_t* dst = sm + SaOff::STG + (ch * SA_CH + r) * 64 + (pc - 8) * 16;
            if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st->data) + slot * 64 + (pc - 8) * 16);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
          } else {
            float* dst = reinterpret_cast<float*>(sm + SaOff::SCL) + ch * SA_CH + r;
            if (slot >= 0)
              asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                           "l"(st->scale + slot)
                           : "memory");
            else *dst = 0.f;
          }
        }
        cp_async_commit();
      }
      // rows of the round's last chunk past nr read as zeros (masked below)
    } else {
      issue_gather(r0, nr);
    }
    // zero the unused tail of the last chunk (its rows are masked, but must be finite)
    for (int u = tid; u < (nch * SA_CH - nr) * 16; u += SA_THREADS) {
      const int jj = nr + u / 16, pc = u % 16;
      const int ch = jj / SA_CH, r = jj % SA_CH;
      *reinterpret_cast<uint4*>(sm + SaOff::KV + ch * 16384 + (pc >> 3) * 8192 + r * 128 +
                                (((pc & 7) ^ (r & 7)) << 4)) = make_uint4(0, 0, 0, 0);
    }
    // visibility bits: row jj of the round is valid when listed and not NO_ROW
    for (int w0 = 0; w0 < nch * SA_CH; w0 += SA_THREADS) {
      const int jj = w0 + tid;
      const bool v = jj < nr && rows[r0 + jj] != NO_ROW;
      const uint32_t bits = __ballot_sync(0xffffffffu, v);
      if (lane == 0 && jj < nch * SA_CH) visw[jj >> 5] = bits;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (p.comp.fmt == HCL_FP8SPLIT) {
      for (int u = tid; u < nr * 8; u += SA_THREADS) {
        const int jj = u >> 3, cc = u & 7, ch = jj / SA_CH, r = jj % SA_CH;
        const uint2 codes = *reinterpret_cast<const uint2*>(sm + SaOff::STG + (ch * SA_CH + r) * 64 + cc * 8);
        const float sc = reinterpret_cast<const float*>(sm + SaOff::SCL)[ch * SA_CH + r];
        uint4 v;
        v.x = e4m3x2_bf16x2(uint16_t(codes.x & 0xffff), sc);
        v.y = e4m3x2_bf16x2(uint16_t(codes.x >> 16), sc);
        v.z = e4m3x2_bf16x2(uint16_t(codes.y & 0xffff), sc);
        v.w = e4m3x2_bf16x2(uint16_t(codes.y >> 16), sc);
        *reinterpret_cast<uint4*>(sm + SaOff::KV + ch * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    // S_c = Q K_c^T (M = 128 heads, N = 64 rows, K = 128 dims in 8 steps of 16)
    if (tid == 0) {
      const uint32_t aq = smem_u32(sm + SaOff::Q);
      for (int ch = 0; ch < nch; ch++) {
        const uint32_t ak = smem_u32(sm + SaOff::KV + ch * 16384);
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
          const uint32_t h = ks >> 2, kk = ks & 3;
          umma_bf16(tbase + ch * SA_CH, make_sdesc(aq + h * 16384 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                    make_sdesc(ak + h * 8192 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                    idesc_bf16(128, SA_CH), ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(bar_s);
    }
    __syncwarp();   // warp 0 reconverges before waiting (the issuing lane is not left behind)
    ok = ok && mbar_wait(bar_s, rd & 1, p.limit, nullptr);
    tc_fence_after();
    // softmax of the round: this thread holds columns 32*hc .. 32*hc+31 of every chunk
    uint32_t sv[SA_RCH][32];
#pragma unroll
    for (int ch = 0; ch < SA_RCH; ch++)
      if (ch < nch) {
        tmem_ld16(trow + ch * SA_CH + hc * 32, *reinterpret_cast<uint32_t(*)[16]>(&sv[ch][0]));
        tmem_ld16(trow + ch * SA_CH + hc * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[ch][16]));
      }
    tmem_ld_wait();
    float lmax = -INFINITY;
#pragma unroll
    for (int ch = 0; ch < SA_RCH; ch++)
      if (ch < nch) {
        const uint32_t vb = visw[2 * ch + hc];
#pragma unroll
        for (int j = 0; j < 32; j++)
          if ((vb >> j) & 1u) lmax = fmaxf(lmax, __uint_as_float(sv[ch][j]) * p.scale_log2);
      }
    xch[tid] = lmax;
    __syncthreads();
    const float m_new = fmaxf(m_run, fmaxf(xch[row], xch[row + SA_ROWS]));
    const float muse = m_new == -INFINITY ? 0.f : m_new;
    float lsum = 0.f;
#pragma unroll
    for (int ch = 0; ch < SA_RCH; ch++)
      if (ch < nch) {
        const uint32_t vb = visw[2 * ch + hc];
        uint8_t* prow = sm + SaOff::P + ch * 16384 + row * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; q4++) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const int j = q4 * 8 + i;
            const float p0 = ((vb >> j) & 1u) ? exp2f(__uint_as_float(sv[ch][j]) * p.scale_log2 - muse) : 0.f;
            const float p1 = ((vb >> (j + 1)) & 1u) ? exp2f(__uint_as_float(sv[ch][j + 1]) * p.scale_log2 - muse) : 0.f;
            lsum += p0 + p1;
            pk[i >> 1] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + (((hc * 4 + q4) ^ (row & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // O_round = sum_c P_c V_c (V is the MN-major operand of the same tile)
    if (tid == 0) {
      for (int ch = 0; ch < nch; ch++) {
        const uint32_t ap = smem_u32(sm + SaOff::P + ch * 16384);
        const uint32_t av = smem_u32(sm + SaOff::KV + ch * 16384);
#pragma unroll
        for (int ks = 0; ks < 4; ks++)
          umma_bf16(tbase + ocol, make_sdesc(ap + ks * 32, 16, 1024, SMEM_SWIZZLE_128B),
                    make_sdesc(av + ks * 2048, 8192, 1024, SMEM_SWIZZLE_128B),
                    idesc_bf16(128, SA_D) | (1u << 16), (ch > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(bar_o);
    }
    __syncwarp();
    ok = ok && mbar_wait(bar_o, rd & 1, p.limit, nullptr);
    tc_fence_after();
    {
      uint32_t r64[64];
#pragma unroll
      for (int q4 = 0; q4 < 4; q4++)
        tmem_ld16(trow + ocol + hc * 64 + q4 * 16, *reinterpret_cast<uint32_t(*)[16]>(&r64[q4 * 16]));
      tmem_ld_wait();
      const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
#pragma unroll
      for (int i = 0; i < 64; i++) o_acc[i] = o_acc[i] * alpha + __uint_as_float(r64[i]);
      l_run = l_run * alpha + lsum;
      m_run = m_new;
    }
    tc_fence_before();
    __syncthreads();   // the round's TMEM and shared tiles may be reused
  }
  if (!ok) report(p.status, HCL_ERR_TIMEOUT);
  xch[SA_THREADS + tid] = l_run;
  __syncthreads();
  const float l_tot = xch[SA_THREADS + row] + xch[SA_THREADS + row + SA_ROWS];
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }

  // ---- 6. merge of the S partials (head h -> CTA h % S, slot h / S) -------------------
  const bool hv = row < p.H;
  const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
  const float lse2 = l_tot > 0.f ? m_run + log2f(l_tot) : -INFINITY;
  if (S == 1) {
    float f = inv_l, m2 = m_run, l2 = l_tot;
    if (p.sink) {
      const float s2 = p.sink[min(row, p.H - 1)] * SA_LOG2E;
      const float mm = fmaxf(m2, s2);
      const float fa = l2 > 0.f ? exp2f(m2 - mm) : 0.f;
      const float l3 = l2 * fa + exp2f(s2 - mm);
      f = l3 > 0.f ? fa / l3 : 0.f;
      l2 = l3;
      m2 = mm;
    }
    if (hv) {
      __nv_bfloat16* dst = p.out + ((size_t)b * p.H + row) * SA_D + hc * 64;
#pragma unroll
      for (int i = 0; i < 64; i += 8)
        *reinterpret_cast<uint4*>(dst + i) =
            make_uint4(pack_bf16x2(o_acc[i] * f, o_acc[i + 1] * f), pack_bf16x2(o_acc[i + 2] * f, o_acc[i + 3] * f),
                       pack_bf16x2(o_acc[i + 4] * f, o_acc[i + 5] * f), pack_bf16x2(o_acc[i + 6] * f, o_acc[i + 7] * f));
      if (hc == 0 && p.lse) p.lse[(size_t)b * p.H + row] = l2 > 0.f ? (m2 + log2f(l2)) * SA_LN2 : -INFINITY;
    }
    return;
  }
  if (hv) {
    const int owner = row % S, slot = row / S;
    float* dst = cl.map_shared_rank(recv, owner) + ((size_t)slot * S + c) * SA_D + hc * 64;
#pragma unroll
    for (int i = 0; i < 64; i += 4)
      *reinterpret_cast<float4*>(dst + i) =
          make_float4(o_acc[i] * inv_l, o_acc[i + 1] * inv_l, o_acc[i + 2] * inv_l, o_acc[i + 3] * inv_l);
    if (hc == 0) *(cl.map_shared_rank(recv_lse, owner) + slot * S + c) = lse2;
  }
  cl.sync();
  const int rpo = (SA_ROWS + S - 1) / S;
  for (int slot = warp; slot < rpo; slot += SA_WARPS) {
    const int h = c + S * slot;
    if (h >= p.H) break;
    const float ls = lane < S ? recv_lse[slot * S + lane] : -INFINITY;
    float M = ls;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
    float s2 = -INFINITY;
    if (p.sink) {
      s2 = p.sink[h] * SA_LOG2E;
      M = fmaxf(M, s2);
    }
    const float wl = (ls == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ls - M);
    float den = wl;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o2);
    if (p.sink && M > -INFINITY) den += exp2f(s2 - M);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* part = reinterpret_cast<const float4*>(recv + (size_t)slot * S * SA_D);
#pragma unroll
    for (int s = 0; s < SA_MAXS; s++) {
      const float wgt = __shfl_sync(0xffffffffu, wl, s);
      if (s < S && wgt != 0.f) {
        const float4 v = part[s * (SA_D / 4) + lane];
        acc.x += wgt * v.x; acc.y += wgt * v.y; acc.z += wgt * v.z; acc.w += wgt * v.w;
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const size_t orow = (size_t)b * p.H + h;
    reinterpret_cast<uint2*>(p.out + orow * SA_D)[lane] =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    if (p.lse && lane == 0) p.lse[orow] = den > 0.f ? (M + log2f(den)) * SA_LN2 : -INFINITY;
  }
}

}  // namespace

// Cluster shape of the fused decode selection + attention for Nc entries: S CTAs of 256
// threads, each owning G = 256 * gpt groups of 16 entries (gpt a power of two <= 16), S <= 16.
// A function of Nc only.
bool select_attn_shape(int Nc, int* S_out, int* gpt_out) {
  const int ngp = gmax_row_stride(Nc);
  int gpt = 1;
  while (gpt < 16 && (long long)SA_USE_S * SA_THREADS * gpt < ngp) gpt <<= 1;
  if ((long long)SA_USE_S * SA_THREADS * gpt < ngp) return false;
  const int G = SA_THREADS * gpt;
  const int S = (ngp + G - 1) / G;
  *S_out = S;
  *gpt_out = gpt;
  return true;
}

bool select_attn_supported(int Nc, int H, int k, int W, int comp_fmt) {
  int S, gpt;
  return select_attn_shape(Nc, &S, &gpt) && H >= 1 && H <= SA_ROWS && k >= 1 && k <= 4096 &&
         W >= 0 && (W + S - 1) / S <= 256 && (comp_fmt == HCL_BF16 || comp_fmt == HCL_FP8SPLIT);
}

hcl_status_t launch_select_attn(const SelectAttnArgs& a, cudaStream_t st) {
  int S, gpt;
  if (!select_attn_shape(a.Nc, &S, &gpt)) return fail(HCL_ERR_UNSUPPORTED, "select_attn: Nc too large");
  auto kern = select_attn_kernel;
  const int smem = (int)SaOff::TOTAL + 1024;
  hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, true);
  if (e != HCL_OK) return e;
  SaParams p;
  p.scores = static_cast<const uint16_t*>(a.scores);
  p.gmax = a.gmax;
  p.g2nd = a.g2nd;
  p.garg = a.garg;
  p.Nc = a.Nc;
  p.NGP = gmax_row_stride(a.Nc);
  p.gpt = gpt;
  p.G = SA_THREADS * gpt;
  p.q_pos = a.q_pos;
  p.m = a.m;
  p.k = a.k;
  p.idx = a.idx;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.H = a.H;
  p.comp = a.comp;
  p.raw = a.raw;
  p.W = a.W;
  p.scale_log2 = a.scale * SA_LOG2E;
  p.sink = a.sink;
  p.q_gamma = a.q_gamma;
  p.q_eps = a.q_eps;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.status = a.status;
  p.limit = wait_limit_cycles();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(a.B * S));
  cfg.blockDim = dim3(SA_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, p), "select_attn launch");
}

}  // namespace hcl
