// topk.cu -- per-query-row exact top-k by radix selection.
//
// [Tripbot §3.1] After the lightning indexer scores every compressed entry, only the top-k
// entries (k = 1024 for V4-Pro, 512 for V4-Flash) enter the attention; [CSDN §1.4] scoring
// in BF16 instead of FP32 halves the selection work.  Ties go to the lower entry index and
// the k indices are written in ascending order (padded with -1 when fewer are visible).
//
// Design (B200): one thread-block cluster of C blocks per score row (C = 1..16).  Each block
// copies its contiguous slice of the row into shared memory as order-preserving unsigned
// keys, then the cluster runs a most-significant-digit radix select (16-bit keys: digits of
// 12 + 4 bits; 32-bit keys: 12 + 12 + 8): every block histograms its slice (shared-memory
// atomics), adds its non-zero bins into block 0's histogram through distributed shared
// memory, block 0 finds the digit holding the k-th largest key, and all blocks read it back.
// Cluster barriers are hardware barriers between co-scheduled blocks (no spin loops).  The
// exact threshold key T and the number of T-valued keys to take then give each block, from
// the blocks before it, the output positions of its selected keys; warps emit them in index
// order with ballots.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace cg = cooperative_groups;

namespace hcl {
namespace {

constexpr int TK_THREADS = 1024;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int MAX_BINS = 4096;

__device__ __forceinline__ uint32_t ordered_key_f32(uint32_t bits) {
  return bits ^ ((bits & 0x80000000u) ? 0xFFFFFFFFu : 0x80000000u);
}
__device__ __forceinline__ uint32_t ordered_key_bf16(uint16_t bits) {
  return uint32_t(bits ^ ((bits & 0x8000u) ? 0xFFFFu : 0x8000u));
}

struct TkShared {
  uint32_t hist[MAX_BINS];   // this block's histogram (block 0: also the merged one)
  uint32_t merged[MAX_BINS];
  uint32_t bcast[4];         // block 0 -> all: digit, count above
  uint32_t cnt[4];           // this block's (#greater, #equal); then the blocks-before sums
  uint32_t wsum[2][TK_WARPS];
  uint32_t scan_tmp[TK_WARPS];
};

// Exclusive scan of one value per thread over the block (1024 threads).
__device__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    const uint32_t t = tmp[lane];
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s - t;
  }
  __syncthreads();
  const uint32_t res = tmp[w] + x - v;
  __syncthreads();
  return res;
}

// Final step shared by both selection kernels: with the exact threshold key T and krem, the
// number of T-valued keys to take (lowest indices first), every block counts its keys > T and
// == T, learns from the blocks before it (DSMEM) where its output starts, and its warps write
// the selected indices in ascending order with ballots.  Ends with a cluster barrier so no
// block exits while another may still read its shared memory.
template <class KeyAt>
__device__ void emit_ordered(cg::cluster_group& cluster, uint32_t (*wsum)[TK_WARPS], uint32_t* cnt,
                             KeyAt key_at, int n, int lo, uint32_t T, uint32_t krem, int k,
                             int32_t* out, int32_t* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster.block_rank();
  const int seg = (n + TK_WARPS - 1) / TK_WARPS;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  uint32_t g = 0, e = 0;
  for (int j = s0 + lane; j < s1; j += 32) {
    const uint32_t key = key_at(j);
    g += key > T;
    e += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    g += __shfl_xor_sync(0xffffffffu, g, o);
    e += __shfl_xor_sync(0xffffffffu, e, o);
  }
  if (lane == 0) { wsum[0][warp] = g; wsum[1][warp] = e; }
  __syncthreads();
  if (tid == 0) {
    uint32_t tg = 0, te = 0;
    for (int w = 0; w < TK_WARPS; w++) { tg += wsum[0][w]; te += wsum[1][w]; }
    cnt[0] = tg;
    cnt[1] = te;
  }
  cluster.sync();
  // counts of the blocks before this one: lane r of warp 0 reads block r (one round trip),
  // warp-sums them and shares the result through shared memory
  if (warp == 0) {
    uint32_t cg_ = 0, ce_ = 0;
    if (lane < rank) {
      const uint32_t* c = cluster.map_shared_rank(cnt, lane);
      cg_ = c[0];
      ce_ = c[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cg_ += __shfl_xor_sync(0xffffffffu, cg_, o);
      ce_ += __shfl_xor_sync(0xffffffffu, ce_, o);
    }
    if (lane == 0) { cnt[2] = cg_; cnt[3] = ce_; }
  }
  __syncthreads();
  const uint32_t gt_before = cnt[2], eq_before = cnt[3];
  const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, cnt[1]) : 0u;
  uint32_t wg_before = 0, we_before = 0;
  for (int w = 0; w < warp; w++) { wg_before += wsum[0][w]; we_before += wsum[1][w]; }
  uint32_t pos_out = gt_before + min(eq_before, krem) + wg_before + min(we_before, eq_take);
  uint32_t eq_seen = we_before;
  for (int j0 = s0; j0 < s1; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < s1 ? key_at(j) : 0u;
    const bool is_eq = j < s1 && key == T;
    const bool is_gt = j < s1 && key > T;
    const uint32_t eqmask = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t my_eq_rank = eq_seen + __popc(eqmask & ((1u << lane) - 1));
    const bool sel = is_gt || (is_eq && my_eq_rank < eq_take);
    const uint32_t selmask = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const uint32_t slot = pos_out + __popc(selmask & ((1u << lane) - 1));
      if (slot < (uint32_t)k) out[slot] = lo + j;
      else report(status, HCL_ERR_DEVICE_FAULT);
    }
    pos_out += __popc(selmask);
    eq_seen += __popc(eqmask);
  }
  cluster.sync();
}

template <bool BF16>
__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_kernel(const void* __restrict__ scores, int Tq, int Nc, const int32_t* __restrict__ q_pos,
                int m, int k, int32_t* __restrict__ idx, int chunk_cap,
                int32_t* status) {
  cg::cluster_group cluster = cg::this_cluster();
  pdl_enter();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const long long row = blockIdx.x / C;
  extern __shared__ __align__(16) uint8_t tk_smem[];
  TkShared& S = *reinterpret_cast<TkShared*>(tk_smem);
  uint32_t* keys32 = reinterpret_cast<uint32_t*>(tk_smem + sizeof(TkShared));
  uint16_t* keys16 = reinterpret_cast<uint16_t*>(tk_smem + sizeof(TkShared));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int pos = q_pos[row];
  const int nvis = pos < 0 ? 0 : min(Nc, (pos + 1) / m);
  int32_t* out = idx + row * k;
  if (nvis <= k) {
    // every visible entry is selected; uniform over the cluster, no barrier needed
    for (int j = rank * TK_THREADS + tid; j < k; j += C * TK_THREADS) out[j] = j < nvis ? j : -1;
    return;
  }
  const int chunk = (nvis + C - 1) / C;
  const int lo = min(nvis, rank * chunk);
  const int n = min(nvis, lo + chunk) - lo;
  const bool resident = n <= chunk_cap;

  auto key_at = [&](int j) -> uint32_t {
    if (resident) return BF16 ? uint32_t(keys16[j]) : keys32[j];
    if (BF16) {
      const uint16_t* s = static_cast<const uint16_t*>(scores) + row * (long long)Nc + lo;
      return ordered_key_bf16(s[j]);
    }
    const uint32_t* s = static_cast<const uint32_t*>(scores) + row * (long long)Nc + lo;
    return ordered_key_f32(s[j]);
  };

  if (resident) {
    if (BF16) {
      const uint16_t* s = static_cast<const uint16_t*>(scores) + row * (long long)Nc + lo;
      for (int j = tid; j < n; j += TK_THREADS) keys16[j] = uint16_t(ordered_key_bf16(s[j]));
    } else {
      const uint32_t* s = static_cast<const uint32_t*>(scores) + row * (long long)Nc + lo;
      for (int j = tid; j < n; j += TK_THREADS) keys32[j] = ordered_key_f32(s[j]);
    }
  }

  constexpr int NPASS = BF16 ? 2 : 3;
  const int shifts[3] = {BF16 ? 4 : 20, BF16 ? 0 : 8, 0};
  const int widths[3] = {12, BF16 ? 4 : 12, 8};
  uint32_t prefix = 0, pmask = 0;
  uint32_t krem = (uint32_t)k;
  uint32_t* merged0 = cluster.map_shared_rank(S.merged, 0);
  uint32_t* bcast0 = cluster.map_shared_rank(S.bcast, 0);

  for (int ps = 0; ps < NPASS; ps++) {
    const int shift = shifts[ps], bins = 1 << widths[ps];
    for (int i = tid; i < bins; i += TK_THREADS) {
      S.hist[i] = 0;
      if (rank == 0) S.merged[i] = 0;
    }
    cluster.sync();  // also orders the key loads above before their use
    for (int j = tid; j < n; j += TK_THREADS) {
      const uint32_t key = key_at(j);
      if ((key & pmask) == prefix) atomicAdd(&S.hist[(key >> shift) & (bins - 1)], 1u);
    }
    __syncthreads();
    for (int i = tid; i < bins; i += TK_THREADS)
      if (S.hist[i]) atomicAdd(merged0 + i, S.hist[i]);
    cluster.sync();
    if (rank == 0) {
      // find the digit d with count(above d) < krem <= count(above d) + cnt[d]
      const int per = (bins + TK_THREADS - 1) / TK_THREADS;
      // thread t covers bins from the top: [bins-1-t*per .. bins-t*per-per]
      uint32_t local = 0;
      for (int u = 0; u < per; u++) {
        int bin = bins - 1 - (tid * per + u);
        if (bin >= 0) local += S.merged[bin];
      }
      const uint32_t before = block_excl_scan(local, S.scan_tmp);
      if (before < krem && krem <= before + local) {
        uint32_t acc = before;
        for (int u = 0; u < per; u++) {
          int bin = bins - 1 - (tid * per + u);
          uint32_t c = S.merged[bin];
          if (acc + c >= krem) {
            S.bcast[0] = (uint32_t)bin;
            S.bcast[1] = acc;
            break;
          }
          acc += c;
        }
      }
    }
    cluster.sync();
    const uint32_t dig = bcast0[0], above = bcast0[1];
    prefix |= dig << shift;
    pmask |= uint32_t(bins - 1) << shift;
    krem -= above;
  }
  emit_ordered(cluster, S.wsum, S.cnt, key_at, n, lo, prefix, krem, k, out, status);
}

// ---------------------------------------------------------------------------------------
// Exact 16-bit first digit.  bf16 scores are concentrated in a few exponents, so a 12-bit
// first digit piles most keys onto a handful of shared-memory counters; with the whole top
// 16 bits as the digit (65536 u16 counters packed in pairs, 128 KB) collisions only happen
// between equal keys.  Each block first finds its local threshold t_r: the largest digit with
// at least ceil(k/C) of its keys at or above it (capped by its key count).  T0 = min_r t_r is
// a provable lower bound of the global k-th key (every block has >= ceil(k/C) keys >= T0), so
// block 0 only sums the cluster's histograms over [T0, 65535] -- a few hundred digits in
// practice -- reading them through distributed shared memory.  32-bit (fp32) keys then resolve
// the low 16 bits among the keys of the chosen digit with two 8-bit passes.

struct Tk16Shared {
  uint32_t hist[32768];  // 65536 u16 counters of the top-16-bit digit, two per word; only the
                         // words [wlo, whi] spanned by this block's keys are valid
  uint32_t hist8[256];   // 8-bit digit histogram (32-bit keys, low half)
  uint32_t merged8[256];
  uint32_t res[4];       // suffix-search result: digit, count above, found flag
  uint32_t tloc;         // this block's local threshold digit (NONE: no constraint)
  int wlo, whi;          // word range of this block's keys (wlo > whi: no keys)
  uint32_t bcast[4];
  uint32_t cnt[4];
  uint32_t wsum[2][TK_WARPS];
  uint32_t scan_tmp[TK_WARPS + 1];
  uint32_t* srcs[16];    // block 0: the cluster's histograms and their word ranges
  int los[16], his[16];
  uint32_t t0;
};
constexpr uint32_t NONE = 0xFFFFFFFFu;

// Exclusive block scan (1024 threads) returning the block total in `total`.
__device__ uint32_t block_scan_total(uint32_t v, uint32_t* tmp, uint32_t& total) {
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
    const uint32_t t = tmp[lane];
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s - t;
    if (lane == 31) tmp[TK_WARPS] = s;
  }
  __syncthreads();
  const uint32_t res = tmp[w] + x - v;
  total = tmp[TK_WARPS];
  __syncthreads();
  return res;
}

// Largest digit t >= t_min with sum_{d >= t} cnt(d) >= target, where cnt(d) adds the packed
// u16 counters of `nsrc` histograms (this block's or, through DSMEM, the cluster's), source r
// valid on words [wlo[r], whi[r]].  Scans 1024 words (2048 digits) per round down from the
// highest valid word and stops at the round that crosses.
// Result in res[0] (digit), res[1] (count above the digit), res[2] (1 if found).
__device__ void suffix_find(uint32_t* const* srcs, const int* wlo, const int* whi, int nsrc,
                            uint32_t t_min, uint32_t target, uint32_t* tmp, uint32_t* res) {
  const int tid = threadIdx.x;
  const int w_min = int(t_min >> 1);
  int w_top = -1;
  for (int r = 0; r < nsrc; r++) w_top = max(w_top, whi[r]);
  if (tid == 0) res[2] = 0;
  __syncthreads();
  uint32_t run = 0;
  for (int wtop = w_top; wtop >= w_min; wtop -= TK_THREADS) {
    const int word = wtop - tid;
    uint32_t c_lo = 0, c_hi = 0;
    if (word >= w_min) {
      // unrolled so the (remote) loads of all sources are in flight together
#pragma unroll
      for (int r = 0; r < 16; r++) {
        if (r < nsrc && word >= wlo[r] && word <= whi[r]) {
          const uint32_t v = srcs[r][word];
          c_lo += v & 0xFFFFu;
          c_hi += v >> 16;
        }
      }
      if (uint32_t(2 * word) < t_min) c_lo = 0;
      if (uint32_t(2 * word + 1) < t_min) c_hi = 0;
    }
    const uint32_t c = c_lo + c_hi;
    uint32_t total;
    const uint32_t excl = block_scan_total(c, tmp, total);
    const uint32_t before = run + excl;
    if (before < target && target <= before + c) {   // the crossing is in this word
      if (before + c_hi >= target) { res[0] = 2 * word + 1; res[1] = before; }
      else { res[0] = 2 * word; res[1] = before + c_hi; }
      res[2] = 1;
    }
    __syncthreads();
    if (res[2]) break;
    run += total;
  }
  __syncthreads();
}

template <bool BF16>
__global__ void __launch_bounds__(TK_THREADS, 1)
    topk16_kernel(const void* __restrict__ scores, int Tq, int Nc, const int32_t* __restrict__ q_pos,
                  int m, int k, int32_t* __restrict__ idx, int32_t* status) {
  cg::cluster_group cluster = cg::this_cluster();
  pdl_enter();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const long long row = blockIdx.x / C;
  extern __shared__ __align__(16) uint8_t tk_smem[];
  Tk16Shared& S = *reinterpret_cast<Tk16Shared*>(tk_smem);
  uint16_t* keys16 = reinterpret_cast<uint16_t*>(tk_smem + sizeof(Tk16Shared));
  uint32_t* keys32 = reinterpret_cast<uint32_t*>(tk_smem + sizeof(Tk16Shared));
  const int tid = threadIdx.x;

  const int pos = q_pos[row];
  const int nvis = pos < 0 ? 0 : min(Nc, (pos + 1) / m);
  int32_t* out = idx + row * k;
  if (nvis <= k) {
    for (int j = rank * TK_THREADS + tid; j < k; j += C * TK_THREADS) out[j] = j < nvis ? j : -1;
    return;
  }
  const int chunk = (nvis + C - 1) / C;
  const int lo = min(nvis, rank * chunk);
  const int n = min(nvis, lo + chunk) - lo;
  auto key_at = [&](int j) -> uint32_t { return BF16 ? uint32_t(keys16[j]) : keys32[j]; };
  constexpr int SH = BF16 ? 0 : 16;

  uint32_t dmin = 0xFFFFFFFFu, dmax = 0;
  {
    // 16-byte vector loads where the slice is aligned (several in flight per thread), scalar
    // loads for the unaligned head and the tail
    constexpr int EPV = BF16 ? 8 : 4;            // keys per 16-byte vector
    constexpr int ESZ = BF16 ? 2 : 4;
    const long long base = row * (long long)Nc + lo;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(scores) + uintptr_t(base) * ESZ;
    const int head = min(n, int(((16 - (addr & 15)) & 15) / ESZ));
    const int nvec = (n - head) / EPV;
    auto put = [&](int j, uint32_t raw) {
      const uint32_t key = BF16 ? ordered_key_bf16(uint16_t(raw)) : ordered_key_f32(raw);
      if (BF16) keys16[j] = uint16_t(key);
      else keys32[j] = key;
      dmin = min(dmin, key >> SH);
      dmax = max(dmax, key >> SH);
    };
    const uint16_t* s16 = static_cast<const uint16_t*>(scores) + base;
    const uint32_t* s32 = static_cast<const uint32_t*>(scores) + base;
    for (int j = tid; j < head; j += TK_THREADS) put(j, BF16 ? s16[j] : s32[j]);
    const uint4* v = reinterpret_cast<const uint4*>(BF16 ? (const void*)(s16 + head)
                                                         : (const void*)(s32 + head));
#pragma unroll 4
    for (int u = tid; u < nvec; u += TK_THREADS) {
      const uint4 x = __ldg(v + u);
      const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; e++) {
        if (BF16) {
          put(head + u * 8 + 2 * e, w4[e] & 0xFFFFu);
          put(head + u * 8 + 2 * e + 1, w4[e] >> 16);
        } else {
          put(head + u * 4 + e, w4[e]);
        }
      }
    }
    for (int j = head + nvec * EPV + tid; j < n; j += TK_THREADS) put(j, BF16 ? s16[j] : s32[j]);
  }
  if (tid == 0) { S.wlo = 0x7fffffff; S.whi = -1; }
  __syncthreads();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dmin = min(dmin, __shfl_xor_sync(0xffffffffu, dmin, o));
    dmax = max(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
  }
  if ((tid & 31) == 0 && dmin <= dmax) {
    atomicMin(&S.wlo, int(dmin >> 1));
    atomicMax(&S.whi, int(dmax >> 1));
  }
  __syncthreads();
  const int wlo = S.wlo, whi = S.whi;
  for (int i = wlo + tid; i <= whi; i += TK_THREADS) S.hist[i] = 0;   // only the spanned words
  __syncthreads();
  for (int j = tid; j < n; j += TK_THREADS) {
    const uint32_t d = key_at(j) >> SH;
    atomicAdd(&S.hist[d >> 1], 1u << ((d & 1) << 4));
  }
  __syncthreads();
  // local threshold: at least ceil(k / C) of this block's keys at or above it
  const uint32_t kc = min((uint32_t)n, (uint32_t)((k + C - 1) / C));
  uint32_t* self[1] = {S.hist};
  if (kc > 0) {
    suffix_find(self, &wlo, &whi, 1, 0, kc, S.scan_tmp, S.res);
    if (tid == 0) S.tloc = S.res[2] ? S.res[0] : 0u;
  } else if (tid == 0) {
    S.tloc = NONE;
  }
  cluster.sync();
  if (rank == 0) {
    // warp 0: lane r fetches block r's threshold and word range (one DSMEM round trip)
    if (tid < 32) {
      uint32_t t = NONE;
      if (tid < C) {
        S.srcs[tid] = cluster.map_shared_rank(S.hist, tid);
        t = *cluster.map_shared_rank(&S.tloc, tid);
        S.los[tid] = *cluster.map_shared_rank(&S.wlo, tid);
        S.his[tid] = *cluster.map_shared_rank(&S.whi, tid);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t = min(t, __shfl_xor_sync(0xffffffffu, t, o));
      if (tid == 0) S.t0 = t == NONE ? 0u : t;
    }
    __syncthreads();
    const uint32_t t0 = S.t0;
    suffix_find(S.srcs, S.los, S.his, C, t0, (uint32_t)k, S.scan_tmp, S.res);
    if (!S.res[2] && t0 > 0) suffix_find(S.srcs, S.los, S.his, C, 0, (uint32_t)k, S.scan_tmp, S.res);
    if (tid == 0) {
      S.bcast[0] = S.res[2] ? S.res[0] : 0u;
      S.bcast[1] = S.res[2] ? S.res[1] : 0u;
    }
  }
  cluster.sync();
  const uint32_t* b0 = cluster.map_shared_rank(S.bcast, 0);
  uint32_t prefix = b0[0] << SH;
  uint32_t pmask = 0xFFFFu << SH;
  uint32_t krem = (uint32_t)k - b0[1];
  if (!BF16) {
    uint32_t* merged0 = cluster.map_shared_rank(S.merged8, 0);
    for (int ps = 0; ps < 2; ps++) {
      const int shift = 8 - 8 * ps;
      for (int i = tid; i < 256; i += TK_THREADS) {
        S.hist8[i] = 0;
        if (rank == 0) S.merged8[i] = 0;
      }
      cluster.sync();
      for (int j = tid; j < n; j += TK_THREADS) {
        const uint32_t key = key_at(j);
        if ((key & pmask) == prefix) atomicAdd(&S.hist8[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      for (int i = tid; i < 256; i += TK_THREADS)
        if (S.hist8[i]) atomicAdd(merged0 + i, S.hist8[i]);
      cluster.sync();
      if (rank == 0 && tid < 32) {
        // one warp: 8 bins per lane from the top, warp scan, crossing lane resolves
        uint32_t c[8], loc = 0;
#pragma unroll
        for (int u = 0; u < 8; u++) { c[u] = S.merged8[255 - (tid * 8 + u)]; loc += c[u]; }
        uint32_t x = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
          if (tid >= o) x += y;
        }
        const uint32_t before = x - loc;
        if (before < krem && krem <= x) {
          uint32_t acc = before;
          for (int u = 0; u < 8; u++) {
            if (acc + c[u] >= krem) { S.bcast[2] = 255 - (tid * 8 + u); S.bcast[3] = acc; break; }
            acc += c[u];
          }
        }
      }
      cluster.sync();
      prefix |= b0[2] << shift;
      pmask |= 255u << shift;
      krem -= b0[3];
    }
  }
  emit_ordered(cluster, S.wsum, S.cnt, key_at, n, lo, prefix, krem, k, out, status);
}

// Cluster size: enough blocks that a slice fits in shared memory and, while slices stay
// long (>= 4096 keys), enough clusters to cover the SMs.
int choose_cluster(long long rows, int nvis_max, size_t cap_keys) {
  int C = 1;
  while (C < 16) {
    const long long chunk = (nvis_max + C - 1) / C;
    const bool too_long = (size_t)chunk > cap_keys;
    const bool too_few = rows * C < (long long)num_sms() && chunk >= 8192;
    if (!too_long && !too_few) break;
    C <<= 1;
  }
  return C;
}

template <bool BF16>
hcl_status_t run_topk(const TopkArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.Tq;
  const int key_bytes = BF16 ? 2 : 4;
  const size_t cap_keys = (200 * 1024 - sizeof(TkShared)) / key_bytes;
  int C = choose_cluster(rows, a.Nc, cap_keys);
  auto kern = topk_kernel<BF16>;
  hcl_status_t e = check_cuda(
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1),
      "topk cluster attribute");
  if (e != HCL_OK) return e;
  for (;;) {
    const size_t chunk = (size_t)(a.Nc + C - 1) / C;
    const int chunk_cap = (int)std::min(chunk, cap_keys);
    const size_t smem = sizeof(TkShared) + ((size_t)chunk_cap * key_bytes + 15) / 16 * 16;
    e = check_cuda(
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
        "topk smem attribute");
    if (e != HCL_OK) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(TK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    int nclusters = 0;
    cudaError_t qe = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if ((qe != cudaSuccess || nclusters < 1) && C > 1) {
      cudaGetLastError();  // clear the query's error and retry with a smaller cluster
      C >>= 1;
      continue;
    }
    return check_cuda(cudaLaunchKernelEx(&cfg, kern, a.scores, a.Tq, a.Nc, a.q_pos, a.m, a.k,
                                         a.idx, chunk_cap, a.status),
                      "topk launch");
  }
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int, int) { return 0; }

// Exact-16-bit-digit selection when a cluster of <= 16 blocks can hold the row's keys next to
// the 128 KB histogram; the cluster size gives >= ~1 block per SM on few long rows.
template <bool BF16>
hcl_status_t run_topk16(const TopkArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  const long long rows = (long long)a.B * a.Tq;
  const int key_bytes = BF16 ? 2 : 4;
  const size_t cap_keys = (226 * 1024 - sizeof(Tk16Shared)) / key_bytes;
  int C = 1;
  while (C < 16 && ((size_t)(a.Nc + C - 1) / C > cap_keys ||
                    (rows * C < (long long)num_sms() && (a.Nc + C - 1) / C >= 8192)))
    C <<= 1;
  if ((size_t)(a.Nc + C - 1) / C > cap_keys) return HCL_OK;   // too long: radix-12 path
  auto kern = topk16_kernel<BF16>;
  // attributes and the schedulability of each cluster size are set / queried once
  static bool attr_done = false;
  static int smem_set = 0;
  static int cluster_ok[17] = {0};   // 0 unknown, 1 ok, -1 not schedulable
  hcl_status_t e;
  if (!attr_done) {
    e = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1),
                   "topk cluster attribute");
    if (e != HCL_OK) return e;
    e = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        226 * 1024),
                   "topk smem attribute");
    if (e != HCL_OK) return e;
    smem_set = 226 * 1024;
    attr_done = true;
  }
  for (;;) {
    const size_t chunk = (size_t)(a.Nc + C - 1) / C;
    const size_t smem = sizeof(Tk16Shared) + (chunk * key_bytes + 15) / 16 * 16;
    if (chunk > cap_keys || (int)smem > smem_set) return HCL_OK;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(TK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cluster_ok[C] == 0) {
      // co-resident clusters of this size (at the largest shared memory the kernel may use)
      cudaLaunchConfig_t q = cfg;
      q.dynamicSmemBytes = smem_set;
      int nclusters = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&nclusters, kern, &q);
      if (qe != cudaSuccess) cudaGetLastError();
      cluster_ok[C] = (qe == cudaSuccess && nclusters >= 1) ? nclusters : -1;
    }
    // not schedulable, or more rows than co-resident clusters (a second wave costs a whole
    // kernel's latency): halve the cluster while the slices still fit
    const bool two_waves = cluster_ok[C] > 0 && rows > cluster_ok[C];
    if (C > 1 && (cluster_ok[C] < 0 || two_waves) &&
        (size_t)(a.Nc + C / 2 - 1) / (C / 2) <= cap_keys) {
      C >>= 1;
      continue;
    }
    if (cluster_ok[C] < 0 && C > 1) {
      C >>= 1;
      continue;
    }
    *used = true;
    return check_cuda(cudaLaunchKernelEx(&cfg, kern, a.scores, a.Tq, a.Nc, a.q_pos, a.m, a.k,
                                         a.idx, a.status),
                      "topk launch");
  }
}

hcl_status_t launch_topk(const TopkArgs& a, void*, size_t, cudaStream_t st) {
  if ((long long)a.B * a.Tq == 0 || a.k == 0) return HCL_OK;
  bool used = false;
  hcl_status_t e = a.score_fmt == HCL_BF16 ? run_topk16<true>(a, st, &used)
                                           : run_topk16<false>(a, st, &used);
  if (e != HCL_OK || used) return e;
  if (a.score_fmt == HCL_BF16) return run_topk<true>(a, st);
  return run_topk<false>(a, st);
}

}  // namespace hcl
