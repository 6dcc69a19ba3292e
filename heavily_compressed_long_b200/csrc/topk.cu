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
#include <map>
#include <mutex>

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

// Emission, shared by the selection kernels.  With the exact threshold key T and krem, the
// number of T-valued keys to take (lowest indices first), a block's selected keys are its keys
// > T and its first eq_take keys == T; given the counts of the blocks before it (gt_before,
// eq_before), its warps write the selected indices in ascending order with ballots.
//
// count_pass: per-warp counts of keys > T and == T over the warp's segment, into wsum.
template <class KeyAt>
__device__ void count_pass(uint32_t (*wsum)[TK_WARPS], KeyAt key_at, int n, uint32_t T) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
}

// write_pass: after count_pass and a block barrier.
template <class KeyAt>
__device__ void write_pass(const uint32_t (*wsum)[TK_WARPS], KeyAt key_at, int n, int lo, uint32_t T,
                           uint32_t krem, int k, uint32_t gt_before, uint32_t eq_before,
                           int32_t* out, int32_t* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (n + TK_WARPS - 1) / TK_WARPS;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  uint32_t own_eq = 0, wg_before = 0, we_before = 0;
  for (int w = 0; w < TK_WARPS; w++) {
    own_eq += wsum[1][w];
    if (w < warp) { wg_before += wsum[0][w]; we_before += wsum[1][w]; }
  }
  const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, own_eq) : 0u;
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
}

// Emission when the blocks' counts are not known yet: every block counts, publishes its totals,
// reads those of the blocks before it through DSMEM (lane r of warp 0 reads block r), then
// writes.  Ends with a cluster barrier so no block exits while another may still read its
// shared memory.
template <class KeyAt>
__device__ void emit_ordered(cg::cluster_group& cluster, uint32_t (*wsum)[TK_WARPS], uint32_t* cnt,
                             KeyAt key_at, int n, int lo, uint32_t T, uint32_t krem, int k,
                             int32_t* out, int32_t* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster.block_rank();
  count_pass(wsum, key_at, n, T);
  __syncthreads();
  if (tid == 0) {
    uint32_t tg = 0, te = 0;
    for (int w = 0; w < TK_WARPS; w++) { tg += wsum[0][w]; te += wsum[1][w]; }
    cnt[0] = tg;
    cnt[1] = te;
  }
  cluster.sync();
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
  write_pass(wsum, key_at, n, lo, T, krem, k, cnt[2], cnt[3], out, status);
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
  const int tid = threadIdx.x;

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
// between equal keys.  After one cluster barrier every block reads all the cluster's
// histograms through distributed shared memory, from the top digit down, and finds the digit
// T of the k-th largest key itself (no broadcast round).  For bf16 keys the digit is the whole
// key, so the same pass also yields the number of keys > T and == T in the blocks before this
// one, which places this block's output without another exchange: the block signals the
// cluster barrier once its remote reads are done and writes its indices while the others
// finish.  32-bit (fp32) keys resolve their low 16 bits among the keys of digit T with two
// 8-bit passes and emit after a count exchange.

struct alignas(16) Tk16Shared {
  uint32_t hist[32768];  // 65536 u16 counters of the top-16-bit digit, two per word; only the
                         // words [wlo, whi] spanned by this block's keys are valid
  uint32_t hist8[256];   // 8-bit digit histogram (32-bit keys, low half)
  uint32_t merged8[256];
  uint32_t res[8];       // digit search: digit, count above, found, gt_before, eq_before
  int wlo, whi;          // word range of this block's keys (wlo > whi: no keys)
  uint32_t bcast[4];
  uint32_t cnt[4];
  uint32_t wsum[2][TK_WARPS];
  uint32_t scan_tmp[TK_WARPS + 1];
  uint32_t red[2][TK_WARPS];
  uint32_t* srcs[16];    // the cluster's histograms and their word ranges
  int los[16], his[16];
};

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

// Largest digit T with sum_{d >= T} cnt(d) >= target, where cnt(d) adds the packed u16 counters
// of the cluster's `nsrc` histograms (source r valid on words [wlo[r], whi[r]]).  Scans 1024
// words (2048 digits) per round down from the highest valid word and stops at the round that
// crosses.  res[0] = T, res[1] = number of keys with digit > T, res[2] = 1 if found; and over
// the sources r < me only: res[3] = keys with digit > T, res[4] = keys with digit == T.
__device__ void suffix_find(uint32_t* const* srcs, const int* wlo, const int* whi, int nsrc, int me,
                            uint32_t target, uint32_t* tmp, uint32_t (*red)[TK_WARPS],
                            uint32_t* res, int w_start = 0x7fffffff, uint32_t run0 = 0,
                            uint32_t acc0 = 0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int w_top = -1, w_bot = 0x7fffffff;
  for (int r = 0; r < nsrc; r++) {
    if (wlo[r] <= whi[r]) { w_top = max(w_top, whi[r]); w_bot = min(w_bot, wlo[r]); }
  }
  w_top = min(w_top, w_start);   // continue a search below the words already scanned
  __syncthreads();               // (callers may still read res)
  if (tid == 0) { res[2] = 0; res[3] = 0; res[4] = 0; }
  __syncthreads();
  uint32_t run = run0, acc_gt = tid == 0 ? acc0 : 0u;   // acc_gt: summed over the block
  for (int wtop = w_top; wtop >= w_bot; wtop -= TK_THREADS) {
    const int word = wtop - tid;
    uint32_t c_lo = 0, c_hi = 0, b_lo = 0, b_hi = 0;
    if (word >= w_bot) {
      // unrolled so the (remote) loads of all sources are in flight together
#pragma unroll
      for (int r = 0; r < 16; r++) {
        if (r < nsrc && word >= wlo[r] && word <= whi[r]) {
          const uint32_t v = srcs[r][word];
          c_lo += v & 0xFFFFu;
          c_hi += v >> 16;
          if (r < me) { b_lo += v & 0xFFFFu; b_hi += v >> 16; }
        }
      }
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
    if (res[2]) {
      // the earlier rounds lie wholly above T; in this round split each word at T
      const uint32_t T = res[0];
      uint32_t gt = acc_gt, eq = 0;
      if (word >= w_bot) {
        if (uint32_t(2 * word) > T) gt += b_lo;
        else if (uint32_t(2 * word) == T) eq += b_lo;
        if (uint32_t(2 * word + 1) > T) gt += b_hi;
        else if (uint32_t(2 * word + 1) == T) eq += b_hi;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
      }
      if (lane == 0) { red[0][warp] = gt; red[1][warp] = eq; }
      __syncthreads();
      if (warp == 0) {
        uint32_t g = red[0][lane], e = red[1][lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          g += __shfl_xor_sync(0xffffffffu, g, o);
          e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) { res[3] = g; res[4] = e; }
      }
      break;
    }
    run += total;
    acc_gt += b_lo + b_hi;
  }
  __syncthreads();
}

// Warp-inclusive scan.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Warp-level variant of suffix_find for narrow searches: warp 0 scans 128 words (256 digits)
// per round, each lane reading 4 words of every source with one 16-byte load, so a round costs
// one remote round trip and 32 x nsrc requests; after WARP_ROUNDS rounds without the crossing
// the block-wide suffix_find takes over below.  Same results as suffix_find (res[0..4]).
constexpr int WARP_ROUNDS = 4;

__device__ void suffix_find_top(uint32_t* const* srcs, const int* wlo, const int* whi, int nsrc,
                                int me, uint32_t target, uint32_t* tmp, uint32_t (*red)[TK_WARPS],
                                uint32_t* res) {
  const int tid = threadIdx.x, lane = tid & 31;
  int w_top = -1, w_bot = 0x7fffffff;
  for (int r = 0; r < nsrc; r++) {
    if (wlo[r] <= whi[r]) { w_top = max(w_top, whi[r]); w_bot = min(w_bot, wlo[r]); }
  }
  if (tid < 32) {
    uint32_t run = 0, acc_gt = 0;
    bool found = false;
    int gtop = w_top >> 2;
    for (int round = 0; round < WARP_ROUNDS && !found && gtop >= (w_bot >> 2); round++, gtop -= 32) {
      const int gi = gtop - lane;   // this lane's words 4gi .. 4gi+3 (digits 8gi .. 8gi+7)
      uint32_t c[8], bc[8];         // index i <-> digit 8gi + 7 - i (descending)
#pragma unroll
      for (int i = 0; i < 8; i++) c[i] = bc[i] = 0u;
      if (gi >= (w_bot >> 2)) {
#pragma unroll
        for (int r = 0; r < 16; r++) {
          if (r < nsrc && 4 * gi + 3 >= wlo[r] && 4 * gi <= whi[r]) {
            const uint4 v = *reinterpret_cast<const uint4*>(srcs[r] + 4 * gi);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int w = 0; w < 4; w++) {
              const int word = 4 * gi + w;
              if (word >= wlo[r] && word <= whi[r]) {
                c[7 - 2 * w] += w4[w] & 0xFFFFu;   // digit 2*word
                c[6 - 2 * w] += w4[w] >> 16;       // digit 2*word + 1
                if (r < me) { bc[7 - 2 * w] += w4[w] & 0xFFFFu; bc[6 - 2 * w] += w4[w] >> 16; }
              }
            }
          }
        }
      }
      uint32_t tot = 0, btot = 0;
#pragma unroll
      for (int i = 0; i < 8; i++) { tot += c[i]; btot += bc[i]; }
      const uint32_t incl = warp_incl_scan(tot);
      const uint32_t before = run + incl - tot;
      const bool cross = before < target && target <= before + tot;
      const uint32_t cm = __ballot_sync(0xffffffffu, cross);
      if (cm) {
        const int cl = __ffs(cm) - 1;
        uint32_t T = 0, above = 0, gt = 0, eq = 0;
        if (lane == cl) {
          uint32_t acc = before;
          int ti = 7;
#pragma unroll
          for (int i = 0; i < 8; i++) {
            if (acc + c[i] >= target) { ti = i; break; }
            acc += c[i];
          }
          T = uint32_t(8 * gi + 7 - ti);
          above = acc;
#pragma unroll
          for (int i = 0; i < 8; i++) {
            if (i < ti) gt += bc[i];
            else if (i == ti) eq += bc[i];
          }
        } else if (lane < cl) {
          gt = btot;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          gt += __shfl_xor_sync(0xffffffffu, gt, o);
          eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        T = __shfl_sync(0xffffffffu, T, cl);
        above = __shfl_sync(0xffffffffu, above, cl);
        if (lane == 0) { res[0] = T; res[1] = above; res[2] = 1; res[3] = acc_gt + gt; res[4] = eq; }
        found = true;
      } else {
        run += __shfl_sync(0xffffffffu, incl, 31);
        uint32_t bt = btot;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bt += __shfl_xor_sync(0xffffffffu, bt, o);
        acc_gt += bt;
      }
    }
    if (lane == 0) {
      if (!found) { res[2] = 0; res[5] = run; res[6] = acc_gt; res[7] = uint32_t(gtop); }
      else res[7] = 0xFFFFFFFFu;
    }
  }
  __syncthreads();
  if (res[7] != 0xFFFFFFFFu && int(res[7]) >= (w_bot >> 2)) {
    // not within the first rounds: the block-wide search continues below the scanned words
    suffix_find(srcs, wlo, whi, nsrc, me, target, tmp, red, res, 4 * int(res[7]) + 3, res[5],
                res[6]);
  }
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// Arrive without release: only used once this block's remote reads have all returned their
// values (the barrier then only keeps the other blocks' shared memory alive).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---- bf16 rows, vectorised: keys live in shared memory as 8 u16 per 16-byte vector, placed
// so that vector u matches the 16-byte-aligned global vector it came from.  Position p of
// the block's key array holds key j = p - off of the slice (valid for 0 <= j < n); the other
// positions of the first and last vector are padding and are masked out.

// Bits e (0..7) of vector u whose key is valid.
__device__ __forceinline__ uint32_t valid8(int u, int off, int n) {
  const int p0 = 8 * u;
  const int a = max(0, off - p0), b = min(8, off + n - p0);
  return b > a ? ((0xFFu >> (8 - (b - a))) << a) : 0u;
}

// Per-key masks (bit e for element e) of keys > T and == T among 8 packed u16 keys.
__device__ __forceinline__ void cmp8(const uint4& x, uint32_t T, uint32_t& gt, uint32_t& eq) {
  const uint32_t TT = T | (T << 16);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  gt = 0;
  eq = 0;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const uint32_t g = __vcmpgtu2(w[i], TT), e = __vcmpeq2(w[i], TT);
    gt |= ((g & 1u) | ((g >> 15) & 2u)) << (2 * i);
    eq |= ((e & 1u) | ((e >> 15) & 2u)) << (2 * i);
  }
}

// Order-preserving keys of two packed bf16 values: x ^ 0x8000 for positive, ~x for negative.
__device__ __forceinline__ uint32_t ordered_key_bf16x2(uint32_t x) {
  return x ^ 0x80008000u ^ (((x >> 15) & 0x00010001u) * 0x7FFFu);
}

// Count pass over warp w's vectors [w*V, min(nv, (w+1)*V)): keys > T and == T, into wsum.
__device__ void count16(uint32_t (*wsum)[TK_WARPS], const uint4* kv, int nv, int off, int n,
                        uint32_t T) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int V = (nv + TK_WARPS - 1) / TK_WARPS;
  const int u0 = min(nv, warp * V), u1 = min(nv, u0 + V);
  uint32_t g = 0, e = 0;
  for (int u = u0 + lane; u < u1; u += 32) {
    uint32_t gm, em;
    cmp8(kv[u], T, gm, em);
    const uint32_t vm = valid8(u, off, n);
    g += __popc(gm & vm);
    e += __popc(em & vm);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    g += __shfl_xor_sync(0xffffffffu, g, o);
    e += __shfl_xor_sync(0xffffffffu, e, o);
  }
  if (lane == 0) { wsum[0][warp] = g; wsum[1][warp] = e; }
}

// Write pass (after count16 and a block barrier): the block's selected keys, in index order,
// from output slot gt_before + min(eq_before, krem) on.
__device__ void write16(const uint32_t (*wsum)[TK_WARPS], const uint4* kv, int nv, int off, int n,
                        int lo, uint32_t T, uint32_t krem, int k, uint32_t gt_before,
                        uint32_t eq_before, int32_t* out, int32_t* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int V = (nv + TK_WARPS - 1) / TK_WARPS;
  const int u0 = min(nv, warp * V), u1 = min(nv, u0 + V);
  uint32_t own_eq = 0, wg_before = 0, we_before = 0;
  for (int w = 0; w < TK_WARPS; w++) {
    own_eq += wsum[1][w];
    if (w < warp) { wg_before += wsum[0][w]; we_before += wsum[1][w]; }
  }
  const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, own_eq) : 0u;
  uint32_t pos_out = gt_before + min(eq_before, krem) + wg_before + min(we_before, eq_take);
  uint32_t eq_seen = we_before;
  for (int ub = u0; ub < u1; ub += 32) {
    const int u = ub + lane;
    uint32_t gm = 0, em = 0;
    if (u < u1) {
      cmp8(kv[u], T, gm, em);
      const uint32_t vm = valid8(u, off, n);
      gm &= vm;
      em &= vm;
    }
    if (__ballot_sync(0xffffffffu, (gm | em) != 0u) == 0u) continue;
    const uint32_t ne = __popc(em);
    const uint32_t e_incl = warp_incl_scan(ne);
    const uint32_t e_before = eq_seen + e_incl - ne;   // ties before this lane's keys
    uint32_t take = eq_take > e_before ? min(eq_take - e_before, ne) : 0u;
    uint32_t sel = gm;
    for (uint32_t m = em; take > 0; take--) {          // the lane's first `take` ties
      const uint32_t low = m & (0u - m);
      sel |= low;
      m ^= low;
    }
    const uint32_t ns = __popc(sel);
    const uint32_t s_incl = warp_incl_scan(ns);
    uint32_t slot = pos_out + s_incl - ns;
    for (uint32_t m = sel; m != 0u; m &= m - 1u) {
      const int e = __ffs(m) - 1;
      if (slot < (uint32_t)k) out[slot] = lo + (8 * u + e - off);
      else report(status, HCL_ERR_DEVICE_FAULT);
      slot++;
    }
    pos_out += __shfl_sync(0xffffffffu, s_incl, 31);
    eq_seen += __shfl_sync(0xffffffffu, e_incl, 31);
  }
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
  int off = 0, nv = 0;                     // bf16: vector layout of the keys (see valid8)
  const uint4* kv = reinterpret_cast<const uint4*>(keys16);
  if constexpr (BF16) {
    const uint16_t* s16 = static_cast<const uint16_t*>(scores) + row * (long long)Nc + lo;
    off = int((reinterpret_cast<uintptr_t>(s16) & 15) >> 1);
    nv = (off + n + 7) >> 3;
    const uint4* g = reinterpret_cast<const uint4*>(s16 - off);   // 16-byte aligned
    uint4* kw = reinterpret_cast<uint4*>(keys16);
    uint32_t vmin = 0xFFFFFFFFu, vmax = 0u;                        // packed pairs
#pragma unroll 4
    for (int u = tid; u < nv; u += TK_THREADS) {
      const uint32_t vm = valid8(u, off, n);
      uint4 y;
      if (vm == 0xFFu) {
        const uint4 x = __ldg(g + u);
        y = make_uint4(ordered_key_bf16x2(x.x), ordered_key_bf16x2(x.y), ordered_key_bf16x2(x.z),
                       ordered_key_bf16x2(x.w));
        vmin = __vminu2(vmin, __vminu2(__vminu2(y.x, y.y), __vminu2(y.z, y.w)));
        vmax = __vmaxu2(vmax, __vmaxu2(__vmaxu2(y.x, y.y), __vmaxu2(y.z, y.w)));
      } else {
        // first / last vector of the slice: only its valid elements are read
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; e++) {
          if ((vm >> e) & 1u) {
            const uint32_t key = ordered_key_bf16(s16[8 * u + e - off]);
            w[e >> 1] |= key << ((e & 1) * 16);
            dmin = min(dmin, key);
            dmax = max(dmax, key);
          }
        }
        y = make_uint4(w[0], w[1], w[2], w[3]);
      }
      kw[u] = y;
    }
    dmin = min(dmin, min(vmin & 0xFFFFu, vmin >> 16));
    dmax = max(dmax, max(vmax & 0xFFFFu, vmax >> 16));
  } else {
    // 16-byte vector loads where the slice is aligned (several in flight per thread), scalar
    // loads for the unaligned head and the tail
    const long long base = row * (long long)Nc + lo;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(scores) + uintptr_t(base) * 4;
    const int head = min(n, int(((16 - (addr & 15)) & 15) / 4));
    const int nvec = (n - head) / 4;
    auto put = [&](int j, uint32_t raw) {
      const uint32_t key = ordered_key_f32(raw);
      keys32[j] = key;
      dmin = min(dmin, key >> SH);
      dmax = max(dmax, key >> SH);
    };
    const uint32_t* s32 = static_cast<const uint32_t*>(scores) + base;
    for (int j = tid; j < head; j += TK_THREADS) put(j, s32[j]);
    const uint4* v = reinterpret_cast<const uint4*>(s32 + head);
#pragma unroll 4
    for (int u = tid; u < nvec; u += TK_THREADS) {
      const uint4 x = __ldg(v + u);
      put(head + u * 4 + 0, x.x);
      put(head + u * 4 + 1, x.y);
      put(head + u * 4 + 2, x.z);
      put(head + u * 4 + 3, x.w);
    }
    for (int j = head + nvec * 4 + tid; j < n; j += TK_THREADS) put(j, s32[j]);
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
  if constexpr (BF16) {
    for (int u = tid; u < nv; u += TK_THREADS) {
      const uint4 x = kv[u];
      const uint32_t vm = valid8(u, off, n);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 8; e++) {
        if ((vm >> e) & 1u) {
          const uint32_t d = (w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
          atomicAdd(&S.hist[d >> 1], 1u << ((d & 1) << 4));
        }
      }
    }
  } else {
    for (int j = tid; j < n; j += TK_THREADS) {
      const uint32_t d = key_at(j) >> SH;
      atomicAdd(&S.hist[d >> 1], 1u << ((d & 1) << 4));
    }
  }
  cluster.sync();
  // every block: lane r of warp 0 fetches block r's histogram address and word range (one
  // DSMEM round trip), then the digit search over all of them
  if (tid < 32) {
    if (tid < C) {
      S.srcs[tid] = cluster.map_shared_rank(S.hist, tid);
      S.los[tid] = *cluster.map_shared_rank(&S.wlo, tid);
      S.his[tid] = *cluster.map_shared_rank(&S.whi, tid);
    }
  }
  __syncthreads();
  suffix_find(S.srcs, S.los, S.his, C, rank, (uint32_t)k, S.scan_tmp, S.red, S.res);
  // (nvis > k keys are present, so the search always finds its digit)
  const uint32_t digit = S.res[2] ? S.res[0] : 0u;
  const uint32_t above = S.res[2] ? S.res[1] : 0u;
  if (BF16) {
    const uint32_t gt_before = S.res[3], eq_before = S.res[4];
    cluster_arrive_release();      // this block reads no remote shared memory from here on
    count16(S.wsum, kv, nv, off, n, digit);
    __syncthreads();
    write16(S.wsum, kv, nv, off, n, lo, digit, (uint32_t)k - above, k, gt_before, eq_before, out,
            status);
    cluster_wait_acquire();        // keep this block's histogram alive for the others
    return;
  }
  uint32_t prefix = digit << SH;
  uint32_t pmask = 0xFFFFu << SH;
  uint32_t krem = (uint32_t)k - above;
  {
    const uint32_t* b0 = cluster.map_shared_rank(S.bcast, 0);
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

// ---------------------------------------------------------------------------------------
// Register-resident bf16 selection (slices of up to 32 K keys per block, 1024 threads).
// Every thread holds up to 4 x 8 consecutive keys in registers.  The k-th largest of the
// threads' maxima is a lower bound L of the row's k-th largest key: the maxima are keys of
// distinct threads, so at least k keys are >= L.  The cluster finds L from one histogram
// count per thread (instead of one per key), then histograms only the candidate keys >= L
// (about k of them per row on typical data) over the digit window [L, max] and finds the
// exact threshold T, together with this block's counts before it, in a second search.  The
// block's selected indices are then placed by one packed block scan and written straight
// from registers.  Two cluster barriers in all; the last remote read is followed by a
// split arrive so that the writes overlap the other blocks' searches.

constexpr int TR_VPT = 4;                                   // 16-byte vectors per thread
constexpr int TR_MAX_KEYS = TK_THREADS * TR_VPT * 8 - 7;    // slice limit (any alignment)
constexpr int TR_CWORDS = 4096;                             // candidate window: 8192 digits

struct alignas(16) TrShared {
  uint32_t hist[32768];       // u16 pairs over all 65536 digits: thread maxima, then (when the
                              // candidate window is too wide) the candidates
  uint32_t histc[TR_CWORDS];  // u16 pairs over digits [cbase, cbase + 8192): the candidates
  uint32_t scan_tmp[TK_WARPS + 1];
  uint32_t red[2][TK_WARPS];
  uint32_t res[8];
  uint32_t dmax;              // this block's largest key (0 with no keys)
  uint32_t nmax;              // threads of this block holding at least one key
  uint32_t pdmax[16];         // every block's dmax / nmax, pushed by that block
  uint32_t pnmax[16];
  uint32_t* srcs[16];
  int los[16], his[16];
};

__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_reg_kernel(const __nv_bfloat16* __restrict__ scores, int Nc,
                    const int32_t* __restrict__ q_pos, int m, int k, int32_t* __restrict__ idx,
                    int32_t* status, int prewait) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t tk_smem[];
  TrShared& S = *reinterpret_cast<TrShared*>(tk_smem);
  const int tid = threadIdx.x, lane = tid & 31;
  // shared memory only: may overlap the previous kernel's tail
  for (int i = tid; i < 32768; i += TK_THREADS) S.hist[i] = 0u;
  if (tid == 0) S.dmax = 0u;
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const long long row = blockIdx.x / C;
  // q_pos may be read before waiting for the previous kernel when it does not write it
  if (!prewait) pdl_enter();
  const int pos = q_pos[row];
  if (prewait) pdl_enter();
  const int nvis = pos < 0 ? 0 : min(Nc, (pos + 1) / m);
  int32_t* out = idx + row * k;
  if (nvis <= k) {
    for (int j = rank * TK_THREADS + tid; j < k; j += C * TK_THREADS) out[j] = j < nvis ? j : -1;
    return;
  }
  const int chunk = (nvis + C - 1) / C;
  const int lo = min(nvis, rank * chunk);
  const int n = min(nvis, lo + chunk) - lo;

  // ---- keys of this thread: vectors [v0, v1) of the slice's 16-byte-aligned vectors
  const uint16_t* s16 = reinterpret_cast<const uint16_t*>(scores) + row * (long long)Nc + lo;
  const int off = int((reinterpret_cast<uintptr_t>(s16) & 15) >> 1);
  const int nv = (off + n + 7) >> 3;
  const int v0 = int((long long)tid * nv / TK_THREADS);
  const int v1 = int((long long)(tid + 1) * nv / TK_THREADS);
  const uint4* g = reinterpret_cast<const uint4*>(s16 - off);
  uint4 x[TR_VPT];
  uint32_t vmask[TR_VPT];
#pragma unroll
  for (int i = 0; i < TR_VPT; i++) {
    const int u = v0 + i;
    vmask[i] = u < v1 ? valid8(u, off, n) : 0u;
    if (vmask[i] == 0xFFu) {
      x[i] = __ldg(g + u);
    } else {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; e++)
        if ((vmask[i] >> e) & 1u) w[e >> 1] |= uint32_t(s16[8 * u + e - off]) << ((e & 1) * 16);
      x[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  uint32_t tmax = 0u;
  bool any = false;
#pragma unroll
  for (int i = 0; i < TR_VPT; i++) {
    x[i] = make_uint4(ordered_key_bf16x2(x[i].x), ordered_key_bf16x2(x[i].y),
                      ordered_key_bf16x2(x[i].z), ordered_key_bf16x2(x[i].w));
    if (vmask[i] == 0xFFu) {
      const uint32_t mm = __vmaxu2(__vmaxu2(x[i].x, x[i].y), __vmaxu2(x[i].z, x[i].w));
      tmax = max(tmax, max(mm & 0xFFFFu, mm >> 16));
      any = true;
    } else if (vmask[i]) {
      const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
      for (int e = 0; e < 8; e++)
        if ((vmask[i] >> e) & 1u) tmax = max(tmax, (w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
      any = true;
    }
  }
  const int nany = __syncthreads_count(any);   // (also: histogram zeroed)
  if (any) atomicAdd(&S.hist[tmax >> 1], 1u << ((tmax & 1) << 4));
  uint32_t bm = any ? tmax : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bm = max(bm, __shfl_xor_sync(0xffffffffu, bm, o));
  if (lane == 0) atomicMax(&S.dmax, bm);
  __syncthreads();
  if (tid < C) {   // push this block's largest key and maxima count to every block
    cluster.map_shared_rank(S.pdmax, tid)[rank] = S.dmax;
    cluster.map_shared_rank(S.pnmax, tid)[rank] = uint32_t(nany);
  }
  cluster.sync();

  // ---- L: the k-th largest thread maximum (0 when the row has fewer than k maxima)
  if (tid < 32) {
    uint32_t dm = 0u, nm = 0u;
    if (tid < C) {
      S.srcs[tid] = cluster.map_shared_rank(S.hist, tid);
      dm = S.pdmax[tid];
      nm = S.pnmax[tid];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dm = max(dm, __shfl_xor_sync(0xffffffffu, dm, o));
      nm += __shfl_xor_sync(0xffffffffu, nm, o);
    }
    if (tid < 16) { S.los[tid] = 0; S.his[tid] = int(dm >> 1); }
    if (tid == 0) { S.res[6] = dm; S.res[7] = nm; }
  }
  __syncthreads();
  const uint32_t Mx = S.res[6];
  uint32_t L = 0u;                              // fewer than k maxima: every key is a candidate
  if (S.res[7] >= (uint32_t)k) {
    suffix_find_top(S.srcs, S.los, S.his, C, 0, (uint32_t)k, S.scan_tmp, S.red, S.res);
    L = S.res[2] ? S.res[0] : 0u;
  }

  // ---- candidates (keys >= L) into the digit window [cbase, Mx]
  const uint32_t cbase = L & ~1u;
  const bool small = Mx - cbase < 2u * TR_CWORDS;
  uint32_t* H = small ? S.histc : S.hist;
  const uint32_t hb = small ? cbase : 0u;       // digit of word 0 of H
  if (!small) cluster.sync();                   // every block is done reading the maxima
  for (int w = int((cbase - hb) >> 1) + tid; w <= int((Mx - hb) >> 1); w += TK_THREADS) H[w] = 0u;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < TR_VPT; i++) {
    if (vmask[i] == 0u) continue;
    const uint32_t w4[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
    // fast reject: the vector's largest key
    const uint32_t mm = __vmaxu2(__vmaxu2(w4[0], w4[1]), __vmaxu2(w4[2], w4[3]));
    if (max(mm & 0xFFFFu, mm >> 16) < L) continue;
#pragma unroll
    for (int e = 0; e < 8; e++) {
      const uint32_t key = (w4[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
      if (((vmask[i] >> e) & 1u) && key >= L) {
        const uint32_t d = key - hb;
        atomicAdd(&H[d >> 1], 1u << ((d & 1) << 4));
      }
    }
  }
  cluster.sync();
  if (tid < 16) {
    if (tid < C) S.srcs[tid] = cluster.map_shared_rank(H, tid);
    S.los[tid] = int((cbase - hb) >> 1);
    S.his[tid] = int((Mx - hb) >> 1);
  }
  __syncthreads();
  suffix_find_top(S.srcs, S.los, S.his, C, rank, (uint32_t)k, S.scan_tmp, S.red, S.res);
  const uint32_t T = (S.res[2] ? S.res[0] : 0u) + hb;
  const uint32_t above = S.res[2] ? S.res[1] : 0u;
  const uint32_t gt_before = S.res[3], eq_before = S.res[4];
  const uint32_t krem = (uint32_t)k - above;
  cluster_arrive_relaxed();                     // no remote shared-memory reads from here on

  // ---- emission: one packed scan (keys == T in the high half, > T in the low half)
  uint32_t gm[TR_VPT], em[TR_VPT], gt = 0u, eq = 0u;
#pragma unroll
  for (int i = 0; i < TR_VPT; i++) {
    cmp8(x[i], T, gm[i], em[i]);
    gm[i] &= vmask[i];
    em[i] &= vmask[i];
    gt += __popc(gm[i]);
    eq += __popc(em[i]);
  }
  uint32_t total;
  const uint32_t excl = block_scan_total((eq << 16) | gt, S.scan_tmp, total);
  const uint32_t own_eq = total >> 16;
  const uint32_t e_before = excl >> 16, g_before = excl & 0xFFFFu;
  const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, own_eq) : 0u;
  uint32_t slot = gt_before + min(eq_before, krem) + g_before + min(e_before, eq_take);
  uint32_t take = eq_take > e_before ? min(eq_take - e_before, eq) : 0u;
#pragma unroll
  for (int i = 0; i < TR_VPT; i++) {
    uint32_t sel = gm[i];
    for (uint32_t mm = em[i]; take > 0u && mm != 0u; take--) {
      const uint32_t low = mm & (0u - mm);
      sel |= low;
      mm ^= low;
    }
    for (; sel != 0u; sel &= sel - 1u) {
      const int e = __ffs(sel) - 1;
      if (slot < (uint32_t)k) out[slot] = lo + (8 * (v0 + i) + e - off);
      else report(status, HCL_ERR_DEVICE_FAULT);
      slot++;
    }
  }
  cluster_wait_acquire();                       // keep this block's histograms for the others
}

// ---------------------------------------------------------------------------------------
// Decode selection from group summaries (inside the fused decode step, bf16 scores).  The indexer
// also writes, for every group of 16 entries, a summary of its visible scores as
// order-preserving keys: the largest, the second largest and the position of the largest.  The
// k-th largest of the maxima, L, is a lower bound of the row's k-th largest score (the maxima
// are scores of k distinct entries), so only groups whose maximum reaches L can hold selected
// entries -- on typical data about k groups, a few per cent of the row -- and a group whose
// second largest key is below L holds exactly one candidate, known from the summary.  One block
// per row: histogram of the maxima -> L; histogram of the candidate keys (scores read only for
// the few groups with two or more) -> the exact threshold T; then an index-ordered scan places
// every selected entry.  No cluster, no exchange between blocks.

constexpr int GM_G = 16;         // entries per group
constexpr int GM_GPT = 16;       // groups per thread: rows of up to 16 x 1024 groups
constexpr int GM_MAX_GROUPS = GM_GPT * TK_THREADS;

constexpr int GM_WWORDS = 4096;  // window histogram: 8192 digits
constexpr int GM_POOL = 512;     // groups with several candidates staged in shared memory
constexpr int GM_FLAT = 5120;    // candidates listed flat for the emission (more: per-thread loops)

struct alignas(16) GmShared {
  union {
    uint16_t list[GM_MAX_GROUPS];    // candidate group ids, in index order (fallback)
    uint32_t praw[GM_POOL][8];       // scores of the pooled groups as copied (bf16 pairs)
    struct {                         // the candidates in index order (emission)
      uint32_t fent[GM_FLAT];        // entry index
      uint16_t fkey[GM_FLAT];        // order-preserving key
    };
  };
  uint4 gms[2][TK_THREADS];      // thread t's 16 group maxima (0: no visible entry),
  uint4 g2s[2][TK_THREADS];      // their second maxima
  uint4 gas[TK_THREADS];         // and the positions of the maxima (low 4 bits of a byte)
  uint32_t wh[GM_WWORDS];        // u16 pairs over the digit window [wb, wb + 8191]: maxima
  uint32_t wc[GM_WWORDS];        // the same over the candidate keys
  uint32_t pent[GM_POOL][GM_G];  // candidates of the pooled groups: key << 4 | position
  uint32_t pcnt[GM_POOL];        // and their number
  uint16_t pgrp[GM_POOL];        // and the group of each slot
  uint32_t ncand;                // candidate keys in the row
  uint32_t npool;                // pool slots asked for
  uint32_t wcnt[TK_WARPS][16];   // per-warp digit counts of one radix pass
  uint32_t scan_tmp[TK_WARPS + 1];
  uint32_t red[2][TK_WARPS];
  uint32_t res[8];
  unsigned long long tmp64[TK_WARPS + 1];
};

// Exclusive block scan of 64-bit values (1024 threads), block total in `total`.
__device__ unsigned long long block_scan64(unsigned long long v, unsigned long long* tmp,
                                           unsigned long long& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    const unsigned long long t = tmp[lane];
    unsigned long long s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s - t;
    if (lane == 31) tmp[TK_WARPS] = s;
  }
  __syncthreads();
  const unsigned long long res = tmp[w] + x - v;
  total = tmp[TK_WARPS];
  __syncthreads();
  return res;
}

// Suffix search over one histogram of u16 digit pairs (word w: digit 2w low, 2w+1 high)
// between words w_bot and w_top, done by one warp from the top down in chunks of 128 words
// (4 per lane) and stopping at the chunk that holds the target: the keys sit near the top of
// the window, so a chunk or two usually suffices.  res[0] = digit T of the target-th largest
// counted key, res[1] = keys in digits above T, res[2] = 1 if found.  The caller publishes
// res with a barrier.
__device__ void warp_suffix(const uint32_t* hist, int w_top, int w_bot, uint32_t target,
                            uint32_t* res) {
  const int lane = threadIdx.x & 31;
  uint32_t run = 0;
  for (int ghi = w_top >> 2; ghi >= (w_bot >> 2); ghi -= 32) {
    const int gi = ghi - lane;
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; i++) c[i] = 0u;
    if (gi >= (w_bot >> 2)) {
      const uint4 v = *reinterpret_cast<const uint4*>(hist + 4 * gi);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int w = 0; w < 4; w++) {
        const int word = 4 * gi + w;
        if (word >= w_bot && word <= w_top) {
          c[7 - 2 * w] = w4[w] & 0xFFFFu;   // digit 2*word
          c[6 - 2 * w] = w4[w] >> 16;       // digit 2*word + 1
        }
      }
    }
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) tot += c[i];
    uint32_t inc = tot;                     // lanes in descending digit order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t before = run + inc - tot;
    const bool hit = before < target && target <= before + tot;
    if (hit) {
      uint32_t acc = before;
      int ti = 7;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        if (acc + c[i] >= target) { ti = i; break; }
        acc += c[i];
      }
      res[0] = uint32_t(8 * gi + 7 - ti);
      res[1] = acc;
      res[2] = 1;
    }
    if (__ballot_sync(0xffffffffu, hit)) return;
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) res[2] = 0;
}

// The same search by the whole block in one step: thread t counts the 8 digits of words
// w_top - 4t - 3 .. w_top - 4t (every word of a window of <= 4 x 1024 words), one block scan
// gives the keys above each thread's digits, and the thread whose digits hold the target-th
// largest key writes res[0..2] as warp_suffix does.  All threads call it; res is published.
__device__ void block_window_select(const uint32_t* hist, int w_top, int w_bot, uint32_t target,
                                    uint32_t* scan_tmp, uint32_t* res) {
  const int hi = w_top - 4 * (int)threadIdx.x;          // this thread's highest word
  uint32_t c[8];                                          // descending digits
  uint32_t tot = 0;
#pragma unroll
  for (int j = 0; j < 4; j++) {
    const int w = hi - j;
    const uint32_t v = (w >= w_bot) ? hist[w] : 0u;
    c[2 * j] = v >> 16;                                   // digit 2w + 1
    c[2 * j + 1] = v & 0xFFFFu;                           // digit 2w
    tot += c[2 * j] + c[2 * j + 1];
  }
  if (threadIdx.x == 0) res[2] = 0;
  uint32_t total;
  const uint32_t before = block_scan_total(tot, scan_tmp, total);
  if (before < target && target <= before + tot) {
    uint32_t acc = before;
    int ti = 7;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      if (acc + c[i] >= target) { ti = i; break; }
      acc += c[i];
    }
    res[0] = uint32_t(2 * (hi - (ti >> 1)) + ((ti & 1) ? 0 : 1));
    res[1] = acc;
    res[2] = 1;
  }
  __syncthreads();
}

// Radix-4 selection over 16-bit keys spread across the block, without atomics: each thread
// counts its keys per 4-bit digit in four 64-bit words (16-bit fields, digit d in word d/4,
// field d%4), warps add the words with shuffles, and warp 0 sums the 32 warps' counts.
struct Digits4 {
  unsigned long long c0 = 0, c1 = 0, c2 = 0, c3 = 0;
  __device__ __forceinline__ void add(uint32_t d) {
    const unsigned long long inc = 1ull << (16 * (d & 3u));
    if (d < 4u) c0 += inc;
    else if (d < 8u) c1 += inc;
    else if (d < 12u) c2 += inc;
    else c3 += inc;
  }
};

// Block part of one pass: returns the digit holding the target-th largest counted key and
// updates target (its rank within the digit) and above (counted keys in higher digits).
__device__ uint32_t radix4_reduce(Digits4 c, uint32_t& target, uint32_t& above,
                                  uint32_t (*wcnt)[16], uint32_t* res) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c.c0 += __shfl_xor_sync(0xffffffffu, c.c0, o);
    c.c1 += __shfl_xor_sync(0xffffffffu, c.c1, o);
    c.c2 += __shfl_xor_sync(0xffffffffu, c.c2, o);
    c.c3 += __shfl_xor_sync(0xffffffffu, c.c3, o);
  }
  if (lane < 16) {
    const unsigned long long wsel = lane < 4 ? c.c0 : lane < 8 ? c.c1 : lane < 12 ? c.c2 : c.c3;
    wcnt[warp][lane] = uint32_t((wsel >> (16 * (lane & 3))) & 0xFFFFull);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t t = 0;
    if (lane < 16) {
#pragma unroll 8
      for (int w = 0; w < TK_WARPS; w++) t += wcnt[w][lane];
    }
    uint32_t suf = t;                     // keys in digits >= lane (lanes lane .. 15)
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 16) suf += y;
    }
    const uint32_t above_d = suf - t;
    const bool hit = lane < 16 && above_d < target && target <= suf;
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    const int d = m ? __ffs(m) - 1 : 0;
    const uint32_t ad = __shfl_sync(0xffffffffu, above_d, d);
    if (lane == 0) { res[0] = uint32_t(d); res[1] = ad; }
  }
  __syncthreads();
  const uint32_t d = res[0], ad = res[1];
  __syncthreads();
  target -= ad;
  above += ad;
  return d;
}

// The 16 order-preserving keys of group g (entries 16g .. 16g+15 of the row), packed in pairs.
__device__ __forceinline__ void load_group(const uint16_t* sr, bool al, int g, int nvis,
                                           uint32_t (&kk)[8]) {
  if (al && GM_G * g + GM_G <= nvis) {
    const uint4* v = reinterpret_cast<const uint4*>(sr + GM_G * g);
    const uint4 a = __ldg(v), b = __ldg(v + 1);
    kk[0] = ordered_key_bf16x2(a.x); kk[1] = ordered_key_bf16x2(a.y);
    kk[2] = ordered_key_bf16x2(a.z); kk[3] = ordered_key_bf16x2(a.w);
    kk[4] = ordered_key_bf16x2(b.x); kk[5] = ordered_key_bf16x2(b.y);
    kk[6] = ordered_key_bf16x2(b.z); kk[7] = ordered_key_bf16x2(b.w);
  } else {
    // unaligned row or the row's last, partial group: invisible entries get key 0
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int e = GM_G * g + 2 * i;
      const uint32_t lo = e < nvis ? ordered_key_bf16(sr[e]) : 0u;
      const uint32_t hi = e + 1 < nvis ? ordered_key_bf16(sr[e + 1]) : 0u;
      kk[i] = lo | (hi << 16);
    }
  }
}

__device__ __forceinline__ uint32_t key_of(const uint32_t (&kk)[8], int i) {
  return (kk[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu;
}

// gmax rows have a stride of NGP = round_up(ceil(Nc / 16), 16) groups, so the 16 maxima of a
// thread never straddle a row.
__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_gm_kernel(const __nv_bfloat16* __restrict__ scores, const uint16_t* __restrict__ gmax,
                   const uint16_t* __restrict__ g2nd, const uint8_t* __restrict__ garg,
                   int Nc, int NGP, const int32_t* __restrict__ q_pos, int m, int k,
                   int32_t* __restrict__ idx, int32_t* status, int prewait) {
  extern __shared__ __align__(16) uint8_t tk_smem[];
  GmShared& S = *reinterpret_cast<GmShared*>(tk_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row = blockIdx.x;
  if (!prewait) pdl_enter();
  const int pos = q_pos[row];
  const int nvis = pos < 0 ? 0 : min(Nc, (pos + 1) / m);
  const int ngv = (nvis + GM_G - 1) / GM_G;              // groups with a visible entry
  if (prewait) pdl_enter();
  int32_t* out = idx + row * k;
  if (nvis <= k) {
    for (int j = tid; j < k; j += TK_THREADS) out[j] = j < nvis ? j : -1;
    return;
  }
  const uint16_t* sr = reinterpret_cast<const uint16_t*>(scores) + row * (long long)Nc;
  const bool al = (reinterpret_cast<uintptr_t>(sr) & 15) == 0;

  // ---- this thread's 16 group summaries (groups 16t .. 16t+15) in shared memory: maxima
  // (groups past the visible ones read as 0), second maxima, positions of the maxima
  const int g0 = GM_GPT * tid;
  uint32_t gmr[GM_GPT / 2];
  {
    const uint4* v = reinterpret_cast<const uint4*>(gmax + row * (long long)NGP + g0);
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (g0 < ngv) {
      a = __ldg(v);
      b = __ldg(v + 1);
      const long long o = row * (long long)NGP + g0;
      cp_async16(&S.g2s[0][tid], g2nd + o);
      cp_async16(&S.g2s[1][tid], g2nd + o + 8);
      cp_async16(&S.gas[tid], garg + o);
    }
    cp_async_commit();
    gmr[0] = a.x; gmr[1] = a.y; gmr[2] = a.z; gmr[3] = a.w;
    gmr[4] = b.x; gmr[5] = b.y; gmr[6] = b.z; gmr[7] = b.w;
#pragma unroll
    for (int i = 0; i < GM_GPT; i++)
      if (g0 + i >= ngv) gmr[i >> 1] &= (i & 1) ? 0x0000FFFFu : 0xFFFF0000u;
    S.gms[0][tid] = make_uint4(gmr[0], gmr[1], gmr[2], gmr[3]);
    S.gms[1][tid] = make_uint4(gmr[4], gmr[5], gmr[6], gmr[7]);
  }
  auto gm_of = [&](int i) { return (gmr[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu; };
  // maximum and position of the maximum of group 16t+i, i dynamic
  auto gm_sh = [&](int i) {
    return uint32_t(reinterpret_cast<const uint16_t*>(&S.gms[i >> 3][tid])[i & 7]);
  };
  auto arg_sh = [&](int i) {
    return uint32_t(reinterpret_cast<const uint8_t*>(&S.gas[tid])[i]) & 15u;
  };
  static_assert(GM_WWORDS == 4 * TK_THREADS, "one uint4 of the candidate histogram per thread");
  reinterpret_cast<uint4*>(S.wc)[tid] = make_uint4(0, 0, 0, 0);
  reinterpret_cast<uint4*>(S.wh)[tid] = make_uint4(0, 0, 0, 0);
  if (tid == 0) { S.ncand = 0u; S.npool = 0u; }
  // block: number of maxima and the largest (the row's largest visible key)
  uint32_t nz = 0, tmax = 0;
#pragma unroll
  for (int i = 0; i < GM_GPT; i++) { nz += gm_of(i) != 0u; tmax = max(tmax, gm_of(i)); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nz += __shfl_xor_sync(0xffffffffu, nz, o);
    tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
  }
  if (lane == 0) { S.red[0][warp] = nz; S.red[1][warp] = tmax; }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = S.red[0][lane], m2 = S.red[1][lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      m2 = max(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    }
    if (lane == 0) { S.res[5] = a; S.res[6] = m2; }
  }
  __syncthreads();
  const uint32_t Mx = S.res[6];
  // histogram window [wb, Mx] of 8192 digits under the largest key
  const uint32_t wb = Mx >= 8190u ? ((Mx - 8190u) & ~1u) : 0u;

  // ---- L: a lower bound of the row's k-th largest key.  The k-th largest group maximum is
  // one (the maxima are keys of k distinct groups); it is estimated from one maximum per
  // thread (a 1/16 sample), taken a little low, and checked when the candidates are counted:
  // if fewer than k keys reach it, the exact k-th largest maximum is selected instead.
  uint32_t L = 0u;
  bool need_exact = false;
  if (S.res[5] >= (uint32_t)k) {
    const uint32_t ns = (uint32_t)min(TK_THREADS, (ngv + GM_GPT - 1) / GM_GPT);   // samples
    const uint32_t want = (uint32_t)(((unsigned long long)k * ns * 3) / (2ull * (uint32_t)ngv)) + 8u;
    if (want < ns) {
      const uint32_t sv = gm_of(0);             // group 16t: thread t's sample (0: none)
      if (sv != 0u && sv >= wb) atomicAdd(&S.wh[(sv - wb) >> 1], 1u << (((sv - wb) & 1) << 4));
      __syncthreads();
      if (warp == 0) warp_suffix(S.wh, int((Mx - wb) >> 1), 0, want, S.res);
      __syncthreads();
      if (S.res[2]) L = S.res[0] + wb;
    }
    need_exact = L == 0u;
  }

  uint32_t qm = 0, dm = 0;          // bit i: group 16t+i holds one candidate / two or more
  uint32_t ndm = 0, pbase = 0;
  uint32_t c_own = 0;               // this thread's candidate keys
  bool inwin = false;               // every candidate key lies in the window
  for (int pass = 0; pass < 2; pass++) {
    if (need_exact) {
      // the k-th largest of all maxima (radix-4, no atomics)
      uint32_t target = (uint32_t)k, ab = 0u, pmask = 0u;
      L = 0u;
#pragma unroll 1
      for (int shift = 12; shift >= 0; shift -= 4) {
        Digits4 c;
#pragma unroll
        for (int i = 0; i < GM_GPT; i++) {
          const uint32_t v = gm_sh(i);
          if (v != 0u && (v & pmask) == L) c.add((v >> shift) & 15u);
        }
        L |= radix4_reduce(c, target, ab, S.wcnt, S.res) << shift;
        pmask |= 15u << shift;
      }
    }
    // ---- candidates: the visible keys >= L.  Thread t owns groups 16t .. 16t+15, in index
    // order.  A group with one candidate gives it (key, position) from the summary; the scores
    // of a group with more are copied into a pool slot (all copies in flight together) and its
    // candidates listed there.  Every candidate key goes into the window histogram, and the
    // block counts them.
    const uint32_t L1 = max(L, 1u);   // key 0 marks an invisible entry
    inwin = L >= wb;
    cp_async_wait<0>();
    {
      const uint4 m0 = S.gms[0][tid], m1 = S.gms[1][tid], s0 = S.g2s[0][tid], s1 = S.g2s[1][tid];
      const uint32_t mw[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
      const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      uint32_t qa = 0u, sa = 0u;
#pragma unroll
      for (int w = 0; w < 8; w++) {
        qa |= (uint32_t((mw[w] & 0xFFFFu) >= L1) | (uint32_t((mw[w] >> 16) >= L1) << 1)) << (2 * w);
        sa |= (uint32_t((sw[w] & 0xFFFFu) >= L) | (uint32_t((sw[w] >> 16) >= L) << 1)) << (2 * w);
      }
      dm = qa & sa;
      qm = qa & ~sa;
    }
    uint32_t c = __popc(qm);
    if (inwin) {
      for (uint32_t mm = qm; mm; mm &= mm - 1u) {
        const uint32_t d = gm_sh(__ffs(mm) - 1) - wb;
        atomicAdd(&S.wc[d >> 1], 1u << ((d & 1) << 4));
      }
    }
    ndm = __popc(dm);
    pbase = ndm ? atomicAdd(&S.npool, ndm) : 0u;
    if (ndm && pbase + ndm <= GM_POOL) {
      uint32_t sl = pbase;
      for (uint32_t mm = dm; mm; mm &= mm - 1u, sl++) S.pgrp[sl] = uint16_t(g0 + __ffs(mm) - 1);
    }
    __syncthreads();
    // the pooled groups (two or more candidates) one per thread: all their score loads in
    // flight together, the keys >= L listed in the slot and counted in the window histogram
    if (S.npool <= (uint32_t)GM_POOL && tid < (int)S.npool) {
      const int sl = tid;
      const int e0 = GM_G * int(S.pgrp[sl]);
      uint32_t kw[8];
      if (al && e0 + GM_G <= nvis) {
        const uint4 a = *reinterpret_cast<const uint4*>(sr + e0);
        const uint4 b2 = *reinterpret_cast<const uint4*>(sr + e0 + 8);
        kw[0] = a.x; kw[1] = a.y; kw[2] = a.z; kw[3] = a.w;
        kw[4] = b2.x; kw[5] = b2.y; kw[6] = b2.z; kw[7] = b2.w;
      } else {
#pragma unroll
        for (int w = 0; w < 8; w++)
          kw[w] = uint32_t(sr[min(e0 + 2 * w, nvis - 1)]) |
                  (uint32_t(sr[min(e0 + 2 * w + 1, nvis - 1)]) << 16);
      }
      const int nv = nvis - e0;
      uint32_t msk = 0u;
#pragma unroll
      for (int w = 0; w < 8; w++) {
        kw[w] = ordered_key_bf16x2(kw[w]);
        msk |= (uint32_t((kw[w] & 0xFFFFu) >= L1) | (uint32_t((kw[w] >> 16) >= L1) << 1)) << (2 * w);
      }
      if (nv < GM_G) msk &= (1u << nv) - 1u;
      uint32_t n = 0;
#pragma unroll
      for (int j = 0; j < GM_G; j++) {
        if (!((msk >> j) & 1u)) continue;
        const uint32_t key = (kw[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu;
        S.pent[sl][n++] = (key << 4) | uint32_t(j);
        if (inwin) atomicAdd(&S.wc[(key - wb) >> 1], 1u << (((key - wb) & 1) << 4));
      }
      S.pcnt[sl] = n;
    }
    __syncthreads();
    if (ndm && pbase + ndm <= GM_POOL)
      for (uint32_t sl = pbase; sl < pbase + ndm; sl++) c += S.pcnt[sl];
    c_own = c;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0 && c) atomicAdd(&S.ncand, c);
    __syncthreads();
    if (S.ncand >= (uint32_t)k) break;
    // the estimate was too high (an exact L always has k candidates): start over from it
    __syncthreads();
    reinterpret_cast<uint4*>(S.wc)[tid] = make_uint4(0, 0, 0, 0);
    if (tid == 0) { S.ncand = 0u; S.npool = 0u; }
    need_exact = true;
  }

  uint32_t T = 0u, above = 0u;
  // u16 digit counts cannot overflow while the row has fewer than 2^16 candidates
  if (inwin && S.ncand < 65536u && S.npool <= (uint32_t)GM_POOL) {
    // the k-th largest candidate key: all candidate keys lie in [L, Mx], at most 8192 digits,
    // searched by the whole block at once
    block_window_select(S.wc, int((Mx - wb) >> 1), int((L - wb) >> 1), (uint32_t)k, S.scan_tmp,
                        S.res);
    if (S.res[2] && S.ncand <= (uint32_t)GM_FLAT) {
      T = S.res[0] + wb;
      above = S.res[1];
      const uint32_t krem = (uint32_t)k - above;
      // ---- emission from one flat candidate list in index order: every thread writes its
      // candidates at its offset, then takes a contiguous run of at most ceil(ncand / 1024)
      // list entries, so no warp serialises over its lanes' differing candidate counts
      const uint32_t nc = S.ncand;
      uint32_t ntot;
      uint32_t o = block_scan_total(c_own, S.scan_tmp, ntot);
      {
        uint32_t sl = pbase;
        for (uint32_t mm = qm | dm; mm; mm &= mm - 1u) {
          const int i = __ffs(mm) - 1, e0 = GM_G * (GM_GPT * tid + i);
          if ((qm >> i) & 1u) {
            S.fkey[o] = uint16_t(gm_sh(i));
            S.fent[o++] = uint32_t(e0) + arg_sh(i);
          } else {
            const uint32_t n = S.pcnt[sl++];
            for (uint32_t e = 0; e < n; e++) {
              const uint32_t v = S.pent[sl - 1][e];
              S.fkey[o] = uint16_t(v >> 4);
              S.fent[o++] = uint32_t(e0) + (v & 15u);
            }
          }
        }
      }
      __syncthreads();
      const uint32_t per = (nc + TK_THREADS - 1) / TK_THREADS;
      const uint32_t j0 = min(nc, per * tid), j1 = min(nc, j0 + per);
      uint32_t gt = 0, eq = 0;
      for (uint32_t j = j0; j < j1; j++) {
        const uint32_t key = S.fkey[j];
        gt += key > T;
        eq += key == T;
      }
      unsigned long long tot64;
      const unsigned long long ex =
          block_scan64((static_cast<unsigned long long>(eq) << 32) | gt, S.tmp64, tot64);
      uint32_t e_before = uint32_t(ex >> 32);
      uint32_t slot = uint32_t(ex) + min(e_before, krem);
      for (uint32_t j = j0; j < j1; j++) {
        const uint32_t key = S.fkey[j];
        bool sel = key > T;
        if (!sel && key == T) { sel = e_before < krem; e_before++; }
        if (sel) {
          if (slot < (uint32_t)k) S.wh[slot] = S.fent[j];
          else report(status, HCL_ERR_DEVICE_FAULT);
          slot++;
        }
      }
      __syncthreads();
      for (int j = tid; j < k; j += TK_THREADS) out[j] = int32_t(S.wh[j]);
      return;
    }
    if (S.res[2]) {
      T = S.res[0] + wb;
      above = S.res[1];
      const uint32_t krem = (uint32_t)k - above;
      // ---- emission in index order: one packed (ties, above) scan over the threads
      uint32_t gt = 0, eq = 0;
      for (uint32_t mm = qm; mm; mm &= mm - 1u) {
        const uint32_t key = gm_sh(__ffs(mm) - 1);
        gt += key > T;
        eq += key == T;
      }
      for (uint32_t sl = pbase; sl < pbase + ndm; sl++) {
        const uint32_t n = S.pcnt[sl];
        for (uint32_t e = 0; e < n; e++) {
          const uint32_t key = S.pent[sl][e] >> 4;
          gt += key > T;
          eq += key == T;
        }
      }
      unsigned long long tot64;
      const unsigned long long ex =
          block_scan64((static_cast<unsigned long long>(eq) << 32) | gt, S.tmp64, tot64);
      if (gt | eq) {
        uint32_t e_before = uint32_t(ex >> 32);
        uint32_t slot = uint32_t(ex) + min(e_before, krem);
        auto place = [&](uint32_t v, int e0) {
          const uint32_t key = v >> 4;
          bool sel = key > T;
          if (!sel && key == T) { sel = e_before < krem; e_before++; }
          if (sel) {
            if (slot < (uint32_t)k) S.wh[slot] = uint32_t(e0 + int(v & 15u));
            else report(status, HCL_ERR_DEVICE_FAULT);
            slot++;
          }
        };
        uint32_t sl = pbase;
        for (uint32_t mm = qm | dm; mm; mm &= mm - 1u) {
          const int i = __ffs(mm) - 1, e0 = GM_G * (GM_GPT * tid + i);
          if ((qm >> i) & 1u) {
            place((gm_sh(i) << 4) | arg_sh(i), e0);
          } else {
            const uint32_t n = S.pcnt[sl];
            for (uint32_t e = 0; e < n; e++) place(S.pent[sl][e], e0);
            sl++;
          }
        }
      }
      // the k positions are filled (k < visible entries): one coalesced write of the list
      __syncthreads();
      for (int j = tid; j < k; j += TK_THREADS) out[j] = int32_t(S.wh[j]);
      return;
    }
  }
  T = 0u;
  above = 0u;

  // ---- keys spread below the window or 2^16 candidates and more (heavy ties): select over the
  // candidate groups, listed in index order, reloading their keys in every pass
  uint32_t ngc;
  {
    uint32_t nq = 0;
#pragma unroll
    for (int i = 0; i < GM_GPT; i++) nq += (gm_sh(i) != 0u && gm_sh(i) >= L);
    uint32_t o = block_scan_total(nq, S.scan_tmp, ngc);
#pragma unroll
    for (int i = 0; i < GM_GPT; i++)
      if (gm_sh(i) != 0u && gm_sh(i) >= L) S.list[o++] = uint16_t(GM_GPT * tid + i);
  }
  __syncthreads();
  {
    uint32_t target = (uint32_t)k, pmask = 0u;
#pragma unroll 1
    for (int shift = 12; shift >= 0; shift -= 4) {
      Digits4 c;
      for (int j = tid; j < int(ngc); j += TK_THREADS) {
        uint32_t kk[8];
        load_group(sr, al, S.list[j], nvis, kk);
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const uint32_t key = key_of(kk, i);
          if (key != 0u && key >= L && (key & pmask) == T) c.add((key >> shift) & 15u);
        }
      }
      T |= radix4_reduce(c, target, above, S.wcnt, S.res) << shift;
      pmask |= 15u << shift;
    }
  }
  const uint32_t krem = (uint32_t)k - above;
  unsigned long long base = 0;                            // (ties << 32 | above) so far
  for (int j0 = 0; j0 < int(ngc); j0 += TK_THREADS) {
    const int j = j0 + tid;
    uint32_t kk[8];
    uint32_t gt = 0, eq = 0;
    int g = -1;
    if (j < int(ngc)) {
      g = S.list[j];
      load_group(sr, al, g, nvis, kk);
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const uint32_t key = key_of(kk, i);
        gt += key > T;
        eq += key == T;
      }
    }
    unsigned long long tot64;
    const unsigned long long ex =
        base + block_scan64((static_cast<unsigned long long>(eq) << 32) | gt, S.tmp64, tot64);
    base += tot64;
    if (g >= 0 && (gt | eq) != 0u) {
      const uint32_t e_before = uint32_t(ex >> 32), g_before = uint32_t(ex);
      uint32_t slot = g_before + min(e_before, krem);
      uint32_t take = krem > e_before ? min(krem - e_before, eq) : 0u;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const uint32_t key = key_of(kk, i);
        bool sel = key > T;
        if (!sel && key == T && take > 0u) { sel = true; take--; }
        if (sel) {
          if (slot < (uint32_t)k) out[slot] = GM_G * g + i;
          else report(status, HCL_ERR_DEVICE_FAULT);
          slot++;
        }
      }
    }
  }
}

hcl_status_t run_topk_gm(const TopkArgs& a, const uint16_t* gmax, const uint16_t* g2nd,
                        const uint8_t* garg, cudaStream_t st) {
  auto kern = topk_gm_kernel;
  const int smem = (int)sizeof(GmShared);
  hcl_status_t ea = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, false);
  if (ea != HCL_OK) return ea;
  const long long rows = (long long)a.B * a.Tq;
  const int NGP = gmax_row_stride(a.Nc);
  return check_cuda(launch_pdl(kern, dim3((unsigned)rows), dim3(TK_THREADS), (size_t)smem, st, 1,
                               static_cast<const __nv_bfloat16*>(a.scores), gmax, g2nd, garg,
                               a.Nc, NGP,
                               a.q_pos, a.m, a.k, a.idx, a.status, a.prewait),
                    "topk launch");
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

// Co-resident cluster counts of one kernel per cluster size (index C), queried on first use
// and cached per (kernel, CUDA context): 0 unknown, -1 not schedulable.
struct ClusterCounts {
  int n[17] = {0};
  int& operator[](int C) { return n[C]; }
};
ClusterCounts& cluster_counts(const void* kern) {
  static std::mutex mu;
  static std::map<std::pair<const void*, unsigned long long>, ClusterCounts> cache;
  std::lock_guard<std::mutex> lock(mu);
  return cache[std::make_pair(kern, current_ctx_id())];   // map nodes never move
}

template <bool BF16>
hcl_status_t run_topk(const TopkArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.Tq;
  const int key_bytes = BF16 ? 2 : 4;
  const size_t cap_keys = (200 * 1024 - sizeof(TkShared)) / key_bytes;
  int C = choose_cluster(rows, a.Nc, cap_keys);
  auto kern = topk_kernel<BF16>;
  hcl_status_t e;
  for (;;) {
    const size_t chunk = (size_t)(a.Nc + C - 1) / C;
    const int chunk_cap = (int)std::min(chunk, cap_keys);
    const size_t smem = sizeof(TkShared) + ((size_t)chunk_cap * key_bytes + 15) / 16 * 16;
    e = set_kernel_attrs(reinterpret_cast<const void*>(kern), (int)smem, true);
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
  const size_t cap_keys = (226 * 1024 - sizeof(Tk16Shared) - 16) / key_bytes;
  auto kern = topk16_kernel<BF16>;
  // attributes are set once per context; the co-resident cluster count of each size is
  // queried once per context (0 unknown, -1 not schedulable)
  hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(kern), 226 * 1024, true);
  if (e != HCL_OK) return e;
  ClusterCounts& max_clusters = cluster_counts(reinterpret_cast<const void*>(kern));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(TK_THREADS);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  auto clusters_of = [&](int C) {
    if (max_clusters[C] == 0) {
      cudaLaunchConfig_t q = cfg;
      attr[0].val.clusterDim.x = C;
      q.gridDim = dim3((unsigned)C);
      q.dynamicSmemBytes = 226 * 1024;   // the largest the kernel may use
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, kern, &q);
      if (qe != cudaSuccess) cudaGetLastError();
      max_clusters[C] = (qe == cudaSuccess && n >= 1) ? n : -1;
    }
    return max_clusters[C];
  };
  // Cluster size: the slices must fit in shared memory; while slices stay long (>= 8192
  // keys) more blocks per row shorten every phase, as long as all rows' clusters are
  // co-resident (a second wave costs a whole kernel's latency).
  static const int sizes[] = {1, 2, 4, 6, 8, 10, 12, 14, 16};
  int best = 0;
  for (int C : sizes) {
    const size_t chunk = (size_t)(a.Nc + C - 1) / C;
    if (chunk > cap_keys) continue;
    const int nc = clusters_of(C);
    if (nc < 0) continue;
    if (best == 0) best = C;               // smallest that fits: the fallback
    if (rows > nc) break;                  // larger clusters would not fit in one wave
    best = C;
    if (rows * C >= (long long)num_sms() || chunk < 8192) break;
  }
  if (best == 0) return HCL_OK;            // too long for this kernel: radix-12 path
  const int C = best;
  const size_t chunk = (size_t)(a.Nc + C - 1) / C;
  attr[0].val.clusterDim.x = C;
  cfg.gridDim = dim3((unsigned)(rows * C));
  // (+16: bf16 keys may start up to 7 positions into their first vector)
  cfg.dynamicSmemBytes = sizeof(Tk16Shared) + (chunk * key_bytes + 15) / 16 * 16 + 16;
  *used = true;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, a.scores, a.Tq, a.Nc, a.q_pos, a.m, a.k,
                                       a.idx, a.status),
                    "topk launch");
}

// Register-resident bf16 selection for few long rows (decode): the cluster size is the
// largest (up to 16) whose clusters for all rows are co-resident, while slices stay long.
hcl_status_t run_topk_reg(const TopkArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  const long long rows = (long long)a.B * a.Tq;
  if (rows > num_sms()) return HCL_OK;          // many rows: the shared-memory kernels
  auto kern = topk_reg_kernel;
  const int smem = (int)sizeof(TrShared);
  hcl_status_t e = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, true);
  if (e != HCL_OK) return e;
  ClusterCounts& max_clusters = cluster_counts(reinterpret_cast<const void*>(kern));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(TK_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  auto clusters_of = [&](int C) {
    if (max_clusters[C] == 0) {
      attr[0].val.clusterDim.x = C;
      cudaLaunchConfig_t q = cfg;
      q.gridDim = dim3((unsigned)C);
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, kern, &q);
      if (qe != cudaSuccess) cudaGetLastError();
      max_clusters[C] = (qe == cudaSuccess && n >= 1) ? n : -1;
    }
    return max_clusters[C];
  };
  static const int sizes[] = {1, 2, 4, 6, 8, 10, 12, 14, 16};
  int best = 0;
  for (int C : sizes) {
    const long long chunk = ((long long)a.Nc + C - 1) / C;
    if (chunk > TR_MAX_KEYS) continue;
    const int nc = clusters_of(C);
    if (nc < 0 || rows > nc) {
      if (best) break;
      continue;
    }
    best = C;
    if (rows * C >= (long long)num_sms() || chunk < 8192) break;
  }
  if (best == 0) return HCL_OK;
  attr[0].val.clusterDim.x = best;
  cfg.gridDim = dim3((unsigned)(rows * best));
  *used = true;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(a.scores),
                                       a.Nc, a.q_pos, a.m, a.k, a.idx, a.status, a.prewait),
                    "topk launch");
}

bool topk_gmax_supported(int Nc) { return (Nc + GM_G - 1) / GM_G <= GM_MAX_GROUPS; }

hcl_status_t launch_topk_gmax(const TopkArgs& a, const uint16_t* gmax, const uint16_t* g2nd,
                              const uint8_t* garg, cudaStream_t st) {
  if ((long long)a.B * a.Tq == 0 || a.k == 0) return HCL_OK;
  if (!topk_gmax_supported(a.Nc)) return fail(HCL_ERR_UNSUPPORTED, "group-maxima top-k: Nc too large");
  return run_topk_gm(a, gmax, g2nd, garg, st);
}

hcl_status_t launch_topk(const TopkArgs& a, void*, size_t, cudaStream_t st) {
  if ((long long)a.B * a.Tq == 0 || a.k == 0) return HCL_OK;
  bool used = false;
  hcl_status_t e = HCL_OK;
  if (a.score_fmt == HCL_BF16) {
    e = run_topk_reg(a, st, &used);
    if (e != HCL_OK || used) return e;
  }
  e = a.score_fmt == HCL_BF16 ? run_topk16<true>(a, st, &used)
                              : run_topk16<false>(a, st, &used);
  if (e != HCL_OK || used) return e;
  if (a.score_fmt == HCL_BF16) return run_topk<true>(a, st);
  return run_topk<false>(a, st);
}

}  // namespace hcl
