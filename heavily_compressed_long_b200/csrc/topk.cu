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
  uint32_t cnt[2];           // this block's (#greater, #equal)
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

template <bool BF16>
__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_kernel(const void* __restrict__ scores, int Tq, int Nc, const int32_t* __restrict__ q_pos,
                int m, int k, int32_t* __restrict__ idx, int chunk_cap,
                int32_t* status) {
  cg::cluster_group cluster = cg::this_cluster();
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
  const uint32_t T = prefix;

  // counts of keys greater than / equal to the threshold, per warp segment
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
  if (lane == 0) { S.wsum[0][warp] = g; S.wsum[1][warp] = e; }
  __syncthreads();
  if (tid == 0) {
    uint32_t tg = 0, te = 0;
    for (int w = 0; w < TK_WARPS; w++) { tg += S.wsum[0][w]; te += S.wsum[1][w]; }
    S.cnt[0] = tg;
    S.cnt[1] = te;
  }
  cluster.sync();
  uint32_t gt_before = 0, eq_before = 0;
  for (int r = 0; r < rank; r++) {
    const uint32_t* c = cluster.map_shared_rank(S.cnt, r);
    gt_before += c[0];
    eq_before += c[1];
  }
  const uint32_t eq_take = krem > eq_before ? min(krem - eq_before, S.cnt[1]) : 0u;
  uint32_t wg_before = 0, we_before = 0;
  for (int w = 0; w < warp; w++) { wg_before += S.wsum[0][w]; we_before += S.wsum[1][w]; }
  uint32_t pos_out = gt_before + min(eq_before, krem) + wg_before + min(we_before, eq_take);
  uint32_t eq_seen = we_before;
  for (int j0 = s0; j0 < s1; j0 += 32) {
    const int j = j0 + lane;
    uint32_t key = j < s1 ? key_at(j) : 0u;
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
  cluster.sync();  // no block leaves while another may still read its shared memory
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
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(TK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
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

hcl_status_t launch_topk(const TopkArgs& a, void*, size_t, cudaStream_t st) {
  if ((long long)a.B * a.Tq == 0 || a.k == 0) return HCL_OK;
  if (a.score_fmt == HCL_BF16) return run_topk<true>(a, st);
  return run_topk<false>(a, st);
}

}  // namespace hcl
