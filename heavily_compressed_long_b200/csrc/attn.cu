// attn.cu -- attention over compressed entries plus the raw sliding window.
//
// [Tripbot §3.1 step 2] CSA attends over the top-k selected compressed entries;
// [Tripbot §3.2; CSDN §1.2] HCA attends densely over every compressed entry;
// [Tripbot §3.3] both add a branch over the most recent W raw tokens and may add a learnable
// sink that lets the weights sum to less than one.  Per query head h, over the row list J:
//     z_j = scale * q_h . kv_j,   o_h = sum_j softmax(z)_j kv_j,   lse_h = log sum_j e^{z_j}
// Each compressed or raw row serves as both key and value of the one shared KV head.
//
// Design (B200): one block per (sequence, query group, KV split).  A query group is G queries
// x H heads = up to 128 (query, head) rows, 16 per warp; all rows of a group share one KV row
// list (CSA: G = 1, the query's selected entries then its window; HCA: the G consecutive
// queries share the visible-entry prefix and the union of their windows, with per-row
// causal masks).  The list is processed in chunks of 64 rows, gathered with cp.async into a
// double-buffered, XOR-swizzled shared tile (split FP8 rows are staged raw and widened to
// bf16 in shared memory with their per-row scale); QK^T and PV run on tensor cores
// (mma.sync m16n8k16 bf16, fp32 accumulation) with an online softmax in registers.  With
// several KV splits each block writes a normalised partial (o, lse) to the caller's
// workspace and a merge kernel combines them by log-sum-exp.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace cg = cooperative_groups;

namespace hcl {
namespace {

constexpr int D = 128;
constexpr int KVB = 64;
constexpr int MAX_CLUSTER_ROWS = 16;   // largest cluster of splits merged through DSMEM
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnParams {
  const __nv_bfloat16* q;
  int B, Tq, H;
  hcl_kv_t comp;
  int n_comp, mh;
  const int32_t* idx;
  int k;
  hcl_kv_t raw;
  int W;
  const int32_t* q_pos;
  float scale_log2;
  const float* sink;
  const float* q_gamma;  // RMSNorm of every query head row (fp32 [d]), or null
  float q_eps;
  __nv_bfloat16* out;
  float* lse;
  float* ws_o;
  float* ws_lse;
  int G, n_groups, splits, cps, rows_pad;
  int cmerge;  // 1: the splits of a group form one cluster and merge through DSMEM
  int hsplit;  // blocks sharing one group's (query, head) rows (cluster merge only)
  int prewait; // 1: q, q_pos and the raw window store are not written by the previous kernel in
               // the stream, so they may be read before waiting for it (fused decode step only)
  int32_t* status;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// byte offset of 16-byte chunk `c` (0..15) of tile row `r` (256-byte rows, XOR swizzle)
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return uint32_t(r) * 256u + (uint32_t(c ^ (r & 7)) << 4);
}

// Two E4M3 codes -> two bf16 values times `scale` (exact widening, one rounding).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t codes, float scale) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
  __half2 hv = *reinterpret_cast<__half2*>(&h2);
  float2 f = __half22float2(hv);
  return pack_bf16(f.x * scale, f.y * scale);
}

struct RowSrc {
  long long slot;  // row slot in the store (-1: invalid)
  int from_raw;
};

template <int KVFMT, int MODE, int NW>
__global__ void __launch_bounds__(NW * 32)
    attn_kernel(AttnParams p) {
  // Wait for the previous kernel before the first global read -- or, when q and q_pos are
  // known not to come from it, only before reading the selected indices.
  if (!p.prewait) pdl_enter();
  constexpr int NT = NW * 32;
  extern __shared__ __align__(128) uint8_t at_smem[];
  uint8_t* tiles = at_smem;                              // [2][64][256 B] bf16
  uint8_t* stage = at_smem + 2 * KVB * 256;              // fp8: [2][64][64 B] codes
  float* sscale = reinterpret_cast<float*>(stage + 2 * KVB * 64);  // fp8: [2][64]
  RowSrc* rsrc = reinterpret_cast<RowSrc*>(sscale + 2 * KVB);      // [2][64]
  // cluster merge: the partials of the rows this block merges, pushed here by every split:
  // recv[slot][split][D] and recv_lse[slot][split], slot = row / splits
  float* recv = reinterpret_cast<float*>(rsrc + 2 * KVB);
  const int rpo = (NW * 16 + p.splits - 1) / p.splits;            // rows merged per block
  float* recv_lse = recv + (size_t)rpo * p.splits * D;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int bid = blockIdx.x;
  const int split = bid % p.splits;
  bid /= p.splits;
  const int hpart = bid % p.hsplit;   // which slice of the group's (query, head) rows
  bid /= p.hsplit;
  const int row_base = hpart * NW * 16;
  const int grp = bid % p.n_groups;
  const int b = bid / p.n_groups;
  const int t0 = grp * p.G;
  const int gq = min(p.G, p.Tq - t0);  // queries in this group

  // positions of the group's queries
  int pmin = 0x7fffffff, pmax = -1;
  for (int q = 0; q < gq; q++) {
    int pp = p.q_pos[(size_t)b * p.Tq + t0 + q];
    pmin = min(pmin, pp);
    pmax = max(pmax, pp);
  }
  // row list: [list_a entries] ++ [raw tokens raw_lo .. raw_lo + n_raw - 1]
  int n_a, raw_lo, n_raw;
  if (MODE == 0) {
    n_a = p.k;
    raw_lo = pmax - p.W + 1;  // CSA: G == 1, window of the one query (may start < 0)
    n_raw = p.W;
  } else {
    n_a = pmax < 0 ? 0 : min(p.n_comp, (pmax + 1) / p.mh);
    raw_lo = pmin - p.W + 1;
    n_raw = p.W > 0 ? max(0, pmax - raw_lo + 1) : 0;
  }
  const int total = n_a + n_raw;
  const int n_chunks = (total + KVB - 1) / KVB;
  const int c_begin = split * p.cps;
  // the last split takes every remaining chunk (query groups whose positions are not
  // consecutive may have longer lists than the host planned for)
  const int c_end = split == p.splits - 1 ? n_chunks : min(n_chunks, c_begin + p.cps);

  // this thread's two rows (g, g+8 of the warp's 16) -> query, head, position, visibility
  const int g = lane >> 2, tq = lane & 3;
  int row_q[2], row_h[2], row_p[2], row_nv[2];
  bool row_ok[2];
#pragma unroll
  for (int i = 0; i < 2; i++) {
    const int r = row_base + warp * 16 + g + 8 * i;
    const int q = r / p.H;
    row_q[i] = q;
    row_h[i] = r % p.H;
    row_ok[i] = q < gq;
    row_p[i] = row_ok[i] ? p.q_pos[(size_t)b * p.Tq + t0 + q] : -1;
    row_nv[i] = row_p[i] < 0 ? 0 : min(p.n_comp, (row_p[i] + 1) / max(1, p.mh));
  }

  // Q fragments (A operand, 16 rows x 128 dims = 8 k-steps)
  uint32_t qa[8][4];
  {
    const __nv_bfloat16* qrow[2];
#pragma unroll
    for (int i = 0; i < 2; i++)
      qrow[i] = row_ok[i] ? p.q + (((size_t)b * p.Tq + t0 + row_q[i]) * p.H + row_h[i]) * D
                          : nullptr;
#pragma unroll
    for (int kk = 0; kk < 8; kk++) {
      const int c0 = kk * 16 + tq * 2;
      qa[kk][0] = qrow[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + c0) : 0u;
      qa[kk][1] = qrow[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + c0) : 0u;
      qa[kk][2] = qrow[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + c0 + 8) : 0u;
      qa[kk][3] = qrow[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + c0 + 8) : 0u;
    }
  }
  if (p.q_gamma != nullptr) {
    // RMSNorm of the two query rows [Tripbot §5], fp32, rounded back to the bf16 operand: the
    // four threads of a quad hold a row's 128 dims (fragment j: row j&1, dims c0 + 8*(j>>1))
    float ss[2] = {0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; kk++)
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float lo = __uint_as_float(qa[kk][j] << 16), hi = __uint_as_float(qa[kk][j] & 0xFFFF0000u);
        ss[j & 1] = fmaf(lo, lo, fmaf(hi, hi, ss[j & 1]));
      }
    float rn[2];
#pragma unroll
    for (int i = 0; i < 2; i++) {
      ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], 1);
      ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], 2);
      rn[i] = 1.f / sqrtf(ss[i] / float(D) + p.q_eps);
    }
#pragma unroll
    for (int kk = 0; kk < 8; kk++)
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int c = kk * 16 + tq * 2 + 8 * (j >> 1);
        const float lo = __uint_as_float(qa[kk][j] << 16), hi = __uint_as_float(qa[kk][j] & 0xFFFF0000u);
        qa[kk][j] = pack_bf16(lo * rn[j & 1] * __ldg(p.q_gamma + c),
                              hi * rn[j & 1] * __ldg(p.q_gamma + c + 1));
      }
  }

  // A CSA block whose rows are all window rows needs nothing from the previous kernel (the
  // top-k): with prewait it gathers its rows before waiting.
  const bool early = p.prewait && MODE == 0 && c_begin * KVB >= n_a;
  if (p.prewait && !early) pdl_enter();

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; n++) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

  // ---- gather of one chunk into buffer `buf` ----
  auto resolve_row = [&](int chunk, int buf, int j) {
    {
      const int e = chunk * KVB + j;
      RowSrc rs{-1, 0};
      if (e < n_a) {
        long long ent;
        if (MODE == 0) {
          ent = p.idx[((size_t)b * p.Tq + t0) * p.k + e];
          if (ent < -1 || ent >= p.n_comp) {
            report(p.status, HCL_ERR_DEVICE_FAULT);
            ent = -1;
          }
        } else {
          ent = e;
        }
        if (ent >= 0) rs.slot = (long long)b * p.comp.cap + (ent % p.comp.cap);
      } else if (e < total) {
        const long long u = (long long)raw_lo + (e - n_a);
        if (u >= 0) { rs.slot = (long long)b * p.raw.cap + (u % p.raw.cap); rs.from_raw = 1; }
      }
      rsrc[buf * KVB + j] = rs;
    }
  };
  auto resolve = [&](int chunk, int buf) {
    for (int j = tid; j < KVB; j += NT) resolve_row(chunk, buf, j);
  };
  auto issue = [&](int buf) {
    uint8_t* tile = tiles + buf * KVB * 256;
    if (KVFMT == HCL_BF16) {
      for (int u = tid; u < KVB * 16; u += NT) {
        const int r = u >> 4, c = u & 15;
        const RowSrc rs = rsrc[buf * KVB + r];
        uint8_t* dst = tile + tile_off(r, c);
        if (rs.slot >= 0) {
          const hcl_kv_t& st = rs.from_raw ? p.raw : p.comp;
          cp_async16(dst, static_cast<const uint8_t*>(st.data) + rs.slot * 256 + c * 16);
        } else {
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
      }
    } else {
      // rope half straight into tile columns 64..127; codes and scale into staging
      for (int u = tid; u < KVB * 13; u += NT) {
        const int r = u / 13, c = u % 13;
        const RowSrc rs = rsrc[buf * KVB + r];
        const hcl_kv_t& st = rs.from_raw ? p.raw : p.comp;
        if (c < 8) {
          uint8_t* dst = tile + tile_off(r, 8 + c);
          if (rs.slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.rope) + rs.slot * 128 + c * 16);
          else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        } else if (c < 12) {
          uint8_t* dst = stage + (buf * KVB + r) * 64 + (c - 8) * 16;
          if (rs.slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.data) + rs.slot * 64 + (c - 8) * 16);
          else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        } else {
          float* dst = sscale + buf * KVB + r;
          if (rs.slot >= 0)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                         "l"(st.scale + rs.slot)
                         : "memory");
          else *dst = 0.f;
        }
      }
    }
    cp_async_commit();
  };
  auto widen = [&](int buf) {  // FP8 staging -> bf16 tile columns 0..63
    uint8_t* tile = tiles + buf * KVB * 256;
    for (int u = tid; u < KVB * 8; u += NT) {
      const int r = u >> 3, c = u & 7;  // 8 codes -> one 16-byte bf16 chunk
      const uint2 codes = *reinterpret_cast<const uint2*>(stage + (buf * KVB + r) * 64 + c * 8);
      const float sc = sscale[buf * KVB + r];
      uint4 v;
      v.x = e4m3x2_to_bf16x2(uint16_t(codes.x & 0xffff), sc);
      v.y = e4m3x2_to_bf16x2(uint16_t(codes.x >> 16), sc);
      v.z = e4m3x2_to_bf16x2(uint16_t(codes.y & 0xffff), sc);
      v.w = e4m3x2_to_bf16x2(uint16_t(codes.y >> 16), sc);
      *reinterpret_cast<uint4*>(tile + tile_off(r, c)) = v;
    }
  };

  // Both buffers are filled up front (their index loads and row gathers overlap); afterwards
  // each buffer is refilled with the chunk two ahead as soon as it has been consumed.
  if (c_begin < c_end) {
    if (NT >= 2 * KVB) {
      // both chunks' index loads in flight together: threads [0, 64) and [64, 128)
      if (tid < 2 * KVB) {
        const int ch = c_begin + tid / KVB;
        if (ch < c_end) resolve_row(ch, tid / KVB, tid % KVB);
      }
    } else {
      resolve(c_begin, 0);
      if (c_begin + 1 < c_end) resolve(c_begin + 1, 1);
    }
    __syncthreads();
    issue(0);
    if (c_begin + 1 < c_end) issue(1);
  }
  if (early) pdl_enter();
  for (int c = c_begin; c < c_end; c++) {
    const int buf = (c - c_begin) & 1;
    if (c + 1 < c_end) cp_async_wait<1>();   // chunk c landed; chunk c+1 may be in flight
    else cp_async_wait<0>();
    __syncthreads();
    if (KVFMT == HCL_FP8SPLIT) {
      widen(buf);
      __syncthreads();
    }
    const uint32_t tbase = smem_u32(tiles + buf * KVB * 256);

    // S = Q K^T for this warp's 16 rows x 64 kv rows
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; n++) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int n = 0; n < 8; n++) {
#pragma unroll
      for (int kk = 0; kk < 8; kk += 2) {
        const int mi = lane >> 3, ri = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tbase + tile_off(n * 8 + ri, kk * 2 + mi), b0, b1, b2, b3);
        mma_bf16(s[n], qa[kk], b0, b1);
        mma_bf16(s[n], qa[kk + 1], b2, b3);
      }
    }
    // mask, scale (log2 domain), online softmax
    float cmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; n++) {
#pragma unroll
      for (int e2 = 0; e2 < 4; e2++) {
        const int i = e2 >> 1;
        const int j = n * 8 + tq * 2 + (e2 & 1);
        const RowSrc rs = rsrc[buf * KVB + j];
        const int e = c * KVB + j;
        bool vis = rs.slot >= 0 && row_ok[i];
        if (MODE == 1 && vis) {
          if (e < n_a) vis = e < row_nv[i];
          else {
            const int u = raw_lo + (e - n_a);
            vis = u <= row_p[i] && u > row_p[i] - p.W;
          }
        }
        const float z = vis ? s[n][e2] * p.scale_log2 : -INFINITY;
        s[n][e2] = z;
        cmax[i] = fmaxf(cmax[i], z);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; i++) {
      cmax[i] = fmaxf(cmax[i], __shfl_xor_sync(0xffffffffu, cmax[i], 1));
      cmax[i] = fmaxf(cmax[i], __shfl_xor_sync(0xffffffffu, cmax[i], 2));
    }
    float corr[2], muse[2];
#pragma unroll
    for (int i = 0; i < 2; i++) {
      const float mnew = fmaxf(mrow[i], cmax[i]);
      muse[i] = mnew == -INFINITY ? 0.f : mnew;
      corr[i] = exp2f(mrow[i] - muse[i]);
      mrow[i] = mnew;
    }
    float rsum[2] = {0.f, 0.f};
    uint32_t pa[4][4];
#pragma unroll
    for (int n = 0; n < 8; n++) {
      const float p0 = exp2f(s[n][0] - muse[0]), p1 = exp2f(s[n][1] - muse[0]);
      const float p2 = exp2f(s[n][2] - muse[1]), p3 = exp2f(s[n][3] - muse[1]);
      rsum[0] += p0 + p1;
      rsum[1] += p2 + p3;
      const int kk = n >> 1, hi = n & 1;
      pa[kk][hi * 2 + 0] = pack_bf16(p0, p1);
      pa[kk][hi * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int i = 0; i < 2; i++) lrow[i] = lrow[i] * corr[i] + rsum[i];
#pragma unroll
    for (int n = 0; n < 16; n++) {
      o[n][0] *= corr[0]; o[n][1] *= corr[0];
      o[n][2] *= corr[1]; o[n][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; kk++) {
#pragma unroll
      for (int n = 0; n < 16; n += 2) {
        const int mi = lane >> 3, ri = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(tbase + tile_off(kk * 16 + (mi & 1) * 8 + ri, n + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(o[n], pa[kk], b0, b1);
        mma_bf16(o[n + 1], pa[kk], b2, b3);
      }
    }
    __syncthreads();
    if (c + 2 < c_end) {   // this buffer is free: start the chunk two ahead
      resolve(c + 2, buf);
      __syncthreads();
      issue(buf);
    }
  }

  // row sums across the 4 threads of a row
#pragma unroll
  for (int i = 0; i < 2; i++) {
    lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 1);
    lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 2);
  }
  const size_t item = (size_t)blockIdx.x;
#pragma unroll
  for (int i = 0; i < 2; i++) {
    if (!row_ok[i]) continue;
    const int r = warp * 16 + g + 8 * i;
    float m2 = mrow[i], l2 = lrow[i], f = 1.f;
    if (p.splits == 1) {
      if (p.sink) {
        const float s2 = p.sink[row_h[i]] * LOG2E;
        const float mm = fmaxf(m2, s2);
        f = (l2 > 0.f) ? exp2f(m2 - mm) : 0.f;
        l2 = l2 * f + exp2f(s2 - mm);
        m2 = mm;
      }
      const float inv = l2 > 0.f ? f / l2 : 0.f;
      const size_t orow = ((size_t)b * p.Tq + t0 + row_q[i]) * p.H + row_h[i];
      __nv_bfloat16* dst = p.out + orow * D;
#pragma unroll
      for (int n = 0; n < 16; n++) {
        const int col = n * 8 + tq * 2;
        *reinterpret_cast<uint32_t*>(dst + col) = pack_bf16(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
      }
      if (p.lse && tq == 0) p.lse[orow] = l2 > 0.f ? (m2 + log2f(l2)) * LN2 : -INFINITY;
    } else {
      // normalised partial and its log2-domain LSE: pushed into the shared memory of the
      // block that merges row r (cluster merge: block r % splits, slot r / splits), or to
      // the caller's workspace (merge kernel)
      const float inv = l2 > 0.f ? 1.f / l2 : 0.f;
      const float ls = l2 > 0.f ? m2 + log2f(l2) : -INFINITY;
      float* dst;
      float* dst_lse;
      if (p.cmerge) {
        cg::cluster_group cluster = cg::this_cluster();
        const int owner = r % p.splits, slot = r / p.splits;
        dst = cluster.map_shared_rank(recv, owner) + ((size_t)slot * p.splits + split) * D;
        dst_lse = cluster.map_shared_rank(recv_lse, owner) + slot * p.splits + split;
      } else {
        dst = p.ws_o + (item * p.rows_pad + r) * D;
        dst_lse = p.ws_lse + item * p.rows_pad + r;
      }
      // 16-byte stores: the two threads of a column pair swap halves, and for column block n
      // the even (n even) or odd (n odd) thread of each pair writes four columns.  Both
      // threads of a pair hold the same row, so they skip rows together.
      const unsigned pm = 3u << (lane & ~1);
#pragma unroll
      for (int n = 0; n < 16; n++) {
        const float mx = o[n][2 * i] * inv, my = o[n][2 * i + 1] * inv;
        const float ox = __shfl_xor_sync(pm, mx, 1), oy = __shfl_xor_sync(pm, my, 1);
        if ((tq & 1) == (n & 1)) {
          const float4 v = (tq & 1) ? make_float4(ox, oy, mx, my) : make_float4(mx, my, ox, oy);
          *reinterpret_cast<float4*>(dst + n * 8 + (tq >> 1) * 4) = v;
        }
      }
      if (tq == 0) *dst_lse = ls;
    }
  }
  if (p.cmerge) {
    // The splits of this query group are the blocks of one cluster.  Every block has pushed
    // its partials to the merging blocks; after the barrier (which makes those remote stores
    // visible) block `split` merges rows split, split + S, ... by log-sum-exp from its own
    // shared memory.  No block reads another's shared memory afterwards, so none waits.
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int S = p.splits;
    const int rows_valid = gq * p.H;
    for (int slot = warp; slot < rpo; slot += NW) {
      const int r = split + S * slot;   // row within the block's slice
      const int rg = row_base + r;      // row within the group
      if (r >= NW * 16 || rg >= rows_valid) break;
      const float ls = lane < S ? recv_lse[slot * S + lane] : -INFINITY;
      float M = ls;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
      const int h = rg % p.H;
      float s2 = -INFINITY;
      if (p.sink) {
        s2 = p.sink[h] * LOG2E;
        M = fmaxf(M, s2);
      }
      const float wl = (ls == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ls - M);
      float den = wl;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o2);
      if (p.sink && M > -INFINITY) den += exp2f(s2 - M);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4* part = reinterpret_cast<const float4*>(recv + (size_t)slot * S * D);
#pragma unroll
      for (int s = 0; s < MAX_CLUSTER_ROWS; s++) {
        const float wgt = __shfl_sync(0xffffffffu, wl, s);
        if (s < S && wgt != 0.f) {
          const float4 v = part[s * (D / 4) + lane];
          acc.x += wgt * v.x; acc.y += wgt * v.y; acc.z += wgt * v.z; acc.w += wgt * v.w;
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      const size_t orow = ((size_t)b * p.Tq + t0 + rg / p.H) * p.H + h;
      reinterpret_cast<uint2*>(p.out + orow * D)[lane] =
          make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
      if (p.lse && lane == 0) p.lse[orow] = den > 0.f ? (M + log2f(den)) * LN2 : -INFINITY;
    }
  }
}

// Combine the KV splits of every (query, head) row by log-sum-exp (log2 domain partials).
__global__ void attn_merge_kernel(AttnParams p) {
  pdl_enter();
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)p.B * p.Tq * p.H;
  if (gw >= nrows) return;
  const int h = int(gw % p.H);
  const long long bt = gw / p.H;
  const int t = int(bt % p.Tq);
  const int b = int(bt / p.Tq);
  const int grp = t / p.G;
  const int r = (t - grp * p.G) * p.H + h;
  const size_t item0 = ((size_t)b * p.n_groups + grp) * p.splits;
  // split LSEs: one per lane (32 at a time), reduced with shuffles -- no dependent loads
  float M = -INFINITY;
  for (int s0 = 0; s0 < p.splits; s0 += 32) {
    const int s = s0 + lane;
    const float ls = s < p.splits ? p.ws_lse[(item0 + s) * p.rows_pad + r] : -INFINITY;
    M = fmaxf(M, ls);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float s2 = -INFINITY;
  if (p.sink) {
    s2 = p.sink[h] * LOG2E;
    M = fmaxf(M, s2);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M > -INFINITY) {
    for (int s0 = 0; s0 < p.splits; s0 += 32) {
      const int s = s0 + lane;
      const float ls = s < p.splits ? p.ws_lse[(item0 + s) * p.rows_pad + r] : -INFINITY;
      const float wl = ls == -INFINITY ? 0.f : exp2f(ls - M);    // this lane's split weight
      float dsum = wl;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
      den += dsum;
      const int ns = min(32, p.splits - s0);
#pragma unroll 4
      for (int j = 0; j < ns; j++) {
        const float wgt = __shfl_sync(0xffffffffu, wl, j);
        if (wgt == 0.f) continue;
        const float4 v = __ldg(reinterpret_cast<const float4*>(
                                   p.ws_o + ((item0 + s0 + j) * p.rows_pad + r) * D) + lane);
        acc.x += wgt * v.x; acc.y += wgt * v.y; acc.z += wgt * v.z; acc.w += wgt * v.w;
      }
    }
    if (p.sink) den += exp2f(s2 - M);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = p.out + gw * D + lane * 4;
  reinterpret_cast<uint2*>(dst)[0] = make_uint2(pack_bf16(acc.x * inv, acc.y * inv),
                                                pack_bf16(acc.z * inv, acc.w * inv));
  if (p.lse && lane == 0) p.lse[gw] = den > 0.f ? (M + log2f(den)) * LN2 : -INFINITY;
}

// ---------------------------------------------------------------------------------------
// CSA decode on tcgen05 tensor cores (one query per sequence, up to 128 heads).
// Block = (sequence, KV split of up to TC_MAXC chunks of 64 rows); thread t <-> head t <->
// TMEM lane t.  Shared memory holds Q (128 heads x 128 dims), the gathered KV rows of the
// split and P, all as 128-byte SW128 rows (dims 0-63 and 64-127 in two halves).  The same
// KV tile is the K-major B operand of S = Q K^T (N = 64 rows per chunk) and the MN-major B
// operand of O = P V (K = rows, N = 128 dims), so V needs no transpose.  S (64 fp32 columns
// per chunk) and O (128 columns) live in TMEM.  The softmax is two-pass over the split's
// chunks: row maximum, then exp2 / row sum / P in bf16.  Splits merge as in attn_kernel.
constexpr int TC_MAXC = 4;          // chunks per block with a single split
constexpr int TC_MAXC_MERGE = 2;    // chunks per block when splits merge in a cluster (its KV
                                    // and P tiles, 64 KB, then stage the 128 x 512 B partials)
constexpr int TC_ROWS = 128;        // head rows per block = UMMA M = TMEM lanes
constexpr int TC_THREADS = 256;     // two threads per row (column halves)

struct TcOff {
  uint32_t q, kv, pm, stg, scl, rs, bar, vis, xch, recv, lse, total;
};
__host__ __device__ inline TcOff tc_offsets(int cps, int splits) {
  TcOff o;
  o.q = 0;                                   // 2 halves x 128 rows x 128 B
  o.kv = 32768;                              // cps x (2 halves x 64 rows x 128 B)
  o.pm = o.kv + cps * 16384;                 // cps x (128 rows x 128 B)
  o.stg = o.pm + cps * 16384;                // fp8: cps x 64 rows x 64 B codes
  o.scl = o.stg + cps * 4096;                // fp8: cps x 64 scales
  o.rs = o.scl + cps * 256;                  // cps x 64 RowSrc
  o.bar = o.rs + cps * 64 * (uint32_t)sizeof(RowSrc);   // 2 mbarriers + TMEM base
  o.vis = o.bar + 32;                        // row-visibility bits, 64 per chunk
  o.xch = (o.vis + 8 * cps + 15) & ~15u;     // partial maxima / sums of the two column halves
  o.recv = o.xch + 2 * TC_THREADS * 4;       // cluster merge: splits x rpo x D fp16 partials
  const int rpo = splits > 1 ? (TC_ROWS + splits - 1) / splits : 0;
  o.lse = o.recv + (uint32_t)(rpo * splits * D * 2);
  o.total = o.lse + (uint32_t)(((rpo + 3) & ~3) * splits * 4);   // [splits][rpo rounded to 4]
  return o;
}

template <int KVFMT>
__global__ void __launch_bounds__(TC_THREADS, 1) attn_tc_kernel(AttnParams p) {
  const bool early_ok = p.prewait != 0;
  extern __shared__ __align__(1024) uint8_t tc_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = tid & (TC_ROWS - 1);   // head row = TMEM lane (warps w and w+4 share a quadrant)
  const int hc = tid / TC_ROWS;          // which half of the columns this thread handles
  const int split = blockIdx.x % p.splits;
  const int b = blockIdx.x / p.splits;
  const TcOff off = tc_offsets(p.cps, p.splits);
  uint8_t* sQ = sm + off.q;
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + off.bar);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + off.bar + 16);
  uint32_t* visw = reinterpret_cast<uint32_t*>(sm + off.vis);
  float* xch = reinterpret_cast<float*>(sm + off.xch);   // [2][TC_THREADS]: partial max, sum
  __half* recv_h = reinterpret_cast<__half*>(sm + off.recv);   // [splits][rpo][D] fp16 partials
  float* recv_lse = reinterpret_cast<float*>(sm + off.lse);

  // row list of this split: k selected entries, then the W window rows
  const int n_a = p.k, total = p.k + p.W;
  const int n_chunks = (total + KVB - 1) / KVB;
  const int c_begin = split * p.cps;
  const int c_end = split == p.splits - 1 ? n_chunks : min(n_chunks, c_begin + p.cps);
  const int nch = max(0, min(TC_MAXC, c_end - c_begin));
  const uint32_t ocol = uint32_t(p.cps * 64);              // O columns after the S columns
  const uint32_t ncols = ocol + D <= 256 ? 256u : 512u;

  // splits > 1: the partials of this block's head rows arrive by bulk copies, counted on
  // bar_r: S copies of rows_o rows of 512 bytes (rows_o = this block's rows, see the push)
  uint64_t* bar_r = bar_s + 3;
  const int rpo = p.splits > 1 ? (TC_ROWS + p.splits - 1) / p.splits : 1;
  const int rpo4 = (rpo + 3) & ~3;                          // log-sum-exps per split, 16-byte rows
  auto rows_of = [&](int o) { return max(0, min(rpo, p.H - o * rpo)); };
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    if (p.splits > 1) {
      mbar_init(bar_r, 1);
      mbar_arrive_expect_tx(bar_r, rows_of(split) > 0
                                       ? uint32_t(p.splits * (rows_of(split) * D * 2 + rpo4 * 4))
                                       : 0u);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(sTmem, ncols);
    tmem_relinquish();
  }
  // every block's bar_r is initialised before any block may copy into it (this waits on no
  // other kernel: it runs while the top-k still works)
  if (p.splits > 1) cg::this_cluster().sync();
  const bool early = early_ok && c_begin * KVB >= n_a;     // window rows only
  if (!early_ok) pdl_enter();
  const int pos = p.q_pos[b];
  const int raw_lo = pos - p.W + 1;

  // Q: thread (row, hc) loads dims 64*hc .. 64*hc+63 of head `row` into SW128 half hc
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.H + row) * D) + hc * 8;
    uint4 qv[8];
#pragma unroll
    for (int c = 0; c < 8; c++) qv[c] = row < p.H ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    if (p.q_gamma != nullptr) {
      // RMSNorm of the head's query row [Tripbot §5]: the two threads of a row add their
      // halves' sums of squares through shared memory; fp32, rounded back to bf16
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 8; c++) {
        const uint32_t w4[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          ss = fmaf(lo, lo, fmaf(hi, hi, ss));
        }
      }
      xch[tid] = ss;
      __syncthreads();
      const float rn = 1.f / sqrtf((xch[row] + xch[row + TC_ROWS]) / float(D) + p.q_eps);
#pragma unroll
      for (int c = 0; c < 8; c++) {
        uint32_t w4[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int dim = hc * 64 + c * 8 + 2 * j;
          const float lo = __uint_as_float(w4[j] << 16), hi = __uint_as_float(w4[j] & 0xFFFF0000u);
          w4[j] = pack_bf16(lo * rn * __ldg(p.q_gamma + dim), hi * rn * __ldg(p.q_gamma + dim + 1));
        }
        qv[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; c++)
      *reinterpret_cast<uint4*>(sQ + hc * 16384 + row * 128 + ((c ^ (row & 7)) << 4)) = qv[c];
  }
  if (early_ok && !early) pdl_enter();

  // rows of the split: two threads per row resolve the row's store slot and copy their halves
  // of its 16-byte pieces (rope half / bf16 rows straight into the SW128 tile with cp.async,
  // E4M3 codes and scales into staging); a warp's ballot gives the validity bits of its 16 rows
  const int nrows = nch * KVB;
  for (int j0 = 0; j0 < nrows; j0 += TC_THREADS / 2) {
    const int jj = j0 + (tid >> 1), half = tid & 1;
    const int e = c_begin * KVB + jj;
    long long slot = -1;
    bool from_raw = false;
    if (jj < nrows) {
      if (e < n_a) {
        long long ent = p.idx[(size_t)b * p.k + e];
        if (ent < -1 || ent >= p.n_comp) {
          if (half == 0) report(p.status, HCL_ERR_DEVICE_FAULT);
          ent = -1;
        }
        if (ent >= 0) slot = (long long)b * p.comp.cap + (ent % p.comp.cap);
      } else if (e < total) {
        const long long u = (long long)raw_lo + (e - n_a);
        if (u >= 0) { slot = (long long)b * p.raw.cap + (u % p.raw.cap); from_raw = true; }
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, slot >= 0);
    uint32_t bits16 = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) bits16 |= ((bal >> (2 * i)) & 1u) << i;
    if (lane == 0 && j0 + 16 * warp < nrows)
      reinterpret_cast<uint16_t*>(visw)[(j0 >> 4) + warp] = uint16_t(bits16);
    if (jj >= nrows) continue;
    const int ch = jj / KVB, r = jj % KVB;
    const hcl_kv_t& st = from_raw ? p.raw : p.comp;
    uint8_t* kv = sm + off.kv + ch * 16384;
    if (KVFMT == HCL_BF16) {
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int c = half * 8 + i;
        uint8_t* dst = kv + (c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.data) + slot * 256 + c * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    } else if (half == 0) {        // RoPE dims 64..127: the second half, as stored
#pragma unroll
      for (int c = 0; c < 8; c++) {
        uint8_t* dst = kv + 8192 + r * 128 + ((c ^ (r & 7)) << 4);
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.rope) + slot * 128 + c * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    } else {                       // E4M3 codes of dims 0..63 and the row scale
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint8_t* dst = sm + off.stg + (ch * KVB + r) * 64 + c * 16;
        if (slot >= 0) cp_async16(dst, static_cast<const uint8_t*>(st.data) + slot * 64 + c * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
      float* dst = reinterpret_cast<float*>(sm + off.scl) + ch * KVB + r;
      if (slot >= 0)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                     "l"(st.scale + slot)
                     : "memory");
      else *dst = 0.f;
    }
  }
  cp_async_commit();
  if (early) pdl_enter();
  cp_async_wait<0>();
  __syncthreads();
  if (KVFMT == HCL_FP8SPLIT) {
    // widen: 8 codes x scale -> one 16-byte bf16 chunk of the first half
    for (int u = tid; u < nrows * 8; u += TC_THREADS) {
      const int jj = u >> 3, c = u & 7, ch = jj / KVB, r = jj % KVB;
      const uint2 codes = *reinterpret_cast<const uint2*>(sm + off.stg + (ch * KVB + r) * 64 + c * 8);
      const float sc = reinterpret_cast<const float*>(sm + off.scl)[ch * KVB + r];
      uint4 v;
      v.x = e4m3x2_to_bf16x2(uint16_t(codes.x & 0xffff), sc);
      v.y = e4m3x2_to_bf16x2(uint16_t(codes.x >> 16), sc);
      v.z = e4m3x2_to_bf16x2(uint16_t(codes.y & 0xffff), sc);
      v.w = e4m3x2_to_bf16x2(uint16_t(codes.y >> 16), sc);
      *reinterpret_cast<uint4*>(sm + off.kv + ch * 16384 + r * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
  }
  fence_proxy_async_smem();      // Q, the gathered rows and the widened halves -> UMMA
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const long long limit = 2000000000LL;

  // S_c = Q K_c^T (M = 128 heads, N = 64 rows, K = 128 dims in 8 steps of 16)
  if (tid == 0 && nch > 0) {
    const uint32_t aq = smem_u32(sQ);
    for (int c = 0; c < nch; c++) {
      const uint32_t ak = smem_u32(sm + off.kv + c * 16384);
#pragma unroll
      for (int ks = 0; ks < 8; ks++) {
        const uint32_t h = ks >> 2, kk = ks & 3;
        umma_bf16(tbase + c * 64, make_sdesc(aq + h * 16384 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  make_sdesc(ak + h * 8192 + kk * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  idesc_bf16(128, 64), ks > 0 ? 1u : 0u);
      }
    }
    umma_commit(bar_s);
  }
  __syncwarp();   // warp 0 reconverges before waiting (the issuing lane is not left behind)
  bool ok = nch == 0 || mbar_wait(bar_s, 0, limit, nullptr);
  if (!ok) report(p.status, HCL_ERR_TIMEOUT);
  tc_fence_after();

  // softmax for head `row` over the split's rows (log2 domain); this thread holds columns
  // 32*hc .. 32*hc+31 of every chunk and exchanges its partial maximum and sum with the
  // other half's thread through shared memory
  const uint32_t trow = tbase + (uint32_t((warp & 3) * 32) << 16);
  float lmax = -INFINITY;
  auto cols = [&](int c, uint32_t (&r32)[32]) {
    tmem_ld16(trow + c * 64 + hc * 32, *reinterpret_cast<uint32_t(*)[16]>(&r32[0]));
    tmem_ld16(trow + c * 64 + hc * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r32[16]));
  };
  uint32_t sv[2][32];
  const bool inreg = nch <= 2;
  if (inreg) {
#pragma unroll
    for (int c = 0; c < 2; c++)
      if (c < nch) cols(c, sv[c]);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < 2; c++)
      if (c < nch) {
        const uint32_t vb = visw[2 * c + hc];
#pragma unroll
        for (int j = 0; j < 32; j++)
          if ((vb >> j) & 1u) lmax = fmaxf(lmax, __uint_as_float(sv[c][j]) * p.scale_log2);
      }
  } else {
    for (int c = 0; c < nch; c++) {
      uint32_t r32[32];
      cols(c, r32);
      tmem_ld_wait();
      const uint32_t vb = visw[2 * c + hc];
#pragma unroll
      for (int j = 0; j < 32; j++)
        if ((vb >> j) & 1u) lmax = fmaxf(lmax, __uint_as_float(r32[j]) * p.scale_log2);
    }
  }
  xch[tid] = lmax;
  __syncthreads();
  const float mrow = fmaxf(xch[row], xch[row + TC_ROWS]);
  const float muse = mrow == -INFINITY ? 0.f : mrow;
  float lsum = 0.f;
  const unsigned long long c2x2 = f2_make(p.scale_log2, p.scale_log2);
  const unsigned long long negm = f2_make(-muse, -muse);
  auto emit_p = [&](int c, const uint32_t (&r32)[32]) {
    const uint32_t vb = visw[2 * c + hc];
    uint8_t* prow = sm + off.pm + c * 16384 + row * 128;
    unsigned long long ls2 = 0ull;   // two partial sums (+0.0f each)
#pragma unroll
    for (int q4 = 0; q4 < 4; q4++) {
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int j = q4 * 8 + i;
        // 2^(s * scale - m) for a pair of columns: one paired FMA, two exponentials
        const unsigned long long t =
            f2_fma(f2_make(__uint_as_float(r32[j]), __uint_as_float(r32[j + 1])), c2x2, negm);
        float p0 = ex2_ftz(f2_lo(t)), p1 = ex2_ftz(f2_hi(t));
        if (vb != 0xFFFFFFFFu) {
          p0 = ((vb >> j) & 1u) ? p0 : 0.f;
          p1 = ((vb >> (j + 1)) & 1u) ? p1 : 0.f;
        }
        ls2 = f2_add(ls2, f2_make(p0, p1));
        pk[i >> 1] = pack_bf16(p0, p1);
      }
      *reinterpret_cast<uint4*>(prow + (((hc * 4 + q4) ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    lsum += f2_lo(ls2) + f2_hi(ls2);
  };
  if (inreg) {
#pragma unroll
    for (int c = 0; c < 2; c++)
      if (c < nch) emit_p(c, sv[c]);
  } else {
    for (int c = 0; c < nch; c++) {
      uint32_t r32[32];
      cols(c, r32);
      tmem_ld_wait();
      emit_p(c, r32);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();               // (also: every thread has read the partial maxima)
  xch[TC_THREADS + tid] = lsum;
  tc_fence_after();

  // O = sum_c P_c V_c (M = 128 heads, N = 128 dims, K = 64 rows per chunk in 4 steps of 16);
  // V is MN-major: 64-dim halves 8 KB apart (LBO), 8-row groups 1 KB apart (SBO)
  if (tid == 0 && nch > 0) {
    for (int c = 0; c < nch; c++) {
      const uint32_t ap = smem_u32(sm + off.pm + c * 16384);
      const uint32_t av = smem_u32(sm + off.kv + c * 16384);
#pragma unroll
      for (int ks = 0; ks < 4; ks++)
        umma_bf16(tbase + ocol, make_sdesc(ap + ks * 32, 16, 1024, SMEM_SWIZZLE_128B),
                  make_sdesc(av + ks * 2048, 8192, 1024, SMEM_SWIZZLE_128B),
                  idesc_bf16(128, D) | (1u << 16), (c > 0 || ks > 0) ? 1u : 0u);
    }
    umma_commit(bar_o);
  }
  __syncwarp();
  ok = nch == 0 || mbar_wait(bar_o, 0, limit, nullptr);
  if (!ok) report(p.status, HCL_ERR_TIMEOUT);
  __syncthreads();               // the partial sums
  tc_fence_after();

  // output dims 64*hc .. 64*hc+63 of head `row`: normalised partial (o, lse) or the output
  const bool hv = row < p.H;
  float m2 = mrow, l2 = xch[TC_THREADS + row] + xch[TC_THREADS + row + TC_ROWS];
  const float inv_l = l2 > 0.f ? 1.f / l2 : 0.f;
  // splits > 1: row r is merged by block r / rpo (contiguous head blocks) in its slot r % rpo;
  // the normalised partial rows (|o| <= max |v|: fp16, 11 significant bits, is exact enough for
  // a bf16 output and halves the bytes crossing between blocks) are staged in this block's (now
  // idle) KV tiles, XOR-swizzled in 16-byte chunks, and block o's rows then go to it as one
  // bulk copy
  uint8_t* stage = sm + off.kv;                   // 128 rows x 256 B (KV tiles, cps == 2)
  float* stage_lse = reinterpret_cast<float*>(sm + off.pm);   // [owner][rpo4] (P tiles)
  if (p.splits > 1 && hv && hc == 0)
    stage_lse[(row / rpo) * rpo4 + row % rpo] = l2 > 0.f ? m2 + log2f(l2) : -INFINITY;
  float f = inv_l;
  if (p.splits == 1 && p.sink) {
    const float s2 = p.sink[min(row, p.H - 1)] * LOG2E;
    const float mm = fmaxf(m2, s2);
    const float fa = l2 > 0.f ? exp2f(m2 - mm) : 0.f;
    const float l3 = l2 * fa + exp2f(s2 - mm);
    f = l3 > 0.f ? fa / l3 : 0.f;
    l2 = l3;
    m2 = mm;
  }
  {
    uint32_t r64[64];
#pragma unroll
    for (int q4 = 0; q4 < 4; q4++)
      tmem_ld16(trow + ocol + hc * 64 + q4 * 16, *reinterpret_cast<uint32_t(*)[16]>(&r64[q4 * 16]));
    tmem_ld_wait();
    if (p.splits > 1) {
      // chunk c (16 bytes = 8 fp16) of row `row` at chunk position c ^ (row & 7): conflict-free
#pragma unroll
      for (int i = 0; i < 64; i += 8) {
        const int c = hc * 8 + (i >> 3);
        uint4 v;
        v.x = pack_half2(__uint_as_float(r64[i]) * inv_l, __uint_as_float(r64[i + 1]) * inv_l);
        v.y = pack_half2(__uint_as_float(r64[i + 2]) * inv_l, __uint_as_float(r64[i + 3]) * inv_l);
        v.z = pack_half2(__uint_as_float(r64[i + 4]) * inv_l, __uint_as_float(r64[i + 5]) * inv_l);
        v.w = pack_half2(__uint_as_float(r64[i + 6]) * inv_l, __uint_as_float(r64[i + 7]) * inv_l);
        *reinterpret_cast<uint4*>(stage + row * 256 + ((c ^ (row & 7)) << 4)) = v;
      }
    } else if (hv) {
      {
        __nv_bfloat16* dst = p.out + ((size_t)b * p.H + row) * D + hc * 64;
#pragma unroll
        for (int i = 0; i < 64; i += 8) {
          reinterpret_cast<uint4*>(dst + i)[0] =
              make_uint4(pack_bf16(__uint_as_float(r64[i]) * f, __uint_as_float(r64[i + 1]) * f),
                         pack_bf16(__uint_as_float(r64[i + 2]) * f, __uint_as_float(r64[i + 3]) * f),
                         pack_bf16(__uint_as_float(r64[i + 4]) * f, __uint_as_float(r64[i + 5]) * f),
                         pack_bf16(__uint_as_float(r64[i + 6]) * f, __uint_as_float(r64[i + 7]) * f));
        }
      }
    }
  }
  if (p.splits > 1) {
    fence_proxy_async_smem();                     // staged rows -> the bulk-copy engine
    __syncthreads();
    if (tid == 0) {
      // block o receives rows o*rpo .. o*rpo + rows_of(o) - 1 at recv[split][slot][D], still
      // swizzled (chunk c of row r at c ^ (r & 7))
      for (int o = 0; o < p.splits; o++)
        if (rows_of(o) > 0) {
          bulk_copy_to_cluster(cluster_map(recv_h + (size_t)split * rpo * D, o),
                               stage + (size_t)o * rpo * 256, uint32_t(rows_of(o) * 256),
                               cluster_map(bar_r, o));
          bulk_copy_to_cluster(cluster_map(recv_lse + (size_t)split * rpo4, o),
                               stage_lse + (size_t)o * rpo4, uint32_t(rpo4 * 4),
                               cluster_map(bar_r, o));
        }
    }
  }
  if (p.splits == 1 && hv && hc == 0 && p.lse)
    p.lse[(size_t)b * p.H + row] = l2 > 0.f ? (m2 + log2f(l2)) * LN2 : -INFINITY;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, ncols);
  }
  if (p.splits > 1) {
    // merge the rows this block owns (row r -> block r / rpo, slot r % rpo) once its own
    // copies (partials and log-sum-exps) have landed (bar_r).  Every block arrives on the
    // cluster barrier after that and waits on it only before exiting: when it passes, every
    // block's copies out of this block's shared memory have been received
    if (!mbar_wait(bar_r, 0, limit, nullptr)) report(p.status, HCL_ERR_TIMEOUT);
    asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
    const int S = p.splits;
    // two heads per warp, one per 16-lane half: lane hl holds dims 8 hl .. 8 hl + 7 (16-byte
    // chunk hl of the row, stored at chunk hl ^ (h & 7)) and, for hl < S, split hl's weight
    const int hl = lane & 15, hb = lane & 16;
    for (int slot0 = 2 * warp; slot0 < rpo; slot0 += 2 * (TC_THREADS / 32)) {
      const int slot = min(slot0 + (lane >> 4), rpo - 1);
      const int h = split * rpo + slot;
      const bool act = slot0 + (lane >> 4) < rpo && h < p.H;
      const float ls = (act && hl < S) ? recv_lse[hl * rpo4 + slot] : -INFINITY;
      float M = ls;
#pragma unroll
      for (int o2 = 8; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
      float s2 = -INFINITY;
      if (p.sink) {
        s2 = p.sink[min(h, p.H - 1)] * LOG2E;
        M = fmaxf(M, s2);
      }
      const float wl = (ls == -INFINITY || M == -INFINITY) ? 0.f : ex2_ftz(ls - M);
      float den = wl;
#pragma unroll
      for (int o2 = 8; o2 > 0; o2 >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o2);
      if (p.sink && M > -INFINITY) den += ex2_ftz(s2 - M);
      const uint8_t* part =
          reinterpret_cast<const uint8_t*>(recv_h + (size_t)slot * D) + ((hl ^ (h & 7)) << 4);
      // every split's partial loaded up front (independent loads), then summed in split order
      // (a zero weight adds 0 * v = 0: the partials are finite)
      uint4 hv4[MAX_CLUSTER_ROWS];
#pragma unroll
      for (int s = 0; s < MAX_CLUSTER_ROWS; s++)
        hv4[s] = (act && s < S) ? *reinterpret_cast<const uint4*>(part + (size_t)s * rpo * D * 2)
                                : make_uint4(0u, 0u, 0u, 0u);
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; i++) acc[i] = 0.f;
#pragma unroll
      for (int s = 0; s < MAX_CLUSTER_ROWS; s++) {
        const float wgt = __shfl_sync(0xffffffffu, wl, hb | s);
        if (s < S) {
          const uint32_t w4[4] = {hv4[s].x, hv4[s].y, hv4[s].z, hv4[s].w};
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[i]));
            acc[2 * i] += wgt * f.x;
            acc[2 * i + 1] += wgt * f.y;
          }
        }
      }
      const float inv = den > 0.f ? __fdividef(1.f, den) : 0.f;
      const size_t orow = (size_t)b * p.H + h;
      if (act) {
        reinterpret_cast<uint4*>(p.out + orow * D)[hl] =
            make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                       pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
        if (p.lse && hl == 0) p.lse[orow] = den > 0.f ? (M + __log2f(den)) * LN2 : -INFINITY;
      }
    }
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  }
}

struct Plan {
  int G, NW, n_groups, splits, cps, rows_pad, n_chunks_max, cmerge, hsplit;
};

constexpr int MAX_CLUSTER = 16;

// Blocks: one per (sequence, query group, split).  The split of a query group's row list --
// and so the order in which partial results are merged -- is a function of the per-sequence
// shape only (queries per sequence, heads, list length), never of the batch size or of the
// device: a sequence's output is then bitwise the same whatever batch it is decoded in
// (batch-invariant kernels, [Tripbot §8 infrastructure table]).  A sequence with few query
// groups (decode) splits its list into pieces of SPLIT_CHUNKS chunks so that its rows spread
// over several SMs; with many groups every group is one block.  Splits of a group merge in a
// cluster through DSMEM when they fit one (<= 16 blocks; no workspace, no merge launch),
// otherwise through the caller's workspace and a merge kernel; both merge the splits of a row
// in split order.
constexpr int SPLIT_CHUNKS = 2;
constexpr int FEW_GROUPS = 32;

Plan make_plan(int mode, int B, int Tq, int H, int list_max) {
  Plan pl;
  pl.G = mode == 0 ? 1 : std::max(1, 128 / H);
  pl.G = std::min(pl.G, Tq);
  const int rows = pl.G * H;
  pl.NW = rows <= 16 ? 1 : rows <= 32 ? 2 : rows <= 64 ? 4 : 8;
  pl.rows_pad = pl.NW * 16;
  pl.n_groups = (Tq + pl.G - 1) / pl.G;
  pl.n_chunks_max = std::max(1, (list_max + KVB - 1) / KVB);
  pl.cps = pl.n_groups >= FEW_GROUPS ? pl.n_chunks_max : SPLIT_CHUNKS;
  pl.splits = (pl.n_chunks_max + pl.cps - 1) / pl.cps;
  pl.cmerge = pl.splits > 1 && pl.splits <= MAX_CLUSTER;
  // few clusters of 8-warp blocks leave SMs idle: halve the rows per block instead (each
  // (query, head) row's arithmetic is the same in either shape, so the bits do not change)
  const long long blocks = (long long)B * pl.n_groups;
  pl.hsplit = 1;
  if (pl.cmerge && pl.NW == 8 && blocks * pl.splits * 2 <= num_sms()) {
    pl.hsplit = 2;
    pl.NW = 4;
    pl.rows_pad = 64;
  }
  return pl;
}

template <int KVFMT, int MODE, int NW>
hcl_status_t launch_t(const AttnParams& p, cudaStream_t st, long long grid) {
  auto kern = attn_kernel<KVFMT, MODE, NW>;
  size_t smem = 2 * KVB * 256 + 2 * KVB * 64 + 2 * KVB * 4 + 2 * KVB * sizeof(RowSrc);
  if (!p.cmerge) {
    return check_cuda(launch_pdl(kern, dim3((unsigned)grid), dim3(NW * 32), smem, st, 1, p),
                      "attention launch");
  }
  // receive buffers: ceil(rows / splits) slots x splits partials (+ LSE)
  auto recv_bytes = [](int S) {
    return (size_t)((NW * 16 + S - 1) / S) * S * (D + 1) * sizeof(float);
  };
  size_t recv_max = 0;
  for (int S = 2; S <= MAX_CLUSTER; S++) recv_max = std::max(recv_max, recv_bytes(S));
  const size_t smem_max = smem + recv_max;
  smem += recv_bytes(p.splits);
  // set for the largest cluster need, once per kernel and context
  hcl_status_t ea = set_kernel_attrs(reinterpret_cast<const void*>(kern), (int)smem_max, true);
  if (ea != HCL_OK) return ea;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, p), "attention launch");
}

template <int KVFMT, int MODE>
hcl_status_t launch_nw(const AttnParams& p, int NW, cudaStream_t st, long long grid) {
  switch (NW) {
    case 1: return launch_t<KVFMT, MODE, 1>(p, st, grid);
    case 2: return launch_t<KVFMT, MODE, 2>(p, st, grid);
    case 4: return launch_t<KVFMT, MODE, 4>(p, st, grid);
    default: return launch_t<KVFMT, MODE, 8>(p, st, grid);
  }
}

// CSA decode on tcgen05 when the plan allows it: one query per sequence, all heads in one
// block (up to 128), splits merged in a cluster (or a single split), <= TC_MAXC chunks each.
bool tc_usable(const AttnArgs& a, const Plan& pl) {
  return a.mode == 0 && a.Tq == 1 && a.H <= TC_ROWS &&
         ((pl.splits == 1 && pl.cps <= TC_MAXC) || (pl.cmerge && pl.cps == TC_MAXC_MERGE));
}

template <int KVFMT>
hcl_status_t launch_tc(const AttnParams& p, cudaStream_t st) {
  auto kern = attn_tc_kernel<KVFMT>;
  size_t smem_max = (size_t)tc_offsets(TC_MAXC, 1).total + 1024;
  for (int S = 2; S <= MAX_CLUSTER; S++)
    smem_max = std::max(smem_max, (size_t)tc_offsets(TC_MAXC_MERGE, S).total + 1024);
  hcl_status_t ea = set_kernel_attrs(reinterpret_cast<const void*>(kern), (int)smem_max, true);
  if (ea != HCL_OK) return ea;
  const size_t smem = (size_t)tc_offsets(p.cps, p.splits).total + 1024;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(p.B * p.splits));
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = p.splits > 1 ? 2 : 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, kern, p), "attention launch");
}

// Longest row list a block may process: CSA k selected entries + W window rows; HCA every
// entry (n = Nh) plus the union of the G windows of a query group.  The workspace query and
// the launch both plan from this one number.
int list_max_for(int mode, int B, int Tq, int H, int n, int W) {
  if (mode == 0) return n + std::max(0, W);
  const Plan pl = make_plan(1, B, Tq, H, 0);
  return n + (W > 0 ? W + pl.G - 1 : 0);
}

}  // namespace

size_t attn_workspace_bytes(int mode, int B, int Tq, int H, int n, int W) {
  const Plan pl = make_plan(mode, B, Tq, H, list_max_for(mode, B, Tq, H, n, W));
  if (pl.splits <= 1 || pl.cmerge) return 0;
  const size_t items = (size_t)B * pl.n_groups * pl.splits;
  return items * pl.rows_pad * (D + 1) * sizeof(float);
}

hcl_status_t launch_attn(const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  if ((long long)a.B * a.Tq == 0) return HCL_OK;
  const int list_max = list_max_for(a.mode, a.B, a.Tq, a.H, a.mode == 0 ? a.k : a.n_comp, a.W);
  const Plan pl = make_plan(a.mode, a.B, a.Tq, a.H, list_max);
  AttnParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.B = a.B; p.Tq = a.Tq; p.H = a.H;
  p.comp = a.comp; p.n_comp = a.n_comp; p.mh = a.mode == 0 ? 1 : a.mh;
  p.idx = a.idx; p.k = a.k;
  p.raw = a.raw; p.W = a.W;
  p.q_pos = a.q_pos;
  p.scale_log2 = a.scale * LOG2E;
  p.sink = a.sink;
  p.q_gamma = a.q_gamma;
  p.q_eps = a.q_eps;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.G = pl.G; p.n_groups = pl.n_groups; p.splits = pl.splits; p.cps = pl.cps;
  p.rows_pad = pl.rows_pad;
  p.cmerge = pl.cmerge;
  p.hsplit = pl.hsplit;
  p.prewait = a.prewait;
  p.status = a.status;
  p.ws_o = nullptr;
  p.ws_lse = nullptr;
  if (pl.splits > 1 && !pl.cmerge) {
    const size_t items = (size_t)a.B * pl.n_groups * pl.splits;
    const size_t need = items * pl.rows_pad * (D + 1) * sizeof(float);
    if (ws == nullptr || ws_bytes < need)
      return fail(HCL_ERR_INVALID_ARG, "attention workspace too small: need %zu bytes, got %zu",
                  need, ws_bytes);
    p.ws_o = static_cast<float*>(ws);
    p.ws_lse = p.ws_o + items * pl.rows_pad * D;
  }
  if (hca_flash_usable(a)) return launch_hca_flash(a, st);
  if (tc_usable(a, pl)) {
    return a.comp.fmt == HCL_FP8SPLIT ? launch_tc<HCL_FP8SPLIT>(p, st) : launch_tc<HCL_BF16>(p, st);
  }
  const long long grid = (long long)a.B * pl.n_groups * pl.hsplit * pl.splits;
  hcl_status_t e;
  const bool fp8 = a.comp.fmt == HCL_FP8SPLIT;
  if (a.mode == 0) e = fp8 ? launch_nw<HCL_FP8SPLIT, 0>(p, pl.NW, st, grid)
                           : launch_nw<HCL_BF16, 0>(p, pl.NW, st, grid);
  else e = fp8 ? launch_nw<HCL_FP8SPLIT, 1>(p, pl.NW, st, grid)
               : launch_nw<HCL_BF16, 1>(p, pl.NW, st, grid);
  if (e != HCL_OK || pl.splits == 1 || pl.cmerge) return e;
  const long long threads = (long long)a.B * a.Tq * a.H * 32;
  return check_cuda(launch_pdl(attn_merge_kernel, dim3((unsigned)((threads + 255) / 256)),
                               dim3(256), 0, st, 1, p),
                    "attention merge launch");
}

// ---------------------------------------------------------------------------------------
// Scratch for hcl_csa_sparse_attn_noalloc: a fixed device array in this module, so callers
// that may not allocate device memory still get the split-KV attention.  Every GPU that loads
// the library holds these NOALLOC_SCRATCH_BYTES until the process exits.  All calls share it:
// calls that overlap on the GPU race on it.  Nothing in it has to start at zero -- each
// partial (o, lse) slot the merge reads is written earlier in the same call.
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the calling thread's current CUDA context.  The
// array's name is only a host-side stand-in in host code, so the address is looked up by
// cudaGetSymbolAddress with the device current and cached per device together with the id of
// the context it belongs to: a call in another context (one created after cudaDeviceReset, or
// a non-primary context) finds no cached entry for its context id and looks the address up
// again.  Context ids are never reused within a process.
hcl_status_t noalloc_scratch(void** ptr) {
  static std::mutex mu;
  static unsigned long long ctx_of[64] = {};
  static void* cache[64] = {};
  int dev = 0;
  hcl_status_t e = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (e != HCL_OK) return e;
  if (dev < 0 || dev >= 64) return fail(HCL_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx == 0 || ctx_of[dev] != ctx || cache[dev] == nullptr) {
    void* p = nullptr;
    e = check_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    if (e != HCL_OK) return e;
    cache[dev] = p;
    ctx_of[dev] = current_ctx_id();   // the lookup made the device's context current
  }
  *ptr = cache[dev];
  return HCL_OK;
}

}  // namespace hcl
