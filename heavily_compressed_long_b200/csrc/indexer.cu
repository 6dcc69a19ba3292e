// indexer.cu -- the lightning indexer on tcgen05 tensor cores.
//
// [Tripbot §3.1] A light multi-head dot-product scorer rates every compressed entry for the
// current query; [CSDN §1.4] its QK product runs in FP4 and the scores are quantised from
// FP32 to BF16 before the top-k.  For query t, entry i:
//     s[t, i] = sum_h w[t, h] * max(0, qI[t, h, :] . kI[i, :])      (i visible, else -inf)
//
// Design (B200): the contraction is laid out "keys x query-heads": the UMMA M dimension is
// 128 index keys, N is QT queries x 16 (padded) heads, K = dI = 64.  Each thread of the
// epilogue then owns one key (one TMEM lane) and all heads of its queries, so the ReLU-weighted
// head reduction is thread-local and the score row is written coalesced.
//   - warp 0: TMA producer streaming stages of TPS key tiles (and their E8M0 scales) into a
//             shared-memory ring;
//   - warp 1: allocates TMEM, issues per stage TPS tcgen05.mma (kind::f16 for bf16 operands, or
//             kind::mxf4.block_scale with the key scales copied shared->TMEM by tcgen05.cp),
//             and commits once per stage;
//   - warps 2..: epilogue: tcgen05.ld of the stage's accumulators, ReLU, weighted head sum,
//             mask, optional bf16 rounding, store.
// Decode (one query per sequence) is a pure HBM stream: several 128-key tiles per stage
// amortise the MMA -> commit -> epilogue -> release round trip, and several stage
// accumulators stay in flight in TMEM, so the TMA ring runs ahead.  Prefill uses N = 16
// queries x 16 heads = 256 per tile.  With MXFP4 keys the bf16 index query may be quantised
// in the prologue (same encoder as hcl_quant_mxfp4).  Every wait is bounded; a wait that runs
// out sets HCL_ERR_TIMEOUT in the status word, and the block drains its copies and MMAs,
// frees TMEM and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include <type_traits>

#include "hcl_common.cuh"
#include "hcl_internal.h"
#include "mxfp4.cuh"

namespace hcl {
namespace {

constexpr int KEYS = 128;  // keys per UMMA tile = M
constexpr int HP = 16;     // heads per query, padded = UMMA N per query

struct IdxParams {
  const uint8_t* qI;          // pre-quantised / bf16 operand rows
  const uint8_t* qI_sf;       // MXFP4 scales of qI (when pre-quantised)
  const uint8_t* kI_sf;       // MXFP4 key scales [B, cap, 2] (packed-row decode path)
  const __nv_bfloat16* qI_bf16;  // bf16 index queries to quantise in-kernel (MXFP4 keys), or null
  const float* w;
  const int32_t* q_pos;
  void* scores;
  int score_fmt;
  int B, Tq, HI, Nc, m, cap;
  int vec_ok;                 // Nc % 4 == 0 and scores 16-byte aligned: vector score stores
  uint16_t* gmax;             // packed-row decode, bf16 scores: per-16-entry maxima, or null
  uint16_t* g2nd;             //   second largest per group
  uint8_t* garg;              //   position of the largest in its group
  int NG;                     // gmax row stride in groups
  int n_qt, n_kt, n_kc, kt_per_chunk;
  int32_t* status;
  long long limit;
};

__host__ __device__ constexpr uint32_t tmem_cols_for(uint32_t need) {
  uint32_t c = 32;
  while (c < need) c <<= 1;
  return c;
}

// Operand kinds: 0 = bf16 (one key per 128-byte K-row, SW128); 1 = MXFP4 (one key per 32-byte
// K-row, SW32); 2 = MXFP4 packed rows (decode): four consecutive keys form one 128-byte K-row
// (K = 256 = 4 keys x 64), loaded with SW128 as one 16 KB box of 512 keys.  The query operand
// is block-diagonal (row (j, h) holds q_h in K-segment j), so UMMA k-step j (K = 64) yields
// key 4r+j against every head in accumulator columns j*16 .. j*16+15 of lane r.
template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
struct IdxLayout {
  static constexpr int KPR = KIND == 2 ? 4 : 1;            // keys per operand row
  static constexpr int TK = KEYS * KPR;                     // keys per tile
  static constexpr int N = QT * HP * KPR;
  static constexpr int ROWB = KIND == 1 ? 32 : 128;         // bytes per K-row of an operand
  static constexpr int A_TILE = KEYS * ROWB;
  static constexpr int A_STAGE = TPS * A_TILE;
  static constexpr int SF_TILE = KIND == 0 ? 0 : TK * 2;    // raw E8M0 bytes per tile
  static constexpr int SF_BLOCKS = KIND == 0 ? 0 : KPR;     // 512-byte tcgen05.cp blocks per tile
  static constexpr int BOX_ROWS = (TPS * KEYS) < 256 ? (TPS * KEYS) : 256;
  static constexpr int B_BYTES = ((N * ROWB + 1023) / 1024) * 1024;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr int OFF_SFRAW = OFF_B + B_BYTES;
  static constexpr int OFF_SFEXP = OFF_SFRAW + STAGES * TPS * SF_TILE;
  static constexpr int OFF_SFB = OFF_SFEXP + STAGES * TPS * SF_BLOCKS * 512;
  static constexpr int OFF_W = OFF_SFB + (KIND != 0 ? 512 : 0);
  static constexpr int OFF_NVIS = OFF_W + QT * HP * 4;
  static constexpr int OFF_BAR = ((OFF_NVIS + QT * 4 + 7) / 8) * 8;
  static constexpr int NBAR = 2 * STAGES + 2 * NACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int NT = 64 + 32 * EPI;
  static constexpr int ACC_COLS = NACC * TPS * N;
  static constexpr uint32_t TMEM_COLS =
      tmem_cols_for(ACC_COLS + (KIND != 0 ? 4 * SF_BLOCKS * TPS + 4 : 0));
};

// Two fp32 lanes packed in 64 bits (x in the low word) and their paired fused multiply-add.
__device__ __forceinline__ unsigned long long pack2(float x, float y) {
  return (unsigned long long)__float_as_uint(x) | ((unsigned long long)__float_as_uint(y) << 32);
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
__global__ void __launch_bounds__(64 + 32 * EPI, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmSF,
                   IdxParams p) {
  using Lay = IdxLayout<KIND, QT, TPS, STAGES, NACC, EPI>;
  static_assert(KIND != 2 || (QT == 1 && EPI == 4), "packed rows: one query, 128 epilogue threads");
  constexpr int N = Lay::N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* sA = sm + Lay::OFF_A;
  uint8_t* sB = sm + Lay::OFF_B;
  uint8_t* sSFraw = sm + Lay::OFF_SFRAW;
  uint8_t* sSFexp = sm + Lay::OFF_SFEXP;
  uint8_t* sSFB = sm + Lay::OFF_SFB;
  float* sW = reinterpret_cast<float*>(sm + Lay::OFF_W);
  int* sNvis = reinterpret_cast<int*>(sm + Lay::OFF_NVIS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* accf = bars + 2 * STAGES;
  uint64_t* acce = bars + 2 * STAGES + NACC;
  uint64_t* drain = bars + 2 * STAGES + 2 * NACC;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + Lay::OFF_MISC);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 4);

  const int warp = warp_id(), lane = lane_id();
  int item = blockIdx.x;
  const int kc = item % p.n_kc;
  item /= p.n_kc;
  const int qt = item % p.n_qt;
  const int b = item / p.n_qt;
  const int kt0 = kc * p.kt_per_chunk;                      // multiple of TPS
  const int ntiles = min(p.n_kt, kt0 + p.kt_per_chunk) - kt0;
  const int nstages = (ntiles + TPS - 1) / TPS;
  const int t0 = qt * QT;
  if (ntiles <= 0) return;  // uniform over the block

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < NACC; a++) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 32 * EPI); }
    mbar_init(drain, 1);
    *sAbort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sTmem, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    if (KIND == 1) prefetch_tmap(&tmSF);
  }
  __syncthreads();  // barriers initialised, TMEM allocated
  tc_fence_after();
  // everything above touches no global memory; the rest may read what the previous kernel
  // in the stream wrote.  The producer starts streaming keys as soon as the epilogue warps
  // have issued their few prologue loads (named barrier 3); the MMA warp waits (named
  // barrier 2) until those warps have built the query operand.
  pdl_enter();
  if (threadIdx.x >= 64) {
    // Query operand tile (K-major, swizzled as the UMMA descriptor expects), head weights,
    // visible counts, and (MXFP4) the query scale factors in the tcgen05.cp block layout
    // (line n%32, 32-bit word n/32, bytes 0..1).
    const int et = threadIdx.x - 64, ne = 32 * EPI;
    if (KIND == 0) {
      for (int u = et; u < N * 8; u += ne) {
        const int n = u / 8, c = u % 8;
        const int q = n / HP, h = n % HP, t = t0 + q;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < p.Tq && h < p.HI)
          v = __ldg(reinterpret_cast<const uint4*>(
              p.qI + (((size_t)b * p.Tq + t) * p.HI + h) * 128 + c * 16));
        *reinterpret_cast<uint4*>(sB + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4)) = v;
      }
    } else if (KIND == 2) {
      // Packed rows, one query (EPI = 4: 128 threads).  Thread et holds 8 values of head
      // h = et/8, scale block half = (et/4)&1, part c = et&3; the four threads of a block share
      // its amax by shuffles (max is exact, so the scale matches hcl_quant_mxfp4 bit for bit).
      // Its packed word goes to rows (seg, h) of the block-diagonal operand, chunk 2*seg+half.
      // All global loads are issued before the producer may start (named barrier 3).
      const int h = et >> 3, half = (et >> 2) & 1, c = et & 3;
      const bool valid = t0 < p.Tq && h < p.HI;
      const bool quant = p.qI_bf16 != nullptr;
      const size_t row = ((size_t)b * p.Tq + t0) * p.HI + h;
      uint4 v = make_uint4(0, 0, 0, 0);
      uint32_t word = 0;
      int code = 0;
      if (valid) {
        if (quant) {
          v = __ldg(reinterpret_cast<const uint4*>(p.qI_bf16 + row * 64 + half * 32 + c * 8));
        } else {
          word = __ldg(reinterpret_cast<const uint32_t*>(p.qI + row * 32 + half * 16 + c * 4));
          code = __ldg(p.qI_sf + row * 2 + half);
        }
      }
      float wv = 0.f;
      if (et < HP && t0 < p.Tq && et < p.HI) wv = __ldg(p.w + ((size_t)b * p.Tq + t0) * p.HI + et);
      int pos = -1;
      if (et == 0 && t0 < p.Tq) pos = __ldg(p.q_pos + (size_t)b * p.Tq + t0);
      asm volatile("bar.arrive 3, %0;" ::"r"(32 + 32 * EPI) : "memory");
      if (quant) {
        float amax = bf16x8_amax(v);
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        code = mxfp4_scale_code(amax);
        word = mxfp4_encode8(v, e8m0_value(code));
        if (!valid) { word = 0; code = 0; }
      }
      const int code_other = __shfl_xor_sync(0xffffffffu, code, 4);
#pragma unroll
      for (int seg = 0; seg < 4; seg++) {
        const int n = seg * HP + h;
        const int cc = 2 * seg + half;
        *reinterpret_cast<uint32_t*>(sB + (n >> 3) * 1024 + (n & 7) * 128 +
                                     ((cc ^ (n & 7)) << 4) + c * 4) = word;
      }
      // the six zero chunks of each of the 64 rows
      for (int it = et; it < N * 6; it += ne) {
        const int n = it / 6, j = it % 6, seg = n / HP;
        const int cc = j < 2 * seg ? j : j + 2;
        *reinterpret_cast<uint4*>(sB + (n >> 3) * 1024 + (n & 7) * 128 + ((cc ^ (n & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
      }
      // query scales: word (n%32)*4 + n/32 of row n = (seg, h) holds (s_half0, s_half1);
      // the words of rows 64..127 are zero
      if (half == 0 && c == 0) {
#pragma unroll
        for (int seg = 0; seg < 4; seg++) {
          const int n = seg * HP + h;
          reinterpret_cast<uint32_t*>(sSFB)[(n & 31) * 4 + (n >> 5)] =
              uint32_t(code) | (uint32_t(code_other) << 8);
        }
      }
      if (et < 64) reinterpret_cast<uint32_t*>(sSFB)[4 * (et >> 1) + 2 + (et & 1)] = 0u;
      if (et < HP) sW[et] = wv;
      if (et == 0) sNvis[0] = pos < 0 ? 0 : min(p.Nc, (pos + 1) / p.m);
    } else {
      // Thread et owns the query-scale word et of the tcgen05.cp block (line et/4, word et%4),
      // i.e. operand row n = et/4 + 32*(et%4), and builds that row.  Every global load is
      // issued before the producer may start (named barrier 3), so these few loads are not
      // queued behind the key stream.
      const int n = (et >> 2) + 32 * (et & 3);
      const int seg = KIND == 2 ? n / HP : 0;   // packed rows: K-segment of this B row
      const int q = KIND == 2 ? 0 : n / HP, h = n % HP, t = t0 + q;
      const bool valid = et < 128 && n < N && t < p.Tq && h < p.HI;
      const bool quant = p.qI_bf16 != nullptr;
      const size_t row = ((size_t)b * p.Tq + t) * p.HI + h;
      uint4 v0[4], v1[4];
      uint4 pk0 = make_uint4(0, 0, 0, 0), pk1 = pk0;
      uint32_t s0 = 0, s1 = 0;
      if (valid) {
        if (quant) {
          const uint4* src = reinterpret_cast<const uint4*>(p.qI_bf16 + row * 64);
#pragma unroll
          for (int i = 0; i < 4; i++) { v0[i] = __ldg(src + i); v1[i] = __ldg(src + 4 + i); }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(p.qI + row * 32);
          pk0 = __ldg(src);
          pk1 = __ldg(src + 1);
          s0 = p.qI_sf[row * 2];
          s1 = p.qI_sf[row * 2 + 1];
        }
      }
      float wv = 0.f;
      if (et < QT * HP) {
        const int qw = et / HP, hw = et % HP, tw = t0 + qw;
        if (tw < p.Tq && hw < p.HI) wv = __ldg(p.w + ((size_t)b * p.Tq + tw) * p.HI + hw);
      }
      int pos = -1;
      if (et < QT && t0 + et < p.Tq) pos = __ldg(p.q_pos + (size_t)b * p.Tq + t0 + et);
      asm volatile("bar.arrive 3, %0;" ::"r"(32 + 32 * EPI) : "memory");
      if (valid && quant) {
        s0 = (uint32_t)mxfp4_encode32(v0, pk0);
        s1 = (uint32_t)mxfp4_encode32(v1, pk1);
      }
      if (et < 128 && n < N) {
        if (KIND == 1) {
          const int sw = (n & 7) >> 2;
          uint8_t* rowp = sB + (n >> 3) * 256 + (n & 7) * 32;
          *reinterpret_cast<uint4*>(rowp + ((0 ^ sw) << 4)) = pk0;
          *reinterpret_cast<uint4*>(rowp + ((1 ^ sw) << 4)) = pk1;
        } else {
          // 128-byte SW128 row: q_h's 32 bytes in chunks 2*seg, 2*seg+1, zeros elsewhere
          uint8_t* rowp = sB + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
          for (int c = 0; c < 8; c++) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(rowp + ((c ^ (n & 7)) << 4)) =
                c == 2 * seg ? pk0 : (c == 2 * seg + 1 ? pk1 : z);
          }
        }
      }
      if (et < 128) reinterpret_cast<uint32_t*>(sSFB)[et] = s0 | (s1 << 8);
      if (et < QT * HP) sW[et] = wv;
      if (et < QT) sNvis[et] = pos < 0 ? 0 : min(p.Nc, (pos + 1) / p.m);
    }
    if (KIND == 0) {
      for (int u = et; u < QT * HP; u += ne) {
        const int q = u / HP, h = u % HP, t = t0 + q;
        // (multi-tile prefill keeps w/2: its reduction forms w * relu(x) as (w/2) * (x + |x|))
        const float wv = (t < p.Tq && h < p.HI) ? p.w[((size_t)b * p.Tq + t) * p.HI + h] : 0.f;
        sW[u] = (TPS > 1 && QT > 1) ? 0.5f * wv : wv;
      }
      for (int q = et; q < QT; q += ne) {
        const int t = t0 + q;
        int nv = 0;
        if (t < p.Tq) {
          const int pos = p.q_pos[(size_t)b * p.Tq + t];
          nv = pos < 0 ? 0 : min(p.Nc, (pos + 1) / p.m);
        }
        sNvis[q] = nv;
      }
      asm volatile("bar.arrive 3, %0;" ::"r"(32 + 32 * EPI) : "memory");
    }
    fence_proxy_async_smem();
  }
  if (warp >= 1) asm volatile("bar.sync 2, %0;" ::"r"(32 + 32 * EPI) : "memory");
  const uint32_t tbase = *sTmem;
  const uint32_t sfa_t = tbase + Lay::ACC_COLS;
  const uint32_t sfb_t = tbase + Lay::ACC_COLS + 4 * Lay::SF_BLOCKS * TPS;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    asm volatile("bar.sync 3, %0;" ::"r"(32 + 32 * EPI) : "memory");  // prologue loads issued
    if (lane == 0) {
      // decode streams every key exactly once: keep it from displacing the scores in L2
      const uint64_t pol = l2_evict_first_policy();
      int issued = 0;
      for (int i = 0; i < nstages; i++) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.limit, sAbort)) {
          *sAbort = 1;
          report(p.status, HCL_ERR_TIMEOUT);
          break;
        }
        const int key0 = (kt0 + i * TPS) * Lay::TK;
        // packed rows: the stage's key scales are one contiguous run, copied untiled (its
        // length stops at the buffer's capacity; cap % 8 == 0 keeps it a multiple of 16 B)
        const uint32_t sf_bytes =
            KIND == 2 ? 2u * (uint32_t)min(TPS * Lay::TK, p.cap - key0) : TPS * Lay::SF_TILE;
        mbar_arrive_expect_tx(&full[s], TPS * Lay::A_TILE + sf_bytes);
#pragma unroll
        for (int r = 0; r < TPS * KEYS; r += Lay::BOX_ROWS) {
          if (KIND == 2)
            tma_load_3d_hint(sA + s * Lay::A_STAGE + r * Lay::ROWB, &tmK, &full[s], 0,
                             key0 / Lay::KPR + r, b, pol);
          else
            tma_load_3d(sA + s * Lay::A_STAGE + r * Lay::ROWB, &tmK, &full[s], 0,
                        key0 / Lay::KPR + r, b);
        }
        if (KIND == 1)
          tma_load_3d(sSFraw + s * TPS * 256, &tmSF, &full[s], 0, key0 / 8, b);
        if (KIND == 2)
          bulk_load_hint(sSFraw + s * TPS * Lay::SF_TILE, p.kI_sf + ((size_t)b * p.cap + key0) * 2,
                         sf_bytes, &full[s], pol);
        issued++;
      }
      // Drain: every issued copy has landed before the block may exit.
      for (int i = max(0, issued - STAGES); i < issued; i++)
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.limit, nullptr))
          report(p.status, HCL_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (KIND != 0 && lane == 0)
      tmem_cp_32x128b_x4(sfb_t, make_sdesc(smem_u32(sSFB), 16, 128, SMEM_SWIZZLE_NONE));
    for (int i = 0; i < nstages; i++) {
      const int s = i % STAGES;
      const int a = i % NACC;
      bool ok = mbar_wait(&full[s], (i / STAGES) & 1, p.limit, sAbort);
      ok = ok && mbar_wait(&acce[a], ((i / NACC) & 1) ^ 1, p.limit, sAbort);
      if (!__all_sync(0xffffffffu, ok)) {
        *sAbort = 1;
        report(p.status, HCL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      if (KIND == 1) {
        // E8M0 scales of the stage's key tiles: raw [128 rows x 2 B] per tile -> the
        // 32 x 16 B block layout (line r%32, word r/32, bytes 0..1) tcgen05.cp replicates.
#pragma unroll
        for (int t = 0; t < TPS; t++) {
          const uint16_t* raw = reinterpret_cast<const uint16_t*>(sSFraw + (s * TPS + t) * 256);
          const uint4 v = make_uint4(raw[lane], raw[lane + 32], raw[lane + 64], raw[lane + 96]);
          *reinterpret_cast<uint4*>(sSFexp + (s * TPS + t) * 512 + lane * 16) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (KIND == 2) {
        // packed rows: row r of a tile holds keys 4r..4r+3; k-step j needs key 4r+j's two
        // scales at (line r%32, word r/32) -- raw u16 index 4r+j
#pragma unroll
        for (int t = 0; t < TPS; t++) {
          const uint16_t* raw =
              reinterpret_cast<const uint16_t*>(sSFraw + (s * TPS + t) * Lay::SF_TILE);
#pragma unroll
          for (int j = 0; j < 4; j++) {
            const uint4 v = make_uint4(raw[4 * lane + j], raw[4 * (lane + 32) + j],
                                       raw[4 * (lane + 64) + j], raw[4 * (lane + 96) + j]);
            *reinterpret_cast<uint4*>(sSFexp + ((s * TPS + t) * 4 + j) * 512 + lane * 16) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t aB = smem_u32(sB);
#pragma unroll
        for (int t = 0; t < TPS; t++) {
          const uint32_t d = tbase + (a * TPS + t) * N;
          const uint32_t aA = smem_u32(sA + s * Lay::A_STAGE + t * Lay::A_TILE);
          if (KIND == 0) {
#pragma unroll
            for (int k = 0; k < 4; k++)
              umma_bf16(d, make_sdesc(aA + 32 * k, 16, 1024, SMEM_SWIZZLE_128B),
                        make_sdesc(aB + 32 * k, 16, 1024, SMEM_SWIZZLE_128B), idesc_bf16(KEYS, N),
                        k > 0 ? 1u : 0u);
          } else if (KIND == 2) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
              tmem_cp_32x128b_x4(sfa_t + 4 * (t * 4 + j),
                                 make_sdesc(smem_u32(sSFexp + ((s * TPS + t) * 4 + j) * 512), 16,
                                            128, SMEM_SWIZZLE_NONE));
              umma_mxf4(d, make_sdesc(aA + 32 * j, 16, 1024, SMEM_SWIZZLE_128B),
                        make_sdesc(aB + 32 * j, 16, 1024, SMEM_SWIZZLE_128B), idesc_mxf4(KEYS, N),
                        sfa_t + 4 * (t * 4 + j), sfb_t, j > 0 ? 1u : 0u);
            }
          } else {
            tmem_cp_32x128b_x4(sfa_t + 4 * t, make_sdesc(smem_u32(sSFexp + (s * TPS + t) * 512),
                                                         16, 128, SMEM_SWIZZLE_NONE));
            umma_mxf4(d, make_sdesc(aA, 16, 256, SMEM_SWIZZLE_32B),
                      make_sdesc(aB, 16, 256, SMEM_SWIZZLE_32B), idesc_mxf4(KEYS, N),
                      sfa_t + 4 * t, sfb_t, 0u);
          }
        }
        umma_commit(&empty[s]);
        umma_commit(&accf[a]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(drain);
    __syncwarp();
    if (!mbar_wait(drain, 0, p.limit, nullptr) && lane == 0) report(p.status, HCL_ERR_TIMEOUT);
  } else {
    // ---------------- epilogue ----------------
    // EPI/4 groups of four warps (one warp per TMEM lane quarter) split the tile's queries
    constexpr int NGRP = EPI / 4;
    static_assert(EPI % 4 == 0 && QT % NGRP == 0, "epilogue warps must split the queries evenly");
    constexpr int QPER = QT / NGRP;
    // queries per TMEM load batch (16 fp32 columns each): with 16 epilogue warps the register
    // budget is smaller, and four warps per scheduler hide the load latency instead
    constexpr int LDB = EPI >= 16 ? 2 : 4;
    constexpr bool ALL_AT_ONCE = QPER * TPS <= LDB;  // every column of a stage in one batch
    constexpr int QG = QPER < LDB ? QPER : LDB;      // otherwise: queries per load batch
    const int quarter = warp & 3;
    const int qbeg = ((warp - 2) / 4) * QPER;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;

    auto emit = [&](int tile, int q, const uint32_t (&r)[16]) {
      // ReLU-weighted head sum as two interleaved fp32 chains (paired FMA), the weights read
      // as four 16-byte vectors
      const float4* wq = reinterpret_cast<const float4*>(sW + q * HP);
      unsigned long long acc = 0ull;
#pragma unroll
      for (int h4 = 0; h4 < HP / 4; h4++) {
        const float4 wv = wq[h4];
        acc = fma2(pack2(wv.x, wv.y), pack2(fmaxf(__uint_as_float(r[4 * h4]), 0.f),
                                            fmaxf(__uint_as_float(r[4 * h4 + 1]), 0.f)), acc);
        acc = fma2(pack2(wv.z, wv.w), pack2(fmaxf(__uint_as_float(r[4 * h4 + 2]), 0.f),
                                            fmaxf(__uint_as_float(r[4 * h4 + 3]), 0.f)), acc);
      }
      const float s = __uint_as_float(uint32_t(acc)) + __uint_as_float(uint32_t(acc >> 32));
      const int t = t0 + q;
      const int key = tile * KEYS + quarter * 32 + lane;
      if (t < p.Tq && key < p.Nc) {
        const float v = key < sNvis[q] ? s : -INFINITY;
        const size_t o = ((size_t)b * p.Tq + t) * p.Nc + key;
        if (p.score_fmt == HCL_FP32) static_cast<float*>(p.scores)[o] = v;
        else static_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
      }
    };

    // packed rows (one query): lane r of the tile holds keys 4r..4r+3, stored as one vector
    auto emit4 = [&](int tile, const uint32_t (&r)[4][16]) {
      const int key = tile * Lay::TK + (quarter * 32 + lane) * 4;
      const int nv = sNvis[0];
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < HP; h++) s = fmaf(sW[h], fmaxf(__uint_as_float(r[j][h]), 0.f), s);
        v[j] = key + j < nv ? s : -INFINITY;
      }
      if (t0 >= p.Tq) return;
      if (p.gmax != nullptr) {
        // per 16-entry group (lanes 4q .. 4q+3 hold group key/16), as order-preserving keys of
        // the bf16 scores: the largest visible score, its position in the group (the lowest
        // on ties) and the second largest (equal to the largest when that repeats; 0 when
        // there is none).  The top-k's lower bound and its candidate list come from these.
        uint32_t m1 = 0u, m2 = 0u, a1 = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
          if (key + j < nv) {
            const uint32_t bits = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
            const uint32_t kk = bits ^ ((bits & 0x8000u) ? 0xFFFFu : 0x8000u);
            if (kk > m1) { m2 = m1; m1 = kk; a1 = uint32_t((lane & 3) * 4 + j); }
            else if (kk > m2) { m2 = kk; }
          }
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          const uint32_t n1 = __shfl_xor_sync(0xffffffffu, m1, o);
          const uint32_t n2 = __shfl_xor_sync(0xffffffffu, m2, o);
          const uint32_t b1 = __shfl_xor_sync(0xffffffffu, a1, o);
          const uint32_t second = max(min(m1, n1), max(m2, n2));
          if (n1 > m1 || (n1 == m1 && b1 < a1)) a1 = b1;
          m1 = max(m1, n1);
          m2 = second;
        }
        if ((lane & 3) == 0 && key < p.Nc) {
          const size_t gi = ((size_t)b * p.Tq + t0) * p.NG + (key >> 4);
          p.gmax[gi] = uint16_t(m1);
          p.g2nd[gi] = uint16_t(m2);
          p.garg[gi] = uint8_t(a1);
        }
      }
      const size_t o = ((size_t)b * p.Tq + t0) * p.Nc + key;
      if (p.vec_ok && key + 3 < p.Nc) {
        if (p.score_fmt == HCL_FP32) {
          *reinterpret_cast<float4*>(static_cast<float*>(p.scores) + o) =
              make_float4(v[0], v[1], v[2], v[3]);
        } else {
          __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
          __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
          uint2 u;
          u.x = *reinterpret_cast<uint32_t*>(&lo);
          u.y = *reinterpret_cast<uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.scores) + o) = u;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; j++) {
          if (key + j >= p.Nc) break;
          if (p.score_fmt == HCL_FP32) static_cast<float*>(p.scores)[o + j] = v[j];
          else static_cast<__nv_bfloat16*>(p.scores)[o + j] = __float2bfloat16_rn(v[j]);
        }
      }
    };

    // prefill with several key tiles per stage: this thread's queries are the same in every
    // stage, so their (halved) weights stay in registers, and so does the number of keys that
    // all of them see (lim)
    constexpr bool PRE_MT = KIND == 0 && TPS > 1 && QT > 1;
    float wreg[PRE_MT ? QPER : 1][16];
    int lim = p.Nc;
    if constexpr (PRE_MT) {
#pragma unroll
      for (int g = 0; g < QPER; g++) lim = min(lim, sNvis[qbeg + g]);
#pragma unroll
      for (int g = 0; g < QPER; g++)
#pragma unroll
        for (int h = 0; h < 16; h += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(sW + (qbeg + g) * HP + h);
          wreg[g][h] = w4.x; wreg[g][h + 1] = w4.y; wreg[g][h + 2] = w4.z; wreg[g][h + 3] = w4.w;
        }
    }

    for (int i = 0; i < nstages; i++) {
      const int a = i % NACC;
      bool ok = mbar_wait(&accf[a], (i / NACC) & 1, p.limit, sAbort);
      if (!__all_sync(0xffffffffu, ok)) {
        *sAbort = 1;
        report(p.status, HCL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int tile0 = kt0 + i * TPS;
      const uint32_t tacc = tbase + lane_off + a * TPS * N;
      if constexpr (KIND == 2) {
        uint32_t r[TPS][4][16];
#pragma unroll
        for (int t = 0; t < TPS; t++)
#pragma unroll
          for (int j = 0; j < 4; j++) tmem_ld16(tacc + t * N + j * HP, r[t][j]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&acce[a]);
#pragma unroll
        for (int t = 0; t < TPS; t++) emit4(tile0 + t, r[t]);
      } else if constexpr (KIND == 0 && TPS > 1 && QT > 1) {
        // prefill with several key tiles per stage: query by query, the weights (registers) are
        // applied to this thread's key in every tile of the stage (with 16 epilogue warps the
        // registers do not allow loading the next query's columns ahead; four warps per
        // scheduler hide the load latency instead).  A stage whose keys all of this warp's
        // queries see, with bf16 scores, takes a body without per-score checks.
        constexpr bool ILP2 = true;    // two accumulator chains per (query, tile)
        const int kw = tile0 * KEYS + quarter * 32;
        const bool bf = p.score_fmt != HCL_FP32;
        auto stage = [&](auto fast_c) {
          constexpr bool FAST = decltype(fast_c)::value;
#pragma unroll
          for (int g = 0; g < QPER; g++) {
            const int q = qbeg + g;
            uint32_t r[TPS][16];
#pragma unroll
            for (int t = 0; t < TPS; t++) tmem_ld16(tacc + t * N + q * HP, r[t]);
            tmem_ld_wait();
            if (g + 1 == QPER) {
              tc_fence_before();
              mbar_arrive(&acce[a]);
            }
            const size_t orow = ((size_t)b * p.Tq + t0 + q) * p.Nc;
#pragma unroll
            for (int t = 0; t < TPS; t++) {
              const float* wv = wreg[g];
              // w * relu(x) == (w/2) * (x + |x|) exactly (x + |x| is 2x or 0): an add with an
              // absolute-value operand on the FMA pipe instead of a max on the ALU pipe
              unsigned long long acc0 = 0ull, acc1 = 0ull;
#pragma unroll
              for (int h = 0; h < HP; h += 4) {
                const float x0 = __uint_as_float(r[t][h]), x1 = __uint_as_float(r[t][h + 1]);
                const float x2 = __uint_as_float(r[t][h + 2]), x3 = __uint_as_float(r[t][h + 3]);
                acc0 = fma2(pack2(wv[h], wv[h + 1]), pack2(x0 + fabsf(x0), x1 + fabsf(x1)), acc0);
                if (ILP2)
                  acc1 = fma2(pack2(wv[h + 2], wv[h + 3]), pack2(x2 + fabsf(x2), x3 + fabsf(x3)), acc1);
                else
                  acc0 = fma2(pack2(wv[h + 2], wv[h + 3]), pack2(x2 + fabsf(x2), x3 + fabsf(x3)), acc0);
              }
              const unsigned long long acc = ILP2 ? add2(acc0, acc1) : acc0;
              const float sc = __uint_as_float(uint32_t(acc)) + __uint_as_float(uint32_t(acc >> 32));
              const int key = (tile0 + t) * KEYS + quarter * 32 + lane;
              if constexpr (FAST) {
                static_cast<__nv_bfloat16*>(p.scores)[orow + key] = __float2bfloat16_rn(sc);
              } else if (t0 + q < p.Tq && key < p.Nc) {
                const float v = key < sNvis[q] ? sc : -INFINITY;
                if (!bf) static_cast<float*>(p.scores)[orow + key] = v;
                else static_cast<__nv_bfloat16*>(p.scores)[orow + key] = __float2bfloat16_rn(v);
              }
            }
          }
        };
        if (bf && kw + (TPS - 1) * KEYS + 32 <= lim) stage(std::integral_constant<bool, true>{});
        else stage(std::integral_constant<bool, false>{});
      } else if (ALL_AT_ONCE) {
        uint32_t r[TPS * QPER][16];
#pragma unroll
        for (int t = 0; t < TPS; t++)
#pragma unroll
          for (int g = 0; g < QPER; g++) tmem_ld16(tacc + t * N + (qbeg + g) * HP, r[t * QPER + g]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&acce[a]);
#pragma unroll
        for (int t = 0; t < TPS; t++)
#pragma unroll
          for (int g = 0; g < QPER; g++) emit(tile0 + t, qbeg + g, r[t * QPER + g]);
      } else {
#pragma unroll 1
        for (int t = 0; t < TPS; t++) {
#pragma unroll 1
          for (int q0 = 0; q0 < QPER; q0 += QG) {
            uint32_t r[QG][16];
#pragma unroll
            for (int g = 0; g < QG; g++) tmem_ld16(tacc + t * N + (qbeg + q0 + g) * HP, r[g]);
            tmem_ld_wait();
            if (t == TPS - 1 && q0 + QG >= QPER) {
              tc_fence_before();
              mbar_arrive(&acce[a]);
            }
#pragma unroll
            for (int g = 0; g < QG; g++) emit(tile0 + t, qbeg + q0 + g, r[g]);
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Lay::TMEM_COLS);
  }
}

int smem_per_sm() {
  int dev = 0, b = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&b, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  return b > 0 ? b : 228 * 1024;
}

template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
hcl_status_t run(const IndexerArgs& a, const void* qI_bf16, const CUtensorMap& tmK,
                 const CUtensorMap& tmSF, cudaStream_t st, int min_smem) {
  using Lay = IdxLayout<KIND, QT, TPS, STAGES, NACC, EPI>;
  auto kern = indexer_kernel<KIND, QT, TPS, STAGES, NACC, EPI>;
  const int smem = std::max(Lay::BYTES + 1024, min_smem);
  hcl_status_t ea = set_kernel_attrs(reinterpret_cast<const void*>(kern), smem, false);
  if (ea != HCL_OK) return ea;
  // blocks per SM: shared memory (+1 KB reserved per block), TMEM (512 columns), threads
  int per_sm = smem_per_sm() / (smem + 1024);
  per_sm = std::max(1, std::min({per_sm, int(512 / Lay::TMEM_COLS), 2048 / Lay::NT}));
  IdxParams p;
  p.qI = static_cast<const uint8_t*>(a.qI);
  p.qI_sf = static_cast<const uint8_t*>(a.qI_sf);
  p.qI_bf16 = static_cast<const __nv_bfloat16*>(qI_bf16);
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.scores = a.scores;
  p.score_fmt = a.score_fmt;
  p.kI_sf = static_cast<const uint8_t*>(a.kI_sf);
  p.B = a.B; p.Tq = a.Tq; p.HI = a.HI; p.Nc = a.Nc; p.m = a.m; p.cap = a.kI_cap;
  p.vec_ok = (a.Nc % 4 == 0) && (reinterpret_cast<uintptr_t>(a.scores) % 16 == 0);
  p.gmax = (KIND == 2 && a.score_fmt == HCL_BF16) ? a.gmax : nullptr;
  p.g2nd = a.g2nd;
  p.garg = a.garg;
  p.NG = gmax_row_stride(a.Nc);
  p.n_qt = (a.Tq + QT - 1) / QT;
  p.n_kt = (a.Nc + Lay::TK - 1) / Lay::TK;
  // key chunks per (sequence, query tile): as many as fill the co-resident slots without
  // spilling into a second wave
  const long long target = (long long)num_sms() * per_sm;
  const long long base = (long long)a.B * p.n_qt;
  const int n_stages_total = (p.n_kt + TPS - 1) / TPS;
  int n_kc = (int)std::max(1LL, std::min<long long>(n_stages_total, target / base));
  if (base > target) {
    // more (query tile) blocks than slots: split the keys so that the last wave is nearly
    // full, as long as every block keeps >= 32 stages to amortise its prologue
    for (int c = 1; c <= 8 && n_stages_total / c >= 32; c++) {
      const long long blocks = base * c, waves = (blocks + target - 1) / target;
      if (blocks * 100 >= waves * target * 95) { n_kc = c; break; }
    }
  }
  const int st_per_chunk = (n_stages_total + n_kc - 1) / n_kc;
  p.kt_per_chunk = st_per_chunk * TPS;
  p.n_kc = (p.n_kt + p.kt_per_chunk - 1) / p.kt_per_chunk;
  p.status = a.status;
  p.limit = wait_limit_cycles();
  const long long grid = base * p.n_kc;
  if (grid == 0) return HCL_OK;
  return check_cuda(launch_pdl(kern, dim3((unsigned)grid), dim3(Lay::NT), (size_t)smem, st, 1,
                               tmK, tmSF, p),
                    "index_scores launch");
}

hcl_status_t make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, cuuint64_t d0,
                      cuuint64_t d1, cuuint64_t d2, cuuint64_t s1, cuuint64_t s2, cuuint32_t b0,
                      cuuint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return fail(HCL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HCL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return HCL_OK;
}

// Decode configurations: stage = TPS tiles; box rows = min(256, TPS*128).
constexpr int DEC_BF16_TPS = 2;
// bf16 prefill: 8 queries x 16 heads (N = 128) against two 128-key tiles per stage
constexpr int PRE_BF16_TPS = 2;

}  // namespace

hcl_status_t launch_indexer_q(const IndexerArgs& a, const void* qI_bf16, cudaStream_t st) {
  if (a.B == 0 || a.Tq == 0 || a.Nc == 0) return HCL_OK;
  CUtensorMap tmK, tmSF;
  memset(&tmSF, 0, sizeof(tmSF));
  hcl_status_t e;
  const bool mx = a.op_fmt == HCL_MXFP4;
  const bool decode = a.Tq <= 2;
  if (!mx) {
    const cuuint32_t rows = std::min(256, (decode ? DEC_BF16_TPS : PRE_BF16_TPS) * KEYS);
    e = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.kI, 64, a.kI_cap, a.B, 128,
                 (cuuint64_t)a.kI_cap * 128, 64, rows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != HCL_OK) return e;
    if (decode) return run<0, 1, DEC_BF16_TPS, 3, 3, 4>(a, nullptr, tmK, tmSF, st, 0);
    return run<0, 8, PRE_BF16_TPS, 4, 2, 16>(a, nullptr, tmK, tmSF, st, 0);
  }
  if (decode) {
    // packed rows: [B, cap/4, 128 B] (four keys per row), 16 KB boxes with SW128; the key
    // scales are fetched by untiled bulk copies
    e = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.kI, 128, a.kI_cap / 4, a.B, 128,
                 (cuuint64_t)a.kI_cap * 32, 128, KEYS, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != HCL_OK) return e;
    return run<2, 1, 1, 5, 3, 4>(a, qI_bf16, tmK, tmSF, st, 0);
  }
  e = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.kI, 32, a.kI_cap, a.B, 32,
               (cuuint64_t)a.kI_cap * 32, 32, KEYS, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != HCL_OK) return e;
  e = make_map(&tmSF, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.kI_sf, 16, a.kI_cap / 8, a.B, 16,
               (cuuint64_t)a.kI_cap * 2, 16, KEYS / 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != HCL_OK) return e;
  return run<1, 8, 1, 8, 2, 8>(a, qI_bf16, tmK, tmSF, st, 120 * 1024);
}

hcl_status_t launch_indexer(const IndexerArgs& a, cudaStream_t st) {
  return launch_indexer_q(a, nullptr, st);
}

}  // namespace hcl
