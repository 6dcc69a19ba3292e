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
  const __nv_bfloat16* qI_bf16;  // bf16 index queries to quantise in-kernel (MXFP4 keys), or null
  const float* w;
  const int32_t* q_pos;
  void* scores;
  int score_fmt;
  int B, Tq, HI, Nc, m;
  int n_qt, n_kt, n_kc, kt_per_chunk;
  int32_t* status;
  long long limit;
};

__host__ __device__ constexpr uint32_t tmem_cols_for(uint32_t need) {
  uint32_t c = 32;
  while (c < need) c <<= 1;
  return c;
}

template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
struct IdxLayout {
  static constexpr int N = QT * HP;
  static constexpr int ROWB = KIND == 0 ? 128 : 32;       // bytes per K-row of an operand
  static constexpr int A_TILE = KEYS * ROWB;
  static constexpr int A_STAGE = TPS * A_TILE;
  static constexpr int SF_TILE = KIND == 1 ? KEYS * 2 : 0;
  static constexpr int BOX_ROWS = (TPS * KEYS) < 256 ? (TPS * KEYS) : 256;
  static constexpr int B_BYTES = ((N * ROWB + 1023) / 1024) * 1024;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr int OFF_SFRAW = OFF_B + B_BYTES;
  static constexpr int OFF_SFEXP = OFF_SFRAW + (KIND == 1 ? STAGES * TPS * 256 : 0);
  static constexpr int OFF_SFB = OFF_SFEXP + (KIND == 1 ? STAGES * TPS * 512 : 0);
  static constexpr int OFF_W = OFF_SFB + (KIND == 1 ? 512 : 0);
  static constexpr int OFF_NVIS = OFF_W + QT * HP * 4;
  static constexpr int OFF_BAR = ((OFF_NVIS + QT * 4 + 7) / 8) * 8;
  static constexpr int NBAR = 2 * STAGES + 2 * NACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int NT = 64 + 32 * EPI;
  static constexpr int ACC_COLS = NACC * TPS * N;
  static constexpr uint32_t TMEM_COLS = tmem_cols_for(ACC_COLS + (KIND == 1 ? 4 * TPS + 4 : 0));
};

__device__ __forceinline__ void epi_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
__global__ void __launch_bounds__(64 + 32 * EPI, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmSF,
                   IdxParams p) {
  using Lay = IdxLayout<KIND, QT, TPS, STAGES, NACC, EPI>;
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
  // everything above touches no global memory; the rest may read what the previous kernel
  // in the stream wrote
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
    } else {
      for (int u = et; u < 128; u += ne) reinterpret_cast<uint32_t*>(sSFB)[u] = 0u;
      epi_bar(ne);
      for (int n = et; n < N; n += ne) {
        const int q = n / HP, h = n % HP, t = t0 + q;
        uint4 pk0 = make_uint4(0, 0, 0, 0), pk1 = pk0;
        uint32_t s0 = 0, s1 = 0;
        if (t < p.Tq && h < p.HI) {
          const size_t row = ((size_t)b * p.Tq + t) * p.HI + h;
          if (p.qI_bf16 != nullptr) {
            const uint4* src = reinterpret_cast<const uint4*>(p.qI_bf16 + row * 64);
            uint4 v0[4], v1[4];
#pragma unroll
            for (int i = 0; i < 4; i++) { v0[i] = __ldg(src + i); v1[i] = __ldg(src + 4 + i); }
            s0 = (uint32_t)mxfp4_encode32(v0, pk0);
            s1 = (uint32_t)mxfp4_encode32(v1, pk1);
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(p.qI + row * 32);
            pk0 = __ldg(src);
            pk1 = __ldg(src + 1);
            s0 = p.qI_sf[row * 2];
            s1 = p.qI_sf[row * 2 + 1];
          }
        }
        const int sw = (n & 7) >> 2;
        uint8_t* rowp = sB + (n >> 3) * 256 + (n & 7) * 32;
        *reinterpret_cast<uint4*>(rowp + ((0 ^ sw) << 4)) = pk0;
        *reinterpret_cast<uint4*>(rowp + ((1 ^ sw) << 4)) = pk1;
        sSFB[(n & 31) * 16 + (n >> 5) * 4 + 0] = uint8_t(s0);
        sSFB[(n & 31) * 16 + (n >> 5) * 4 + 1] = uint8_t(s1);
      }
    }
    for (int u = et; u < QT * HP; u += ne) {
      const int q = u / HP, h = u % HP, t = t0 + q;
      sW[u] = (t < p.Tq && h < p.HI) ? p.w[((size_t)b * p.Tq + t) * p.HI + h] : 0.f;
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
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const uint32_t sfa_t = tbase + Lay::ACC_COLS;
  const uint32_t sfb_t = tbase + Lay::ACC_COLS + 4 * TPS;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nstages; i++) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.limit, sAbort)) {
          *sAbort = 1;
          report(p.status, HCL_ERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&full[s], TPS * (Lay::A_TILE + Lay::SF_TILE));
        const int row0 = (kt0 + i * TPS) * KEYS;
#pragma unroll
        for (int r = 0; r < TPS * KEYS; r += Lay::BOX_ROWS)
          tma_load_3d(sA + s * Lay::A_STAGE + r * Lay::ROWB, &tmK, &full[s], 0, row0 + r, b);
        if (KIND == 1)
          tma_load_3d(sSFraw + s * TPS * 256, &tmSF, &full[s], 0, row0 / 8, b);
        issued++;
      }
      // Drain: every issued copy has landed before the block may exit.
      for (int i = max(0, issued - STAGES); i < issued; i++)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.limit, nullptr);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (KIND == 1 && lane == 0)
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
    mbar_wait(drain, 0, p.limit, nullptr);
  } else {
    // ---------------- epilogue ----------------
    constexpr int QPER = EPI >= 8 ? QT / 2 : QT;
    constexpr bool ALL_AT_ONCE = QPER * TPS <= 4;   // every column of a stage in one batch
    constexpr int QG = QPER < 4 ? QPER : 4;          // otherwise: queries per load batch
    const int quarter = warp & 3;
    const int qbeg = ((warp - 2) / 4) * QPER;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;

    auto emit = [&](int tile, int q, const uint32_t (&r)[16]) {
      const float* wq = sW + q * HP;
      float s = 0.f;
#pragma unroll
      for (int h = 0; h < HP; h++) s = fmaf(wq[h], fmaxf(__uint_as_float(r[h]), 0.f), s);
      const int t = t0 + q;
      const int key = tile * KEYS + quarter * 32 + lane;
      if (t < p.Tq && key < p.Nc) {
        const float v = key < sNvis[q] ? s : -INFINITY;
        const size_t o = ((size_t)b * p.Tq + t) * p.Nc + key;
        if (p.score_fmt == HCL_FP32) static_cast<float*>(p.scores)[o] = v;
        else static_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
      }
    };

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
      if (ALL_AT_ONCE) {
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
  static int v = 0;
  if (v == 0) {
    int dev = 0, b = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&b, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    v = b > 0 ? b : 228 * 1024;
  }
  return v;
}

template <int KIND, int QT, int TPS, int STAGES, int NACC, int EPI>
hcl_status_t run(const IndexerArgs& a, const void* qI_bf16, const CUtensorMap& tmK,
                 const CUtensorMap& tmSF, cudaStream_t st, int min_smem) {
  using Lay = IdxLayout<KIND, QT, TPS, STAGES, NACC, EPI>;
  auto kern = indexer_kernel<KIND, QT, TPS, STAGES, NACC, EPI>;
  const int smem = std::max(Lay::BYTES + 1024, min_smem);
  static int configured_smem = -1;  // per instantiation
  if (configured_smem != smem) {
    hcl_status_t e = check_cuda(
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
        "indexer smem attribute");
    if (e != HCL_OK) return e;
    configured_smem = smem;
  }
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
  p.B = a.B; p.Tq = a.Tq; p.HI = a.HI; p.Nc = a.Nc; p.m = a.m;
  p.n_qt = (a.Tq + QT - 1) / QT;
  p.n_kt = (a.Nc + KEYS - 1) / KEYS;
  const long long target = (long long)num_sms() * per_sm;
  const long long base = (long long)a.B * p.n_qt;
  const int n_stages_total = (p.n_kt + TPS - 1) / TPS;
  int n_kc = (int)std::max(1LL, std::min<long long>(n_stages_total, (target + base - 1) / base));
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
constexpr int DEC_BF16_TPS = 2, DEC_MX_TPS = 4;

}  // namespace

hcl_status_t launch_indexer_q(const IndexerArgs& a, const void* qI_bf16, cudaStream_t st) {
  if (a.B == 0 || a.Tq == 0 || a.Nc == 0) return HCL_OK;
  CUtensorMap tmK, tmSF;
  memset(&tmSF, 0, sizeof(tmSF));
  hcl_status_t e;
  const bool mx = a.op_fmt == HCL_MXFP4;
  const bool decode = a.Tq <= 2;
  if (!mx) {
    const cuuint32_t rows = decode ? std::min(256, DEC_BF16_TPS * KEYS) : KEYS;
    e = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.kI, 64, a.kI_cap, a.B, 128,
                 (cuuint64_t)a.kI_cap * 128, 64, rows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != HCL_OK) return e;
    if (decode) return run<0, 1, DEC_BF16_TPS, 3, 3, 4>(a, nullptr, tmK, tmSF, st, 0);
    return run<0, 16, 1, 4, 2, 8>(a, nullptr, tmK, tmSF, st, 120 * 1024);
  }
  const int tps = decode ? DEC_MX_TPS : 1;
  const cuuint32_t rows = std::min(256, tps * KEYS);
  e = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.kI, 32, a.kI_cap, a.B, 32,
               (cuuint64_t)a.kI_cap * 32, 32, rows, CU_TENSOR_MAP_SWIZZLE_32B);
  if (e != HCL_OK) return e;
  e = make_map(&tmSF, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.kI_sf, 16, a.kI_cap / 8, a.B, 16,
               (cuuint64_t)a.kI_cap * 2, 16, tps * KEYS / 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != HCL_OK) return e;
  if (decode) return run<1, 1, DEC_MX_TPS, 5, 3, 4>(a, qI_bf16, tmK, tmSF, st, 0);
  return run<1, 8, 1, 8, 2, 8>(a, qI_bf16, tmK, tmSF, st, 120 * 1024);
}

hcl_status_t launch_indexer(const IndexerArgs& a, cudaStream_t st) {
  return launch_indexer_q(a, nullptr, st);
}

}  // namespace hcl
