// api.cu -- the extern "C" boundary of libhcl: argument validation, error reporting and the
// composition of the hot-path steps.  Every entry point validates on the host and enqueues
// nothing when it returns an error.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace hcl {

static thread_local char g_err[512] = "";

hcl_status_t fail(hcl_status_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

hcl_status_t check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HCL_OK;
  return fail(HCL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

hcl_status_t check_launch(const char* what) { return check_cuda(cudaGetLastError(), what); }

static int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = current_device();
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

static long long clock_khz() {
  static long long cache[64] = {0};
  int dev = current_device();
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int khz = 0;
    cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
    cache[dev] = khz > 0 ? khz : 2000000;
  }
  return cache[dev];
}

long long wait_limit_cycles() { return clock_khz() * 1000LL; }  // about one second

unsigned long long current_ctx_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext c = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  return get_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

hcl_status_t set_kernel_attrs(const void* kern, int smem, bool nonportable_cluster) {
  // The maximum dynamic shared memory is one value per kernel and context: it is only ever
  // raised (a smaller later request must not lower the limit a larger launch relies on).
  static std::mutex mu;
  static std::map<std::pair<const void*, unsigned long long>, std::pair<int, bool>> done;
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx != 0) {
    auto it = done.find(std::make_pair(kern, ctx));
    if (it != done.end() && it->second.first >= smem && (it->second.second || !nonportable_cluster))
      return HCL_OK;
  }
  int want = smem;
  bool cluster = nonportable_cluster;
  if (ctx != 0) {
    auto it = done.find(std::make_pair(kern, ctx));
    if (it != done.end()) {
      want = std::max(want, it->second.first);
      cluster = cluster || it->second.second;
    }
  }
  hcl_status_t e = check_cuda(
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want),
      "kernel shared-memory attribute");
  if (e != HCL_OK) return e;
  if (cluster) {
    e = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1),
                   "kernel cluster attribute");
    if (e != HCL_OK) return e;
  }
  // the attribute call makes a context current if none was; record under its id
  const unsigned long long now = current_ctx_id();
  if (now != 0) done[std::make_pair(kern, now)] = std::make_pair(want, cluster);
  return HCL_OK;
}

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

namespace {

__global__ void selftest_wait_kernel(int32_t* status, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up and report.
  if (!mbar_wait(&bar, 0, limit, nullptr)) report(status, HCL_ERR_TIMEOUT);
}

}  // namespace

hcl_status_t launch_selftest_wait(int32_t* status, int limit_us, cudaStream_t st) {
  const long long limit = clock_khz() * (long long)limit_us / 1000LL;
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit);
  return check_launch("selftest");
}

}  // namespace hcl

using namespace hcl;

#define HCL_REQUIRE(cond, ...)                                       \
  do {                                                               \
    if (!(cond)) return fail(HCL_ERR_INVALID_ARG, __VA_ARGS__);      \
  } while (0)

static cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

static hcl_status_t check_kv(const hcl_kv_t* kv, int d, const char* name) {
  HCL_REQUIRE(kv != nullptr, "%s: descriptor is NULL", name);
  HCL_REQUIRE(kv->cap > 0, "%s: cap must be positive", name);
  HCL_REQUIRE(kv->data != nullptr && aligned16(kv->data), "%s: data must be 16-byte aligned", name);
  if (kv->fmt == HCL_FP8SPLIT) {
    HCL_REQUIRE(kv->scale != nullptr && kv->rope != nullptr && aligned16(kv->rope),
                "%s: FP8SPLIT needs scale and 16-byte aligned rope", name);
  } else {
    HCL_REQUIRE(kv->fmt == HCL_BF16, "%s: fmt must be HCL_BF16 or HCL_FP8SPLIT", name);
  }
  (void)d;
  return HCL_OK;
}

extern "C" {

const char* hcl_version(void) { return "libhcl 0.1 (sm_100a)"; }
const char* hcl_last_error(void) { return g_err; }

static hcl_status_t compress_common(const void* kv, const void* gate, const float* bias, int B,
                                    int L, int d, int m, int overlap, int e0, int e1, void* out,
                                    int out_fmt, int out_cap, const float* gamma, float eps,
                                    void* stream, int max_m) {
  HCL_REQUIRE(B >= 0 && L >= 0, "B and L must be non-negative");
  HCL_REQUIRE(d > 0 && d % 8 == 0 && d <= 1024, "d must be a positive multiple of 8, <= 1024");
  HCL_REQUIRE(m >= 1 && m <= max_m, "m must be in [1, %d]", max_m);
  const long long n_ent = (L + (long long)m - 1) / m;
  HCL_REQUIRE(0 <= e0 && e0 <= e1 && e1 <= n_ent && e1 <= out_cap,
              "need 0 <= entry_begin <= entry_end <= min(ceil(L/m)=%lld, out_cap=%d)", n_ent,
              out_cap);
  HCL_REQUIRE(out_fmt == HCL_FP32 || out_fmt == HCL_BF16, "out_fmt must be HCL_FP32 or HCL_BF16");
  if (gamma != nullptr) {
    HCL_REQUIRE(eps > 0.f && eps < 1e30f, "eps must be a positive number");
    // the RMSNorm reduction runs over the d/8 threads of an entry (a power of two <= 32) or,
    // for HCA with d/8 dividing 256, over a block
    const int G = d / 8;
    const bool small = overlap || 256 % G != 0;
    if (small && (G > 32 || (G & (G - 1)) != 0))
      return fail(HCL_ERR_UNSUPPORTED, "RMSNorm epilogue needs d/8 a power of two <= 32 (d=%d)", d);
  }
  if (e1 == e0 || B == 0) return HCL_OK;
  HCL_REQUIRE(kv && gate && bias && out, "NULL pointer");
  HCL_REQUIRE(aligned16(kv) && aligned16(gate) && aligned16(out), "kv, gate, out must be 16-byte aligned");
  return launch_compress(kv, gate, bias, B, L, d, m, overlap, e0, e1, out, out_fmt, out_cap,
                         gamma, eps, as_stream(stream));
}

hcl_status_t hcl_csa_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                              int d, int m, int entry_begin, int entry_end, void* out,
                              int out_fmt, int out_cap, const float* gamma, float eps,
                              void* stream) {
  return compress_common(kv, gate, bias, B, L, d, m, 1, entry_begin, entry_end, out, out_fmt,
                         out_cap, gamma, eps, stream, 64);
}

hcl_status_t hcl_hca_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                              int d, int m, int entry_begin, int entry_end, void* out,
                              int out_fmt, int out_cap, const float* gamma, float eps,
                              void* stream) {
  return compress_common(kv, gate, bias, B, L, d, m, 0, entry_begin, entry_end, out, out_fmt,
                         out_cap, gamma, eps, stream, 1024);
}

hcl_status_t hcl_quant_kv_fp8(const void* kv, int64_t rows, int d, void* nope, float* scale,
                              void* rope, void* stream) {
  HCL_REQUIRE(rows >= 0, "rows must be non-negative");
  HCL_REQUIRE(d >= 16 && d <= 256 && (d & (d - 1)) == 0, "d must be a power of two in [16, 256]");
  if (rows == 0) return HCL_OK;
  HCL_REQUIRE(kv && nope && scale && rope, "NULL pointer");
  HCL_REQUIRE(aligned16(kv) && aligned16(rope) && ((uintptr_t)nope & 7) == 0,
              "kv, rope must be 16-byte aligned and nope 8-byte aligned");
  return launch_quant_kv_fp8(kv, rows, d, nope, scale, rope, as_stream(stream));
}

hcl_status_t hcl_quant_mxfp4(const void* x, int64_t rows, int cols, void* packed, void* e8m0,
                             void* stream) {
  HCL_REQUIRE(rows >= 0, "rows must be non-negative");
  HCL_REQUIRE(cols > 0 && cols % 32 == 0, "cols must be a positive multiple of 32");
  if (rows == 0) return HCL_OK;
  HCL_REQUIRE(x && packed && e8m0, "NULL pointer");
  HCL_REQUIRE(aligned16(x) && aligned16(packed), "x and packed must be 16-byte aligned");
  return launch_quant_mxfp4(x, rows, cols, packed, e8m0, as_stream(stream));
}

// Validation + launch of the indexer.  qI_bf16 (MXFP4 keys only): the bf16 index query, to be
// quantised inside the indexer instead of taking pre-quantised qI / qI_sf.
static hcl_status_t index_scores_impl(int op_fmt, const void* qI, const void* qI_sf,
                                      const void* qI_bf16, const float* w, const void* kI,
                                      const void* kI_sf, int B, int Tq, int HI, int dI, int Nc,
                                      int kI_cap, const int32_t* q_pos, int m, void* scores,
                                      int score_fmt, int32_t* status, void* stream,
                                      uint16_t* gmax = nullptr, uint16_t* g2nd = nullptr,
                                      uint8_t* garg = nullptr) {
  HCL_REQUIRE(op_fmt == HCL_BF16 || op_fmt == HCL_MXFP4, "op_fmt must be HCL_BF16 or HCL_MXFP4");
  HCL_REQUIRE(score_fmt == HCL_FP32 || score_fmt == HCL_BF16, "score_fmt must be HCL_FP32 or HCL_BF16");
  HCL_REQUIRE(B >= 0 && Tq >= 0 && Nc >= 0, "negative size");
  if (dI != 64) return fail(HCL_ERR_UNSUPPORTED, "only dI == 64 is supported (got %d)", dI);
  HCL_REQUIRE(HI >= 1 && HI <= 16, "HI must be in [1, 16]");
  HCL_REQUIRE(m >= 1, "m must be >= 1");
  HCL_REQUIRE(Nc <= kI_cap, "Nc must be <= kI_cap");
  if (op_fmt == HCL_MXFP4) HCL_REQUIRE(kI_cap % 8 == 0, "MXFP4 keys need kI_cap % 8 == 0");
  if ((long long)B * Tq * Nc == 0) return HCL_OK;
  const void* q_any = qI_bf16 ? qI_bf16 : qI;
  HCL_REQUIRE(q_any && w && kI && q_pos && scores, "NULL pointer");
  HCL_REQUIRE(aligned16(q_any) && aligned16(kI), "qI and kI must be 16-byte aligned");
  if (op_fmt == HCL_MXFP4)
    HCL_REQUIRE((qI_bf16 || qI_sf) && kI_sf && aligned16(kI_sf),
                "MXFP4 needs 16-byte aligned scale arrays");
  IndexerArgs a{op_fmt, qI, qI_sf, w, kI, kI_sf, B, Tq, HI, dI, Nc, kI_cap, q_pos, m, scores,
                score_fmt, status, gmax, g2nd, garg};
  return launch_indexer_q(a, qI_bf16, as_stream(stream));
}

hcl_status_t hcl_csa_index_scores(int op_fmt, const void* qI, const void* qI_sf, const float* w,
                                  const void* kI, const void* kI_sf, int B, int Tq, int HI,
                                  int dI, int Nc, int kI_cap, const int32_t* q_pos, int m,
                                  void* scores, int score_fmt, int32_t* status, void* stream) {
  return index_scores_impl(op_fmt, qI, qI_sf, nullptr, w, kI, kI_sf, B, Tq, HI, dI, Nc, kI_cap,
                           q_pos, m, scores, score_fmt, status, stream);
}

size_t hcl_csa_topk_workspace_bytes(int B, int Tq, int Nc, int k, int score_fmt) {
  return topk_workspace_bytes(B, Tq, Nc, k, score_fmt);
}

static hcl_status_t topk_common(const void* scores, int score_fmt, int B, int Tq, int Nc,
                               const int32_t* q_pos, int m, int k, int32_t* idx, void* ws,
                               size_t ws_bytes, int32_t* status, void* stream, int prewait) {
  HCL_REQUIRE(score_fmt == HCL_FP32 || score_fmt == HCL_BF16, "score_fmt must be HCL_FP32 or HCL_BF16");
  HCL_REQUIRE(B >= 0 && Tq >= 0 && Nc >= 0, "negative size");
  HCL_REQUIRE(k >= 1 && k <= 4096, "k must be in [1, 4096]");
  HCL_REQUIRE(Nc <= (1 << 22), "Nc must be <= 2^22");
  HCL_REQUIRE(m >= 1, "m must be >= 1");
  HCL_REQUIRE(ws_bytes >= topk_workspace_bytes(B, Tq, Nc, k, score_fmt), "workspace too small");
  if ((long long)B * Tq == 0) return HCL_OK;
  HCL_REQUIRE(q_pos && idx && (scores || Nc == 0), "NULL pointer");
  TopkArgs a{scores, score_fmt, B, Tq, Nc, q_pos, m, k, idx, status, prewait};
  return launch_topk(a, ws, ws_bytes, as_stream(stream));
}

hcl_status_t hcl_csa_topk(const void* scores, int score_fmt, int B, int Tq, int Nc,
                          const int32_t* q_pos, int m, int k, int32_t* idx, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream) {
  return topk_common(scores, score_fmt, B, Tq, Nc, q_pos, m, k, idx, ws, ws_bytes, status, stream,
                     0);
}

static hcl_status_t attn_common(int mode, const void* q, int B, int Tq, int H, int d,
                                const hcl_kv_t* comp, int n_comp, int mh, const int32_t* idx,
                                int k, const hcl_kv_t* raw, int L, int W, const int32_t* q_pos,
                                float scale, const float* sink, const float* q_gamma,
                                float q_eps, void* out, float* lse, void* ws, size_t ws_bytes,
                                int32_t* status, void* stream, int prewait = 0) {
  HCL_REQUIRE(B >= 0 && Tq >= 0, "negative size");
  if (d != 128) return fail(HCL_ERR_UNSUPPORTED, "only d == 128 is supported (got %d)", d);
  HCL_REQUIRE(H >= 1 && H <= 128, "H must be in [1, 128]");
  HCL_REQUIRE(W >= 0 && n_comp >= 0 && L >= 0, "negative size");
  if (mode == 0) HCL_REQUIRE(k >= 0 && (k == 0 || idx != nullptr), "k must be >= 0 with idx given");
  else HCL_REQUIRE(mh >= 1, "mh must be >= 1");
  if ((long long)B * Tq == 0) return HCL_OK;
  HCL_REQUIRE(q && out && q_pos, "NULL pointer");
  if (q_gamma != nullptr) HCL_REQUIRE(q_eps > 0.f && q_eps < 1e30f, "q_eps must be a positive number");
  HCL_REQUIRE(aligned16(q) && aligned16(out), "q and out must be 16-byte aligned");
  hcl_status_t e = check_kv(comp, d, mode == 0 ? "kvc" : "kvh");
  if (e != HCL_OK) return e;
  e = check_kv(raw, d, "raw");
  if (e != HCL_OK) return e;
  HCL_REQUIRE(comp->fmt == raw->fmt, "compressed and raw stores must share one format");
  HCL_REQUIRE(comp->cap >= n_comp || mode == 0, "kvh cap must be >= Nh");
  const size_t need = hcl::attn_workspace_bytes(mode, B, Tq, H, mode == 0 ? k : n_comp, W);
  HCL_REQUIRE(ws_bytes >= need, "workspace too small: need %zu bytes", need);
  AttnArgs a;
  a.mode = mode; a.q = q; a.B = B; a.Tq = Tq; a.H = H; a.d = d;
  a.comp = *comp; a.n_comp = n_comp; a.mh = mh; a.idx = idx; a.k = k;
  a.raw = *raw; a.L = L; a.W = W; a.q_pos = q_pos; a.scale = scale; a.sink = sink;
  a.out = out; a.lse = lse; a.status = status; a.prewait = prewait;
  a.q_gamma = q_gamma; a.q_eps = q_eps;
  return launch_attn(a, ws, ws_bytes, as_stream(stream));
}

size_t hcl_csa_sparse_attn_workspace_bytes(int B, int Tq, int H, int k, int W) {
  return hcl::attn_workspace_bytes(0, B, Tq, H, k, W);
}

hcl_status_t hcl_csa_sparse_attn(const void* q, int B, int Tq, int H, int d, const hcl_kv_t* kvc,
                                 int Nc, const int32_t* idx, int k, const hcl_kv_t* raw, int L,
                                 int W, const int32_t* q_pos, float scale, const float* sink,
                                 const float* q_gamma, float q_eps, void* out, float* lse,
                                 void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return attn_common(0, q, B, Tq, H, d, kvc, Nc, 1, idx, k, raw, L, W, q_pos, scale, sink,
                     q_gamma, q_eps, out, lse, ws, ws_bytes, status, stream);
}

// The CSA attention with its split-KV partials in the library's fixed scratch array instead
// of a caller workspace, for callers that may not allocate device memory (see hcl.h).
hcl_status_t hcl_csa_sparse_attn_noalloc(const void* q, int B, int Tq, int H, int d,
                                         const hcl_kv_t* kvc, int Nc, const int32_t* idx, int k,
                                         const hcl_kv_t* raw, int L, int W,
                                         const int32_t* q_pos, float scale, const float* sink,
                                         void* out, float* lse, int32_t* status, void* stream) {
  static_assert(HCL_NOALLOC_SCRATCH_BYTES == hcl::NOALLOC_SCRATCH_BYTES, "scratch size");
  HCL_REQUIRE(B >= 0 && Tq >= 0 && H >= 1 && k >= 0 && W >= 0, "invalid size");
  const size_t need = hcl::attn_workspace_bytes(0, B, Tq, H, k, W);
  HCL_REQUIRE(need <= hcl::NOALLOC_SCRATCH_BYTES,
              "hcl_csa_sparse_attn_noalloc: this problem needs %zu bytes of split-KV scratch, "
              "more than the library's fixed %zu bytes; use hcl_csa_sparse_attn with a workspace",
              need, hcl::NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    hcl_status_t e = hcl::noalloc_scratch(&scratch);
    if (e != HCL_OK) return e;
  }
  return attn_common(0, q, B, Tq, H, d, kvc, Nc, 1, idx, k, raw, L, W, q_pos, scale, sink,
                     nullptr, 0.f, out, lse, scratch, need > 0 ? hcl::NOALLOC_SCRATCH_BYTES : 0,
                     status, stream);
}

size_t hcl_hca_dense_attn_workspace_bytes(int B, int Tq, int H, int Nh, int W) {
  return hcl::attn_workspace_bytes(1, B, Tq, H, Nh, W);
}

hcl_status_t hcl_hca_dense_attn(const void* q, int B, int Tq, int H, int d, const hcl_kv_t* kvh,
                                int Nh, int mh, const hcl_kv_t* raw, int L, int W,
                                const int32_t* q_pos, float scale, const float* sink,
                                const float* q_gamma, float q_eps, void* out, float* lse,
                                void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return attn_common(1, q, B, Tq, H, d, kvh, Nh, mh, nullptr, 0, raw, L, W, q_pos, scale, sink,
                     q_gamma, q_eps, out, lse, ws, ws_bytes, status, stream);
}

// ---- fused decode step -----------------------------------------------------------------

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DecodeWs {
  size_t q_packed, q_sf, scores, gmax, idx, attn, total;
};

// The decode step selects from the indexer's per-16-entry maxima when the keys are MXFP4 and
// the scores bf16 (the indexer's packed-row decode path writes them).
static bool decode_uses_gmax(int op_fmt, int score_fmt, int Nc) {
  return op_fmt == HCL_MXFP4 && score_fmt == HCL_BF16 && hcl::topk_gmax_supported(Nc);
}

static DecodeWs decode_ws_layout(int B, int H, int HI, int Nc, int k, int W, int op_fmt,
                                 int score_fmt, int dI) {
  DecodeWs l;
  size_t off = 0;
  l.q_packed = off;
  if (op_fmt == HCL_MXFP4) off += align256((size_t)B * HI * dI / 2);
  l.q_sf = off;
  if (op_fmt == HCL_MXFP4) off += align256((size_t)B * HI * dI / 32);
  l.scores = off;
  off += align256((size_t)B * Nc * (score_fmt == HCL_BF16 ? 2 : 4));
  l.gmax = off;
  // group maxima, second maxima (u16) and positions (u8)
  if (decode_uses_gmax(op_fmt, score_fmt, Nc)) off += align256((size_t)B * hcl::gmax_row_stride(Nc) * 5);
  l.idx = off;
  off += align256((size_t)B * k * 4);
  l.attn = off;
  off += align256(hcl::attn_workspace_bytes(0, B, 1, H, k, W));
  l.total = off;
  return l;
}

size_t hcl_csa_decode_step_workspace_bytes(int B, int H, int HI, int Nc, int k, int W,
                                           int op_fmt, int score_fmt) {
  return decode_ws_layout(B, H, HI, Nc, k, W, op_fmt, score_fmt, 64).total;
}

int hcl_csa_decode_step_kernels(int B, int H, int HI, int Nc, int k, int W, int op_fmt,
                                int score_fmt, int kv_fmt) {
  (void)HI;
  if (B <= 0) return 0;
  (void)op_fmt; (void)score_fmt; (void)Nc; (void)kv_fmt;
  const size_t ws = hcl::attn_workspace_bytes(0, B, 1, H, k, W);
  return 3 + (ws > 0 ? 1 : 0);  // indexer, top-k, attention (+ split merge)
}

hcl_status_t hcl_csa_decode_step(const void* q, const void* qI_bf16, const float* w, int op_fmt,
                                 const void* kI, const void* kI_sf, int kI_cap, int score_fmt,
                                 int B, int H, int HI, int dI, int d, const hcl_kv_t* kvc,
                                 int Nc, int m, int k, const hcl_kv_t* raw, int L, int W,
                                 const int32_t* q_pos, float scale, const float* sink,
                                 const float* q_gamma, float q_eps, void* out, float* lse,
                                 int32_t* idx_out, void* ws, size_t ws_bytes, int32_t* status,
                                 void* stream) {
  if (dI != 64) return fail(HCL_ERR_UNSUPPORTED, "only dI == 64 is supported");
  const DecodeWs l = decode_ws_layout(B, H, HI, Nc, k, W, op_fmt, score_fmt, dI);
  HCL_REQUIRE(ws != nullptr && aligned16(ws) && ws_bytes >= l.total,
              "decode workspace too small: need %zu bytes", l.total);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  hcl_status_t e;
  // MXFP4 keys: the bf16 index query is quantised inside the indexer (no separate launch)
  void* scores = wsb + l.scores;
  uint16_t* gmax =
      decode_uses_gmax(op_fmt, score_fmt, Nc) ? reinterpret_cast<uint16_t*>(wsb + l.gmax) : nullptr;
  const size_t ngs = (size_t)B * hcl::gmax_row_stride(Nc);
  uint16_t* g2nd = gmax ? gmax + ngs : nullptr;
  uint8_t* garg = gmax ? reinterpret_cast<uint8_t*>(g2nd + ngs) : nullptr;
  if (op_fmt == HCL_MXFP4)
    e = index_scores_impl(op_fmt, nullptr, nullptr, qI_bf16, w, kI, kI_sf, B, 1, HI, dI, Nc,
                          kI_cap, q_pos, m, scores, score_fmt, status, stream, gmax, g2nd, garg);
  else
    e = index_scores_impl(op_fmt, qI_bf16, nullptr, nullptr, w, kI, kI_sf, B, 1, HI, dI, Nc,
                          kI_cap, q_pos, m, scores, score_fmt, status, stream);
  if (e != HCL_OK) return e;
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + l.idx);
  // the top-k's predecessor is the indexer above, which does not write q_pos
  if (gmax != nullptr) {
    HCL_REQUIRE(k >= 1 && k <= 4096, "k must be in [1, 4096]");
    TopkArgs ta{scores, score_fmt, B, 1, Nc, q_pos, m, k, idx, status, 1};
    e = launch_topk_gmax(ta, gmax, g2nd, garg, as_stream(stream));
  } else {
    e = topk_common(scores, score_fmt, B, 1, Nc, q_pos, m, k, idx, nullptr, 0, status, stream, 1);
  }
  if (e != HCL_OK) return e;
  // the attention's predecessor is the top-k above, which writes neither q, q_pos nor the raw
  // window: the attention may load those before waiting for it
  return attn_common(0, q, B, 1, H, d, kvc, Nc, 1, idx, k, raw, L, W, q_pos, scale, sink, q_gamma,
                     q_eps, out, lse, wsb + l.attn, ws_bytes - l.attn, status, stream, 1);
}

hcl_status_t hcl_cache_append(const void* kv_new, const void* gate_new, const void* kI_new,
                              const int32_t* t_new, int B, int d, int dI, void* stage_kv,
                              void* stage_gate, int stage_cap, const hcl_kv_t* raw,
                              const hcl_kv_t* kvc, const float* bias_csa, int m, int kI_fmt,
                              void* kI, void* kI_sf, int kI_cap, const hcl_kv_t* kvh,
                              const float* bias_hca, int mh, const float* gamma, float eps,
                              int32_t* status, void* stream) {
  (void)status;
  HCL_REQUIRE(B >= 0, "B must be non-negative");
  if (d != 128) return fail(HCL_ERR_UNSUPPORTED, "cache append: only d == 128 is supported");
  if (B == 0) return HCL_OK;
  HCL_REQUIRE(kv_new && gate_new && t_new && stage_kv && stage_gate, "NULL pointer");
  HCL_REQUIRE(aligned16(kv_new) && aligned16(gate_new) && aligned16(stage_kv) &&
                  aligned16(stage_gate),
              "kv_new, gate_new and the staging rings must be 16-byte aligned");
  hcl_status_t e = check_kv(raw, d, "raw");
  if (e != HCL_OK) return e;
  if (raw->fmt == HCL_FP8SPLIT) HCL_REQUIRE(((uintptr_t)raw->data & 7) == 0, "raw: codes must be 8-byte aligned");
  int need_stage = 1;
  if (kvc != nullptr) {
    e = check_kv(kvc, d, "kvc");
    if (e != HCL_OK) return e;
    HCL_REQUIRE(m >= 1 && m <= 8, "m must be in [1, 8]");
    HCL_REQUIRE(bias_csa != nullptr, "bias_csa must be given with kvc");
    need_stage = 2 * m;
    if (kI != nullptr) {
      if (dI != 64) return fail(HCL_ERR_UNSUPPORTED, "cache append: only dI == 64 is supported");
      HCL_REQUIRE(kI_new != nullptr && aligned16(kI_new) && aligned16(kI), "kI_new and kI must be 16-byte aligned");
      HCL_REQUIRE(kI_cap >= 1, "kI_cap must be positive");
      HCL_REQUIRE(kI_fmt == HCL_BF16 || (kI_fmt == HCL_MXFP4 && kI_sf != nullptr),
                  "kI_fmt must be HCL_BF16, or HCL_MXFP4 with kI_sf");
    }
  }
  if (kvh != nullptr) {
    e = check_kv(kvh, d, "kvh");
    if (e != HCL_OK) return e;
    HCL_REQUIRE(mh >= 1 && mh <= 1024, "mh must be in [1, 1024]");
    HCL_REQUIRE(bias_hca != nullptr, "bias_hca must be given with kvh");
    if (mh > need_stage) need_stage = mh;
  }
  HCL_REQUIRE(stage_cap >= need_stage, "stage_cap must be >= %d (2m and mh)", need_stage);
  if (gamma != nullptr) HCL_REQUIRE(eps > 0.f && eps < 1e30f, "eps must be a positive number");
  CacheAppendArgs a{kv_new, gate_new, kI_new, t_new, B, stage_kv, stage_gate, stage_cap, *raw,
                    kvc, bias_csa, m, kI_fmt, kI, kI_sf, kI_cap, kvh, bias_hca, mh, gamma, eps};
  return launch_cache_append(a, as_stream(stream));
}

hcl_status_t hcl_cp_candidates(const void* scores, int score_fmt, const int32_t* idx, int B,
                               int Nc_local, int k, int e0, float* cand_scores,
                               int32_t* cand_idx, int32_t* status, void* stream) {
  HCL_REQUIRE(score_fmt == HCL_FP32 || score_fmt == HCL_BF16, "score_fmt must be HCL_FP32 or HCL_BF16");
  HCL_REQUIRE(B >= 0 && Nc_local >= 0 && k >= 1 && e0 >= 0, "invalid size");
  if (B == 0) return HCL_OK;
  HCL_REQUIRE(idx && cand_scores && cand_idx && (scores || Nc_local == 0), "NULL pointer");
  return launch_cp_candidates(scores, score_fmt, idx, B, Nc_local, k, e0, cand_scores, cand_idx,
                              status, as_stream(stream));
}

hcl_status_t hcl_cp_own(const int32_t* pos, const int32_t* gathered_idx, int B, int n, int k,
                        int e0, int e1, int32_t* sel_out, int32_t* own_out, void* stream) {
  HCL_REQUIRE(B >= 0 && n >= 0 && k >= 1 && 0 <= e0 && e0 <= e1, "invalid size");
  if (B == 0) return HCL_OK;
  HCL_REQUIRE(pos && gathered_idx && sel_out && own_out, "NULL pointer");
  return launch_cp_own(pos, gathered_idx, B, n, k, e0, e1, sel_out, own_out, as_stream(stream));
}

hcl_status_t hcl_lse_merge(const void* o_parts, const float* lse_parts, int G, int64_t rows, int d,
                           int H, const float* sink, void* out, float* lse_out, void* stream) {
  HCL_REQUIRE(G >= 1 && rows >= 0 && H >= 1, "invalid size");
  HCL_REQUIRE(d >= 2 && d % 2 == 0 && d <= 1024, "d must be even, <= 1024");
  if (rows == 0) return HCL_OK;
  HCL_REQUIRE(o_parts && lse_parts && out, "NULL pointer");
  HCL_REQUIRE(((uintptr_t)o_parts & 3) == 0 && ((uintptr_t)out & 3) == 0, "o_parts and out must be 4-byte aligned");
  return launch_lse_merge(o_parts, lse_parts, G, (long long)rows, d, H, sink, out, lse_out,
                          as_stream(stream));
}

hcl_status_t hcl_selftest_bounded_wait(int32_t* status, int limit_us, void* stream) {
  HCL_REQUIRE(status != nullptr, "status must be given");
  HCL_REQUIRE(limit_us >= 1 && limit_us <= 10 * 1000 * 1000, "limit_us must be in [1, 1e7]");
  return launch_selftest_wait(status, limit_us, as_stream(stream));
}

}  // extern "C"
