// hcl_internal.h -- host-side declarations shared by the libhcl translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/hcl.h"

namespace hcl {

// Thread-local error message of the last failing call; returns `code`.
hcl_status_t fail(hcl_status_t code, const char* fmt, ...);
// Maps a pending launch / runtime error to HCL_ERR_CUDA with a message.
hcl_status_t check_cuda(cudaError_t e, const char* what);
hcl_status_t check_launch(const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Launches `kern` with programmatic dependent launch allowed (the kernel must begin with
// pdl_enter() / pdl_wait()), and as clusters of `cluster_x` blocks when cluster_x > 1.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  n++;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    n++;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Number of SMs of the current device (cached per device).
int num_sms();
// Id of the calling thread's current CUDA context, 0 when none is current yet.  Ids are never
// reused within a process (a context created after cudaDeviceReset gets a new one), so they
// key per-context caches safely, unlike device numbers or context handles.
unsigned long long current_ctx_id();
// Makes `kern`'s maximum dynamic shared memory at least `smem` bytes (and, with
// nonportable_cluster, allows cluster sizes above 8), per (kernel, CUDA context): function
// attributes belong to a context, so every device -- and a context re-created after a reset --
// gets its own.  The limit is only ever raised, so launches of one kernel with different
// shared-memory sizes do not undo each other.  Thread-safe.
hcl_status_t set_kernel_attrs(const void* kern, int smem, bool nonportable_cluster);
// Bounded-wait budget for device spin loops, in SM clock cycles (about one second).
long long wait_limit_cycles();

// cuTensorMapEncodeTiled obtained from the driver at run time (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// ---- launchers (each validates nothing; the extern "C" layer does) ----

// gamma (fp32 [d]) non-null: RMSNorm epilogue with epsilon eps.
hcl_status_t launch_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                             int d, int m, int overlap, int e0, int e1, void* out, int out_fmt,
                             int out_cap, const float* gamma, float eps, cudaStream_t st);

hcl_status_t launch_quant_kv_fp8(const void* kv, int64_t rows, int d, void* nope, float* scale,
                                 void* rope, cudaStream_t st);
hcl_status_t launch_quant_mxfp4(const void* x, int64_t rows, int cols, void* packed, void* sf,
                                cudaStream_t st);

struct IndexerArgs {
  int op_fmt;
  const void* qI;
  const void* qI_sf;
  const float* w;
  const void* kI;
  const void* kI_sf;
  int B, Tq, HI, dI, Nc, kI_cap;
  const int32_t* q_pos;
  int m;
  void* scores;
  int score_fmt;
  int32_t* status;
  // optional (decode with MXFP4 keys and bf16 scores): per group of 16 entries, the largest
  // visible score as an order-preserving 16-bit key (0: no visible entry), rows of
  // gmax_row_stride(Nc) groups
  uint16_t* gmax = nullptr;
  uint16_t* g2nd = nullptr;   // with gmax: the second largest per group
  uint8_t* garg = nullptr;    // with gmax: the largest's position in its group (0..15)
};
hcl_status_t launch_indexer(const IndexerArgs& a, cudaStream_t st);
// MXFP4 keys with the bf16 index query [B, Tq, HI, 64] quantised inside the indexer's prologue
// (bit-identical to hcl_quant_mxfp4); a.qI / a.qI_sf are then unused.
hcl_status_t launch_indexer_q(const IndexerArgs& a, const void* qI_bf16, cudaStream_t st);

struct TopkArgs {
  const void* scores;
  int score_fmt;
  int B, Tq, Nc;
  const int32_t* q_pos;
  int m, k;
  int32_t* idx;
  int32_t* status;
  int prewait = 0;  // 1: q_pos does not come from the previous kernel in the stream
};
size_t topk_workspace_bytes(int B, int Tq, int Nc, int k, int score_fmt);
hcl_status_t launch_topk(const TopkArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);
// Decode rows (bf16 scores) whose per-16-entry maxima the indexer wrote (IndexerArgs::gmax);
// rows of gmax_row_stride(Nc) groups (a multiple of 16 groups), for Nc with
// topk_gmax_supported(Nc).
inline int gmax_row_stride(int Nc) { return ((Nc + 15) / 16 + 15) / 16 * 16; }
bool topk_gmax_supported(int Nc);
hcl_status_t launch_topk_gmax(const TopkArgs& a, const uint16_t* gmax, const uint16_t* g2nd,
                              const uint8_t* garg, cudaStream_t st);

// One attention launch: CSA (selected entries + window) or HCA (visible entries + window).
struct AttnArgs {
  int mode;  // 0 = CSA, 1 = HCA
  const void* q;
  int B, Tq, H, d;
  hcl_kv_t comp;  // compressed entries
  int n_comp;     // CSA: Nc; HCA: Nh
  int mh;         // HCA ratio
  const int32_t* idx;
  int k;
  hcl_kv_t raw;
  int L, W;
  const int32_t* q_pos;
  float scale;
  const float* sink;
  void* out;
  float* lse;
  int32_t* status;
  int prewait = 0;  // 1: q, q_pos and raw do not come from the previous kernel in the stream
  const float* q_gamma = nullptr;  // RMSNorm of the query rows (fp32 [d]), or null
  float q_eps = 0.f;
};
// n = k (CSA) or Nh (HCA)
size_t attn_workspace_bytes(int mode, int B, int Tq, int H, int n, int W);
// HCA prefill (many query groups, no KV split) on tcgen05 (attn_flash.cu).
bool hca_flash_usable(const AttnArgs& a);
hcl_status_t launch_hca_flash(const AttnArgs& a, cudaStream_t st);
hcl_status_t launch_attn(const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);

// Decode-time cache append (one token per sequence); kvc / kvh null: no CSA / HCA store.
struct CacheAppendArgs {
  const void* kv_new;
  const void* gate_new;
  const void* kI_new;
  const int32_t* t_new;
  int B;
  void* stage_kv;
  void* stage_gate;
  int stage_cap;
  hcl_kv_t raw;
  const hcl_kv_t* kvc;
  const float* bias_csa;
  int m;
  int kI_fmt;
  void* kI;
  void* kI_sf;
  int kI_cap;
  const hcl_kv_t* kvh;
  const float* bias_hca;
  int mh;
  const float* gamma;
  float eps;
};
hcl_status_t launch_cache_append(const CacheAppendArgs& a, cudaStream_t st);

// Context-parallel decode data steps (cp.cu).
hcl_status_t launch_cp_candidates(const void* scores, int score_fmt, const int32_t* idx, int B,
                                  int Nc_local, int k, int e0, float* cand_s, int32_t* cand_i,
                                  int32_t* status, cudaStream_t st);
hcl_status_t launch_cp_own(const int32_t* pos, const int32_t* gidx, int B, int n, int k, int e0,
                           int e1, int32_t* sel_out, int32_t* own_out, cudaStream_t st);
hcl_status_t launch_lse_merge(const void* o, const float* lse, int G, long long rows, int d, int H,
                              const float* sink, void* out, float* lse_out, cudaStream_t st);

// Fixed device scratch of hcl_csa_sparse_attn_noalloc (split-KV partials), and its device
// address on the current device (looked up once per device).
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(16) << 20;
hcl_status_t noalloc_scratch(void** ptr);

hcl_status_t launch_selftest_wait(int32_t* status, int limit_us, cudaStream_t st);

}  // namespace hcl
