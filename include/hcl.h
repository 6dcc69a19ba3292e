/*
 * hcl.h -- C ABI of libhcl: the CSA / HCA hybrid-attention hot path on one NVIDIA B200
 * (sm_100a).
 *
 * The method (web write-ups of the DeepSeek-V4 technical report):
 *   [Tripbot] "论文解读｜DeepSeek-V4：百万 token 上下文的效率革命", blog.tripbot.top:
 *             §3.1 CSA (4:1 softmax-gated pooling with a learned position bias; a lightning
 *             indexer scores all compressed entries with a multi-head dot product; a per-query
 *             top-k keeps k of them), §3.2 HCA (128:1 pooling, dense attention over all
 *             entries), §3.3 (a 128-token raw sliding-window branch on both; attention sink).
 *   [CSDN]    "从论文出发，逐层剖析 CSA / HCA 混合注意力、mHC 残差连接与 Muon 优化器",
 *             gitcode.csdn.net: §1.1 "工程细节" (overlapped compression: entry i pools the
 *             current m tokens C^a and the previous window's last m tokens C^b), §1.2 HCA,
 *             §1.4 (KV: RoPE dims BF16, other dims FP8; indexer QK product in FP4; index
 *             scores quantised from FP32 to BF16 before top-k).
 *   [Austery] DeepSeek-V4 talk notes, austery.github.io, infrastructure section (MXFP4 on the
 *             indexer QK path).
 *
 * Conventions for every call:
 *   - All tensor pointers are CALLER-OWNED DEVICE memory on the current CUDA device,
 *     row-major and contiguous, with the base address 16-byte aligned.  The library never
 *     allocates device memory; calls that need scratch space take a caller-owned workspace
 *     whose size a *_workspace_bytes() query returns.
 *   - bf16 is IEEE binary32's upper half; e4m3 is OFP8 E4M3 ("fn", max 448); MXFP4 is OCP MX
 *     v1.0 E2M1 elements (two per byte, element 2j in the low nibble) with one E8M0 scale
 *     byte per 32 elements.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream; results are ready when the stream is.
 *   - Every call validates its arguments on the host first and returns HCL_OK, or an error
 *     code with nothing enqueued; hcl_last_error() then returns a message (thread-local).
 *   - Errors detected on the device (an index out of range, a bounded wait that ran out)
 *     are OR-ed as hcl_status_t bits into the optional caller-owned device word `status`
 *     (int32); the kernel skips the faulty access instead of trapping.  Check it after
 *     synchronising.
 *   - Results are bitwise deterministic for fixed inputs and launch shapes.
 *   - Query position p: absolute token position of a query; raw token t is visible to it
 *     when p - W + 1 <= t <= p (window) and compressed entry i of ratio r when its last token
 *     r*i + r - 1 <= p ("causal at entry granularity").
 */
#ifndef HCL_H_
#define HCL_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HCL_API __attribute__((visibility("default")))
#else
#define HCL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HCL_OK = 0,
  HCL_ERR_INVALID_ARG = 1,   /* a shape, pointer, alignment or format was rejected */
  HCL_ERR_UNSUPPORTED = 2,   /* a valid combination this build does not implement */
  HCL_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  HCL_ERR_TIMEOUT = 8,       /* (device status bit) a bounded wait ran out */
  HCL_ERR_DEVICE_FAULT = 16  /* (device status bit) an out-of-range index was skipped */
} hcl_status_t;

typedef enum {
  HCL_BF16 = 0,      /* bf16 values */
  HCL_FP32 = 1,      /* fp32 values */
  HCL_FP8SPLIT = 2,  /* KV rows: d/2 e4m3 codes x per-row fp32 scale, then d/2 bf16 RoPE dims */
  HCL_MXFP4 = 3      /* MXFP4: packed E2M1 pairs + one E8M0 scale per 32 elements */
} hcl_fmt_t;

/*
 * A KV store: compressed entries (one row per entry) or raw tokens (one row per token).
 * Each row is both key and value of the one KV head shared by all query heads.
 *   fmt == HCL_BF16:      data  = bf16 [B, cap, d]
 *   fmt == HCL_FP8SPLIT:  data  = e4m3 [B, cap, d/2]  (dims 0 .. d/2-1, quantised)
 *                         scale = fp32 [B, cap]       (value = code * scale)
 *                         rope  = bf16 [B, cap, d/2]  (dims d/2 .. d-1, the RoPE dims)
 * Row t of sequence b is stored at slot b*cap + (t mod cap): cap equal to the context length
 * is plain linear storage; a smaller cap is a ring (the sliding-window cache), valid as long
 * as every row a call reads is resident.
 */
typedef struct {
  int32_t fmt;
  int32_t cap;
  const void* data;
  const float* scale;
  const void* rope;
} hcl_kv_t;

HCL_API const char* hcl_version(void);
HCL_API const char* hcl_last_error(void);

/* ---------------------------------------------------------------------------------------
 * a1 -- CSA compressor [Tripbot §3.1; CSDN §1.1 工程细节].
 * Entry i (entry_begin <= i < entry_end) pools the 2m raw tokens t_j = m(i-1)+j, j=0..2m-1
 * (C^b = previous window's last m tokens, then C^a = the current m tokens); slots with t_j
 * outside [0, L) are left out.  Per channel c:
 *     out[b, i, c] = sum_j softmax_j( gate[b,t_j,c] + bias[j] ) * kv[b,t_j,c]
 * kv, gate: bf16 [B, L, d]; bias: fp32 [2m]; out: [B, out_cap, d] in out_fmt (HCL_FP32 or
 * HCL_BF16), entry i written at row i.  Requires 0 <= entry_begin <= entry_end <=
 * min(ceil(L/m), out_cap), d % 8 == 0, 1 <= m <= 64.  Accumulates in fp32.
 * RMSNorm of the entries [Tripbot §5: compressed KV entries are RMS-normalised]: with gamma
 * (fp32 [d]) given, each pooled entry c is written as c / sqrt(mean_ch(c^2) + eps) * gamma,
 * computed in fp32 before the output rounding (NULL: no normalisation; eps >= 0).  With
 * gamma, d/8 must be a power of two <= 32 (d = 8 .. 256); otherwise HCL_ERR_UNSUPPORTED.
 */
HCL_API hcl_status_t hcl_csa_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                              int d, int m, int entry_begin, int entry_end, void* out,
                              int out_fmt, int out_cap, const float* gamma, float eps,
                              void* stream);

/* a2 -- HCA compressor [Tripbot §3.2; CSDN §1.2]: as above with span m (no overlap):
 * entry i pools tokens m*i .. m*i+m-1; bias: fp32 [m]; 1 <= m <= 1024; the same optional
 * RMSNorm epilogue (gamma, eps). */
HCL_API hcl_status_t hcl_hca_compress(const void* kv, const void* gate, const float* bias, int B, int L,
                              int d, int m, int entry_begin, int entry_end, void* out,
                              int out_fmt, int out_cap, const float* gamma, float eps,
                              void* stream);

/* ---------------------------------------------------------------------------------------
 * a3 -- cache quantisers [CSDN §1.4; Austery infra].
 * hcl_quant_kv_fp8: kv bf16 [rows, d] -> nope e4m3 [rows, d/2], scale fp32 [rows],
 *   rope bf16 [rows, d/2].  scale = amax(|kv[r, 0:d/2]|)/448 (1 when the amax is 0), code =
 *   E4M3 round-to-nearest-even, saturating, of the fp32 quotient kv/scale; the RoPE half is
 *   copied.  d % 16 == 0, d <= 256.
 * hcl_quant_mxfp4: x bf16 [rows, cols] -> packed [rows, cols/2] and e8m0 [rows, cols/32]:
 *   per block of 32, X = 2^(floor(log2 amax) - 2) (E8M0 code clamped to 0..254; amax 0 ->
 *   code 127); element = E2M1 nearest-even of x/X, saturating at 6, sign kept.
 *   cols % 32 == 0.
 */
HCL_API hcl_status_t hcl_quant_kv_fp8(const void* kv, int64_t rows, int d, void* nope, float* scale,
                              void* rope, void* stream);
HCL_API hcl_status_t hcl_quant_mxfp4(const void* x, int64_t rows, int cols, void* packed, void* e8m0,
                             void* stream);

/* ---------------------------------------------------------------------------------------
 * a4 -- lightning indexer [Tripbot §3.1; CSDN §1.4].
 *   scores[b, t, i] = sum_h w[b,t,h] * max(0, qI[b,t,h,:] . kI[b,i,:])   if i < nvis(b,t)
 *                   = -inf                                                 otherwise
 * with nvis = min(Nc, floor((q_pos[b,t] + 1) / m)).  Dense contraction on tcgen05 tensor
 * cores (fp32 accumulation).
 *   op_fmt HCL_BF16:  qI bf16 [B, Tq, HI, dI]; kI bf16 [B, kI_cap, dI]; qI_sf = kI_sf = NULL.
 *   op_fmt HCL_MXFP4: qI [B, Tq, HI, dI/2] + qI_sf [B, Tq, HI, dI/32];
 *                     kI [B, kI_cap, dI/2] + kI_sf [B, kI_cap, dI/32]; kI_cap % 8 == 0.
 *   w fp32 [B, Tq, HI]; q_pos int32 [B, Tq]; scores [B, Tq, Nc] in score_fmt (HCL_FP32, or
 *   HCL_BF16 = the fp32 score rounded to nearest even).  status: optional device word.
 * Supported: dI == 64, 1 <= HI <= 16, Nc <= kI_cap.
 */
HCL_API hcl_status_t hcl_csa_index_scores(int op_fmt, const void* qI, const void* qI_sf, const float* w,
                                  const void* kI, const void* kI_sf, int B, int Tq, int HI,
                                  int dI, int Nc, int kI_cap, const int32_t* q_pos, int m,
                                  void* scores, int score_fmt, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * a5 -- per-query top-k [Tripbot §3.1].  For each row (b, t): the indices of the k largest
 * scores among the visible entries [0, nvis(b,t)), equal scores going to the lower index,
 * written in ascending index order to idx int32 [B, Tq, k], padded with -1 when nvis < k.
 * scores: [B, Tq, Nc] in score_fmt (HCL_FP32 or HCL_BF16).  Exact radix selection on the
 * order-preserving integer image of the scores (NaN scores are not supported).
 * Supported: 1 <= k <= 4096, Nc <= 2^22.  ws: hcl_csa_topk_workspace_bytes() bytes.
 */
HCL_API size_t hcl_csa_topk_workspace_bytes(int B, int Tq, int Nc, int k, int score_fmt);
HCL_API hcl_status_t hcl_csa_topk(const void* scores, int score_fmt, int B, int Tq, int Nc,
                          const int32_t* q_pos, int m, int k, int32_t* idx, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * a6 -- CSA attention [Tripbot §3.1 step 2, §3.3].  For query (b, t) at p = q_pos[b,t] and
 * each head h, one softmax over the rows J = { kvc entry idx[b,t,j] : idx >= 0 } followed by
 * the window { raw token u : max(0, p-W+1) <= u <= p }:
 *     z_j = scale * q[b,t,h,:] . row_j;  out = sum_j softmax(z)_j row_j;  lse = log sum exp z
 * With a sink (fp32 [H] logits, or NULL) the softmax denominator also has exp(sink[h]) and
 * the sink contributes no value.  No rows and no sink: out = 0, lse = -inf.
 * Query RMSNorm [Tripbot §5: queries are RMS-normalised before attention]: with q_gamma
 * (fp32 [d]) given, every query head row is used as q / sqrt(mean(q^2) + q_eps) * q_gamma,
 * computed in fp32 and rounded to bf16 (the tensor-core operand) before the dot products
 * (NULL: q as given; q_eps > 0).
 *   q bf16 [B, Tq, H, d]; idx int32 [B, Tq, k] (entries < Nc; -1 = none); out bf16
 *   [B, Tq, H, d]; lse fp32 [B, Tq, H] or NULL.  d == 128, 1 <= H <= 128.
 *   ws: hcl_csa_sparse_attn_workspace_bytes() bytes (split-KV partial results).
 * Out-of-range indices set HCL_ERR_DEVICE_FAULT in *status (if given) and are skipped.
 */
HCL_API size_t hcl_csa_sparse_attn_workspace_bytes(int B, int Tq, int H, int k, int W);
HCL_API hcl_status_t hcl_csa_sparse_attn(const void* q, int B, int Tq, int H, int d, const hcl_kv_t* kvc,
                                 int Nc, const int32_t* idx, int k, const hcl_kv_t* raw, int L,
                                 int W, const int32_t* q_pos, float scale, const float* sink,
                                 const float* q_gamma, float q_eps, void* out, float* lse,
                                 void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * hcl_csa_sparse_attn_noalloc -- the CSA attention above for callers that cannot allocate
 * device memory (without the query RMSNorm).  (The paper has no counterpart; this is a
 * deployment variant.)
 * Some callers may not call cudaMalloc at all: serving runtimes that reserve the device's
 * memory up front for their own pool and forbid allocation on the request path (cudaMalloc
 * can synchronise the device and fail once the pool owns the memory), and plugin hosts that
 * hand a kernel only its inputs and outputs.  This entry point takes the same arguments as
 * hcl_csa_sparse_attn minus the workspace and allocates nothing: the split-KV partial results
 * live in a fixed array inside the library, HCL_NOALLOC_SCRATCH_BYTES (16 MiB) on every GPU
 * that loads the library, held until the process exits.  A problem whose partials need more
 * (hcl_csa_sparse_attn_workspace_bytes() > 16 MiB) is rejected with HCL_ERR_INVALID_ARG and
 * a message naming the limit.  The first call on a device looks the array's device address
 * up (cudaGetSymbolAddress) and caches it for that device's current CUDA context; make that
 * first call before any stream capture.  A call made in a different context (for example
 * after cudaDeviceReset, which destroys the old one) looks the address up again, so it is
 * again a first call.  All calls share the array and leave their partials in it; calls that
 * overlap on the GPU (different streams, or threads) race on it, so serialise them.  Nothing
 * in the array needs clearing: each call writes every slot it later reads.
 */
#define HCL_NOALLOC_SCRATCH_BYTES (16u << 20)
HCL_API hcl_status_t hcl_csa_sparse_attn_noalloc(const void* q, int B, int Tq, int H, int d,
                                         const hcl_kv_t* kvc, int Nc, const int32_t* idx, int k,
                                         const hcl_kv_t* raw, int L, int W,
                                         const int32_t* q_pos, float scale, const float* sink,
                                         void* out, float* lse, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * a7 -- HCA attention [Tripbot §3.2, §3.3; CSDN §1.2].  As a6 (sink, query RMSNorm) with
 * J = { kvh entry i : 0 <= i < Nh, mh*(i+1) - 1 <= p } followed by the window: dense, no
 * selection.
 *   kvh: [B, cap, d] rows (cap >= Nh).  d == 128, 1 <= H <= 128.
 */
HCL_API size_t hcl_hca_dense_attn_workspace_bytes(int B, int Tq, int H, int Nh, int W);
HCL_API hcl_status_t hcl_hca_dense_attn(const void* q, int B, int Tq, int H, int d, const hcl_kv_t* kvh,
                                int Nh, int mh, const hcl_kv_t* raw, int L, int W,
                                const int32_t* q_pos, float scale, const float* sink,
                                const float* q_gamma, float q_eps, void* out, float* lse,
                                void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * Fused CSA decode step [Tripbot §3.1]: for each sequence, the new query's index queries are
 * quantised (MXFP4 operands only), scored against all entries, the top-k kept, and
 * attention run over them plus the window -- a4 -> a5 -> a6 enqueued back to back on
 * `stream`.  Arguments as in the individual calls; qI_bf16 is the unquantised bf16 index
 * query [B, 1, HI, dI]; Tq == 1.  ws: hcl_csa_decode_step_workspace_bytes() bytes; it holds
 * the scores and, with MXFP4 operands and bf16 scores, a 5-byte summary per 16-entry group
 * (largest and second largest score as order-preserving keys, position of the largest) that
 * the indexer writes and the top-k reads instead of most of the scores.  The workspace is
 * scratch owned by the caller; its contents after the call are unspecified.
 */
HCL_API size_t hcl_csa_decode_step_workspace_bytes(int B, int H, int HI, int Nc, int k, int W,
                                           int op_fmt, int score_fmt);
/* The number of kernels one hcl_csa_decode_step call with these shapes and formats launches
 * (kv_fmt: the compressed / raw store format): the indexer, the top-k, the attention, and a
 * split merge when the attention needs a workspace. */
HCL_API int hcl_csa_decode_step_kernels(int B, int H, int HI, int Nc, int k, int W, int op_fmt,
                                        int score_fmt, int kv_fmt);
HCL_API hcl_status_t hcl_csa_decode_step(const void* q, const void* qI_bf16, const float* w, int op_fmt,
                                 const void* kI, const void* kI_sf, int kI_cap, int score_fmt,
                                 int B, int H, int HI, int dI, int d, const hcl_kv_t* kvc,
                                 int Nc, int m, int k, const hcl_kv_t* raw, int L, int W,
                                 const int32_t* q_pos, float scale, const float* sink,
                                 const float* q_gamma, float q_eps, void* out, float* lse,
                                 int32_t* idx_out, void* ws, size_t ws_bytes, int32_t* status,
                                 void* stream);

/* ---------------------------------------------------------------------------------------
 * Decode-time cache maintenance [Yanbaoke §5 KV cache management: a heterogeneous KV cache;
 * Austery's talk notes, infrastructure section].  Appends one new raw token per sequence to
 * one layer's cache, on `stream`, before that step's attention reads it:
 *   kv_new, gate_new: bf16 [B, d], the token's KV row and gate logits; t_new: int32 [B], its
 *   absolute position (< 0: the sequence appends nothing this step).
 *   stage_kv, stage_gate: bf16 [B, stage_cap, d], caller-owned staging rings holding the token
 *   rows the compressors still need; token u lives at slot u mod stage_cap.  stage_cap >= 2m
 *   (with kvc) and >= mh (with kvh); before the first call the rings must hold the tokens
 *   before t_new that the next entries pool (the last 2m - 1 / mh - 1 tokens).
 *   raw: the raw sliding-window store (hcl_kv_t, HCL_BF16 or HCL_FP8SPLIT); token t is written
 *   at slot t mod raw->cap (split rows: E4M3 codes with scale amax/448 and the bf16 RoPE half,
 *   bit-identical to hcl_quant_kv_fp8).
 *   kvc (or NULL, an HCA layer): the CSA entry store.  When (t+1) % m == 0, entry i = t/m is
 *   pooled from tokens m(i-1) .. m*i+m-1 with bias_csa (fp32 [2m]) exactly as
 *   hcl_csa_compress computes it, optionally RMS-normalised (gamma, eps as in
 *   hcl_csa_compress), rounded to bf16 and written at slot i mod kvc->cap (split rows
 *   quantised as above).  With kI non-NULL the entry's index key kI_new (bf16 [B, dI]) is
 *   written at slot i mod kI_cap of kI: HCL_BF16 rows [B, kI_cap, dI], or HCL_MXFP4 packed
 *   [B, kI_cap, dI/2] + kI_sf E8M0 [B, kI_cap, dI/32] (bit-identical to hcl_quant_mxfp4).
 *   1 <= m <= 8; dI == 64.
 *   kvh (or NULL, a CSA layer): the HCA entry store.  When (t+1) % mh == 0, entry i = t/mh is
 *   pooled from tokens mh*i .. mh*i+mh-1 with bias_hca (fp32 [mh]) as hcl_hca_compress
 *   computes it (and normalised with gamma), written at slot i mod kvh->cap.  1 <= mh <= 1024.
 * d == 128.  The call writes through the store pointers of raw, kvc and kvh (their `const`
 * only means the attention calls read them).  Sequences are independent; two calls that
 * overlap on the GPU on the same cache race.  status: unused (may be NULL).
 */
HCL_API hcl_status_t hcl_cache_append(const void* kv_new, const void* gate_new,
                                      const void* kI_new, const int32_t* t_new, int B, int d,
                                      int dI, void* stage_kv, void* stage_gate, int stage_cap,
                                      const hcl_kv_t* raw, const hcl_kv_t* kvc,
                                      const float* bias_csa, int m, int kI_fmt, void* kI,
                                      void* kI_sf, int kI_cap, const hcl_kv_t* kvh,
                                      const float* bias_hca, int mh, const float* gamma,
                                      float eps, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------------------
 * Context-parallel CSA decode [Austery's talk notes, infrastructure section: context
 * parallelism]: one sequence's compressed entries sharded over ranks, rank r holding entries
 * [e0, e1).  The ranks' collectives (all-gathers) are issued by the caller between these
 * calls; the data steps are:
 *   hcl_cp_candidates: a rank's local top-k (idx int32 [B, k], ascending local indices, -1
 *     padded, as hcl_csa_topk writes them over the rank's scores [B, Nc_local] in score_fmt)
 *     -> candidates: cand_scores fp32 [B, k] (the bf16 / fp32 score, exactly) and cand_idx
 *     int32 [B, k] = e0 + local index (padding: -inf and -1).  Gathered in rank order the
 *     candidates are in ascending global index order, so the k best of the gathered list
 *     (hcl_csa_topk over the n = ranks * k scores, visible count n: q_pos = n - 1 with m = 1)
 *     are the global top-k with ties to the lower global index.
 *   hcl_cp_own: pos int32 [B, k] (the ascending positions hcl_csa_topk selected in the gathered
 *     list) and gathered_idx int32 [B, n] -> sel_out int32 [B, k], the selected global indices,
 *     ascending, -1 padded; own_out int32 [B, k], those in [e0, e1) as local indices (minus e0),
 *     ascending, -1 padded -- the rank's share of the attention, to pass to
 *     hcl_csa_sparse_attn over its slice (the window on the rank holding the last tokens).
 *   hcl_lse_merge: the ranks' partial attention outputs o_parts bf16 [G, rows, d] and
 *     lse_parts fp32 [G, rows] (natural log; rows = B * Tq * H, head h = row % H) ->
 *     out bf16 [rows, d] = sum_r w_r o_r / sum_r w_r with w_r = exp(lse_r - M), and lse_out
 *     fp32 [rows] (or NULL) = M + log sum_r w_r, M the largest lse; a sink (fp32 [H] logits or
 *     NULL) adds exp(sink[h] - M) to the denominator only.  Partials with lse = -inf weigh 0.
 */
HCL_API hcl_status_t hcl_cp_candidates(const void* scores, int score_fmt, const int32_t* idx, int B,
                                       int Nc_local, int k, int e0, float* cand_scores,
                                       int32_t* cand_idx, int32_t* status, void* stream);
HCL_API hcl_status_t hcl_cp_own(const int32_t* pos, const int32_t* gathered_idx, int B, int n, int k,
                                int e0, int e1, int32_t* sel_out, int32_t* own_out, void* stream);
HCL_API hcl_status_t hcl_lse_merge(const void* o_parts, const float* lse_parts, int G, int64_t rows,
                                   int d, int H, const float* sink, void* out, float* lse_out,
                                   void* stream);

/* ---------------------------------------------------------------------------------------
 * Failure-detection self-test: launches one block whose bounded wait on an mbarrier that
 * nothing signals gives up after about `limit_us` microseconds and ORs HCL_ERR_TIMEOUT
 * into *status.  Exercises the same bounded-wait path the pipelined kernels use.
 */
HCL_API hcl_status_t hcl_selftest_bounded_wait(int32_t* status, int limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HCL_H_ */
