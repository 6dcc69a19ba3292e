// cp.cu -- the data steps of context-parallel CSA decode (one sequence's entries sharded over
// ranks; the exchanges themselves are collectives issued by the caller).
//
// [Austery's talk notes, infrastructure section: context parallelism for the compressed
// attention] Rank r holds entries [e0_r, e1_r) of the sequence.  The global top-k lies in the
// union of the ranks' local top-k (an entry among the k best overall is among the k best of its
// own slice, ties going to the lower index in both), so each rank contributes its local
// selection as (score, global index) candidates, all ranks gather them in rank order (= global
// index order), select the k best of the gathered list, and each attends over the selected
// entries it owns; the partial (o, lse) of the ranks combine by log-sum-exp:
//     M = max_r lse_r,  w_r = exp(lse_r - M),  o = sum_r w_r o_r / sum_r w_r,
//     lse = M + log sum_r w_r     (an attention sink enters as one more term with o = 0).
#include <cuda_bf16.h>

#include "hcl_common.cuh"
#include "hcl_internal.h"

namespace hcl {
namespace {

// (local index, score) -> (fp32 score, global index); -inf / -1 for padding.
__global__ void cp_candidates_kernel(const void* __restrict__ scores, int score_fmt,
                                     const int32_t* __restrict__ idx, int B, int Nc_local, int k,
                                     int e0, float* __restrict__ cand_s, int32_t* __restrict__ cand_i,
                                     int32_t* status) {
  pdl_enter();
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * k) return;
  const long long b = t / k;
  const int li = idx[t];
  float s = -INFINITY;
  int gi = -1;
  if (li >= 0 && li < Nc_local) {
    const long long o = b * Nc_local + li;
    s = score_fmt == HCL_FP32 ? static_cast<const float*>(scores)[o]
                              : __uint_as_float(uint32_t(static_cast<const uint16_t*>(scores)[o]) << 16);
    gi = e0 + li;
  } else if (li >= Nc_local) {
    report(status, HCL_ERR_DEVICE_FAULT);
  }
  cand_s[t] = s;
  cand_i[t] = gi;
}

// One block per sequence.  pos: ascending positions (into the gathered list of n candidates)
// of the k selected, -1 padded; the selected global indices (gathered_idx at those positions,
// -1 for padding candidates) are written ascending and compacted to sel_out [k], and this
// rank's own entries -- the contiguous run of the selection inside [e0, e1) -- as local
// indices to own_out [k], -1 padded.
__global__ void cp_own_kernel(const int32_t* __restrict__ pos, const int32_t* __restrict__ gidx,
                              int n, int k, int e0, int e1, int32_t* __restrict__ sel_out,
                              int32_t* __restrict__ own_out) {
  pdl_enter();
  __shared__ int cnt[2];
  const int b = blockIdx.x;
  const int32_t* pr = pos + (size_t)b * k;
  const int32_t* gr = gidx + (size_t)b * n;
  int32_t* so = sel_out + (size_t)b * k;
  int32_t* oo = own_out + (size_t)b * k;
  // the valid selected (global index >= 0) are a prefix of pos order except for padding
  // candidates scattered among them: compact with a block-wide count per tile
  if (threadIdx.x == 0) { cnt[0] = 0; cnt[1] = 0; }
  __syncthreads();
  // 1) count selected with a valid global index before each position (serial tiles of 1024)
  for (int j0 = 0; j0 < k; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    int g = -1;
    if (j < k && pr[j] >= 0 && pr[j] < n) g = gr[pr[j]];
    const bool valid = g >= 0;
    const bool own = valid && g >= e0 && g < e1;
    // exclusive ranks by warp ballots and a block scan over warps
    __shared__ int wv[32], wo[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const unsigned bv = __ballot_sync(0xffffffffu, valid), bo = __ballot_sync(0xffffffffu, own);
    if (lane == 0) { wv[w] = __popc(bv); wo[w] = __popc(bo); }
    __syncthreads();
    int bvx = 0, box = 0;
    for (int u = 0; u < w; u++) { bvx += wv[u]; box += wo[u]; }
    const int rv = cnt[0] + bvx + __popc(bv & ((1u << lane) - 1u));
    const int ro = cnt[1] + box + __popc(bo & ((1u << lane) - 1u));
    if (valid) so[rv] = g;
    if (own) oo[ro] = g - e0;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tv = 0, to = 0;
      for (int u = 0; u < (int)(blockDim.x >> 5); u++) { tv += wv[u]; to += wo[u]; }
      cnt[0] += tv;
      cnt[1] += to;
    }
    __syncthreads();
  }
  for (int j = cnt[0] + threadIdx.x; j < k; j += blockDim.x) so[j] = -1;
  for (int j = cnt[1] + threadIdx.x; j < k; j += blockDim.x) oo[j] = -1;
}

// One warp per (row = sequence x head): G partials o [G, rows, d] bf16, lse [G, rows] fp32
// (natural log) -> out [rows, d] bf16, lse_out [rows].
__global__ void lse_merge_kernel(const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse,
                                 int G, long long rows, int d, int H, const float* __restrict__ sink,
                                 __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out) {
  pdl_enter();
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float M = -INFINITY;
  for (int g = 0; g < G; g++) M = fmaxf(M, lse[g * rows + r]);
  const float s = sink ? sink[r % H] : -INFINITY;
  M = fmaxf(M, s);
  float den = 0.f;
  for (int g = 0; g < G; g++) {
    const float l = lse[g * rows + r];
    if (l > -INFINITY) den += __expf(l - M);
  }
  if (s > -INFINITY) den += __expf(s - M);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int c = lane * 2; c < d; c += 64) {
    float a0 = 0.f, a1 = 0.f;
    for (int g = 0; g < G; g++) {
      const float l = lse[g * rows + r];
      if (!(l > -INFINITY)) continue;
      const float wgt = __expf(l - M);
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(o + ((size_t)g * rows + r) * d + c);
      a0 = fmaf(wgt, __bfloat162float(v.x), a0);
      a1 = fmaf(wgt, __bfloat162float(v.y), a1);
    }
    *reinterpret_cast<__nv_bfloat162*>(out + (size_t)r * d + c) = __floats2bfloat162_rn(a0 * inv, a1 * inv);
  }
  if (lane == 0 && lse_out) lse_out[r] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace

hcl_status_t launch_cp_candidates(const void* scores, int score_fmt, const int32_t* idx, int B,
                                  int Nc_local, int k, int e0, float* cand_s, int32_t* cand_i,
                                  int32_t* status, cudaStream_t st) {
  const long long n = (long long)B * k;
  if (n == 0) return HCL_OK;
  return check_cuda(launch_pdl(cp_candidates_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                               st, 1, scores, score_fmt, idx, B, Nc_local, k, e0, cand_s, cand_i,
                               status),
                    "cp candidates launch");
}

hcl_status_t launch_cp_own(const int32_t* pos, const int32_t* gidx, int B, int n, int k, int e0,
                           int e1, int32_t* sel_out, int32_t* own_out, cudaStream_t st) {
  if (B == 0) return HCL_OK;
  return check_cuda(launch_pdl(cp_own_kernel, dim3((unsigned)B), dim3(1024), 0, st, 1, pos, gidx, n,
                               k, e0, e1, sel_out, own_out),
                    "cp own launch");
}

hcl_status_t launch_lse_merge(const void* o, const float* lse, int G, long long rows, int d, int H,
                              const float* sink, void* out, float* lse_out, cudaStream_t st) {
  if (rows == 0) return HCL_OK;
  const long long threads = rows * 32;
  return check_cuda(launch_pdl(lse_merge_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256),
                               0, st, 1, static_cast<const __nv_bfloat16*>(o), lse, G, rows, d, H,
                               sink, static_cast<__nv_bfloat16*>(out), lse_out),
                    "lse merge launch");
}

}  // namespace hcl
