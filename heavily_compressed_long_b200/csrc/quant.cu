// quant.cu -- cache-write quantisers.
//
// [CSDN §1.4] KV rows keep the RoPE dims in BF16 and store the other dims in FP8: here E4M3
// with one fp32 scale per row, scale = amax / 448 (448 = E4M3's largest finite value).
// [CSDN §1.4; Austery infra] the lightning indexer's QK operands are MXFP4 (OCP MX v1.0):
// per block of 32 values, an E8M0 shared scale X = 2^(floor(log2 amax) - 2) and E2M1
// elements rounded to nearest even, saturating at 6.
#include <cuda_bf16.h>

#include "hcl_common.cuh"
#include "hcl_internal.h"
#include "mxfp4.cuh"

namespace hcl {
namespace {

// One group of d/8 threads per row: the first half of the group holds dims 0..d/2-1.
__global__ void quant_kv_fp8_kernel(const __nv_bfloat16* __restrict__ kv, long long rows, int d,
                                    uint8_t* __restrict__ nope, float* __restrict__ scale,
                                    __nv_bfloat16* __restrict__ rope) {
  const int G = d >> 3;          // threads per row (power of two, <= 32)
  const int H = G >> 1;          // threads covering the quantised half
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long r = gt / G;
  const int c = int(gt % G);
  const bool active = r < rows;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (active) v = __ldg(reinterpret_cast<const uint4*>(kv + r * d + c * 8));
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&v);
  float a = 0.f;
  if (c < H) {
#pragma unroll
    for (int i = 0; i < 8; i++) a = fmaxf(a, fabsf(bf2f(x[i])));
  }
  // max over the H threads of this row's quantised half (groups are aligned in the warp)
  for (int o = 1; o < H; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (!active) return;
  const float sc = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
  if (c < H) {
    uint16_t p[4];
#pragma unroll
    for (int i = 0; i < 4; i++)
      p[i] = cvt_e4m3x2(__fdiv_rn(bf2f(x[2 * i]), sc), __fdiv_rn(bf2f(x[2 * i + 1]), sc));
    uint2 out = make_uint2(uint32_t(p[0]) | (uint32_t(p[1]) << 16),
                           uint32_t(p[2]) | (uint32_t(p[3]) << 16));
    *reinterpret_cast<uint2*>(nope + r * (d / 2) + c * 8) = out;
    if (c == 0) scale[r] = sc;
  } else {
    *reinterpret_cast<uint4*>(rope + r * (d / 2) + (c - H) * 8) = v;
  }
}

// One thread per block of 32 values.
__global__ void quant_mxfp4_kernel(const __nv_bfloat16* __restrict__ x, long long rows, int cols,
                                   uint8_t* __restrict__ packed, uint8_t* __restrict__ sf) {
  const int nb = cols >> 5;
  const long long blk = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= rows * nb) return;
  const long long r = blk / nb;
  const int j = int(blk % nb);
  const uint4* src = reinterpret_cast<const uint4*>(x + r * cols + j * 32);
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; i++) v[i] = __ldg(src + i);
  uint4 pk;
  const int code = mxfp4_encode32(v, pk);
  *reinterpret_cast<uint4*>(packed + r * (cols / 2) + j * 16) = pk;
  sf[r * nb + j] = uint8_t(code);
}

}  // namespace

hcl_status_t launch_quant_kv_fp8(const void* kv, int64_t rows, int d, void* nope, float* scale,
                                 void* rope, cudaStream_t st) {
  if (rows == 0) return HCL_OK;
  long long threads = rows * (d / 8);
  int blk = 256;
  quant_kv_fp8_kernel<<<(unsigned)((threads + blk - 1) / blk), blk, 0, st>>>(
      static_cast<const __nv_bfloat16*>(kv), rows, d, static_cast<uint8_t*>(nope), scale,
      static_cast<__nv_bfloat16*>(rope));
  return check_launch("quant_kv_fp8");
}

hcl_status_t launch_quant_mxfp4(const void* x, int64_t rows, int cols, void* packed, void* sf,
                                cudaStream_t st) {
  if (rows == 0) return HCL_OK;
  long long blocks = rows * (cols / 32);
  int blk = 256;
  quant_mxfp4_kernel<<<(unsigned)((blocks + blk - 1) / blk), blk, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, static_cast<uint8_t*>(packed),
      static_cast<uint8_t*>(sf));
  return check_launch("quant_mxfp4");
}

}  // namespace hcl
