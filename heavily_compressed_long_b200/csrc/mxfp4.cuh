// mxfp4.cuh -- MXFP4 (OCP Microscaling v1.0) block encoder shared by the quantiser kernel and
// the indexer's in-kernel query quantisation, so both produce identical bits.
//
// [CSDN §1.4; Austery infra] the indexer's QK operands are MXFP4: per block of 32 values an
// E8M0 shared scale X = 2^(floor(log2 amax) - 2) (2 = E2M1's largest exponent) and E2M1
// elements rounded to nearest even, saturating at 6.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace hcl {

// E2M1 code of |q| by comparison against the midpoints of 0, .5, 1, 1.5, 2, 3, 4, 6; a value
// exactly on a midpoint goes to the even code; beyond 6 saturates to code 7; sign kept.
__device__ __forceinline__ uint32_t e2m1_code(float q) {
  const float a = fabsf(q);
  const uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                     (a >= 3.5f) + (a > 5.0f);
  return c | (signbit(q) ? 8u : 0u);
}

// floor(log2(a)) for a finite a > 0 (normal or subnormal binary32).
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = int(b >> 23);
  if (e > 0) return e - 127;
  return (31 - __clz(b & 0x7FFFFFu)) - 149;
}

// E8M0 code of a block's shared scale given the block's amax (127 when amax is 0).
__device__ __forceinline__ int mxfp4_scale_code(float amax) {
  if (!(amax > 0.f)) return 127;
  const int code = floor_log2(amax) - 2 + 127;
  return code < 0 ? 0 : (code > 254 ? 254 : code);
}

// 2^(code-127) as a binary32 (code 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_value(int code) {
  return code >= 1 ? __uint_as_float(uint32_t(code) << 23) : __uint_as_float(0x00400000u);
}

// Largest magnitude among 8 bf16 values (one 16-byte vector).
__device__ __forceinline__ float bf16x8_amax(const uint4& v) {
  const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; i++) amax = fmaxf(amax, fabsf(__bfloat162float(e[i])));
  return amax;
}

// E2M1 codes of 8 bf16 values divided by the block scale X, packed into 4 bytes (element 2j in
// the low nibble of byte j).
__device__ __forceinline__ uint32_t mxfp4_encode8(const uint4& v, float X) {
  const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
  uint32_t acc = 0;
#pragma unroll
  for (int k = 0; k < 8; k++) acc |= e2m1_code(__fdiv_rn(__bfloat162float(e[k]), X)) << (4 * k);
  return acc;
}

// Encode 32 bf16 values (four 16-byte vectors) into 16 packed bytes and return the E8M0 scale
// code.
__device__ __forceinline__ int mxfp4_encode32(const uint4 (&v)[4], uint4& packed) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; i++) amax = fmaxf(amax, bf16x8_amax(v[i]));
  const int code = mxfp4_scale_code(amax);
  const float X = e8m0_value(code);
  packed = make_uint4(mxfp4_encode8(v[0], X), mxfp4_encode8(v[1], X), mxfp4_encode8(v[2], X),
                      mxfp4_encode8(v[3], X));
  return code;
}

}  // namespace hcl
