// codec.cuh -- bf16 -> E4M3 / E2M1 encoding steps of the FP8 quantize
// kernel, of the GEMM epilogue that writes NVFP4 output and of the encoder
// test hook, and the NVFP4 tensor factors shared with the NVFP4 quantize
// kernels.  Those compute the same steps on packed pairs (bf16x2 maxima,
// f32x2 products; each half rounded as the scalar operation), so all produce
// the same codes from the same bf16 values.  Every float step is an explicitly rounded IEEE
// operation; the encodes are the hardware's round-to-nearest-even saturating
// conversions (cvt.rn.satfinite).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace qlb {

__device__ __forceinline__ float absmax8(const uint4& v) {
  // |bf16| max over 8 values, done on the bit patterns' float images
  float m = fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w))));
  return m;
}

__device__ __forceinline__ uint32_t e4m3_pair(uint32_t w, float inv) {
  // bf16x2 word -> 2 E4M3 codes (element 0 in the low byte)
  return cvt_e4m3x2(__fmul_rn(bf16hi(w), inv), __fmul_rn(bf16lo(w), inv));
}

__device__ __forceinline__ uint2 e4m3_8(const uint4& v, float inv) {
  uint2 r;
  r.x = e4m3_pair(v.x, inv) | (e4m3_pair(v.y, inv) << 16);
  r.y = e4m3_pair(v.z, inv) | (e4m3_pair(v.w, inv) << 16);
  return r;
}

__device__ __forceinline__ uint32_t e2m1_4(const uint2& w, float inv) {
  // 4 bf16 -> 4 E2M1 codes packed in 16 bits (element 0 in the low nibble)
  uint32_t b0 = cvt_e2m1x2(__fmul_rn(bf16hi(w.x), inv), __fmul_rn(bf16lo(w.x), inv));
  uint32_t b1 = cvt_e2m1x2(__fmul_rn(bf16hi(w.y), inv), __fmul_rn(bf16lo(w.y), inv));
  return b0 | (b1 << 8);
}

// NVFP4 tensor factors from the tensor amax A: the global (decode) scale
// G = A/2688 (2688 = 448 * 6, the largest E4M3 block scale times the largest
// E2M1 value) and the block-scale encode factor enc = 448/A (0 when A is 0).
__device__ __forceinline__ void nvfp4_tensor_factors(float A, float& G, float& enc) {
  G = __fdiv_rn(A, 2688.f);
  enc = A > 0.f ? __fdiv_rn(448.f, A) : 0.f;
}

// NVFP4 block of 16 elements (v0: elements 0-7, v1: 8-15) against the tensor
// factors G = A/2688 and enc = 448/A: E4M3 block scale sb = E4M3(amax_b * enc),
// element factor inv = 1/(dec(sb) * G) (0 when that is 0), 8 bytes of codes;
// amb returns the block's max |x|.
__device__ __forceinline__ uint32_t nvfp4_block(const uint4& v0, const uint4& v1, float enc,
                                                float G, uint2& codes, float& amb) {
  amb = fmaxf(absmax8(v0), absmax8(v1));
  const uint32_t sb = cvt_e4m3x2(0.f, __fmul_rn(amb, enc)) & 0xFF;
  const float den = __fmul_rn(e4m3_to_f32(sb), G);
  const float inv = den > 0.f ? __fdiv_rn(1.f, den) : 0.f;
  codes.x = e2m1_4(make_uint2(v0.x, v0.y), inv) | (e2m1_4(make_uint2(v0.z, v0.w), inv) << 16);
  codes.y = e2m1_4(make_uint2(v1.x, v1.y), inv) | (e2m1_4(make_uint2(v1.z, v1.w), inv) << 16);
  return sb;
}

}  // namespace qlb
