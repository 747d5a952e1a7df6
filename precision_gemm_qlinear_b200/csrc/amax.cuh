// amax.cuh -- max |x| over bf16 data for the quantize kernels (the tensor
// amax of NVFP4's two-level scaling and the NVFP4 block maxima).  The maxima
// are taken on bf16 pairs: the sign bits cleared, then max.bf16x2, which is
// exact and, like fmaxf, returns the other operand when one is NaN.  The
// result is the same float fmaxf over the widened values gives.
#pragma once

#include <cstdint>

namespace qlb {

// max(|a|, |b|) of two bf16 pairs, pair by pair
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a & 0x7FFF7FFFu), "r"(b & 0x7FFF7FFFu));
  return r;
}

// the larger half of such a pair, as a float
__device__ __forceinline__ float bf16x2_hmax(uint32_t m) {
  return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
}

// max |x| over the 8 values of a 16-byte vector, as a bf16 pair
__device__ __forceinline__ uint32_t absmax8_pair(const uint4& v) {
  return bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w));
}

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// This thread's share of a grid-stride max |x| over nvec 16-byte vectors:
// U loads in flight per thread, one running bf16-pair maximum per load slot.
template <int U>
__device__ __forceinline__ float grid_stride_absmax(const uint4* __restrict__ x, int64_t nvec) {
  uint32_t m[U];
#pragma unroll
  for (int u = 0; u < U; ++u) m[u] = 0u;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + (U - 1) * stride < nvec; i += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = ld_nc_v4(x + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) m[u] = bf16x2_absmax(m[u], absmax8_pair(v[u]));
  }
  for (; i < nvec; i += stride) m[0] = bf16x2_absmax(m[0], absmax8_pair(ld_nc_v4(x + i)));
#pragma unroll
  for (int u = 1; u < U; ++u) m[0] = bf16x2_absmax(m[0], m[u]);
  return bf16x2_hmax(m[0]);
}

// The maximum of a non-negative float over the CTA (as its bit pattern,
// which orders like an unsigned integer), valid in thread 0.
__device__ __forceinline__ uint32_t cta_max_bits(float v) {
  __shared__ uint32_t red[32];
  const uint32_t a = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  uint32_t b = 0;
  if (threadIdx.x == 0)
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = max(b, red[w]);
  return b;
}

// CTA launch bound of the amax passes: 8 loads in flight per thread keep
// them at 40 registers, so six CTAs of 256 threads fit on an SM and a grid
// of six CTAs an SM is one wave.
constexpr int kAmaxLoads = 8;
constexpr int kAmaxCtasPerSm = 6;

}  // namespace qlb
