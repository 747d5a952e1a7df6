// quant.cu -- dynamic activation / weight quantization kernels (HBM bound).
//
//  * quant_fp8_rows: per-token (per-row) FP8-E4M3.  One pass over the row:
//    128-bit loads kept in registers, warp-shuffle (redux) amax, scale
//    s = amax/448, inverse 448/amax, codes E4M3(x * inv) written as 64-bit
//    stores.  "Cuantizacion Dinamica FP8", wavespeed.ai "Solucion de WaveSpeed
//    para Acelerar la Generacion de Imagenes FLUX.1-dev".
//  * tensor_amax + quant_nvfp4: NVFP4 two-level scaling (algoritmulzilei.ro,
//    "Accelerarea generarii de imagini cu FLUX 3 Image Klein"; bytechap.com
//    "Como funciona"): global scale G = A/2688 over the tensor, E4M3 block
//    scale per 16 K-elements, packed E2M1 codes; block scales are written
//    straight into the GEMM's scale-factor atom layout.
//
// Every float step is an explicitly rounded IEEE operation (__fmul_rn,
// __fdiv_rn, __frcp_rn, or mul.rn.f32x2, whose halves round as the scalar
// multiply) so no FMA contraction changes a code.  The NVFP4 kernels take maxima of |x|
// on bf16 pairs (max.bf16x2): exact, and like fmaxf they ignore a NaN
// operand.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "amax.cuh"
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace qlb {

namespace {

// ------------------------------------------------------ FP8 per-token quant

// A team of T threads handles one row; 256 / T rows per CTA iteration.  Up to
// VPL 16-byte vectors per thread stay in registers between the amax and the
// cast; longer rows re-read the remainder (L2-resident by then).
// __launch_bounds__(256, 4): at most 64 registers, so that four CTAs (32
// warps) fit on an SM and a FLUX-sized activation (4608 rows of 3072 = 1152
// CTAs of 4 rows) needs about two short waves with 16 rows in flight per SM.
template <int T, int VPL>
__global__ void __launch_bounds__(256, 4) quant_fp8_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                             int64_t M, int64_t K, int64_t ldx,
                                                             uint8_t* __restrict__ q,
                                                             float* __restrict__ s, RowMap map) {
  constexpr int TEAMS = 256 / T;
  constexpr int WPT = T / 32;  // warps per team
  __shared__ uint32_t red[8];
  const int team = threadIdx.x / T;
  const int tt = threadIdx.x % T;
  const int nvec = static_cast<int>(K >> 3);  // 16-byte vectors per row (K < 2^24)
  grid_dep_wait();               // x may come from the previous kernel
  grid_dep_launch_dependents();  // the GEMM may start its prologue
  for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * TEAMS; row0 < M;
       row0 += static_cast<int64_t>(gridDim.x) * TEAMS) {
    const int64_t row = row0 + team;
    const bool valid = row < M;  // uniform across a warp (T >= 32)
    const uint4* xr = reinterpret_cast<const uint4*>(x + (valid ? map(row) : 0) * ldx);
    uint4 v[VPL];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = tt + i * T;
      if (valid && idx < nvec) {
        v[i] = ld_nc_v4(xr + idx);
        amax = fmaxf(amax, absmax8(v[i]));
      }
    }
    for (int idx = tt + VPL * T; valid && idx < nvec; idx += T)
      amax = fmaxf(amax, absmax8(ld_nc_v4(xr + idx)));
    // amax >= 0, so the float bit patterns order like unsigned integers
    uint32_t a = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if constexpr (WPT > 1) {
      if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
      __syncthreads();
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < WPT; ++w) m = max(m, red[team * WPT + w]);
      a = m;
      __syncthreads();
    }
    const float am = __uint_as_float(a);
    const float scale = __fdiv_rn(am, 448.f);
    const float inv = am > 0.f ? __fdiv_rn(448.f, am) : 0.f;
    if (valid && tt == 0) s[row] = scale;
    uint2* qr = reinterpret_cast<uint2*>(q + row * K);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = tt + i * T;
      if (valid && idx < nvec) qr[idx] = e4m3_8(v[i], inv);
    }
    for (int idx = tt + VPL * T; valid && idx < nvec; idx += T)
      qr[idx] = e4m3_8(ld_nc_v4(xr + idx), inv);
  }
}

// ------------------------------------------------------------ tensor amax

// Grid-stride |x| maximum (grid_stride_absmax: U loads in flight per
// thread, bf16-pair maxima), then the CTA maximum and one atomicMax on the
// float bits (amax >= 0, so they order as integers).
template <int U, int CTAS_PER_SM>
__global__ void __launch_bounds__(256, CTAS_PER_SM) tensor_amax_kernel(const uint4* __restrict__ x,
                                                                       int64_t nvec,
                                                                       uint32_t* amax_bits) {
  grid_dep_wait();
  grid_dep_launch_dependents();
  const uint32_t b = cta_max_bits(grid_stride_absmax<U>(x, nvec));
  if (threadIdx.x == 0) atomicMax(amax_bits, b);
}

// ------------------------------------------------------- NVFP4 block quant

// One warp per row of the padded grid [mpad rows, nks * 256 columns]: in each
// step a lane takes one 16-byte vector (8 elements), so a warp reads 512
// contiguous bytes per load; the two lanes of a 16-element block exchange
// their maxima with one shuffle, and the 4 scale bytes of a 64-element group
// (lanes 8i, 8i+2, 8i+4, 8i+6) are gathered into one word.  U steps of loads
// are issued before any is used.  Rows are taken in reverse order so that the
// first ones processed are the tensor's tail, which the amax pass read last
// and which is still in L2.  Padding rows and K groups get zero scales.
//
// The kernel is issue-bound unless each element costs few instructions, so:
// the block maximum is taken on bf16 pairs (sign bits cleared, max.bf16x2,
// which like fmaxf ignores a NaN operand), the element products
// fl(x * inv_b) are packed f32x2 multiplies (each half rounded as the scalar
// __fmul_rn), and inv_b = fl(1 / fl(dec(sb) * G)) is looked up in a
// 128-entry table that every CTA fills once from the tensor factors (sb is a
// non-negative E4M3 code, 0..0x7F) -- the same values the per-block division
// gives.  Full steps (all 32 lanes inside the row) run without predicates.
// packed f32x2 helpers: one instruction per pair, each half rounded as the
// scalar operation
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_splat(float a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
  return r;
}
// the two values of a bf16x2 word as an f32 pair (element 0 in the low half)
__device__ __forceinline__ uint64_t bf16x2_f32x2(uint32_t w) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  return r;
}
// 8 bf16 values times inv (per element, rounded) -> 8 E2M1 codes, element 0
// in the low nibble
__device__ __forceinline__ uint32_t e2m1_8(const uint4& v, uint64_t inv2) {
  const uint64_t p0 = mul_f32x2(bf16x2_f32x2(v.x), inv2), p1 = mul_f32x2(bf16x2_f32x2(v.y), inv2);
  const uint64_t p2 = mul_f32x2(bf16x2_f32x2(v.z), inv2), p3 = mul_f32x2(bf16x2_f32x2(v.w), inv2);
  uint32_t r;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t.reg .f32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
      "mov.b64 {l0, h0}, %1;\n\tmov.b64 {l1, h1}, %2;\n\t"
      "mov.b64 {l2, h2}, %3;\n\tmov.b64 {l3, h3}, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, h3, l3;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(r)
      : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
  return r;
}

template <int U, int LAYOUT>
__global__ void __launch_bounds__(256) quant_nvfp4_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
    uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int64_t bn, int64_t nks, int64_t mpad,
    const uint32_t* __restrict__ amax_bits, float* g_out, RowMap map) {
  __shared__ float inv_tab[128];
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  grid_dep_wait();  // the tensor amax of the previous kernel
  grid_dep_launch_dependents();
  float G, enc;
  nvfp4_tensor_factors(__uint_as_float(*amax_bits), G, enc);
  if (threadIdx.x < 128) {
    const float den = __fmul_rn(e4m3_to_f32(threadIdx.x), G);
    inv_tab[threadIdx.x] = den > 0.f ? __frcp_rn(den) : 0.f;  // fl(1/den), correctly rounded
  }
  __syncthreads();
  if (w >= mpad) return;  // warp-uniform
  const int64_t row = mpad - 1 - w;
  if (w == 0 && lane == 0 && g_out != nullptr) *g_out = G;
  // The lane's scale word of step s: activation atoms, 4 groups (2048 bytes)
  // per step; weights: the replicated chunks (four copies per word).
  uint32_t* sfa = nullptr;
  if constexpr (LAYOUT == 0)
    sfa = reinterpret_cast<uint32_t*>(sf + sf_offset(row, (lane >> 3) * 4, nks * 4));
  auto put_scale = [&](int64_t s, uint32_t word) {
    if constexpr (LAYOUT == 0) {
      sfa[s * 512] = word;
    } else {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint32_t*>(sf + sfb_word_offset(row, s, lane >> 3, q4, nks, bn)) = word;
    }
  };
  if (row >= M) {  // padding row: zero scales
    if ((lane & 7) == 0)
      for (int64_t s = 0; s < nks; ++s) put_scale(s, 0u);
    return;
  }
  const int64_t nvec = K >> 3;  // 16-byte vectors of a row
  const uint4* xr = reinterpret_cast<const uint4*>(x + map(row) * ldx);
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + row * (K >> 1));
  // one step: block scale, codes, scale word
  auto step = [&](int64_t s, const uint4& v, bool code_ok) {
    float amb = bf16x2_hmax(absmax8_pair(v));
    amb = fmaxf(amb, __shfl_xor_sync(0xffffffffu, amb, 1));  // the block's other half
    const uint32_t sb = cvt_e4m3x2(0.f, __fmul_rn(amb, enc)) & 0x7F;
    const float inv = inv_tab[sb];
    const uint64_t inv2 = f32x2_splat(inv);
    if (code_ok) qr[s * 32 + lane] = e2m1_8(v, inv2);
    const uint32_t b1 = __shfl_down_sync(0xffffffffu, sb, 2);
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, sb, 4);
    const uint32_t b3 = __shfl_down_sync(0xffffffffu, sb, 6);
    if ((lane & 7) == 0) put_scale(s, sb | (b1 << 8) | (b2 << 16) | (b3 << 24));
  };
  const int64_t nfull = nvec >> 5;  // steps with all 32 lanes inside the row
  int64_t s0 = 0;
  for (; s0 + U <= nfull; s0 += U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = ld_nc_v4(xr + (s0 + u) * 32 + lane);
#pragma unroll
    for (int u = 0; u < U; ++u) step(s0 + u, v[u], true);
  }
  for (; s0 < nks; ++s0) {  // the rest: partial steps, zero past the row
    const int64_t vi = s0 * 32 + lane;
    const bool in = vi < nvec;
    step(s0, in ? ld_nc_v4(xr + vi) : make_uint4(0u, 0u, 0u, 0u), in);
  }
}

// ------------------------------------------------------------- test hook

// The device encoders on given values, for tests that compare them with a
// reference encoder value by value: mode 0 E4M3 and mode 1 E2M1 (one code per
// byte) of fp32 inputs, one thread per value, through the conversions the
// quantize kernels use; mode 2 NVFP4 16-element bf16 blocks against the
// tensor amax *amax, one thread per block, through the block encoder of the
// NVFP4-output GEMM epilogue (8 code bytes per block, then one scale byte
// per block after all the codes).
__global__ void debug_encode_kernel(int mode, const void* __restrict__ in, int64_t n,
                                    const float* __restrict__ amax, uint8_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (mode != 2) {
    if (i >= n) return;
    const float v = static_cast<const float*>(in)[i];
    out[i] = static_cast<uint8_t>(mode == 0 ? (cvt_e4m3x2(0.f, v) & 0xFF) : (cvt_e2m1x2(0.f, v) & 0xF));
    return;
  }
  const int64_t nb = n >> 4;
  if (i >= nb) return;
  const uint4* x = static_cast<const uint4*>(in) + 2 * i;
  float G, enc, amb;
  nvfp4_tensor_factors(*amax, G, enc);
  uint2 codes;
  const uint32_t sb = nvfp4_block(x[0], x[1], enc, G, codes, amb);
  reinterpret_cast<uint2*>(out)[i] = codes;
  out[8 * nb + i] = static_cast<uint8_t>(sb);
}

// ---------------------------------------------------- pre-quantized import

// Row n of the GEMM's weight operand is logical row map(n) (SwiGLU
// interleave); rows of `row_bytes` bytes, 16 bytes per thread.
__global__ void import_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                   int64_t N, int64_t row_vecs, RowMap map) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= N * row_vecs) return;
  const int64_t n = i / row_vecs, v = i - n * row_vecs;
  dst[i] = src[map(n) * row_vecs + v];
}

__global__ void import_row_scales_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                         int64_t N, RowMap map) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n < N) dst[n] = src[map(n)];
}

// Logical NVFP4 block scales [N, K/16] -> the replicated weight layout, one
// thread per (row, group of 4 blocks), the same words the weight quantizer
// writes (blocks past K/16 are 0).
__global__ void import_block_scales_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ sf,
                                           int64_t N, int64_t K, int64_t bn, RowMap map) {
  const int64_t nks = sfb_stages(K);
  const int64_t ngp = nks * 4;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * ngp) return;
  const int64_t row = idx / ngp, g = idx - row * ngp;
  const int64_t nb = K >> 4;
  const uint8_t* sr = src + map(row) * nb;
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (g * 4 + i < nb) word |= static_cast<uint32_t>(sr[g * 4 + i]) << (8 * i);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
    *reinterpret_cast<uint32_t*>(sf + sfb_word_offset(row, g >> 2, g & 3, q4, nks, bn)) = word;
}

// QKV epilogue norm weights: bf16 q and k vectors of 128 -> fp32 [2][128]
// (1.0 where a pointer is null).
__global__ void qk_weights_kernel(const __nv_bfloat16* __restrict__ qw,
                                  const __nv_bfloat16* __restrict__ kw, float* __restrict__ dst) {
  const int i = threadIdx.x;  // 0..255
  const __nv_bfloat16* src = i < QKV_HEAD_DIM ? qw : kw;
  const int j = i & (QKV_HEAD_DIM - 1);
  dst[i] = src ? __bfloat162float(src[j]) : 1.0f;
}

// The bias widened to fp32 (exact) in the GEMM's row order, so the epilogue
// adds it without unpacking bf16.
__global__ void permute_bias_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst,
                                    int64_t N, RowMap map) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < N) dst[i] = src ? __bfloat162float(src[map(i)]) : 0.f;
}

}  // namespace

// ---------------------------------------------------------------- launchers

cudaError_t launch_quant_fp8_rows(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                  float* s, RowMap map, int num_sms, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  constexpr int VPL = 8;  // 64 bf16 per thread in registers
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  auto grid_for = [&](int teams) {
    int64_t blocks = (M + teams - 1) / teams;
    int64_t cap = static_cast<int64_t>(num_sms) * 16;
    return static_cast<unsigned>(blocks < cap ? blocks : cap);
  };
  const int64_t per_warp = 32 * VPL * 8;
  cudaLaunchAttribute at[1];
  if (K <= per_warp) {
    cudaLaunchConfig_t c = pdl_config(grid_for(8), 256, 0, st, at, 0);
    return cudaLaunchKernelEx(&c, quant_fp8_rows_kernel<32, VPL>, xb, M, K, ldx, q, s, map);
  } else if (K <= 2 * per_warp) {
    cudaLaunchConfig_t c = pdl_config(grid_for(4), 256, 0, st, at, 0);
    return cudaLaunchKernelEx(&c, quant_fp8_rows_kernel<64, VPL>, xb, M, K, ldx, q, s, map);
  } else if (K <= 4 * per_warp) {
    cudaLaunchConfig_t c = pdl_config(grid_for(2), 256, 0, st, at, 0);
    return cudaLaunchKernelEx(&c, quant_fp8_rows_kernel<128, VPL>, xb, M, K, ldx, q, s, map);
  }
  cudaLaunchConfig_t c = pdl_config(grid_for(1), 256, 0, st, at, 0);
  return cudaLaunchKernelEx(&c, quant_fp8_rows_kernel<256, VPL>, xb, M, K, ldx, q, s, map);
}

cudaError_t launch_import_weights(int fmt, const void* codes, const void* scales, int64_t N,
                                  int64_t K, int64_t bn, uint8_t* wcodes, void* wscales, RowMap map,
                                  cudaStream_t st) {
  const int64_t row_vecs = (fmt == 1 ? K / 2 : K) / 16;
  const int64_t nv = N * row_vecs;
  import_rows_kernel<<<static_cast<unsigned>((nv + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(codes), reinterpret_cast<uint4*>(wcodes), N, row_vecs, map);
  if (fmt == 0) {
    import_row_scales_kernel<<<static_cast<unsigned>((N + 255) / 256), 256, 0, st>>>(
        static_cast<const float*>(scales), static_cast<float*>(wscales), N, map);
  } else {
    const int64_t nt = N * sfb_stages(K) * 4;
    import_block_scales_kernel<<<static_cast<unsigned>((nt + 255) / 256), 256, 0, st>>>(
        static_cast<const uint8_t*>(scales), static_cast<uint8_t*>(wscales), N, K, bn, map);
  }
  return cudaGetLastError();
}

cudaError_t launch_tensor_amax(const void* x, int64_t n_elems, uint32_t* amax_bits, int num_sms,
                               cudaStream_t st) {
  if (n_elems <= 0) return cudaSuccess;
  const int64_t nvec = n_elems >> 3;
  // one wave: the grid-stride loop covers the rest
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * kAmaxCtasPerSm;
  if (blocks > cap) blocks = cap;
  cudaLaunchAttribute at[1];
  cudaLaunchConfig_t c = pdl_config(static_cast<unsigned>(blocks), 256, 0, st, at, 0);
  return cudaLaunchKernelEx(&c, tensor_amax_kernel<kAmaxLoads, kAmaxCtasPerSm>,
                            static_cast<const uint4*>(x), nvec, amax_bits);
}

cudaError_t launch_quant_nvfp4(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                               uint8_t* sf, int sf_layout, int64_t bn, const uint32_t* amax_bits,
                               float* g_out, RowMap map, cudaStream_t st) {
  // weights (layout 1) pad rows to the N tile, activations to 128
  const int64_t mpad = sf_layout == 1 ? ((M + bn - 1) / bn) * bn : ((M + 127) / 128) * 128;
  const int64_t nks = sfb_stages(K);  // == sf_kchunks(K) / 4
  if (mpad <= 0 || nks <= 0) return cudaSuccess;
  const int64_t blocks = (mpad + 7) / 8;  // 8 warps (rows) per CTA
  cudaLaunchAttribute at[1];
  cudaLaunchConfig_t c = pdl_config(static_cast<unsigned>(blocks), 256, 0, st, at, 0);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (sf_layout == 1)  // weights, once per layer
    return cudaLaunchKernelEx(&c, quant_nvfp4_kernel<4, 1>, xb, M, K, ldx, q, sf, bn, nks, mpad,
                              amax_bits, g_out, map);
  // Activations: as many loads in flight as divide the row's 256-element
  // steps evenly (a remainder runs one step at a time), 8 (76 registers,
  // 3 CTAs an SM) or 6 (64 registers, 4 CTAs) before 4: e.g. K = 3072
  // (12 steps) takes 6, K = 8192 and 12288 take 8.
  const int64_t nfull = K >> 8;  // steps with all 32 lanes inside the row
  if (nfull >= 8 && nfull % 8 == 0)
    return cudaLaunchKernelEx(&c, quant_nvfp4_kernel<8, 0>, xb, M, K, ldx, q, sf, bn, nks, mpad,
                              amax_bits, g_out, map);
  if (nfull >= 6 && nfull % 6 == 0)
    return cudaLaunchKernelEx(&c, quant_nvfp4_kernel<6, 0>, xb, M, K, ldx, q, sf, bn, nks, mpad,
                              amax_bits, g_out, map);
  return cudaLaunchKernelEx(&c, quant_nvfp4_kernel<4, 0>, xb, M, K, ldx, q, sf, bn, nks, mpad,
                            amax_bits, g_out, map);
}

cudaError_t launch_debug_encode(int mode, const void* in, int64_t n, const float* amax,
                                uint8_t* out, cudaStream_t st) {
  const int64_t threads = mode == 2 ? (n >> 4) : n;
  if (threads <= 0) return cudaSuccess;
  debug_encode_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(mode, in, n,
                                                                                     amax, out);
  return cudaGetLastError();
}

cudaError_t launch_qk_weights(const void* q_bf16, const void* k_bf16, float* dst,
                              cudaStream_t st) {
  qk_weights_kernel<<<1, 2 * QKV_HEAD_DIM, 0, st>>>(static_cast<const __nv_bfloat16*>(q_bf16),
                                                     static_cast<const __nv_bfloat16*>(k_bf16), dst);
  return cudaGetLastError();
}

cudaError_t launch_permute_bias(const void* src, float* dst, int64_t N, RowMap map,
                                cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  permute_bias_kernel<<<static_cast<unsigned>((N + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(src), dst, N, map);
  return cudaGetLastError();
}

}  // namespace qlb
