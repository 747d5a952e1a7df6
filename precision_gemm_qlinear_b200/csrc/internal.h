// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlb {

// Row order used when quantizing weights for the SwiGLU epilogue: within
// every 256-row block of the GEMM's N dimension, rows [0,128) are gate rows
// and rows [128,256) are the matching up rows, so one N tile of the GEMM holds
// both halves of 128 output columns.
struct RowMap {
  int64_t nout;   // SwiGLU output columns (gate rows are [0,nout), up rows [nout,2*nout))
  int32_t mode;   // 0 = identity, 1 = SwiGLU interleave
  __host__ __device__ __forceinline__ int64_t operator()(int64_t p) const {
    if (mode == 0) return p;
    int64_t t = p >> 8, r = p & 255;
    return r < 128 ? t * 128 + r : nout + t * 128 + (r - 128);
  }
};

// Scale-factor layout of the block-scaled GEMM ("SF atoms"): for a [rows, K]
// NVFP4 operand with one E4M3 scale per 16 K-elements, rows are grouped in
// blocks of 128 and K in chunks of 64 (4 scales).  Each (row block, K chunk)
// is a 512-byte atom; inside it the scale of row r (0..127) and K-block j
// (0..3) sits at byte (r % 32) * 16 + (r / 32) * 4 + j.  Atoms are stored
// K-chunk fastest; the number of K chunks per row block is padded to a
// multiple of 4 (one pipeline stage of 256 K-elements), padding scales are 0.
__host__ __device__ __forceinline__ int64_t sf_kchunks(int64_t K) { return ((K + 255) / 256) * 4; }
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t row, int64_t kb, int64_t kchunks) {
  return ((row >> 7) * kchunks + (kb >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (kb & 3);
}
__host__ __device__ __forceinline__ int64_t sf_bytes(int64_t rows, int64_t K) {
  return ((rows + 127) / 128) * sf_kchunks(K) * 512;
}

// -------------------------------------------------------------- quantize

cudaError_t launch_quant_fp8_rows(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                  float* s, RowMap map, int num_sms, cudaStream_t st);
cudaError_t launch_tensor_amax(const void* x, int64_t n_elems, uint32_t* amax_bits, int num_sms,
                               cudaStream_t st);
cudaError_t launch_quant_nvfp4(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                               uint8_t* sf, const uint32_t* amax_bits, float* g_out, RowMap map,
                               cudaStream_t st);
cudaError_t launch_permute_bias(const void* src, void* dst, int64_t N, RowMap map,
                                cudaStream_t st);

// ------------------------------------------------------------------ GEMM

enum Epi : int32_t { EPI_BIAS = 0, EPI_BIAS_GELU = 1, EPI_SWIGLU = 2, EPI_GATED_RES = 3,
                     EPI_SPLIT = 4 };

struct alignas(64) GemmParams {
  CUtensorMap tmA;  // activation codes [M, K(/2)] bytes, box 128 x 128 B, 128B swizzle
  CUtensorMap tmB;  // weight codes [N, K(/2)] bytes, box 128 B x 256 rows, 128B swizzle
  CUtensorMap tmC;  // output [M, Nout] bf16, box 32 x 32, 64B swizzle
  const float* sa;        // FP8: per-row activation scale [M]
  const float* sw;        // FP8: per-column weight scale [N]
  const uint8_t* sfa;     // NVFP4: activation SF atoms
  const uint8_t* sfb;     // NVFP4: weight SF atoms
  const float* ga;        // NVFP4: activation global scale (device scalar)
  const float* gw;        // NVFP4: weight global scale (device scalar)
  const __nv_bfloat16* bias;      // [N] (zeros when the layer has no bias)
  const __nv_bfloat16* residual;  // [M, Nout] or null
  const __nv_bfloat16* gate;      // [Nout] or null
  uint32_t* err;          // device error word of the handle
  int32_t M, N, Nout, split_col;
  int32_t k_blocks;       // number of 128-byte K stages
  int32_t tiles_m, tiles_n, group_m;
  int32_t sf_kchunks_a, sf_kchunks_b;
  int32_t fault_mode;     // test hook: 0 = none
};

cudaError_t launch_gemm(int fmt, int epi, const GemmParams& p, int num_sms, cudaStream_t st);

// Error codes written to the device error word by the GEMM watchdog.
enum : uint32_t { ERR_WAIT_PRODUCER = 1u, ERR_WAIT_MMA = 2u, ERR_WAIT_EPI = 4u };

}  // namespace qlb
