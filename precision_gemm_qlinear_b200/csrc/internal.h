// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
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

// Scale-factor layout of the weight (B) operand, fed to TMEM by one
// tcgen05.cp.128x256b per 64-element MMA step: for every N tile of `bn` rows
// (the GEMM tile N, 256), every stage of 256 K-elements and every MMA step j (0..3)
// there is a 4096-byte chunk of 128 rows x 32 bytes.  Row (TMEM lane)
// l = 32 q + r0 holds, in word w (0..7), the 4 scales of weight row
// bn * tile + 32 w + r0 for that step -- the same for every q (the
// replication across the four TMEM sub-partitions that the MMA reads).
// Chunks are ordered [tile][stage][j]; the 32-byte rows are stored in the
// unswizzled K-major core-matrix order the copy expects: 8-row groups 256
// bytes apart, the two 16-byte halves of a row 128 bytes apart, rows of a
// group 16 bytes apart.  Words of rows past N (and of rows past bn, for a
// tile narrower than 256) are zero.
__host__ __device__ __forceinline__ int64_t sfb_stages(int64_t K) { return (K + 255) / 256; }
__host__ __device__ __forceinline__ int64_t sfb_bytes(int64_t rows, int64_t K, int64_t bn) {
  return ((rows + bn - 1) / bn) * sfb_stages(K) * 4 * 4096;
}
// byte offset of the scale word of weight row n, stage ks, step j, replica q
__host__ __device__ __forceinline__ int64_t sfb_word_offset(int64_t n, int64_t ks, int64_t j,
                                                            int64_t q, int64_t nks, int64_t bn) {
  const int64_t tile = n / bn, loc = n - tile * bn;
  const int64_t l = q * 32 + (loc & 31), w = loc >> 5;
  return ((tile * nks + ks) * 4 + j) * 4096 + (l >> 3) * 256 + (w >> 2) * 128 + (l & 7) * 16 +
         (w & 3) * 4;
}

// Launch configuration with programmatic stream serialization: the kernel may
// start while the previous kernel in the stream finishes; it calls
// grid_dep_wait() before touching anything that kernel produced.
inline cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                     cudaLaunchAttribute* attrs, unsigned nattrs_before) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attrs[nattrs_before].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[nattrs_before].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = nattrs_before + 1;
  return cfg;
}

// -------------------------------------------------------------- quantize

cudaError_t launch_quant_fp8_rows(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                  float* s, RowMap map, int num_sms, cudaStream_t st);
// Pre-quantized weights in logical order (fmt 0: codes [N, K], fp32 row scales
// [N]; fmt 1: codes [N, K/2], block scales [N, K/16]) -> the GEMM's layout
// (rows permuted by map; NVFP4 scales replicated as the quantizer writes them,
// into a zeroed region).
cudaError_t launch_import_weights(int fmt, const void* codes, const void* scales, int64_t N,
                                  int64_t K, int64_t bn, uint8_t* wcodes, void* wscales, RowMap map,
                                  cudaStream_t st);
// QKV epilogue norm weights (bf16 [128] each, null = all 1) -> fp32 [2][128].
cudaError_t launch_qk_weights(const void* q_bf16, const void* k_bf16, float* dst,
                              cudaStream_t st);
cudaError_t launch_tensor_amax(const void* x, int64_t n_elems, uint32_t* amax_bits, int num_sms,
                               cudaStream_t st);
// sf_layout: 0 = activation (A operand) atoms [sf_offset], 1 = weight (B
// operand) replicated chunks [sfb_word_offset] for N tiles of `bn` rows.
cudaError_t launch_quant_nvfp4(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                               uint8_t* sf, int sf_layout, int64_t bn, const uint32_t* amax_bits,
                               float* g_out, RowMap map, cudaStream_t st);
// Test hook: mode 0 / 1 E4M3 / E2M1 codes of fp32 in[n]; mode 2 NVFP4 blocks
// of bf16 in[n] (n % 16 == 0) against the tensor amax *amax (codes, then
// the block scales).
cudaError_t launch_debug_encode(int mode, const void* in, int64_t n, const float* amax,
                                uint8_t* out, cudaStream_t st);
// bf16 bias [N] (or null = zeros) -> fp32 [N] in the GEMM's row order.
cudaError_t launch_permute_bias(const void* src, float* dst, int64_t N, RowMap map,
                                cudaStream_t st);

// ------------------------------------------------------------------ GEMM

enum Epi : int32_t { EPI_BIAS = 0, EPI_BIAS_GELU = 1, EPI_SWIGLU = 2, EPI_GATED_RES = 3,
                     EPI_SPLIT = 4, EPI_QKV = 5 };

// Head dimension of the QKV epilogue (per-head RMS normalization + rotary
// embedding of q and k).
constexpr int QKV_HEAD_DIM = 128;

struct alignas(64) GemmParams {
  CUtensorMap tmA;  // activation codes [M, K(/2)] bytes, box 128 x 128 B, 128B swizzle
  CUtensorMap tmB;  // weight codes [N, K(/2)] bytes, box 128 B x (256 / CG) rows, 128B swizzle
  CUtensorMap tmC;  // output [M, Nout] bf16, box 32 x 32, 64B swizzle
  CUtensorMap tmSFA;  // NVFP4 pair mode: activation SF atoms as rows of 2048 bytes
  CUtensorMap tmSFB;  // NVFP4 pair mode: weight SF chunks as rows of 2048 bytes
  const float* sa;        // FP8: per-row activation scale [M]
  const float* sw;        // FP8: per-column weight scale [N]
  const uint8_t* sfa;     // NVFP4: activation SF atoms (sf_offset layout)
  const uint8_t* sfb;     // NVFP4: weight SF chunks (sfb_word_offset layout)
  const float* ga;        // NVFP4: activation global scale (device scalar)
  const float* gw;        // NVFP4: weight global scale (device scalar)
  const float* bias;              // fp32 [N] (zeros when the layer has no bias)
  const __nv_bfloat16* residual;  // [M, Nout] or null
  const __nv_bfloat16* gate;      // [Nout] or null
  __nv_bfloat16* out;             // [M, Nout] (the TMA store map tmC covers the same buffer)
  uint32_t* err;          // device error word of the handle
  int32_t M, N, Nout, split_col;
  int32_t k_blocks;       // number of 128-byte K stages
  int32_t tiles_m, tiles_n, group_m;
  int32_t sf_kchunks_a, sfb_nstages;
  int32_t fault_mode;     // test hook: 0 = none
  int32_t gate_rows;      // gated residual: 0 = one gate [Nout]; else gate [M/gate_rows, Nout]
  // QKV epilogue: columns [0, k_col0) are q heads, [k_col0, qk_cols) k heads,
  // the rest v; qk_w = fp32 norm weights [2][128] (q then k); rope tables
  // fp32 [M][64] (cos, sin of each token's angle per pair)
  const float* qk_w;
  const float* rope_cos;
  const float* rope_sin;
  int32_t k_col0, qk_cols;
  float qk_eps;
  // NVFP4 output (instead of bf16): the epilogue's bf16 values quantized for a
  // next layer with K = Nout, against the tensor amax *q_amax supplied by the
  // caller.  Codes [M, Nout/2]; block scales in the sf_offset layout (padded
  // rows [M, q_mpad) get zero scales); *q_g = G; *q_obs = max |value| seen.
  uint8_t* q_codes;
  uint8_t* q_sf;
  const float* q_amax;
  float* q_g;
  uint32_t* q_obs;
  int32_t q_kchunks, q_mpad;
};

// cg = 1: one CTA per 128 x 256 tile; cg = 2: a CTA pair per 256 x 256 tile.
// outq = 1: NVFP4 output through the q_* fields (NVFP4 layers only).
cudaError_t launch_gemm(int fmt, int epi, int cg, int outq, const GemmParams& p, int num_sms,
                        cudaStream_t st);
// N of the GEMM tile for a format / epilogue (the weight scale layout uses it).
int gemm_tile_n(int fmt, int epi);

// Error codes written to the device error word by the GEMM watchdog.
enum : uint32_t { ERR_WAIT_PRODUCER = 1u, ERR_WAIT_MMA = 2u, ERR_WAIT_EPI = 4u };

}  // namespace qlb
