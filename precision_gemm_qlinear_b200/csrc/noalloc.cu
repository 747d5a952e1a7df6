// noalloc.cu -- activation quantization for callers that cannot allocate.
//
// Some callers of this library cannot call cudaMalloc at all: code running
// inside another framework's memory pool, a plugin that is handed only the
// tensors of one operator, or a CUDA-graph replay path that must not touch
// the allocator.  qlinear_quantize_act_noalloc serves them.  For NVFP4 its
// only working memory (one partial amax per 128-row block and the tensor
// amax) lives in a file-scope device array that is part of this library, so
// the caller passes nothing but the input and the two output buffers.
//
// The array is shared by every call on a device and keeps the last call's
// contents.  Nothing in it has to start at zero: each call writes every
// partial it later reads before reading it.  Calls that overlap on the GPU
// (different streams, or different host threads on one device) race on it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qlinear.h"
#include "internal.h"
#include "ptx.cuh"

namespace qlb {

namespace {

// Maximum number of 128-row blocks of one call (M <= 128 * 4096 = 524288 tokens).
constexpr int kMaxRowBlocks = QL_NOALLOC_MAX_ROWS / 128;

// [0, kMaxRowBlocks): partial amax bits per row block; [kMaxRowBlocks]: tensor amax.
static __device__ __align__(256) uint32_t g_noalloc_scratch[kMaxRowBlocks + 64];

// Device address of g_noalloc_scratch per device, found once per device with
// that device current (the array's name in host code is only a stand-in).
uint32_t* scratch_ptr(int dev) {
  static std::mutex mu;
  static uint32_t* ptrs[64] = {nullptr};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  return ptrs[dev];
}

__device__ __forceinline__ float absmax8_bits(const uint4& v) {
  float m = fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))));
  m = fmaxf(m, fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w))));
  return m;
}

// One CTA per 128-row block: max |x| over the block, written (not
// accumulated) to partial[blockIdx.x].
__global__ void __launch_bounds__(256) rowblock_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                            int64_t M, int64_t K,
                                                            uint32_t* __restrict__ partial) {
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int64_t rows = (M - r0) < 128 ? (M - r0) : 128;
  const int64_t nvec = rows * K / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x + r0 * K);
  float m = 0.f;
  for (int64_t i = threadIdx.x; i < nvec; i += blockDim.x) m = fmaxf(m, absmax8_bits(__ldg(xv + i)));
  uint32_t a = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = max(b, red[w]);
    partial[blockIdx.x] = b;
  }
}

// One CTA: tensor amax = max over the nblocks partials, written to *out.
__global__ void __launch_bounds__(256) reduce_amax_kernel(const uint32_t* __restrict__ partial,
                                                          int nblocks, uint32_t* __restrict__ out) {
  uint32_t m = 0;
  for (int i = threadIdx.x; i < nblocks; i += blockDim.x) m = max(m, partial[i]);
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = max(b, red[w]);
    *out = b;
  }
}

}  // namespace

ql_status quantize_act_noalloc(int fmt, int64_t K, int num_sms, const void* x, int64_t M,
                               void* codes, void* scales, cudaStream_t st) {
  if (fmt == QL_W8A16) {
    // weight-only layers keep bf16 activations: a copy, no working memory
    if (cudaMemcpyAsync(codes, x, static_cast<size_t>(M) * K * 2, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess) {
      cudaGetLastError();
      return QL_ERR_CUDA;
    }
    return QL_OK;
  }
  if (fmt == QL_FP8_E4M3) {
    // per-token FP8 is a single pass with no working memory at all
    cudaError_t e = launch_quant_fp8_rows(x, M, K, K, static_cast<uint8_t*>(codes),
                                          static_cast<float*>(scales), RowMap{0, 0}, num_sms, st);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return QL_ERR_CUDA;
    }
    return QL_OK;
  }
  if (M > QL_NOALLOC_MAX_ROWS) return QL_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  uint32_t* scratch = scratch_ptr(dev);
  if (scratch == nullptr) return QL_ERR_CUDA;
  const int nrb = static_cast<int>((M + 127) / 128);
  uint8_t* sf = static_cast<uint8_t*>(scales);
  float* g = reinterpret_cast<float*>(sf + sf_bytes(M, K));
  rowblock_amax_kernel<<<nrb, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), M, K, scratch);
  reduce_amax_kernel<<<1, 256, 0, st>>>(scratch, nrb, scratch + kMaxRowBlocks);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_quant_nvfp4(x, M, K, K, static_cast<uint8_t*>(codes), sf, 0, 128,
                           scratch + kMaxRowBlocks,
                           g, RowMap{0, 0}, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace qlb
