// noalloc.cu -- activation quantization for callers that cannot allocate.
//
// Some callers of this library cannot call cudaMalloc at all: code running
// inside another framework's memory pool, a plugin that is handed only the
// tensors of one operator, or a CUDA-graph replay path that must not touch
// the allocator.  qlinear_quantize_act_noalloc serves them.  For NVFP4 its
// only working memory (the partial maxima of the amax pass and the tensor
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
#include "amax.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace qlb {

namespace {

// Number of partial maxima the array holds (the amax pass runs at most this
// many CTAs); M <= QL_NOALLOC_MAX_ROWS keeps every call's scales tail and
// sizes within what the rest of the library checks.
constexpr int kMaxPartials = QL_NOALLOC_MAX_ROWS / 128;

// [0, kMaxPartials): partial amax bits, one per CTA of the amax pass;
// [kMaxPartials]: tensor amax.
static __device__ __align__(256) uint32_t g_noalloc_scratch[kMaxPartials + 64];

// Device address of g_noalloc_scratch per device, found once per device with
// that device current (the array's name in host code is only a stand-in).
// Devices 0..63 are cached; the caller rejects higher ordinals.
constexpr int kMaxDevices = 64;
uint32_t* scratch_ptr(int dev) {
  static std::mutex mu;
  static uint32_t* ptrs[kMaxDevices] = {nullptr};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
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

// Grid-stride max |x| over the whole tensor (M * K / 8 vectors of 8, the
// same pass as the tensor amax of qlinear_quantize_act): each CTA writes (does
// not accumulate) its maximum to partial[blockIdx.x], so no entry has to
// start at zero.
__global__ void __launch_bounds__(256, kAmaxCtasPerSm) partial_amax_kernel(
    const uint4* __restrict__ xv, int64_t nvec, uint32_t* __restrict__ partial) {
  const uint32_t b = cta_max_bits(grid_stride_absmax<kAmaxLoads>(xv, nvec));
  if (threadIdx.x == 0) partial[blockIdx.x] = b;
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
  if (dev >= kMaxDevices) return QL_ERR_UNSUPPORTED;
  uint32_t* scratch = scratch_ptr(dev);
  if (scratch == nullptr) return QL_ERR_CUDA;
  // amax pass: one wave of up to kAmaxCtasPerSm CTAs an SM (never more than
  // the array's partials), grid-stride over the tensor
  const int64_t nvec = M * K / 8;
  int64_t nblk = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * kAmaxCtasPerSm < kMaxPartials
                          ? static_cast<int64_t>(num_sms) * kAmaxCtasPerSm
                          : static_cast<int64_t>(kMaxPartials);
  if (nblk > cap) nblk = cap;
  uint8_t* sf = static_cast<uint8_t*>(scales);
  float* g = reinterpret_cast<float*>(sf + sf_bytes(M, K));
  // Plain launches on purpose (no programmatic overlap): this call
  // overwrites the tensor amax that the quantize kernel of a previous call on
  // the stream reads, so these kernels may only start once that kernel has
  // finished.
  partial_amax_kernel<<<static_cast<unsigned>(nblk), 256, 0, st>>>(static_cast<const uint4*>(x),
                                                                   nvec, scratch);
  reduce_amax_kernel<<<1, 256, 0, st>>>(scratch, static_cast<int>(nblk), scratch + kMaxPartials);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_quant_nvfp4(x, M, K, K, static_cast<uint8_t*>(codes), sf, 0, 128,
                           scratch + kMaxPartials, g, RowMap{0, 0}, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace qlb
