// qlinear_api.cu -- the C ABI (include/qlinear.h): argument checks, weight
// workspace layout, tensor-map encoding and kernel launches.  No device
// allocation and no host synchronization in the launch calls.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/qlinear.h"
#include "internal.h"

using namespace qlb;

namespace qlb {
ql_status quantize_act_noalloc(int fmt, int64_t K, int num_sms, const void* x, int64_t M,
                               void* codes, void* scales, cudaStream_t st);
}

struct qlinear_s {
  ql_desc d;
  int64_t N, K, Nout;
  int device, num_sms;
  uint8_t* ws;
  size_t ws_bytes;
  // workspace views
  uint32_t* err;
  uint8_t* wcodes;
  float* wscale;     // FP8 per-channel scales [N]
  uint8_t* wsf;      // NVFP4 scale-factor atoms
  float* wG;         // NVFP4 global scale (device scalar)
  uint32_t* wamax;   // NVFP4 amax word used while quantizing W
  float* bias;       // fp32 [N] in the GEMM's row order
  float* qk_w;         // QKV epilogue: fp32 norm weights [2][128] (q, then k)
  float qk_eps;        // QKV epilogue: RMS normalization epsilon
  RowMap map;
  int32_t fault_mode;  // test hook, see qlinear_debug_set_fault
  int32_t bn;          // N of the GEMM tile (256)
  CUtensorMap tmB1;    // weight codes, box 128 B x 256 rows (one CTA per tile)
  CUtensorMap tmB2;    // weight codes, box 128 B x 128 rows (CTA pair per tile)
  CUtensorMap tmSFB;   // NVFP4: weight SF atoms as 2048-byte rows (CTA pair)
};

namespace {

constexpr int32_t kAbiVersion = 1;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct WsLayout {
  size_t err, codes, scales, bias, qk, total;
};

// Weight workspace: [control 1 KB][codes][scales (+16 B tail for NVFP4)][fp32 bias]
WsLayout ws_layout(const ql_desc& d) {
  WsLayout L;
  L.err = 0;
  size_t off = 1024;
  L.codes = off;
  const size_t code_bytes = d.fmt == QL_NVFP4 ? static_cast<size_t>(d.N) * d.K / 2
                                              : static_cast<size_t>(d.N) * d.K;
  off = align_up(off + code_bytes, 1024);
  L.scales = off;
  const size_t sc_bytes = d.fmt == QL_NVFP4
                              ? static_cast<size_t>(sfb_bytes(d.N, d.K, gemm_tile_n(d.fmt, d.epi))) + 16
                                            : static_cast<size_t>(d.N) * 4;
  off = align_up(off + sc_bytes, 1024);
  L.bias = off;
  off = align_up(off + static_cast<size_t>(d.N) * 4, 1024);
  L.qk = off;  // QKV epilogue: q and k norm weights (fp32, 2 x 128)
  if (d.epi == QL_EPI_QKV_NORM_ROPE) off += 1024;
  L.total = off;
  return L;
}

ql_status check_desc(const ql_desc* d) {
  if (!d) return QL_ERR_INVALID_ARG;
  if (d->fmt != QL_FP8_E4M3 && d->fmt != QL_NVFP4 && d->fmt != QL_W8A16)
    return QL_ERR_INVALID_ARG;
  if (d->epi < QL_EPI_BIAS || d->epi > QL_EPI_QKV_NORM_ROPE) return QL_ERR_INVALID_ARG;
  if (d->flags != 0 || d->variant < 0 || d->variant > 2) return QL_ERR_INVALID_ARG;
  if (d->N < 1 || d->K < 1 || d->N > (1 << 24) || d->K > (1 << 24)) return QL_ERR_INVALID_ARG;
  if (d->N % 32 != 0) return QL_ERR_INVALID_ARG;
  if (d->fmt != QL_NVFP4 && d->K % 16 != 0) return QL_ERR_INVALID_ARG;
  if (d->fmt == QL_NVFP4 && d->K % 32 != 0) return QL_ERR_INVALID_ARG;
  if (d->epi == QL_EPI_SWIGLU && d->N % 256 != 0) return QL_ERR_INVALID_ARG;
  // q | k | v of 128-column heads, each part a whole number of 256-column tiles
  if (d->epi == QL_EPI_QKV_NORM_ROPE && d->N % 768 != 0) return QL_ERR_INVALID_ARG;
  if (d->epi == QL_EPI_SPLIT_BIAS_GELU &&
      (d->split_col < 0 || d->split_col > d->N || d->split_col % 32 != 0))
    return QL_ERR_INVALID_ARG;
  return QL_OK;
}

struct DevInfo {
  int device = -1;
  int num_sms = 0;
  int major = 0, minor = 0;
};

ql_status current_device(DevInfo* out) {
  static std::mutex mu;
  static std::vector<DevInfo> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  for (auto& c : cache)
    if (c.device == dev) {
      *out = c;
      return QL_OK;
    }
  DevInfo di;
  di.device = dev;
  if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&di.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  cache.push_back(di);
  *out = di;
  return QL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D tensor map over a row-major [outer, inner] array.
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scale-factor buffers viewed as rows of 2048 bytes: uint64 elements, 256 per
// row, box = `box_rows` rows (activation atoms: 1 row = one pipeline stage of
// one 128-row block; weight chunks: 8 rows = one stage of one 256-row tile).
bool make_sf_tmap(CUtensorMap* m, const void* base, int64_t bytes, uint32_t box_rows) {
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, base, 256, bytes / 2048, 2048, 256,
                   box_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
}

ql_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return QL_OK;
  return QL_ERR_CUDA;
}

size_t act_code_bytes(const qlinear_s* h, int64_t M) {
  if (h->d.fmt == QL_W8A16) return static_cast<size_t>(M) * h->K * 2;  // the bf16 values
  return h->d.fmt == QL_NVFP4 ? static_cast<size_t>(M) * h->K / 2 : static_cast<size_t>(M) * h->K;
}

size_t act_scale_bytes(const qlinear_s* h, int64_t M) {
  if (h->d.fmt == QL_NVFP4) return static_cast<size_t>(sf_bytes(M, h->K)) + 16;
  if (h->d.fmt == QL_W8A16) return 16;  // no activation scales
  return align_up(static_cast<size_t>(M) * 4, 16);
}

}  // namespace

namespace {

// NVFP4 output of qlinear_forward_nvfp4_out.
struct QOut {
  void* codes;
  void* scales;
  const float* amax;
};

ql_status forward_impl(qlinear_t h, const void* codes, const void* scales, int64_t M,
                       const void* residual, const void* gate, int64_t gate_rows, void* out_bf16,
                       const QOut* q, const float* rope_cos, const float* rope_sin,
                       void* stream) {
  if (!h || M < 0 || M > 0x7FFFFFFF) return QL_ERR_INVALID_ARG;
  if (M == 0) return QL_OK;
  const bool w16 = h->d.fmt == QL_W8A16;  // activations are bf16, no scales
  if (!codes || (!scales && !w16) || (!q && !out_bf16)) return QL_ERR_INVALID_ARG;
  const bool gated = h->d.epi == QL_EPI_BIAS_GATED_RESIDUAL;
  if (gated && (!residual || !gate)) return QL_ERR_INVALID_ARG;
  if (gate_rows < 0 || gate_rows > 0x7FFFFFFF || (gate_rows > 0 && !gated))
    return QL_ERR_INVALID_ARG;
  const bool qkv = h->d.epi == QL_EPI_QKV_NORM_ROPE;
  if (qkv != (rope_cos != nullptr) || qkv != (rope_sin != nullptr)) return QL_ERR_INVALID_ARG;
  if (qkv && (!aligned16(rope_cos) || !aligned16(rope_sin))) return QL_ERR_ALIGNMENT;
  if (qkv && q) return QL_ERR_UNSUPPORTED;
  if (!aligned16(codes) || !aligned16(scales) || (!q && !aligned16(out_bf16)))
    return QL_ERR_ALIGNMENT;
  if (gated && (!aligned16(residual) || !aligned16(gate))) return QL_ERR_ALIGNMENT;
  if (h->Nout % 8 != 0) return QL_ERR_ALIGNMENT;
  const bool nv = h->d.fmt == QL_NVFP4;
  if (q) {
    if (!nv || h->Nout % 256 != 0) return QL_ERR_UNSUPPORTED;
    if (!q->codes || !q->scales || !q->amax) return QL_ERR_INVALID_ARG;
    if (!aligned16(q->codes) || !aligned16(q->scales) ||
        (reinterpret_cast<uintptr_t>(q->amax) & 3) != 0)
      return QL_ERR_ALIGNMENT;
  }

  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t kbytes = nv ? h->K / 2 : (w16 ? h->K * 2 : h->K);  // A bytes per row
  // one CTA per 128-row tile for a single M tile, else CTA pairs on 256 rows
  const int cg = h->d.variant == 1 ? 1 : (h->d.variant == 2 ? 2 : (M > 128 ? 2 : 1));
  const bool amap = w16 ? make_tmap(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, codes, h->K, M, kbytes,
                                    64, 128, CU_TENSOR_MAP_SWIZZLE_128B)
                        : make_tmap(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, kbytes, M, kbytes,
                                    128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!amap) return QL_ERR_CUDA;
  if (!q && !make_tmap(&p.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out_bf16, h->Nout, M,
                       h->Nout * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return QL_ERR_CUDA;
  p.tmB = cg == 2 ? h->tmB2 : h->tmB1;
  if (nv && cg == 2) {
    if (!make_sf_tmap(&p.tmSFA, scales, sf_bytes(M, h->K), 1)) return QL_ERR_CUDA;
    p.tmSFB = h->tmSFB;
  }
  if (nv) {
    p.sfa = static_cast<const uint8_t*>(scales);
    p.ga = reinterpret_cast<const float*>(p.sfa + sf_bytes(M, h->K));
    p.sfb = h->wsf;
    p.gw = h->wG;
  } else {
    p.sa = static_cast<const float*>(scales);
    p.sw = h->wscale;
  }
  p.bias = h->bias;
  p.residual = static_cast<const __nv_bfloat16*>(residual);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out = static_cast<__nv_bfloat16*>(out_bf16);
  p.err = h->err;
  p.M = static_cast<int32_t>(M);
  p.N = static_cast<int32_t>(h->N);
  p.Nout = static_cast<int32_t>(h->Nout);
  p.split_col = static_cast<int32_t>(h->d.split_col);
  p.k_blocks = static_cast<int32_t>((kbytes + 127) / 128);
  const int64_t tile_rows = 128 * cg;
  p.tiles_m = static_cast<int32_t>((M + tile_rows - 1) / tile_rows);
  p.tiles_n = static_cast<int32_t>((h->N + h->bn - 1) / h->bn);
  p.group_m = 8;
  p.sf_kchunks_a = static_cast<int32_t>(sf_kchunks(h->K));
  p.sfb_nstages = static_cast<int32_t>(sfb_stages(h->K));
  p.fault_mode = h->fault_mode;
  p.gate_rows = static_cast<int32_t>(gate_rows);
  p.qk_w = h->qk_w;
  p.rope_cos = rope_cos;
  p.rope_sin = rope_sin;
  p.k_col0 = static_cast<int32_t>(h->N / 3);
  p.qk_cols = static_cast<int32_t>(2 * (h->N / 3));
  p.qk_eps = h->qk_eps;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (q) {
    uint8_t* sf = static_cast<uint8_t*>(q->scales);
    p.q_codes = static_cast<uint8_t*>(q->codes);
    p.q_sf = sf;
    p.q_amax = q->amax;
    p.q_g = reinterpret_cast<float*>(sf + sf_bytes(M, h->Nout));
    p.q_obs = reinterpret_cast<uint32_t*>(p.q_g + 1);
    p.q_kchunks = static_cast<int32_t>(sf_kchunks(h->Nout));
    p.q_mpad = static_cast<int32_t>((M + 127) / 128 * 128);
    if (cudaMemsetAsync(p.q_obs, 0, 4, st) != cudaSuccess) {
      cudaGetLastError();
      return QL_ERR_CUDA;
    }
  }
  cudaError_t e = launch_gemm(h->d.fmt, h->d.epi, cg, q ? 1 : 0, p, h->num_sms, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace

namespace {

// Checks shared by both ways of creating a layer, then the handle with its
// workspace pointers (nothing launched yet).
ql_status begin_create(const ql_desc* desc, const void* bias_bf16, void* weight_ws,
                       size_t ws_bytes, qlinear_s** hp) {
  ql_status s = check_desc(desc);
  if (s != QL_OK) return s;
  if (!weight_ws) return QL_ERR_INVALID_ARG;
  if ((bias_bf16 && !aligned16(bias_bf16)) || (reinterpret_cast<uintptr_t>(weight_ws) & 255) != 0)
    return QL_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(*desc);
  if (ws_bytes < L.total) return QL_ERR_INVALID_ARG;
  DevInfo di;
  if ((s = current_device(&di)) != QL_OK) return s;
  if (di.major != 10) return QL_ERR_UNSUPPORTED;

  qlinear_s* h = new (std::nothrow) qlinear_s();
  if (!h) return QL_ERR_INVALID_ARG;
  h->d = *desc;
  h->N = desc->N;
  h->K = desc->K;
  h->Nout = desc->epi == QL_EPI_SWIGLU ? desc->N / 2 : desc->N;
  h->device = di.device;
  h->num_sms = di.num_sms;
  h->ws = static_cast<uint8_t*>(weight_ws);
  h->ws_bytes = ws_bytes;
  h->err = reinterpret_cast<uint32_t*>(h->ws + L.err);
  h->wcodes = h->ws + L.codes;
  h->bias = reinterpret_cast<float*>(h->ws + L.bias);
  h->qk_w = reinterpret_cast<float*>(h->ws + L.qk);
  h->qk_eps = 1e-6f;
  h->map.nout = h->Nout;
  h->map.mode = desc->epi == QL_EPI_SWIGLU ? 1 : 0;
  h->bn = gemm_tile_n(desc->fmt, desc->epi);
  if (desc->fmt != QL_NVFP4) {  // FP8 weights (QL_FP8_E4M3, QL_W8A16)
    h->wscale = reinterpret_cast<float*>(h->ws + L.scales);
  } else {
    h->wsf = h->ws + L.scales;
    h->wG = reinterpret_cast<float*>(h->wsf + sfb_bytes(h->N, h->K, h->bn));
    h->wamax = reinterpret_cast<uint32_t*>(h->wG + 1);
  }
  *hp = h;
  return QL_OK;
}

// The bias and the tensor maps of the weight operand; frees the handle when
// anything failed (including the weight kernels' launch status `e`).
ql_status finish_create(qlinear_s* h, cudaError_t e, const void* bias_bf16, cudaStream_t st,
                        qlinear_t* out) {
  if (e == cudaSuccess) e = launch_permute_bias(bias_bf16, h->bias, h->N, h->map, st);
  if (e == cudaSuccess && h->d.epi == QL_EPI_QKV_NORM_ROPE)
    e = launch_qk_weights(nullptr, nullptr, h->qk_w, st);  // weights 1 until set
  if (e != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return QL_ERR_CUDA;
  }
  const uint64_t kbytes = h->d.fmt == QL_NVFP4 ? h->K / 2 : h->K;
  // W8A16: 64 weights per stage land unswizzled for the converter warps
  const bool w16 = h->d.fmt == QL_W8A16;
  const uint32_t box = w16 ? 64 : 128;
  const CUtensorMapSwizzle sw = w16 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_tmap(&h->tmB1, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->wcodes, kbytes, h->N, kbytes, box,
                      h->bn, sw) &&
            make_tmap(&h->tmB2, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->wcodes, kbytes, h->N, kbytes, box,
                      h->bn / 2, sw);
  if (ok && h->d.fmt == QL_NVFP4)
    ok = make_sf_tmap(&h->tmSFB, h->wsf, sfb_bytes(h->N, h->K, h->bn), 8);
  if (!ok) {
    delete h;
    return QL_ERR_CUDA;
  }
  *out = h;
  return QL_OK;
}

}  // namespace

extern "C" {

int32_t qlinear_abi_version(void) { return kAbiVersion; }

const char* qlinear_status_string(ql_status s) {
  switch (s) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument";
    case QL_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case QL_ERR_UNSUPPORTED: return "unsupported device or configuration";
    case QL_ERR_CUDA: return "CUDA error";
    case QL_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

ql_status qlinear_weight_bytes(const ql_desc* desc, size_t* bytes) {
  if (!bytes) return QL_ERR_INVALID_ARG;
  ql_status s = check_desc(desc);
  if (s != QL_OK) return s;
  *bytes = ws_layout(*desc).total;
  return QL_OK;
}

ql_status qlinear_create(const ql_desc* desc, const void* w_bf16, const void* bias_bf16,
                         void* weight_ws, size_t ws_bytes, void* stream, qlinear_t* out) {
  if (!out) return QL_ERR_INVALID_ARG;
  *out = nullptr;
  if (!w_bf16) return QL_ERR_INVALID_ARG;
  if (!aligned16(w_bf16)) return QL_ERR_ALIGNMENT;
  qlinear_s* h = nullptr;
  ql_status s = begin_create(desc, bias_bf16, weight_ws, ws_bytes, &h);
  if (s != QL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(h->ws, 0, 1024, st);
  if (e == cudaSuccess && desc->fmt != QL_NVFP4) {
    e = launch_quant_fp8_rows(w_bf16, h->N, h->K, h->K, h->wcodes, h->wscale, h->map, h->num_sms,
                              st);
  } else if (e == cudaSuccess) {
    // unused scale words (rows past N) stay zero
    e = cudaMemsetAsync(h->wsf, 0, sfb_bytes(h->N, h->K, h->bn) + 16, st);
    if (e == cudaSuccess) e = launch_tensor_amax(w_bf16, h->N * h->K, h->wamax, h->num_sms, st);
    if (e == cudaSuccess)
      e = launch_quant_nvfp4(w_bf16, h->N, h->K, h->K, h->wcodes, h->wsf, 1, h->bn, h->wamax, h->wG,
                             h->map, st);
  }
  return finish_create(h, e, bias_bf16, st, out);
}

ql_status qlinear_create_prequantized(const ql_desc* desc, const void* codes, const void* scales,
                                      float global_scale, const void* bias_bf16, void* weight_ws,
                                      size_t ws_bytes, void* stream, qlinear_t* out) {
  if (!out) return QL_ERR_INVALID_ARG;
  *out = nullptr;
  if (!codes || !scales) return QL_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales)) return QL_ERR_ALIGNMENT;
  if (desc && desc->fmt == QL_NVFP4 && !(global_scale >= 0.f && global_scale <= 3.4e38f))
    return QL_ERR_INVALID_ARG;  // negative, infinite or NaN
  qlinear_s* h = nullptr;
  ql_status s = begin_create(desc, bias_bf16, weight_ws, ws_bytes, &h);
  if (s != QL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(h->ws, 0, 1024, st);
  if (e == cudaSuccess && desc->fmt == QL_NVFP4) {
    e = cudaMemsetAsync(h->wsf, 0, sfb_bytes(h->N, h->K, h->bn) + 16, st);
    // G from a host value: the copy is staged before the call returns
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(h->wG, &global_scale, sizeof(float), cudaMemcpyHostToDevice, st);
  }
  if (e == cudaSuccess)
    e = launch_import_weights(desc->fmt == QL_NVFP4 ? 1 : 0, codes, scales, h->N, h->K, h->bn,
                              h->wcodes, desc->fmt == QL_NVFP4 ? static_cast<void*>(h->wsf)
                                                               : static_cast<void*>(h->wscale),
                              h->map, st);
  return finish_create(h, e, bias_bf16, st, out);
}

ql_status qlinear_act_bytes(qlinear_t h, int64_t M, size_t* code_bytes, size_t* scale_bytes) {
  if (!h || M < 0 || M > 0x7FFFFFFF || !code_bytes || !scale_bytes) return QL_ERR_INVALID_ARG;
  *code_bytes = act_code_bytes(h, M);
  *scale_bytes = act_scale_bytes(h, M);
  return QL_OK;
}

ql_status qlinear_out_features(qlinear_t h, int64_t* nout) {
  if (!h || !nout) return QL_ERR_INVALID_ARG;
  *nout = h->Nout;
  return QL_OK;
}

ql_status qlinear_quantize_act(qlinear_t h, const void* x_bf16, int64_t M, void* codes,
                               void* scales, void* stream) {
  if (!h || M < 0 || M > 0x7FFFFFFF) return QL_ERR_INVALID_ARG;
  if (M == 0) return QL_OK;
  if (!x_bf16 || !codes || !scales) return QL_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (h->d.fmt == QL_W8A16) {
    // weight-only quantization: the activations stay bf16 (forward may also
    // be given x itself as `codes`)
    e = cudaMemcpyAsync(codes, x_bf16, static_cast<size_t>(M) * h->K * 2, cudaMemcpyDeviceToDevice,
                        st);
  } else if (h->d.fmt == QL_FP8_E4M3) {
    e = launch_quant_fp8_rows(x_bf16, M, h->K, h->K, static_cast<uint8_t*>(codes),
                              static_cast<float*>(scales), RowMap{0, 0}, h->num_sms, st);
  } else {
    uint8_t* sf = static_cast<uint8_t*>(scales);
    float* g = reinterpret_cast<float*>(sf + sf_bytes(M, h->K));
    uint32_t* amax = reinterpret_cast<uint32_t*>(g + 1);
    e = cudaMemsetAsync(amax, 0, 4, st);
    if (e == cudaSuccess) e = launch_tensor_amax(x_bf16, M * h->K, amax, h->num_sms, st);
    if (e == cudaSuccess)
      e = launch_quant_nvfp4(x_bf16, M, h->K, h->K, static_cast<uint8_t*>(codes), sf, 0, 128, amax, g,
                             RowMap{0, 0}, st);
  }
  if (e != cudaSuccess) cudaGetLastError();
  return from_cuda(e);
}

ql_status qlinear_quantize_act_noalloc(qlinear_t h, const void* x_bf16, int64_t M, void* codes,
                                       void* scales, void* stream) {
  if (!h || M < 0 || M > 0x7FFFFFFF) return QL_ERR_INVALID_ARG;
  if (h->d.fmt == QL_NVFP4 && M > QL_NOALLOC_MAX_ROWS) return QL_ERR_INVALID_ARG;
  if (M == 0) return QL_OK;
  if (!x_bf16 || !codes || !scales) return QL_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales)) return QL_ERR_ALIGNMENT;
  return qlb::quantize_act_noalloc(h->d.fmt, h->K, h->num_sms, x_bf16, M, codes, scales,
                                   static_cast<cudaStream_t>(stream));
}

ql_status qlinear_forward(qlinear_t h, const void* codes, const void* scales, int64_t M,
                          const void* residual, const void* gate, void* out_bf16, void* stream) {
  return forward_impl(h, codes, scales, M, residual, gate, 0, out_bf16, nullptr, nullptr, nullptr,
                      stream);
}

ql_status qlinear_forward_rope(qlinear_t h, const void* codes, const void* scales, int64_t M,
                               const float* rope_cos, const float* rope_sin, void* out_bf16,
                               void* stream) {
  if (!rope_cos || !rope_sin) return QL_ERR_INVALID_ARG;
  return forward_impl(h, codes, scales, M, nullptr, nullptr, 0, out_bf16, nullptr, rope_cos,
                      rope_sin, stream);
}

ql_status qlinear_set_qk_norm(qlinear_t h, const void* q_weight_bf16, const void* k_weight_bf16,
                              float eps, void* stream) {
  if (!h || h->d.epi != QL_EPI_QKV_NORM_ROPE || !q_weight_bf16 || !k_weight_bf16)
    return QL_ERR_INVALID_ARG;
  if (!(eps >= 0.f && eps <= 3.4e38f)) return QL_ERR_INVALID_ARG;
  if (!aligned16(q_weight_bf16) || !aligned16(k_weight_bf16)) return QL_ERR_ALIGNMENT;
  cudaError_t e = launch_qk_weights(q_weight_bf16, k_weight_bf16, h->qk_w,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  h->qk_eps = eps;
  return QL_OK;
}

ql_status qlinear_forward_gate_rows(qlinear_t h, const void* codes, const void* scales, int64_t M,
                                    const void* residual, const void* gate, int64_t rows_per_gate,
                                    void* out_bf16, void* stream) {
  if (rows_per_gate < 1) return QL_ERR_INVALID_ARG;
  return forward_impl(h, codes, scales, M, residual, gate, rows_per_gate, out_bf16, nullptr,
                      nullptr, nullptr, stream);
}

ql_status qlinear_forward_nvfp4_out(qlinear_t h, const void* codes, const void* scales, int64_t M,
                                    const void* residual, const void* gate, const float* amax,
                                    void* out_codes, void* out_scales, void* stream) {
  const QOut q{out_codes, out_scales, amax};
  return forward_impl(h, codes, scales, M, residual, gate, 0, nullptr, &q, nullptr, nullptr,
                      stream);
}

ql_status qlinear_export_weights(qlinear_t h, void* codes_host, void* scales_host,
                                 float* global_scale, void* stream) {
  if (!h || !codes_host || !scales_host) return QL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  const bool nv = h->d.fmt == QL_NVFP4;
  const size_t row_bytes = nv ? h->K / 2 : h->K;
  std::vector<uint8_t> codes(static_cast<size_t>(h->N) * row_bytes);
  if (cudaMemcpy(codes.data(), h->wcodes, codes.size(), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  uint8_t* ch = static_cast<uint8_t*>(codes_host);
  for (int64_t p = 0; p < h->N; ++p)
    std::memcpy(ch + h->map(p) * row_bytes, codes.data() + p * row_bytes, row_bytes);
  if (!nv) {
    std::vector<float> sc(h->N);
    if (cudaMemcpy(sc.data(), h->wscale, h->N * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaGetLastError();
      return QL_ERR_CUDA;
    }
    float* sh = static_cast<float*>(scales_host);
    for (int64_t p = 0; p < h->N; ++p) sh[h->map(p)] = sc[p];
  } else {
    std::vector<uint8_t> sf(sfb_bytes(h->N, h->K, h->bn));
    float g = 0.f;
    if (cudaMemcpy(sf.data(), h->wsf, sf.size(), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&g, h->wG, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaGetLastError();
      return QL_ERR_CUDA;
    }
    const int64_t nb = h->K / 16, nks = sfb_stages(h->K);
    uint8_t* sh = static_cast<uint8_t*>(scales_host);
    for (int64_t p = 0; p < h->N; ++p)
      for (int64_t b = 0; b < nb; ++b)
        sh[h->map(p) * nb + b] =
            sf[sfb_word_offset(p, b / 16, (b / 4) & 3, 0, nks, h->bn) + (b & 3)];
    if (global_scale) *global_scale = g;
  }
  return QL_OK;
}

ql_status qlinear_check(qlinear_t h, void* stream) {
  if (!h) return QL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  uint32_t err = 0;
  if (cudaMemcpy(&err, h->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  if (err != 0) {
    uint32_t zero = 0;
    cudaMemcpy(h->err, &zero, 4, cudaMemcpyHostToDevice);
    return QL_ERR_TIMEOUT;
  }
  return QL_OK;
}

ql_status qlinear_debug_set_fault(qlinear_t h, int32_t mode) {
  if (!h || mode < 0 || mode > 1) return QL_ERR_INVALID_ARG;
  h->fault_mode = mode;
  return QL_OK;
}

ql_status qlinear_debug_encode(int32_t mode, const void* in, int64_t n, const float* amax,
                              void* out, void* stream) {
  if (mode < 0 || mode > 2 || n < 0 || n > (int64_t{1} << 40)) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!in || !out || (mode == 2 && (!amax || n % 16 != 0))) return QL_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out) || (mode == 2 && (reinterpret_cast<uintptr_t>(amax) & 3)))
    return QL_ERR_ALIGNMENT;
  cudaError_t e = launch_debug_encode(mode, in, n, amax, static_cast<uint8_t*>(out),
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) cudaGetLastError();
  return from_cuda(e);
}

ql_status qlinear_destroy(qlinear_t h) {
  if (!h) return QL_ERR_INVALID_ARG;
  delete h;
  return QL_OK;
}

}  // extern "C"
