/*
 * qlinear.h -- C ABI of the B200 (sm_100a) dynamically quantized linear layer.
 *
 * One linear layer of a diffusion-transformer denoising step, in three parts:
 *   1. activation quantization, per call (qlinear_quantize_act):
 *        FP8  : per-token E4M3 codes with an fp32 scale per row (amax/448);
 *        NVFP4: E2M1 codes in 16-element K blocks, an E4M3 scale per block and
 *               an fp32 global scale for the tensor (amax/2688);
 *   2. a block-scaled tensor-core GEMM of those codes against weights that
 *      were quantized once by qlinear_create (same formats; FP8 weights carry
 *      one fp32 scale per output channel);
 *   3. a fused epilogue: dequantization scale, bias, then GELU-tanh, SwiGLU or
 *      an adaLN-gated residual add, and a bf16 store (qlinear_forward).
 *
 * Sources: "Cuantizacion Dinamica FP8" in wavespeed.ai's "Solucion de
 * WaveSpeed para Acelerar la Generacion de Imagenes FLUX.1-dev" (weights and
 * activations lowered to FP8 with run-time scales, matmul on the 8-bit tensor
 * cores); algoritmulzilei.ro, "Accelerarea generarii de imagini cu FLUX 3 Image
 * Klein pe GPU-urile Blackwell" (NVFP4 DiT; GEMMs with fused epilogues such as
 * SwiGLU); bytechap.com, "Optimizacion de la inferencia de FLUX 3 Image Klein",
 * section "Como funciona" (NVFP4 lowers both weights and activations).  The
 * pages give no API; this one follows the three-call structure of the path.
 *
 * Conventions for every call:
 *   - All device memory is owned by the caller.  The library never allocates
 *     device memory and never synchronizes the host in the launch calls
 *     (qlinear_quantize_act, qlinear_forward).
 *   - Device pointers must be 16-byte aligned (QL_ERR_ALIGNMENT otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Argument errors are returned before anything is launched.  Launch
 *     failures return QL_ERR_CUDA.  A device-side bounded wait that expired
 *     (the GEMM's pipeline watchdog, about one second) is reported as
 *     QL_ERR_TIMEOUT by the next qlinear_check on the handle.
 *   - bf16 tensors are row-major with unit inner stride.
 *   - A handle may be used from one host thread at a time.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct qlinear_s* qlinear_t;

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1, /* null pointer, bad shape/enum, size too small      */
  QL_ERR_ALIGNMENT = 2,   /* pointer or leading dimension not 16-byte aligned  */
  QL_ERR_UNSUPPORTED = 3, /* valid but not supported (e.g. no sm_100 device)   */
  QL_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed                 */
  QL_ERR_TIMEOUT = 5      /* a device-side bounded wait expired                */
} ql_status;

/* QL_W8A16: weight-only quantization -- FP8-E4M3 weights (per output channel
 * scales, as QL_FP8_E4M3) against bf16 activations that are not quantized;
 * the GEMM expands each FP8 weight stage to bf16 in shared memory and runs
 * bf16 tensor-core MMAs.  Its "codes" are the bf16 activations themselves
 * ([M, K], qlinear_quantize_act copies them; forward may be given x directly)
 * and it has no activation scales (scales may be NULL in qlinear_forward). */
typedef enum { QL_FP8_E4M3 = 0, QL_NVFP4 = 1, QL_W8A16 = 2 } ql_format;

typedef enum {
  QL_EPI_BIAS = 0,                 /* out = y + b                                  */
  QL_EPI_BIAS_GELU = 1,            /* out = gelu_tanh(y + b)                       */
  QL_EPI_SWIGLU = 2,               /* out[:,j] = silu(y[:,j]+b[j]) * (y[:,Nout+j]+b[Nout+j]),
                                      N = 2*Nout, weight rows [0,Nout) = gate,
                                      [Nout,N) = up                                */
  QL_EPI_BIAS_GATED_RESIDUAL = 3,  /* out = residual + gate[n] * (y + b)  (adaLN)  */
  QL_EPI_SPLIT_BIAS_GELU = 4,      /* n < split_col: y + b ; else gelu_tanh(y + b) */
  QL_EPI_QKV_NORM_ROPE = 5         /* QKV projection: columns [0,N/3) q, [N/3,2N/3) k,
                                      [2N/3,N) v, heads of 128; v: y + b; q, k heads:
                                      RMS-normalized (weights, eps: qlinear_set_qk_norm)
                                      then pairs (2i,2i+1) rotated (qlinear_forward_rope) */
} ql_epilogue;

/* Layer description.  y = dequant(codes_x) @ dequant(codes_w)^T, shape [M, N]. */
typedef struct {
  int32_t fmt;       /* ql_format                                                */
  int32_t epi;       /* ql_epilogue                                              */
  int64_t N;         /* output features of the GEMM (SwiGLU: 2*Nout)             */
  int64_t K;         /* input features                                           */
  int64_t split_col; /* QL_EPI_SPLIT_BIAS_GELU only: first GELU column           */
  int32_t variant;   /* 0 = default kernel configuration                         */
  int32_t flags;     /* must be 0                                                */
} ql_desc;

/* Shape rules (QL_ERR_INVALID_ARG otherwise):
 *   FP8, W8A16: K % 16 == 0, N % 32 == 0;  NVFP4: K % 32 == 0, N % 32 == 0;
 *   SwiGLU: N % 256 == 0;  QKV with norm + RoPE: N % 768 == 0;  1 <= K <= 2^24, 1 <= N <= 2^24, 0 <= M <= 2^31-1;
 *   split_col % 32 == 0 for the split epilogue.
 */

/* Bytes of device workspace the handle needs (weights codes + scales + bias +
 * a small control block).  Host only, no CUDA call. */
QL_API ql_status qlinear_weight_bytes(const ql_desc* desc, size_t* bytes);

/* Quantize W once and lay it out for the GEMM -- the weight half of the
 * dynamic quantization ("Cuantizacion Dinamica FP8", wavespeed.ai "Solucion de
 * WaveSpeed...": weights and activations both lowered to FP8; bytechap.com
 * "Como funciona": NVFP4 lowers weights as well as activations).
 *   w_bf16    : device, [N, K] bf16 master weights (read only during the call's
 *               kernels; may be freed once the stream has passed them).
 *   bias_bf16 : device, [N] bf16, or NULL for zero bias.  Copied into weight_ws.
 *   weight_ws : device, >= qlinear_weight_bytes(desc), 256-byte aligned; must
 *               stay alive and untouched until qlinear_destroy.
 *   ws_bytes  : the size of weight_ws, checked against qlinear_weight_bytes
 *               (QL_ERR_INVALID_ARG if smaller) -- an argument beyond the
 *               three-call outline of the path, so that a short buffer is an
 *               error instead of an out-of-bounds write.
 *   stream    : the kernels are enqueued here; the handle may be used on any
 *               stream ordered after this one.
 *   out       : receives the handle (host object owned by the library).
 * FP8 weights: per output channel n, s_w[n] = amax/448, codes E4M3(w*448/amax).
 * NVFP4 weights: global scale over all of W, 16-element block scales. */
QL_API ql_status qlinear_create(const ql_desc* desc, const void* w_bf16, const void* bias_bf16,
                         void* weight_ws, size_t ws_bytes, void* stream, qlinear_t* out);

/* Build a layer from weights that are already quantized -- a pre-quantized
 * checkpoint (algoritmulzilei.ro, "Accelerarea generarii de imagini cu FLUX 3
 * Image Klein pe GPU-urile Blackwell": the runtime loads BFL's pre-quantized
 * NVFP4 DiT checkpoints; paragraph after Table 1).  The weights come in the
 * logical order that qlinear_export_weights returns, so export followed by
 * this call rebuilds an identical layer:
 *   FP8  : codes [N, K] E4M3 bytes; scales fp32 [N] (s_w per output channel).
 *   NVFP4: codes [N, K/2] bytes (element 2j in the low nibble); scales
 *          [N, K/16] E4M3 block-scale bytes; global_scale = G (host value,
 *          finite and >= 0; ignored for FP8).
 *   codes, scales : device, 16-byte aligned; read by kernels enqueued on
 *                   `stream` (keep them alive until the stream passes them).
 *   Everything else as for qlinear_create (same workspace size and layout;
 *   SwiGLU rows are interleaved by the library, the caller passes gate rows
 *   0..N/2-1 then up rows). */
QL_API ql_status qlinear_create_prequantized(const ql_desc* desc, const void* codes,
                                             const void* scales, float global_scale,
                                             const void* bias_bf16, void* weight_ws,
                                             size_t ws_bytes, void* stream, qlinear_t* out);

/* Sizes of the activation code and scale buffers for M tokens.
 *   FP8  : codes [M, K] bytes; scales fp32 [M] (rounded up to 16 bytes).
 *   NVFP4: codes [M, K/2] bytes (two codes per byte, low nibble first);
 *          scales = block scales in the GEMM's tiled layout
 *          (ceil(M/128) x ceil(K/256)*4 chunks of 512 bytes) followed by a
 *          16-byte tail holding the fp32 global scale and the amax word. */
QL_API ql_status qlinear_act_bytes(qlinear_t h, int64_t M, size_t* code_bytes, size_t* scale_bytes);

/* Number of output columns of qlinear_forward (N, or N/2 for SwiGLU). */
QL_API ql_status qlinear_out_features(qlinear_t h, int64_t* nout);

/* Dynamic activation quantization (no host sync, no allocation): the scales
 * are computed from this call's activations ("Cuantizacion Dinamica FP8",
 * wavespeed.ai "Solucion de WaveSpeed...": scales found at run time;
 * algoritmulzilei.ro FLUX 3 Image Klein page: NVFP4 activations).
 *   x_bf16 : device [M, K] bf16;  codes, scales: device, sized by
 *   qlinear_act_bytes.  FP8: one fused pass (row amax, scale, cast).
 *   NVFP4: a tensor-amax pass, then the block quantize that also writes the
 *   global scale into the scales tail. */
QL_API ql_status qlinear_quantize_act(qlinear_t h, const void* x_bf16, int64_t M, void* codes,
                               void* scales, void* stream);

/* Largest M accepted by qlinear_quantize_act_noalloc for NVFP4 layers. */
#define QL_NOALLOC_MAX_ROWS 524288

/* Activation quantization for callers that cannot allocate device memory.
 * The pages have no counterpart of this call; it exists for callers that are
 * not allowed to call cudaMalloc or to own a scratch buffer -- code running
 * inside another framework's memory pool, an operator plugin that is handed
 * only its input and output tensors, or a graph-replay path that must not
 * touch the allocator.
 *   Arguments and outputs are those of qlinear_quantize_act (the caller still
 *   provides x, codes and scales, sized by qlinear_act_bytes).  FP8 layers use
 *   the same single-pass kernel, which needs no working memory.  For NVFP4
 *   the working memory of the tensor-amax reduction (the partial maxima of a
 *   grid-stride pass, then the tensor maximum) is a fixed array inside the
 *   library (QL_NOALLOC_MAX_ROWS / 128 + 64 words per device, held until the
 *   process exits) instead of the amax word in the scales tail.
 *   M > QL_NOALLOC_MAX_ROWS returns QL_ERR_INVALID_ARG before any launch.
 *   The first call on a device looks up that array's device address (no
 *   allocation) and keeps it for the life of the process; make that first
 *   call before any stream capture.  Device ordinals 64 and above return
 *   QL_ERR_UNSUPPORTED.  The kept address does not survive a reset of the
 *   device's primary context (cudaDeviceReset): do not call this entry
 *   point again in a process after such a reset.
 *   All calls on a device share the array and it keeps the last call's
 *   contents; no entry of it needs to start at zero, because every call
 *   writes the entries it reads.  Calls whose kernels overlap on the GPU
 *   (other streams, other host threads) race on the array: order them.
 *   No device memory is allocated or freed, no host sync. */
QL_API ql_status qlinear_quantize_act_noalloc(qlinear_t h, const void* x_bf16, int64_t M,
                                              void* codes, void* scales, void* stream);

/* GEMM + fused epilogue (no host sync, no allocation): the matmul on the 8-bit
 * / 4-bit tensor cores ("Cuantizacion Dinamica FP8", wavespeed.ai "Solucion de
 * WaveSpeed...") with the epilogue fused into the GEMM (algoritmulzilei.ro
 * FLUX 3 Image Klein page: GEMMs with fused epilogues, SwiGLU among them).
 *   codes, scales : as written by qlinear_quantize_act for the same M.
 *   residual      : device [M, Nout] bf16 for QL_EPI_BIAS_GATED_RESIDUAL, else NULL.
 *   gate          : device [Nout] bf16 for QL_EPI_BIAS_GATED_RESIDUAL, else NULL.
 *   out_bf16      : device [M, Nout] bf16 (Nout % 8 == 0). */
QL_API ql_status qlinear_forward(qlinear_t h, const void* codes, const void* scales, int64_t M,
                          const void* residual, const void* gate, void* out_bf16,
                          void* stream);

/* QL_EPI_QKV_NORM_ROPE: the QKV projection with query/key normalization and
 * rotary position embedding in the epilogue (algoritmulzilei.ro, "Accelerarea
 * generarii de imagini cu FLUX 3 Image Klein pe GPU-urile Blackwell": fused
 * GEMMs include QKV projections with query/key normalization and rotary
 * position embeddings; the page gives no formula).  Readings: every column
 * gets y + b; each 128-column q or k head is RMS-normalized,
 * u = v / sqrt(mean(v^2) + eps) * w  (w = the q or k weight vector), then
 * each pair (u[2i], u[2i+1]) is rotated: (a c - b s, a s + b c) with
 * c = rope_cos[m][i], s = rope_sin[m][i] for token m (fp32 tables
 * [M][64], device, 16-byte aligned; the positions behind the angles are the
 * caller's).  v heads are stored as y + b.
 *   qlinear_set_qk_norm: q and k weight vectors (device bf16 [128] each) and
 *   eps (finite, >= 0); until it is called the weights are 1 and eps 1e-6.
 *   qlinear_forward_rope: the forward call of such a layer (qlinear_forward
 *   returns QL_ERR_INVALID_ARG for it: the tables are required). */
QL_API ql_status qlinear_set_qk_norm(qlinear_t h, const void* q_weight_bf16,
                                     const void* k_weight_bf16, float eps, void* stream);
QL_API ql_status qlinear_forward_rope(qlinear_t h, const void* codes, const void* scales,
                                      int64_t M, const float* rope_cos, const float* rope_sin,
                                      void* out_bf16, void* stream);

/* qlinear_forward for QL_EPI_BIAS_GATED_RESIDUAL layers whose adaLN gate
 * differs between groups of tokens, as when the conditional and the
 * unconditional passes of classifier-free guidance are batched into one M:
 * gate is device [ceil(M / rows_per_gate), Nout] bf16 and token m uses gate
 * row m / rows_per_gate (residual + gate[m / rows_per_gate] * (y + b)).
 * rows_per_gate >= 1; other epilogues return QL_ERR_INVALID_ARG. */
QL_API ql_status qlinear_forward_gate_rows(qlinear_t h, const void* codes, const void* scales,
                                           int64_t M, const void* residual, const void* gate,
                                           int64_t rows_per_gate, void* out_bf16, void* stream);

/* GEMM + fused epilogue whose result is written as the NEXT NVFP4 layer's
 * quantized activation instead of bf16 -- the activation quantization fused
 * into the producing kernel.  Kernel fusion is one of the engine features
 * listed in wavespeed.ai's "Solucion de WaveSpeed para Acelerar la Generacion
 * de Imagenes FLUX.1-dev", section "Marco de Inferencia Propietario de
 * WaveSpeedAI"; the fused-epilogue GEMMs are in algoritmulzilei.ro's FLUX 3
 * Image Klein page.  Each epilogue value is rounded to bf16 exactly as
 * qlinear_forward would store it and then quantized to NVFP4 (16-element
 * blocks along the output columns, E4M3 block scales) with the tensor amax
 * taken from `amax` instead of from this output: G = amax/2688 and block
 * scale E4M3(amax_b * 448/amax), the qlinear_quantize_act formulas with the
 * tensor amax replaced.  Values beyond what `amax` can represent saturate.
 *   Only NVFP4 layers (QL_ERR_UNSUPPORTED otherwise), Nout % 256 == 0.
 *   codes, scales, residual, gate : as for qlinear_forward.
 *   amax       : device fp32 scalar: a calibration value or the amax observed
 *                on the previous step (read by the kernel, not by the host).
 *   out_codes  : device [M, Nout/2] bytes; out_scales: device, the block
 *                scales in the activation layout of a layer with K = Nout,
 *                followed by the 16-byte tail: fp32 G, then the largest
 *                |value| of this output as fp32 bits (the observed amax, for
 *                the next step).  Size both with qlinear_act_bytes of the
 *                next layer (K = Nout).  The pair is the codes/scales input
 *                of that layer's qlinear_forward.
 *   With amax equal to this output's true amax the buffers are byte-identical
 *   to qlinear_quantize_act of the bf16 output.  No host sync, no allocation. */
QL_API ql_status qlinear_forward_nvfp4_out(qlinear_t h, const void* codes, const void* scales,
                                           int64_t M, const void* residual, const void* gate,
                                           const float* amax, void* out_codes, void* out_scales,
                                           void* stream);

/* Copy the quantized weights to host memory in logical order (synchronizes).
 *   FP8  : codes_host [N, K] bytes, scales_host fp32 [N], global_scale ignored.
 *   NVFP4: codes_host [N, K/2] bytes, scales_host [N, K/16] E4M3 block-scale
 *          codes, *global_scale = fp32 global scale. */
QL_API ql_status qlinear_export_weights(qlinear_t h, void* codes_host, void* scales_host,
                                 float* global_scale, void* stream);

/* Synchronize `stream` and report a device-side error recorded for this
 * handle (QL_ERR_TIMEOUT) or a pending CUDA error (QL_ERR_CUDA).  Clears the
 * recorded error. */
QL_API ql_status qlinear_check(qlinear_t h, void* stream);

/* Release the host handle (the caller frees weight_ws afterwards). */
QL_API ql_status qlinear_destroy(qlinear_t h);

/* Test hook for the device-side watchdog (no counterpart on the pages).
 * mode 1: in every later qlinear_forward on this handle, the first CTA's TMA
 * producer leaves its first pipeline stage unfilled, so the MMA thread's
 * bounded wait (about one second) expires; the kernel records the expiry,
 * drains what it issued and exits, and qlinear_check returns QL_ERR_TIMEOUT.
 * The output of such a call is incomplete.  mode 0 restores normal operation.
 * Host only, no CUDA call. */
QL_API ql_status qlinear_debug_set_fault(qlinear_t h, int32_t mode);

/* Test hook for the device encoders (no counterpart on the pages): runs the
 * conversions that the quantize kernels and the NVFP4-output epilogue use on
 * caller-chosen values, so that tests can compare every code with a
 * reference encoder (ties, saturation, subnormals, non-finite inputs).
 *   mode 0: in = device fp32 [n] -> out = device u8 [n], E4M3 codes (round to
 *           nearest even, saturating to +-448; NaN stays NaN);
 *   mode 1: in = device fp32 [n] -> out = device u8 [n], one E2M1 code per
 *           byte (low nibble; saturating to +-6);
 *   mode 2: in = device bf16 [n], n % 16 == 0, 16-element blocks quantized
 *           to NVFP4 against the tensor amax in the device fp32 scalar
 *           `amax` (G = amax/2688, block scale E4M3(amax_b * 448/amax));
 *           out = device u8 [n/2 + n/16]: the codes of every block (8 bytes
 *           each, element 2j in the low nibble), then one block-scale byte
 *           per block.
 *   in and out 16-byte aligned.  Enqueued on `stream`, no host sync. */
QL_API ql_status qlinear_debug_encode(int32_t mode, const void* in, int64_t n, const float* amax,
                                      void* out, void* stream);

/* Static description of a status code. */
QL_API const char* qlinear_status_string(ql_status s);

/* ABI version of this header (incremented on incompatible changes). */
QL_API int32_t qlinear_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
