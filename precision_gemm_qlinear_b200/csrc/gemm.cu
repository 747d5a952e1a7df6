// gemm.cu -- persistent, warp-specialised tcgen05 GEMM with fused epilogue.
//
// Two tile configurations share one kernel template:
//   CG = 2 (default): a cluster of 2 CTAs (a "CTA pair" on two SMs) computes a
//          256 x 256 tile with tcgen05.mma.cta_group::2 (M = 256).  Each CTA
//          TMA-loads its own 128 rows of A and its own 128 rows of B (no
//          multicast); the loads of both CTAs are counted on the leader CTA's
//          mbarrier, and the leader's single MMA thread drives both tensor
//          cores.  Per SM, 32 KB of operands feed 512 cycles of FP8 MMA.
//   CG = 1: one CTA computes a 128 x 256 tile (used when M <= 128).
// Roles (10 warps):
//   warp 0      TMA producer: A / B tiles (128-byte swizzle) and, for NVFP4,
//               the block-scale atoms, into an S-stage shared-memory ring
//               guarded by full/empty mbarriers;
//   warp 1      TMEM allocation (512 columns) and, in the leader CTA, the MMA
//               issuer (kind::f8f6f4 for FP8; kind::mxf4nvf4 with block16 E4M3
//               scales for NVFP4, scales staged to TMEM with tcgen05.cp;
//               kind::f16 for weight-only layers) into a double-buffered fp32
//               TMEM accumulator;
//   warps 2..9  epilogue: tcgen05.ld -> registers -> dequant scale, bias,
//               activation / gated residual -> bf16 -> swizzled shared staging
//               -> TMA store.  Two warps share each TMEM sub-partition (32
//               rows) and split its columns.
//   Weight-only layers: warps 2..5 are the epilogue (one per sub-partition,
//   two passes) and warps 6..9 expand the FP8 weight stages to bf16.
// Tiles are visited in groups of `group_m` M-tiles for L2 reuse.  Every
// mbarrier wait is bounded (one second of %globaltimer); on expiry the CTA
// records an error code, drains what it issued and exits cleanly (no trap).
//
// The method: quantized GEMM with fused epilogues (algoritmulzilei.ro,
// "Accelerarea generarii de imagini cu FLUX 3 Image Klein": GEMMs with fused
// epilogues incl. SwiGLU; wavespeed.ai "Cuantizacion Dinamica FP8": the
// matmul runs on the 8-bit tensor cores).  wavespeed.ai "Arquitectura de GPU
// Blackwell de NVIDIA: B200" names the features used here: TMEM, CTA pairs
// that share tensor-core work, 5th-generation tensor cores with FP8/FP4.
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace qlb {

namespace {

constexpr int BM = 128;                // rows of the tile per CTA
constexpr int BK_BYTES = 128;          // K bytes per pipeline stage
constexpr int A_TILE_BYTES = BM * BK_BYTES;  // one 128-row A box: 16 KB
constexpr int STAGING_BYTES = 32 * 64;  // one 32 x 32 bf16 box
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;  // 1 s

// Instruction descriptors (PTX ISA, "Instruction descriptor" of tcgen05.mma):
//  kind::f8f6f4 : [4,6) D format (1 = f32), [7,10) A fmt (0 = E4M3),
//                 [10,13) B fmt, [15]/[16] A/B major (0 = K), [17,23) N>>3,
//                 [24,29) M>>4.
//  kind::mxf4nvf4: [4,6) B scale id, [7,10) A fmt (1 = E2M1), [10,13) B fmt,
//                 [17,23) N>>3, [23] scale type (0 = UE4M3), [24,29) M>>4,
//                 [29,31) A scale id, [31] K size (0 = 64).
template <int CG, int BN>
constexpr uint32_t idesc_f8() {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((BN >> 3) << 17) | (((BM * CG) >> 4) << 24);
}
template <int CG, int BN>
constexpr uint32_t idesc_bf16() {  // kind::f16 with A and B bf16, fp32 accumulate
  return (1u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | (((BM * CG) >> 4) << 24);
}
template <int CG, int BN>
constexpr uint32_t idesc_f4() {
  return (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | (((BM * CG) >> 4) << 24);
}

template <int FMT, int CG, int EPI>
struct Cfg {
  static constexpr bool NV = (FMT == 1);
  // FMT 2: bf16 activations x FP8 weights.  The FP8 weight stage lands raw
  // (B8) and converter warps expand it to bf16 in the MMA's B layout.
  static constexpr bool W16 = (FMT == 2);
  static constexpr bool PAIR = (CG == 2);
  // Warps: producer, MMA, epilogue, and for FMT 2 the weight-stage
  // converters.  FMT 2 tiles take long enough in the main loop that four
  // epilogue warps (two passes each, over the halves eight warps would
  // share) keep up, which leaves room for four converters at 320 threads.
  static constexpr int EPI_WARPS = W16 ? 4 : 8;
  static constexpr int EPI_PASSES = 8 / EPI_WARPS;
  static constexpr int CONV_WARPS = W16 ? 4 : 0;
  static constexpr int THREADS = 64 + 32 * (EPI_WARPS + CONV_WARPS);
  // Tile N: 256 (NVFP4 included: its eight scale-factor copies per stage
  // cost the same whatever N, so the widest MMA amortizes them best; the
  // two accumulators then overlap in TMEM, see below).
  static constexpr int BN = 256;
  static constexpr int A_BYTES = A_TILE_BYTES;  // this stage's rows of A
  static constexpr int B_BYTES = (BN / CG) * BK_BYTES;  // this CTA's rows of B
  static constexpr int SFA_BYTES = NV ? 2048 : 0;       // 4 atoms (one per MMA K step)
  static constexpr int SFB_BYTES = NV ? 16384 : 0;      // 4 replicated 4 KB chunks (all 256 B rows)
  static constexpr int B8_BYTES = W16 ? (BN / CG) * 64 : 0;  // raw FP8 weights, 64 per row
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES + B8_BYTES;
  static constexpr int STAGES = NV ? (PAIR ? 4 : 3) : (W16 ? (PAIR ? 5 : 3) : (PAIR ? 6 : 4));
  // staging buffers per epilogue warp: two unless that breaks the budget
  static constexpr int NBUF =
      (STAGES * STAGE_BYTES + EPI_WARPS * 2 * STAGING_BYTES + 512 + 1024 <= 232448) ? 2 : 1;
  static constexpr int STAGING_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = STAGING_OFF + EPI_WARPS * NBUF * STAGING_BYTES;
  static_assert(BAR_OFF + 512 + 1024 <= 232448, "shared memory budget");
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;  // + barriers + alignment slack
  // TMEM columns: FP8 -> two disjoint 256-column accumulators.  NVFP4 ->
  // the scale factors of the current stage live in [448, 496) (A in 4 x 4
  // columns, B in 4 x 8, one group per 64-element MMA step) and the two
  // 256-column accumulators are [0,256) and [192,448), overlapping in
  // [192,256); the epilogue reads the shared columns first and releases them
  // early.
  static constexpr bool OVL = NV && BN == 256;
  static constexpr uint32_t ACC1 = OVL ? 192 : BN;
  static constexpr uint32_t SFA_COL = 448;
  static constexpr uint32_t SFB_COL = 464;
  static_assert(!NV || ACC1 + BN <= SFA_COL, "TMEM budget");
  // per tile, at the leader: one per epilogue warp and pass
  static constexpr uint32_t EPI_ARRIVALS = EPI_WARPS * EPI_PASSES * CG;
};

struct SmemBars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t ovl_free;
  uint64_t b8_full[8];    // FMT 2: raw weight stage landed (this CTA)
  uint64_t conv_done[8];  // FMT 2: weight stage converted (both CTAs, at the leader)
  uint64_t drain;
  uint32_t tmem_base;
  volatile int32_t abort_flag;
};
static_assert(sizeof(SmemBars) <= 512, "barrier block exceeds its reservation");

__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.tiles_n;
  const int g = t / per_group;
  const int r = t - g * per_group;
  const int m0 = g * p.group_m;
  const int gm = min(p.group_m, p.tiles_m - m0);
  mb = m0 + r % gm;
  nb = r / gm;
}

// Bounded wait on an mbarrier phase.  Returns false when the CTA is aborting
// (another role gave up) or this wait exceeded the limit (then it raises the
// abort flag and records `code` in the device error word).
template <bool CLUSTER_ACQ = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                         uint32_t* err, uint32_t code) {
  const uint32_t a = smem_u32(bar);
  auto try_wait = [&]() {
    return CLUSTER_ACQ ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity);
  };
  if (try_wait()) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (try_wait()) return true;
    if ((it & 31) == 0) {
      if (sb->abort_flag) return false;
      if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
        sb->abort_flag = 1;
        atomicOr(err, code);
        return false;
      }
    }
  }
}

// GELU and SiLU take two special-function-unit operations per element (the
// base-2 exponential and the reciprocal).  The epilogue warps share their
// schedulers with the MMA-issuing thread, so issue slots are the scarce
// resource there; the SFU itself stays lightly loaded (two operations per
// element at 16 lanes per clock per SM is well under the tile time).
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_sfu(float d) {  // d >= 1; rcp(+inf) = +0
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  return r;
}

// GELU-tanh: 0.5 v (1 + tanh(u)) = v / (1 + e^{-2u}), u = sqrt(2/pi) (v + 0.044715 v^3),
// and e^{-2u} = 2^{v (A + B v^2)} with A = -2 sqrt(2/pi) log2(e), B = 0.044715 A.
// SiLU: g / (1 + e^{-g}), e^{-g} = 2^{-g log2(e)}.  For very negative inputs
// the exponential overflows to +inf and the reciprocal returns 0, which is the
// limit of both functions, so no clamp is needed.
constexpr float kGeluA = -2.302208198144325f;
constexpr float kGeluB = -0.1029432395800235f;
constexpr float kNegLog2e = -1.4426950408889634f;

// Two fp32 values in one 64-bit register (element 0 in the low half) for the
// packed f32x2 arithmetic of sm_100: one instruction per pair, each half
// rounded exactly as the scalar operation (fma.rn / mul.rn / add.rn), so the
// results equal the scalar code's bit for bit with half the instructions.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// bf16x2 word -> the pair of its two values
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// GELU-tanh and SiLU on 16 pairs (the forms above, pair by pair); each phase
// runs over all 16 independent pairs, so consecutive instructions do not
// depend on each other.
__device__ __forceinline__ void gelu_tanh_16x2(uint64_t (&v)[16]) {
  const uint64_t A2 = f2pack(kGeluA, kGeluA), B2 = f2pack(kGeluB, kGeluB);
  const uint64_t one2 = f2pack(1.f, 1.f);
  uint64_t d[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) d[k] = mul2(v[k], fma2(B2, mul2(v[k], v[k]), A2));
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float x0, x1;
    f2unpack(d[k], x0, x1);
    d[k] = add2(f2pack(ex2_sfu(x0), ex2_sfu(x1)), one2);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float y0, y1;
    f2unpack(d[k], y0, y1);
    v[k] = mul2(v[k], f2pack(rcp_sfu(y0), rcp_sfu(y1)));
  }
}

// g <- silu(g) * u, pair by pair
__device__ __forceinline__ void silu_mul_16x2(uint64_t (&g)[16], const uint64_t (&u)[16]) {
  const uint64_t nl2 = f2pack(kNegLog2e, kNegLog2e), one2 = f2pack(1.f, 1.f);
  uint64_t d[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float x0, x1;
    f2unpack(mul2(nl2, g[k]), x0, x1);
    d[k] = add2(f2pack(ex2_sfu(x0), ex2_sfu(x1)), one2);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float y0, y1;
    f2unpack(d[k], y0, y1);
    g[k] = mul2(mul2(g[k], f2pack(rcp_sfu(y0), rcp_sfu(y1))), u[k]);
  }
}

// 32 fp32 values (16 pairs) from global memory, 16 bytes per load
__device__ __forceinline__ void load_f2x16(const float* p, uint64_t (&o)[16]) {
  const ulonglong2* q = reinterpret_cast<const ulonglong2*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const ulonglong2 t = __ldg(q + i);
    o[2 * i] = t.x;
    o[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 32 bf16 kept packed (16 registers).
__device__ __forceinline__ void load_bf16x32_packed(const __nv_bfloat16* p, uint4 (&v)[4]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __ldg(q + i);
}
// OQ = 1: the epilogue writes NVFP4 codes and block scales for the next
// layer instead of bf16 (see GemmParams::q_*).
template <int FMT, int EPI, int CG, int OQ>
__global__ void __launch_bounds__(Cfg<FMT, CG, EPI>::THREADS, 1)
    qgemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<FMT, CG, EPI>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SmemBars* sb = reinterpret_cast<SmemBars*>(smem + C::BAR_OFF);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;  // 0 = leader of the pair
  const int unit = C::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = C::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int num_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&sb->full[s]), 1);
      mbar_init(smem_u32(&sb->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sb->acc_full[b]), 1);
      mbar_init(smem_u32(&sb->acc_empty[b]), C::EPI_ARRIVALS);
    }
    mbar_init(smem_u32(&sb->ovl_free), C::EPI_ARRIVALS);
    for (int s = 0; s < 8; ++s) {
      mbar_init(smem_u32(&sb->b8_full[s]), 1);
      mbar_init(smem_u32(&sb->conv_done[s]), CG);  // one converter warp per CTA
    }
    mbar_init(smem_u32(&sb->drain), 1);
    sb->abort_flag = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(smem_u32(&sb->tmem_base), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&sb->tmem_base), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (C::PAIR)
    cluster_sync_all();  // peer barriers are initialised before any remote arrive
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;
  // everything above overlapped the tail of the kernel that produced the
  // activation codes and scales; from here on they are read
  grid_dep_wait();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&p.tmA);
      prefetch_tmap(&p.tmB);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      bool skipped = false;
      for (int t = unit; t < num_tiles && ok; t += nunits) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int a_row = mb * (BM * CG) + static_cast<int>(rank) * BM;
        const int b_row = nb * BN + static_cast<int>(rank) * (BN / CG);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!wait_bar(&sb->empty[stage], phase ^ 1, sb, p.err, ERR_WAIT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sb->full[stage]);
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          // test hook: the leader never fills its first stage, so the MMA
          // thread's bounded wait must expire
          const bool skip = (p.fault_mode == 1 && blockIdx.x == 0 && !skipped);
          if (skip) {
            skipped = true;
          } else {
            if constexpr (C::PAIR) {
              const uint32_t lfb = mapa_shared(fb, 0);  // the leader's full barrier
              if constexpr (C::W16) {
                // bf16 activations (64 elements = 128 bytes per stage) counted
                // at the leader; the raw FP8 weights on this CTA's own barrier,
                // where this CTA's converter warps wait for them
                if (rank == 0) mbar_arrive_expect_tx(fb, 2 * C::A_BYTES);
                tma_load_2d_pair(smem_u32(st), &p.tmA, lfb, kb * 64, a_row);
                const uint32_t xb = smem_u32(&sb->b8_full[stage]);
                mbar_arrive_expect_tx(xb, C::B8_BYTES);
                tma_load_2d(smem_u32(st + C::A_BYTES + C::B_BYTES), &p.tmB, xb, kb * 64, b_row);
              } else {
              if (rank == 0) mbar_arrive_expect_tx(fb, 2 * C::STAGE_BYTES);
              tma_load_2d_pair(smem_u32(st), &p.tmA, lfb, kb * BK_BYTES, a_row);
              tma_load_2d_pair(smem_u32(st + C::A_BYTES), &p.tmB, lfb, kb * BK_BYTES, b_row);
              }
              if constexpr (C::NV) {
                // scales through 2-D maps of 2048-byte rows (uint64 x 256): the
                // A atoms of this CTA's 128 rows (one row of the map) and the
                // replicated B chunks of all 256 columns of the tile (8 rows;
                // both CTAs need them)
                const uint32_t sfs = smem_u32(st + C::A_BYTES + C::B_BYTES);
                const int ka = p.sf_kchunks_a >> 2;
                tma_load_2d_pair(sfs, &p.tmSFA, lfb, 0, (mb * 2 + static_cast<int>(rank)) * ka + kb);
                tma_load_2d_pair(sfs + C::SFA_BYTES, &p.tmSFB, lfb, 0,
                                 8 * (nb * p.sfb_nstages + kb));
              }
            } else {
              if constexpr (C::W16) {
                mbar_arrive_expect_tx(fb, C::A_BYTES);
                tma_load_2d(smem_u32(st), &p.tmA, fb, kb * 64, a_row);
                const uint32_t xb = smem_u32(&sb->b8_full[stage]);
                mbar_arrive_expect_tx(xb, C::B8_BYTES);
                tma_load_2d(smem_u32(st + C::A_BYTES + C::B_BYTES), &p.tmB, xb, kb * 64, b_row);
              } else {
              mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
              tma_load_2d(smem_u32(st), &p.tmA, fb, kb * BK_BYTES, a_row);
              tma_load_2d(smem_u32(st + C::A_BYTES), &p.tmB, fb, kb * BK_BYTES, b_row);
              }
              if constexpr (C::NV) {
                const uint8_t* sfa =
                    p.sfa + (static_cast<int64_t>(mb) * p.sf_kchunks_a + kb * 4) * 512;
                const uint8_t* sfb =
                    p.sfb + (static_cast<int64_t>(nb) * p.sfb_nstages + kb) * C::SFB_BYTES;
                const uint32_t sfs = smem_u32(st + C::A_BYTES + C::B_BYTES);
                bulk_load(sfs, sfa, C::SFA_BYTES, fb);
                bulk_load(sfs + C::SFA_BYTES, sfb, C::SFB_BYTES, fb);
              }
            }
            issued_mask |= 1u << stage;
            issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (sb->abort_flag && (rank == 0 || C::W16)) {
        // let every load counted on this CTA's barriers land before exit (the
        // leader's full barriers count both CTAs' loads; FMT 2's raw weight
        // loads are counted on each CTA's own b8_full barriers)
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask & (1u << s)) {
            const uint64_t t0 = globaltimer_ns();
            if (rank == 0) {
              const uint32_t a = smem_u32(&sb->full[s]);
              while (!mbar_try_wait(a, (issued_phase >> s) & 1) &&
                     globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
              }
            }
            if constexpr (C::W16) {
              const uint32_t x = smem_u32(&sb->b8_full[s]);
              while (!mbar_try_wait(x, (issued_phase >> s) & 1) &&
                     globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
              }
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any = false;
      int local = 0;
      // The issuing thread shares its scheduler with two epilogue warps, so
      // everything that does not change from stage to stage is computed once:
      // stage-0 operand and scale descriptors, scale-factor TMEM addresses.
      const uint32_t s0 = smem_u32(smem);
      const uint64_t d_a0 = sdesc_k_sw128(s0);
      const uint64_t d_b0 = sdesc_k_sw128(s0 + C::A_BYTES);
      const uint64_t d_sfa0 = sdesc_k_interleave(s0 + C::A_BYTES + C::B_BYTES);
      const uint64_t d_sfb0 =
          sdesc_k_interleave2(s0 + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, 128, 256);
      const uint32_t t_sfa = tmem + C::SFA_COL;
      const uint32_t t_sfb = tmem + C::SFB_COL;
      uint64_t so = 0;  // this stage's descriptor offset (16-byte units)
      // Bring in one pipeline stage: wait for its operands (weight-only
      // layers: and for their bf16 conversion by both CTAs), then, for
      // NVFP4, copy its scale factors into TMEM: per MMA step j the A atom
      // (32 x 128-bit, replicated to the 4 sub-partitions by the copy) and
      // the pre-replicated B chunk (128 x 256-bit).  The copies do not touch
      // the accumulator, so a tile's first stage is brought in before its
      // accumulator is free: the tensor pipe runs those copies while the
      // epilogue still drains the previous tile.
      auto stage_in = [&]() -> bool {
        if (!wait_bar(&sb->full[stage], phase, sb, p.err, ERR_WAIT_MMA)) return false;
        if constexpr (C::W16) {
          if (!wait_bar<true>(&sb->conv_done[stage], phase, sb, p.err, ERR_WAIT_MMA)) return false;
        }
        tc_fence_after();
        // the stage-0 descriptors advanced by the stage offset in the
        // 16-byte start-address field
        so = static_cast<uint64_t>(stage) * (C::STAGE_BYTES >> 4);
        if constexpr (C::NV) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t da = d_sfa0 + so + (512 >> 4) * j;
            const uint64_t db = d_sfb0 + so + (4096 >> 4) * j;
            if constexpr (C::PAIR) {
              tc_cp_32x128b_warpx4_pair(t_sfa + 4 * j, da);
              tc_cp_128x256b_pair(t_sfb + 8 * j, db);
            } else {
              tc_cp_32x128b_warpx4(t_sfa + 4 * j, da);
              tc_cp_128x256b(t_sfb + 8 * j, db);
            }
          }
          any = true;
        }
        return true;
      };
      // The stage's four MMA steps (K = 64 FP4 / 32 FP8 / 16 bf16 elements
      // each, 32 bytes of every operand row), then release the stage.
      auto stage_mma = [&](uint32_t d_tmem, bool first) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t ad = d_a0 + so + (32 >> 4) * j;
          const uint64_t bd = d_b0 + so + (32 >> 4) * j;
          const uint32_t acc = (!first || j > 0) ? 1u : 0u;
          if constexpr (C::NV) {
            if constexpr (C::PAIR)
              mma_mxf4nvf4_pair(d_tmem, ad, bd, idesc_f4<CG, BN>(), t_sfa + 4 * j, t_sfb + 8 * j,
                                acc);
            else
              mma_mxf4nvf4(d_tmem, ad, bd, idesc_f4<CG, BN>(), t_sfa + 4 * j, t_sfb + 8 * j, acc);
          } else if constexpr (C::W16) {
            if constexpr (C::PAIR)
              mma_bf16_pair(d_tmem, ad, bd, idesc_bf16<CG, BN>(), acc);
            else
              mma_bf16(d_tmem, ad, bd, idesc_bf16<CG, BN>(), acc);
          } else {
            if constexpr (C::PAIR)
              mma_f8f6f4_pair(d_tmem, ad, bd, idesc_f8<CG, BN>(), acc);
            else
              mma_f8f6f4(d_tmem, ad, bd, idesc_f8<CG, BN>(), acc);
          }
        }
        any = true;
        if constexpr (C::PAIR)
          tc_commit_pair_mc(smem_u32(&sb->empty[stage]), 0x3);
        else
          tc_commit(smem_u32(&sb->empty[stage]));
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      };
      for (int t = unit; t < num_tiles; t += nunits, ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!stage_in()) break;
        if (!wait_bar(&sb->acc_empty[buf], (use & 1) ^ 1, sb, p.err, ERR_WAIT_MMA)) break;
        if (C::OVL && local > 0 &&
            !wait_bar(&sb->ovl_free, static_cast<uint32_t>(local - 1) & 1, sb, p.err,
                      ERR_WAIT_MMA))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (buf ? C::ACC1 : 0u);
        stage_mma(d_tmem, true);
        for (int kb = 1; kb < p.k_blocks; ++kb) {
          if (!stage_in()) {
            ok = false;
            break;
          }
          stage_mma(d_tmem, false);
        }
        if (!ok) break;
        if constexpr (C::PAIR)
          tc_commit_pair_mc(smem_u32(&sb->acc_full[buf]), 0x3);
        else
          tc_commit(smem_u32(&sb->acc_full[buf]));
      }
      if (sb->abort_flag && any) {
        // no MMA may still be writing TMEM when it is released
        if constexpr (C::PAIR)
          tc_commit_pair_mc(smem_u32(&sb->drain), 0x1);
        else
          tc_commit(smem_u32(&sb->drain));
        const uint32_t a = smem_u32(&sb->drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
    }
  } else if (warp >= 2 + C::EPI_WARPS) {
    // ------------------------ FMT 2: FP8 weight stage -> bf16 MMA operand
    // Four warps per CTA, each owning the stages s with s % 4 == its index
    // (with five stages warp 0 owns two, with three warp 3 has none): a warp
    // converts a whole stage, so the publication of one stage to the tensor
    // core (proxy fence, release, arrive) overlaps the other warps'
    // conversion of the next ones.  Owning whole
    // stages keeps every warp's waits on a stage's barrier in the order of
    // its phases (a parity wait must never run two phases ahead).  Each lane takes
    // 16-byte chunks (16 E4M3 codes) of the raw stage -- consecutive lanes
    // read consecutive chunks, so the shared loads are contiguous -- and
    // writes them as 32 bytes of bf16 (exact) in the 128-byte-swizzled
    // K-major layout the MMA descriptor reads: 16-byte chunk c of row r at
    // B + 128 r + ((c ^ (r & 7)) << 4) (the B region is 1024-byte aligned).
    // Loads are issued in batches of 8 chunks before any of them is
    // converted.
    if constexpr (C::W16) {
      constexpr int NCH = (BN / CG) * 4;  // raw 16-byte chunks per stage
      constexpr int PER = NCH / 32;       // per lane: 8 or 16 (pair), 16 or 32 (one CTA)
      constexpr int BATCH = PER < 8 ? PER : 8;
      const int ct = lane;
      const int cw = warp - (2 + C::EPI_WARPS);  // converter warp: 0 .. CONV_WARPS - 1
      const uint32_t done_l0 = mapa_shared(smem_u32(&sb->conv_done[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = unit; t < num_tiles && ok; t += nunits) {
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (stage % C::CONV_WARPS != cw) {
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          if (!wait_bar(&sb->b8_full[stage], phase, sb, p.err, ERR_WAIT_EPI)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          const uint4* b8 = reinterpret_cast<const uint4*>(st + C::A_BYTES + C::B_BYTES);
          uint8_t* bb = st + C::A_BYTES;
#pragma unroll
          for (int i0 = 0; i0 < PER; i0 += BATCH) {
          uint4 c[BATCH];
#pragma unroll
          for (int i = 0; i < BATCH; ++i) c[i] = b8[ct + 32 * (i0 + i)];
#pragma unroll
          for (int i = 0; i < BATCH; ++i) {
            const int q = ct + 32 * (i0 + i);  // raw chunk: row q / 4, chunk q % 4
            const int r = q >> 2, j = q & 3;
            uint4 lo, hi;  // elements 0-7, 8-15 of the chunk as bf16
            e4m3x4_to_bf16x4(c[i].x, lo.x, lo.y);
            e4m3x4_to_bf16x4(c[i].y, lo.z, lo.w);
            e4m3x4_to_bf16x4(c[i].z, hi.x, hi.y);
            e4m3x4_to_bf16x4(c[i].w, hi.z, hi.w);
            *reinterpret_cast<uint4*>(bb + 128 * r + (((2 * j) ^ (r & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(bb + 128 * r + (((2 * j + 1) ^ (r & 7)) << 4)) = hi;
          }
          }
          fence_proxy_async_smem();  // generic-proxy writes -> the tensor core's reads
          __syncwarp();
          if ((threadIdx.x & 31) == 0) mbar_arrive_cluster_smem_release(done_l0 + 8u * stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int ew = warp - 2;           // 0 .. EPI_WARPS - 1
    const int sp = warp & 3;           // TMEM sub-partition: rows [32 sp, 32 sp + 32) of the CTA tile
    uint8_t* staging = smem + C::STAGING_OFF + ew * C::NBUF * STAGING_BYTES;
    // 32-column output chunks per tile
    constexpr int NCHT = (EPI == EPI_SWIGLU) ? BN / 64 : BN / 32;
    const uint32_t ovl_l0 = mapa_shared(smem_u32(&sb->ovl_free), 0);
    int local = 0;
    uint32_t nstore = 0;
    // NVFP4 output: tensor factors from the supplied amax, and the largest
    // |value| this thread quantizes (for the observed amax)
    float q_G = 0.f, q_enc = 0.f, qmax = 0.f;
    if constexpr (OQ) {
      nvfp4_tensor_factors(__ldg(p.q_amax), q_G, q_enc);
      if (blockIdx.x == 0 && ew == 0 && lane == 0) *p.q_g = q_G;
    }
    for (int t = unit; t < num_tiles; t += nunits, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!wait_bar(&sb->acc_full[buf], use & 1, sb, p.err, ERR_WAIT_EPI)) break;
      tc_fence_after();
      // Each sub-partition's work is split in two halves: with eight
      // epilogue warps the two warps of a sub-partition take one each, with
      // four each warp takes both, one per pass.  A half is alternate
      // 32-column chunks (the head, for QKV).  Every (warp, pass) releases
      // the accumulator once.
#pragma unroll 1
      for (int pass = 0; pass < C::EPI_PASSES; ++pass) {
        const int half = C::EPI_PASSES == 2 ? pass : (ew >> 2);
        const int nch = (NCHT - half + 1) >> 1;  // this half's chunks
        const int row0 = mb * (BM * CG) + static_cast<int>(rank) * BM + sp * 32;  // first row of this warp
        const int m = row0 + lane;
        const bool row_ok = m < p.M;
        const bool slab_ok = row0 < p.M;
        float rs;
        if constexpr (C::NV)
          rs = __ldg(p.ga) * __ldg(p.gw);
        else if constexpr (C::W16)
          rs = 1.f;  // bf16 activations carry no scale
        else
          rs = row_ok ? __ldg(p.sa + m) : 0.f;
        const uint32_t tbase = tmem + (static_cast<uint32_t>(sp * 32) << 16) + (buf ? C::ACC1 : 0u);
        // one 32 x 32 bf16 box: swizzled shared staging, then a TMA store
        auto store_chunk = [&](const uint32_t (&pk)[16], int ocol) {
          uint8_t* sbuf = staging + (nstore % C::NBUF) * STAGING_BYTES;
          if (lane == 0) bulk_wait_group_read<C::NBUF - 1>();
          __syncwarp();
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int sw = (j ^ ((lane >> 1) & 3)) << 4;
            *reinterpret_cast<uint4*>(sbuf + lane * 64 + sw) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && slab_ok) {
            tma_store_2d(&p.tmC, smem_u32(sbuf), ocol, row0);
            bulk_commit_group();
          }
          ++nstore;
        };
        if constexpr (EPI == EPI_QKV) {
          // One 128-column head per warp (head `half` of the tile).  Pass 1:
          // the head's sum of squares (q and k heads); pass 2: re-read TMEM,
          // normalize, weight, rotate the pairs, store.  Both passes recompute
          // v = acc * scale + bias from TMEM instead of keeping 128 values.
          const int h0 = nb * BN + QKV_HEAD_DIM * half;
          const uint32_t hb = tbase + QKV_HEAD_DIM * half;
          const bool hlive = h0 < p.N;
          const bool normed = h0 < p.qk_cols;
          const float* wgt = p.qk_w + (h0 < p.k_col0 ? 0 : QKV_HEAD_DIM);
          const int64_t mrow = row_ok ? m : p.M - 1;  // padded rows read row M-1's angles
          auto values = [&](int k, const uint32_t (&a)[32], float (&v)[32]) {
            const float4* bp = reinterpret_cast<const float4*>(p.bias + h0 + 32 * k);
            const float4* swp = reinterpret_cast<const float4*>(p.sw + h0 + 32 * k);
  #pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
              const float4 b4 = __ldg(bp + i4);
              const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
              float sw4[4] = {1.f, 1.f, 1.f, 1.f};
              if constexpr (!C::NV) {
                const float4 s4 = __ldg(swp + i4);
                sw4[0] = s4.x;
                sw4[1] = s4.y;
                sw4[2] = s4.z;
                sw4[3] = s4.w;
              }
  #pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int i = 4 * i4 + j;
                v[i] = fmaf(__uint_as_float(a[i]), C::NV ? rs : rs * sw4[j], bb[j]);
              }
            }
          };
          if (!hlive) {
            // a head past N (ragged N tile): nothing to read, release at once
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (C::OVL) mbar_arrive_cluster(ovl_l0);
              mbar_arrive_cluster(mapa_shared(smem_u32(&sb->acc_empty[buf]), 0));
            }
            continue;
          }
          // steps: 4 sum-of-squares chunks (q, k heads), then the 4 output
          // chunks; the next step's TMEM load is in flight during each step
          const int nsteps = normed ? 8 : 4;
          uint32_t ha[32], hb2[32];
          tmem_ld_32x32b_x32(hb, ha);
          float ss = 0.f, rn = 1.f;
          auto step = [&](int t, const uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
            const int k = t & 3;
            tmem_wait_ld();
            if (t + 1 < nsteps) tmem_ld_32x32b_x32(hb + 32 * ((t + 1) & 3), nxt);
            if (t == nsteps - 1) {
              // the whole head has been read: release this warp's share of both
              // buffers (the overlap columns of NVFP4's 256-wide tiles included)
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if (C::OVL) mbar_arrive_cluster(ovl_l0);
                mbar_arrive_cluster(mapa_shared(smem_u32(&sb->acc_empty[buf]), 0));
              }
            }
            float v[32];
            values(k, cur, v);
            if (normed && t < 4) {
  #pragma unroll
              for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
              if (k == 3) rn = rsqrtf(fmaf(ss, 1.f / QKV_HEAD_DIM, p.qk_eps));
              return;
            }
            if (normed) {
              const float4* wp = reinterpret_cast<const float4*>(wgt + 32 * k);
              const float4* cp =
                  reinterpret_cast<const float4*>(p.rope_cos + mrow * (QKV_HEAD_DIM / 2) + 16 * k);
              const float4* snp =
                  reinterpret_cast<const float4*>(p.rope_sin + mrow * (QKV_HEAD_DIM / 2) + 16 * k);
  #pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const float4 c4 = __ldg(cp + j4), s4 = __ldg(snp + j4);
                const float4 w0 = __ldg(wp + 2 * j4), w1 = __ldg(wp + 2 * j4 + 1);
                const float cs[4] = {c4.x, c4.y, c4.z, c4.w}, sn[4] = {s4.x, s4.y, s4.z, s4.w};
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  #pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                  const int i = 2 * (4 * j4 + tt);
                  const float x0 = v[i] * rn * wv[2 * tt], x1 = v[i + 1] * rn * wv[2 * tt + 1];
                  v[i] = fmaf(x0, cs[tt], -x1 * sn[tt]);
                  v[i + 1] = fmaf(x0, sn[tt], x1 * cs[tt]);
                }
              }
            }
            uint32_t pk[16];
  #pragma unroll
            for (int i = 0; i < 32; i += 2) pk[i >> 1] = pack_bf16x2(v[i], v[i + 1]);
            store_chunk(pk, h0 + 32 * k);
          };
  #pragma unroll 1
          for (int t = 0; t < nsteps; t += 2) {
            step(t, ha, hb2);
            step(t + 1, hb2, ha);
          }
          continue;
        }
        // chunk processed at step ci.  SwiGLU with overlapping buffers: the
        // shared columns are the up half of output chunks 2, 3 in buffer 0 and
        // the gate half of chunks 0, 1 in buffer 1; every warp holds exactly one
        // of them and reads it first.
        auto chunk_of = [&](int ci) {
          const int k = (C::OVL && buf == 0) ? (nch - 1 - ci) : ci;
          return half + 2 * k;
        };
        constexpr int NCHW = (NCHT + 1) / 2;  // most chunks a warp can have
        uint32_t acc[2][32];                   // double-buffered accumulator chunk
        uint32_t accu[32];                     // SwiGLU: the up half
        tmem_ld_32x32b_x32(tbase + 32 * chunk_of(0), acc[0]);
        if constexpr (EPI == EPI_SWIGLU) tmem_ld_32x32b_x32(tbase + 128 + 32 * chunk_of(0), accu);
  #pragma unroll
        for (int ci = 0; ci < NCHW; ++ci) {
          if (ci >= nch) break;
          const int c = chunk_of(ci);
          const int ncol = nb * BN + 32 * c;  // GEMM column of acc[..][0]
          const int ocol = (EPI == EPI_SWIGLU) ? nb * (BN / 2) + 32 * c : ncol;  // output column
          // SwiGLU (N = 256): gate columns ncol.., up columns ncol + 128..
          const bool live = ncol < p.N;  // past the last column (N % 32 == 0); warp-uniform
          // per-column and per-row operands: issued before the TMEM wait so the
          // two latencies overlap
          uint64_t bias2[16];  // the chunk's 32 bias values as pairs
          uint4 gate_a[4], res_a[4];
          if (live) {
            load_f2x16(p.bias + ncol, bias2);
            if constexpr (EPI == EPI_GATED_RES) {
              // per-batch gates (CFG-batched tokens): row m uses gate row m / gate_rows
              const __nv_bfloat16* gp = p.gate + ocol;
              if (p.gate_rows > 0)
                gp += static_cast<int64_t>((row_ok ? m : p.M - 1) / p.gate_rows) * p.Nout;
              load_bf16x32_packed(gp, gate_a);
              if (row_ok) {
                load_bf16x32_packed(p.residual + static_cast<int64_t>(m) * p.Nout + ocol, res_a);
              } else {
  #pragma unroll
                for (int i = 0; i < 4; ++i) res_a[i] = make_uint4(0u, 0u, 0u, 0u);
              }
            }
          }
          tmem_wait_ld();
          // the next chunk's accumulators stream in while this one is computed
          if constexpr (EPI != EPI_SWIGLU) {
            if (ci + 1 < nch) tmem_ld_32x32b_x32(tbase + 32 * chunk_of(ci + 1), acc[(ci + 1) & 1]);
          }
          if (C::OVL && ci == 0) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(ovl_l0);
          }
          if (ci == nch - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sb->acc_empty[buf]), 0));
          }
          const uint32_t* ra = acc[(EPI == EPI_SWIGLU) ? 0 : (ci & 1)];
          uint32_t packed[16];
          if (live) {
            // y = acc * scale + bias, pair by pair (FP8: scale = s_a[m] * s_w[n];
            // NVFP4: G_a * G_w)
            const uint64_t rs2 = f2pack(rs, rs);
            uint64_t v2[16];
            if constexpr (C::NV) {
  #pragma unroll
              for (int k = 0; k < 16; ++k)
                v2[k] = fma2(f2pack(__uint_as_float(ra[2 * k]), __uint_as_float(ra[2 * k + 1])), rs2,
                             bias2[k]);
            } else {
              uint64_t sw2[16];
              load_f2x16(p.sw + ncol, sw2);
  #pragma unroll
              for (int k = 0; k < 16; ++k)
                v2[k] = fma2(f2pack(__uint_as_float(ra[2 * k]), __uint_as_float(ra[2 * k + 1])),
                             mul2(rs2, sw2[k]), bias2[k]);
            }
            if constexpr (EPI == EPI_SWIGLU) {
              // the up half (columns ncol + 128 ..): its bias (and FP8 column
              // scales) are read here, after the gate half's are consumed
              uint64_t u2[16], t2[16];
              load_f2x16(p.bias + ncol + 128, t2);
              if constexpr (C::NV) {
  #pragma unroll
                for (int k = 0; k < 16; ++k)
                  u2[k] = fma2(f2pack(__uint_as_float(accu[2 * k]), __uint_as_float(accu[2 * k + 1])),
                               rs2, t2[k]);
              } else {
                uint64_t sw2[16];
                load_f2x16(p.sw + ncol + 128, sw2);
  #pragma unroll
                for (int k = 0; k < 16; ++k)
                  u2[k] = fma2(f2pack(__uint_as_float(accu[2 * k]), __uint_as_float(accu[2 * k + 1])),
                               mul2(rs2, sw2[k]), t2[k]);
              }
              silu_mul_16x2(v2, u2);
            } else {
              if constexpr (EPI == EPI_GATED_RES) {
  #pragma unroll
                for (int k = 0; k < 16; ++k) {
                  const uint4& gw = gate_a[k >> 2];
                  const uint4& rw = res_a[k >> 2];
                  const int q = k & 3;
                  const uint32_t g = q == 0 ? gw.x : (q == 1 ? gw.y : (q == 2 ? gw.z : gw.w));
                  const uint32_t r = q == 0 ? rw.x : (q == 1 ? rw.y : (q == 2 ? rw.z : rw.w));
                  v2[k] = fma2(bf16x2_to_f2(g), v2[k], bf16x2_to_f2(r));
                }
              }
              if constexpr (EPI == EPI_BIAS_GELU) {
                gelu_tanh_16x2(v2);
              } else if constexpr (EPI == EPI_SPLIT) {
                if (ncol >= p.split_col) gelu_tanh_16x2(v2);  // uniform per chunk
              }
            }
  #pragma unroll
            for (int k = 0; k < 16; ++k) {
              float lo, hi;
              f2unpack(v2[k], lo, hi);
              packed[k] = pack_bf16x2(lo, hi);
            }
          }
          if constexpr (EPI == EPI_SWIGLU) {
            // SwiGLU holds two halves per chunk; the next pair is loaded here,
            // into the same registers
            if (ci + 1 < nch) {
              const int cn = chunk_of(ci + 1);
              tmem_ld_32x32b_x32(tbase + 32 * cn, acc[0]);
              tmem_ld_32x32b_x32(tbase + 128 + 32 * cn, accu);
            }
          }
          if (!live) continue;
          if constexpr (OQ) {
            // two 16-element blocks of the next layer's K: codes for rows < M,
            // zero scales for the padded rows of the last 128-row block
            uint2 c0, c1;
            float a0, a1;
            const uint32_t sb0 = nvfp4_block(make_uint4(packed[0], packed[1], packed[2], packed[3]),
                                             make_uint4(packed[4], packed[5], packed[6], packed[7]),
                                             q_enc, q_G, c0, a0);
            const uint32_t sb1 =
                nvfp4_block(make_uint4(packed[8], packed[9], packed[10], packed[11]),
                            make_uint4(packed[12], packed[13], packed[14], packed[15]), q_enc, q_G,
                            c1, a1);
            uint16_t* sfp = reinterpret_cast<uint16_t*>(p.q_sf + sf_offset(m, ocol >> 4, p.q_kchunks));
            if (row_ok) {
              *reinterpret_cast<uint4*>(p.q_codes + static_cast<int64_t>(m) * (p.Nout >> 1) +
                                        (ocol >> 1)) = make_uint4(c0.x, c0.y, c1.x, c1.y);
              *sfp = static_cast<uint16_t>(sb0 | (sb1 << 8));
              qmax = fmaxf(qmax, fmaxf(a0, a1));
            } else if (m < p.q_mpad) {
              *sfp = 0;
            }
            continue;
          }
          store_chunk(packed, ocol);
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    if constexpr (OQ) {
      // |values| >= 0: float bit patterns order like unsigned integers
      const uint32_t b = __reduce_max_sync(0xffffffffu, __float_as_uint(qmax));
      if (lane == 0 && b != 0u) atomicMax(p.q_obs, b);
    }
  }

  __syncwarp();
  grid_dep_launch_dependents();
  tc_fence_before();
  if constexpr (C::PAIR)
    cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (C::PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

template <int FMT, int EPI, int CG, int OQ>
cudaError_t launch_one(const GemmParams& p, int num_sms, cudaStream_t st) {
  using C = Cfg<FMT, CG, EPI>;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // for each device this process launches on (devices past 63 every time)
  static std::atomic<uint64_t> attr_devices{0};
  auto kern = qgemm_kernel<FMT, EPI, CG, OQ>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (!(attr_devices.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_devices.fetch_or(bit, std::memory_order_release);
  }
  const int tiles = p.tiles_m * p.tiles_n;
  const int units = num_sms / CG;
  const int grid = (tiles < units ? tiles : units) * CG;
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int gemm_tile_n(int fmt, int epi) {
  if (fmt == 0) return Cfg<0, 2, EPI_BIAS>::BN;
  if (fmt == 2) {
    if (epi == EPI_SWIGLU) return Cfg<2, 2, EPI_SWIGLU>::BN;
    if (epi == EPI_QKV) return Cfg<2, 2, EPI_QKV>::BN;
    return Cfg<2, 2, EPI_BIAS>::BN;
  }
  if (epi == EPI_SWIGLU) return Cfg<1, 2, EPI_SWIGLU>::BN;
  if (epi == EPI_QKV) return Cfg<1, 2, EPI_QKV>::BN;
  return Cfg<1, 2, EPI_BIAS>::BN;
}

cudaError_t launch_gemm(int fmt, int epi, int cg, int outq, const GemmParams& p, int num_sms,
                        cudaStream_t st) {
#define QLB_CASE(F, E)                                                     \
  if (fmt == F && epi == E && !outq) {                                     \
    return cg == 2 ? launch_one<F, E, 2, 0>(p, num_sms, st)                \
                   : launch_one<F, E, 1, 0>(p, num_sms, st);               \
  }
#define QLB_CASE_Q(E)                                                      \
  if (fmt == 1 && epi == E && outq) {                                      \
    return cg == 2 ? launch_one<1, E, 2, 1>(p, num_sms, st)                \
                   : launch_one<1, E, 1, 1>(p, num_sms, st);               \
  }
  QLB_CASE(0, EPI_BIAS)
  QLB_CASE(0, EPI_BIAS_GELU)
  QLB_CASE(0, EPI_SWIGLU)
  QLB_CASE(0, EPI_GATED_RES)
  QLB_CASE(0, EPI_SPLIT)
  QLB_CASE(0, EPI_QKV)
  QLB_CASE(1, EPI_BIAS)
  QLB_CASE(1, EPI_BIAS_GELU)
  QLB_CASE(1, EPI_SWIGLU)
  QLB_CASE(1, EPI_GATED_RES)
  QLB_CASE(1, EPI_SPLIT)
  QLB_CASE(1, EPI_QKV)
  QLB_CASE_Q(EPI_BIAS)
  QLB_CASE_Q(EPI_BIAS_GELU)
  QLB_CASE_Q(EPI_SWIGLU)
  QLB_CASE_Q(EPI_GATED_RES)
  QLB_CASE_Q(EPI_SPLIT)
  QLB_CASE(2, EPI_BIAS)
  QLB_CASE(2, EPI_BIAS_GELU)
  QLB_CASE(2, EPI_SWIGLU)
  QLB_CASE(2, EPI_GATED_RES)
  QLB_CASE(2, EPI_SPLIT)
  QLB_CASE(2, EPI_QKV)
#undef QLB_CASE
#undef QLB_CASE_Q
  return cudaErrorInvalidValue;
}

}  // namespace qlb
