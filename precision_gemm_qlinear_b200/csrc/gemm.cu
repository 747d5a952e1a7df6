// gemm.cu -- persistent, warp-specialised tcgen05 GEMM with fused epilogue.
//
// One CTA per SM (persistent), 6 warps:
//   warp 0      TMA producer: A / B operand tiles (128-byte swizzle) and, for
//               NVFP4, the block-scale atoms (bulk copies) into an S-stage
//               shared-memory ring guarded by full/empty mbarriers;
//   warp 1      MMA issuer: allocates 512 TMEM columns; one elected thread
//               issues tcgen05.mma (kind::f8f6f4 for FP8, kind::mxf4nvf4 with
//               block16 E4M3 scales for NVFP4, scales staged to TMEM with
//               tcgen05.cp) into a double-buffered fp32 TMEM accumulator;
//   warps 2..5  epilogue: tcgen05.ld -> registers -> dequant scale, bias,
//               activation / gated residual -> bf16 -> swizzled shared staging
//               -> TMA store.  Each warp owns the 32 TMEM lanes (= tile rows)
//               of its sub-partition.
// Tile 128 x 256 x (128 bytes of K per stage); tiles are visited in groups of
// `group_m` M-tiles for L2 reuse.  Every mbarrier wait is bounded (about one
// second of %globaltimer); on expiry the CTA records an error code, drains
// what it issued and exits cleanly (no trap).
//
// The method: quantized GEMM with fused epilogues (algoritmulzilei.ro,
// "Accelerarea generarii de imagini cu FLUX 3 Image Klein": GEMMs with fused
// epilogues incl. SwiGLU; wavespeed.ai "Cuantizacion Dinamica FP8": the
// matmul runs on the 8-bit tensor cores).  The pages name the Blackwell
// features this uses (TMEM, 5th-generation tensor cores with FP8/FP4) in
// wavespeed.ai "Arquitectura de GPU Blackwell de NVIDIA: B200".
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace qlb {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;          // K bytes per pipeline stage
constexpr int A_BYTES = BM * BK_BYTES;  // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;  // 32 KB
constexpr int SFA_BYTES = 2048;         // 4 atoms (one per MMA K step)
constexpr int SFB_BYTES = 4096;         // 2 row blocks x 4 atoms
constexpr int NUM_THREADS = 192;
constexpr int STAGING_BYTES = 32 * 64;  // one 32 x 32 bf16 box per epilogue warp
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;  // 1 s

// Instruction descriptors (PTX ISA, "Instruction descriptor" of tcgen05.mma):
//  kind::f8f6f4 : [4,6) D format (1 = f32), [7,10) A fmt (0 = E4M3),
//                 [10,13) B fmt, [15]/[16] A/B major (0 = K), [17,23) N>>3,
//                 [24,29) M>>4.
//  kind::mxf4nvf4: [4,6) B scale id, [7,10) A fmt (1 = E2M1), [10,13) B fmt,
//                 [17,23) N>>3, [23] scale type (0 = UE4M3), [24,29) M>>4,
//                 [29,31) A scale id, [31] K size (0 = 64).
constexpr uint32_t IDESC_F8 = (1u << 4) | (0u << 7) | (0u << 10) | ((BN >> 3) << 17) |
                              ((BM >> 4) << 24);
constexpr uint32_t IDESC_F4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);

template <int FMT>
struct Cfg {
  static constexpr bool NV = (FMT == 1);
  static constexpr int STAGES = NV ? 4 : 4;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + (NV ? SFA_BYTES + SFB_BYTES : 0);
  static constexpr int NBUF = NV ? 1 : 2;  // staging buffers per epilogue warp
  static constexpr int STAGING_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = STAGING_OFF + 4 * NBUF * STAGING_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
  // TMEM columns: FP8 -> two disjoint 256-column accumulators.
  // NVFP4 -> accumulators at 0 and 192 (overlapping in [192,256)); the scale
  // factors of the current stage live in [448, 496).
  static constexpr uint32_t ACC1 = NV ? 192 : 256;
  static constexpr uint32_t SFA_COL = 448;
  static constexpr uint32_t SFB_COL = 464;
  static constexpr bool OVL = NV;
};

struct SmemBars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t ovl_free;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int32_t abort_flag;
};

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
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                         uint32_t* err, uint32_t code) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
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

__device__ __forceinline__ float gelu_tanh_f(float v) {
  // 0.5 v (1 + tanh(u)) = v * sigmoid(2u), u = sqrt(2/pi) (v + 0.044715 v^3)
  const float u2 = 1.5957691216057308f * fmaf(0.044715f * v, v * v, v);
  return __fdividef(v, 1.0f + __expf(-u2));
}

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float (&o)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = __ldg(q + i);
    o[8 * i + 0] = bf16lo(v.x);
    o[8 * i + 1] = bf16hi(v.x);
    o[8 * i + 2] = bf16lo(v.y);
    o[8 * i + 3] = bf16hi(v.y);
    o[8 * i + 4] = bf16lo(v.z);
    o[8 * i + 5] = bf16hi(v.z);
    o[8 * i + 6] = bf16lo(v.w);
    o[8 * i + 7] = bf16hi(v.w);
  }
}

template <int FMT, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1) qgemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SmemBars* sb = reinterpret_cast<SmemBars*>(smem + C::BAR_OFF);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&sb->full[s]), 1);
      mbar_init(smem_u32(&sb->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sb->acc_full[b]), 1);
      mbar_init(smem_u32(&sb->acc_empty[b]), 4);
    }
    mbar_init(smem_u32(&sb->ovl_free), 4);
    mbar_init(smem_u32(&sb->drain), 1);
    sb->abort_flag = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sb->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;

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
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!wait_bar(&sb->empty[stage], phase ^ 1, sb, p.err, ERR_WAIT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sb->full[stage]);
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          // test hook: CTA 0 never fills its first stage, so the consumer's
          // bounded wait must expire
          const bool skip = (p.fault_mode == 1 && blockIdx.x == 0 && !skipped);
          if (skip) {
            skipped = true;
          } else {
            mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
            tma_load_2d(smem_u32(st), &p.tmA, fb, kb * BK_BYTES, mb * BM);
            tma_load_2d(smem_u32(st + A_BYTES), &p.tmB, fb, kb * BK_BYTES, nb * BN);
            if constexpr (C::NV) {
              const uint8_t* sfa = p.sfa + (static_cast<int64_t>(mb) * p.sf_kchunks_a + kb * 4) * 512;
              const uint8_t* sfb0 =
                  p.sfb + (static_cast<int64_t>(2 * nb) * p.sf_kchunks_b + kb * 4) * 512;
              const uint8_t* sfb1 =
                  p.sfb + (static_cast<int64_t>(2 * nb + 1) * p.sf_kchunks_b + kb * 4) * 512;
              const uint32_t sfs = smem_u32(st + A_BYTES + B_BYTES);
              bulk_load(sfs, sfa, SFA_BYTES, fb);
              bulk_load(sfs + SFA_BYTES, sfb0, 2048, fb);
              bulk_load(sfs + SFA_BYTES + 2048, sfb1, 2048, fb);
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
      if (sb->abort_flag) {
        // let every load this thread issued land before the CTA exits
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask & (1u << s)) {
            const uint32_t a = smem_u32(&sb->full[s]);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(a, (issued_phase >> s) & 1) &&
                   globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any = false;
      int local = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!wait_bar(&sb->acc_empty[buf], (use & 1) ^ 1, sb, p.err, ERR_WAIT_MMA)) break;
        if (C::OVL && local > 0 &&
            !wait_bar(&sb->ovl_free, static_cast<uint32_t>(local - 1) & 1, sb, p.err,
                      ERR_WAIT_MMA))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (buf ? C::ACC1 : 0u);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!wait_bar(&sb->full[stage], phase, sb, p.err, ERR_WAIT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          const uint32_t a_addr = smem_u32(st);
          const uint32_t b_addr = smem_u32(st + A_BYTES);
          if constexpr (C::NV) {
            const uint32_t sfs = smem_u32(st + A_BYTES + B_BYTES);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_32x128b_warpx4(tmem + C::SFA_COL + 4 * j, sdesc_k_interleave(sfs + 512 * j));
              tc_cp_32x128b_warpx4(tmem + C::SFB_COL + 8 * j,
                                   sdesc_k_interleave(sfs + SFA_BYTES + 512 * j));
              tc_cp_32x128b_warpx4(tmem + C::SFB_COL + 8 * j + 4,
                                   sdesc_k_interleave(sfs + SFA_BYTES + 2048 + 512 * j));
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = sdesc_k_sw128(a_addr + 32 * j);
            const uint64_t bd = sdesc_k_sw128(b_addr + 32 * j);
            const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
            if constexpr (C::NV)
              mma_mxf4nvf4(d_tmem, ad, bd, IDESC_F4, tmem + C::SFA_COL + 4 * j,
                           tmem + C::SFB_COL + 8 * j, acc);
            else
              mma_f8f6f4(d_tmem, ad, bd, IDESC_F8, acc);
          }
          any = true;
          tc_commit(smem_u32(&sb->empty[stage]));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&sb->acc_full[buf]));
      }
      if (sb->abort_flag && any) {
        // no MMA may still be writing TMEM when it is released
        tc_commit(smem_u32(&sb->drain));
        const uint32_t a = smem_u32(&sb->drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int sp = warp & 3;  // TMEM sub-partition = rows [32 sp, 32 sp + 32) of the tile
    uint8_t* staging = smem + C::STAGING_OFF + (warp - 2) * C::NBUF * STAGING_BYTES;
    constexpr int NCH = (EPI == EPI_SWIGLU) ? 4 : 8;  // output chunks of 32 columns per tile
    int local = 0;
    uint32_t nstore = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!wait_bar(&sb->acc_full[buf], use & 1, sb, p.err, ERR_WAIT_EPI)) break;
      tc_fence_after();
      const int m = mb * BM + sp * 32 + lane;
      const bool row_ok = m < p.M;
      const bool slab_ok = (mb * BM + sp * 32) < p.M;
      float rs;
      if constexpr (C::NV)
        rs = __ldg(p.ga) * __ldg(p.gw);
      else
        rs = row_ok ? __ldg(p.sa + m) : 0.f;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(sp * 32) << 16) + (buf ? C::ACC1 : 0u);
      for (int ci = 0; ci < NCH; ++ci) {
        const int c = (C::OVL && buf == 0) ? (ci + NCH - 2) % NCH : ci;
        uint32_t ra[32];
        tmem_ld_32x32b_x32(tbase + 32 * c, ra);
        uint32_t rb[32];
        if constexpr (EPI == EPI_SWIGLU) tmem_ld_32x32b_x32(tbase + 128 + 32 * c, rb);
        tmem_wait_ld();
        if (C::OVL && ci == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sb->ovl_free));
        }
        if (ci == NCH - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sb->acc_empty[buf]));
        }
        // ---- epilogue math on 32 columns of this thread's row
        const int ncol = nb * BN + 32 * c;                          // GEMM column of ra[0]
        const int ocol = (EPI == EPI_SWIGLU) ? nb * (BN / 2) + 32 * c : ncol;  // output column
        if (ncol >= p.N) continue;  // past the last column (N % 32 == 0); warp-uniform
        uint32_t packed[16];
        float bias_a[32];
        load_bf16x32(p.bias + ncol, bias_a);
        if constexpr (EPI == EPI_SWIGLU) {
          float bias_b[32];
          load_bf16x32(p.bias + ncol + 128, bias_b);
          float sw_a[32], sw_b[32];
          if constexpr (!C::NV) {
            const float4* s4a = reinterpret_cast<const float4*>(p.sw + ncol);
            const float4* s4b = reinterpret_cast<const float4*>(p.sw + ncol + 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 a4 = __ldg(s4a + i), b4 = __ldg(s4b + i);
              sw_a[4 * i] = a4.x; sw_a[4 * i + 1] = a4.y; sw_a[4 * i + 2] = a4.z; sw_a[4 * i + 3] = a4.w;
              sw_b[4 * i] = b4.x; sw_b[4 * i + 1] = b4.y; sw_b[4 * i + 2] = b4.z; sw_b[4 * i + 3] = b4.w;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float o[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float sa_ = C::NV ? rs : rs * sw_a[i + h];
              const float sb_ = C::NV ? rs : rs * sw_b[i + h];
              const float g = __uint_as_float(ra[i + h]) * sa_ + bias_a[i + h];
              const float u = __uint_as_float(rb[i + h]) * sb_ + bias_b[i + h];
              o[h] = silu_f(g) * u;
            }
            packed[i >> 1] = pack_bf16x2(o[0], o[1]);
          }
        } else {
          float sw_a[32];
          if constexpr (!C::NV) {
            const float4* s4a = reinterpret_cast<const float4*>(p.sw + ncol);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 a4 = __ldg(s4a + i);
              sw_a[4 * i] = a4.x; sw_a[4 * i + 1] = a4.y; sw_a[4 * i + 2] = a4.z; sw_a[4 * i + 3] = a4.w;
            }
          }
          float gate_a[32], res_a[32];
          if constexpr (EPI == EPI_GATED_RES) {
            load_bf16x32(p.gate + ocol, gate_a);
            if (row_ok) {
              load_bf16x32(p.residual + static_cast<int64_t>(m) * p.Nout + ocol, res_a);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) res_a[i] = 0.f;
            }
          }
          const bool gelu_chunk = (EPI == EPI_BIAS_GELU) || (EPI == EPI_SPLIT && ncol >= p.split_col);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float o[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float s_ = C::NV ? rs : rs * sw_a[i + h];
              float v = __uint_as_float(ra[i + h]) * s_ + bias_a[i + h];
              if constexpr (EPI == EPI_GATED_RES) v = fmaf(gate_a[i + h], v, res_a[i + h]);
              if (EPI == EPI_BIAS_GELU || EPI == EPI_SPLIT) {
                if (gelu_chunk) v = gelu_tanh_f(v);
              }
              o[h] = v;
            }
            packed[i >> 1] = pack_bf16x2(o[0], o[1]);
          }
        }
        // ---- stage through swizzled shared memory, then one TMA store per warp
        uint8_t* sbuf = staging + (nstore % C::NBUF) * STAGING_BYTES;
        if (lane == 0) {
          if constexpr (C::NBUF == 2)
            bulk_wait_group_read<1>();
          else
            bulk_wait_group_read<0>();
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int sw = (j ^ ((lane >> 1) & 3)) << 4;
          *reinterpret_cast<uint4*>(sbuf + lane * 64 + sw) =
              make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && slab_ok) {
          tma_store_2d(&p.tmC, smem_u32(sbuf), ocol, mb * BM + sp * 32);
          bulk_commit_group();
        }
        ++nstore;
      }
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int FMT, int EPI>
cudaError_t launch_one(const GemmParams& p, int num_sms, cudaStream_t st) {
  using C = Cfg<FMT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(qgemm_kernel<FMT, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < num_sms ? tiles : num_sms;
  if (grid <= 0) return cudaSuccess;
  qgemm_kernel<FMT, EPI><<<grid, NUM_THREADS, C::SMEM_BYTES, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int fmt, int epi, const GemmParams& p, int num_sms, cudaStream_t st) {
#define QLB_CASE(F, E) \
  if (fmt == F && epi == E) return launch_one<F, E>(p, num_sms, st);
  QLB_CASE(0, EPI_BIAS)
  QLB_CASE(0, EPI_BIAS_GELU)
  QLB_CASE(0, EPI_SWIGLU)
  QLB_CASE(0, EPI_GATED_RES)
  QLB_CASE(0, EPI_SPLIT)
  QLB_CASE(1, EPI_BIAS)
  QLB_CASE(1, EPI_BIAS_GELU)
  QLB_CASE(1, EPI_SWIGLU)
  QLB_CASE(1, EPI_GATED_RES)
  QLB_CASE(1, EPI_SPLIT)
#undef QLB_CASE
  return cudaErrorInvalidValue;
}

}  // namespace qlb
