// hq_gemm.cu -- integer GEMM with the fused HadaNorm epilogue on 5th-generation
// tensor cores (tcgen05, kind::i8, int32 accumulator in tensor memory).
//
//   acc[t,n] = sum_k A[t,k] * B[n,k]                 (HaTQ Sec. IV-B Eq. (14))
//   Y[t,n]   = bf16( s_x[t] * s_w[n] * acc[t,n]      (accumulator scale, HaTQ Eq. (18))
//                    + b[n] + mu_t * colsum[n] )      (b~ = b + mu W~, HadaNorm Eq. (1))
//
// A = activation codes [T,K] int8, B = weight codes [N,K] int8, both K-major.
// Persistent CTAs (one per SM) walk output tiles of 128 x BN.  Roles:
//   warp 0      one thread issues TMA tensor loads (128-byte swizzle) of the
//               A and B K-slices into a ring of shared-memory stages;
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               (128 x BN x 32 per instruction) and commits each stage back
//               to the producer and each finished accumulator to the epilogue;
//   warps 2..5  read the accumulator from tensor memory (tcgen05.ld), apply
//               the epilogue in fp32 and store bf16 rows.
// Two accumulators in tensor memory let the epilogue of one tile overlap the
// main loop of the next.  Every wait is bounded; a timeout records
// HQ_ERR_TIMEOUT in the device error word and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "hq_device.cuh"
#include "hq_kernels.h"

namespace hq {

namespace {

constexpr int BM = 128;
constexpr int BK = 128;  // K bytes per stage: one 128-byte swizzle row
constexpr int kGemmThreads = 192;
constexpr int kStageBudget = 216 * 1024;

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kStageBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  // instruction descriptor: D s32 (bits 4-5 = 2), A and B signed int8 (bits
  // 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at 24-28.
  static constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) |
                                    (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static constexpr size_t SMEM = size_t(STAGES) * STAGE_BYTES + 1024 /*align*/ + 256 /*ctl*/;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(B_BYTES % 1024 == 0, "stage bases must stay 1024-byte aligned");
};

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked along M/N (stride byte offset 1024), leading byte offset unused (1),
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;
  d |= uint64_t(1024 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

}  // namespace

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + size_t(C::STAGES) * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + size_t(C::STAGES) * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtl wc{p.err, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.num_m_tiles * p.num_n_tiles;
  const int KB = (p.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_idx = tile % p.num_m_tiles;
        const int n_idx = tile / p.num_m_tiles;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(&empty[stage], phase ^ 1u, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + size_t(stage) * C::A_BYTES, &tmA, kb * BK, m_idx * BM, &full[stage]);
          tma_load_2d(sB + size_t(stage) * C::B_BYTES, &tmB, kb * BK, n_idx * BN, &full[stage]);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let the loads still in flight land before the CTA can exit
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < C::STAGES && i < issued; ++i) {
          if (--s < 0) {
            s = C::STAGES - 1;
            ph ^= 1u;
          }
          (void)mbar_wait(&full[s], ph, wc);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc_iter = 0;
      bool ok = true;
      const uint32_t a_base = smem_u32(sA);
      const uint32_t b_base = smem_u32(sB);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++acc_iter) {
        const int acc = acc_iter & 1;
        const uint32_t acc_phase = (acc_iter >> 1) & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(&full[stage], phase, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(a_base + uint32_t(stage) * C::A_BYTES);
          const uint64_t bdesc = sw128_kmajor_desc(b_base + uint32_t(stage) * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            // advance 32 bytes along K inside the swizzle row (encoded >> 4)
            mma_i8(d_tmem, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), C::IDESC,
                   (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
      }
      // wait for every issued MMA before tensor memory can be released
      mma_commit(drain);
      (void)mbar_wait(drain, 0, wc);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    int acc_iter = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++acc_iter) {
      const int acc = acc_iter & 1;
      const uint32_t acc_phase = (acc_iter >> 1) & 1;
      const bool got = !(*abort_flag) && mbar_wait(&tfull[acc], acc_phase, wc);
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int m_idx = tile % p.num_m_tiles;
      const int n_idx = tile / p.num_m_tiles;
      const int64_t row = int64_t(m_idx) * BM + quarter * 32 + lane;
      const bool row_ok = row < p.T;
      float sx = 0.0f, mt = 0.0f;
      if (row_ok) {
        sx = p.a_scale_per_row ? p.a_scale[row] : p.a_scale[0];
        mt = p.a_mean ? p.a_mean[row] : 0.0f;
      }
      const uint32_t t_row = tmem_base + uint32_t(acc * BN) + (uint32_t(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + uint32_t(c * 32), r);
        tmem_wait_ld();
        const int col0 = n_idx * BN + c * 32;
        if (row_ok && col0 < p.N) {
          uint32_t packed[16];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int col = col0 + 4 * g;
            float4 sw = make_float4(0, 0, 0, 0), cs = make_float4(0, 0, 0, 0),
                   bb = make_float4(0, 0, 0, 0);
            if (col < p.N) {
              sw = __ldg(reinterpret_cast<const float4*>(p.w_scale + col));
              if (p.a_mean) cs = __ldg(reinterpret_cast<const float4*>(p.colsum + col));
              if (p.bias) bb = __ldg(reinterpret_cast<const float4*>(p.bias + col));
            }
            const float sws[4] = {sw.x, sw.y, sw.z, sw.w};
            const float css[4] = {cs.x, cs.y, cs.z, cs.w};
            const float bbs[4] = {bb.x, bb.y, bb.z, bb.w};
            float y[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float accf = __int2float_rn(int(r[4 * g + u]));
              y[u] = __fmaf_rn(accf, __fmul_rn(sx, sws[u]), __fmaf_rn(mt, css[u], bbs[u]));
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(y[0], y[1]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(y[2], y[3]);
            packed[2 * g] = *reinterpret_cast<uint32_t*>(&lo);
            packed[2 * g + 1] = *reinterpret_cast<uint32_t*>(&hi);
          }
          uint16_t* yrow = p.Y + row * p.N;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (col0 + 8 * g < p.N) {
              *reinterpret_cast<uint4*>(yrow + col0 + 8 * g) =
                  make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
            }
          }
          if (p.acc_debug) {
            int32_t* arow = p.acc_debug + row * p.N;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              if (col0 + 4 * g < p.N) {
                *reinterpret_cast<uint4*>(arow + col0 + 4 * g) =
                    make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ launch
template <int BN>
static cudaError_t launch_bn(const void* tmap_a, const void* tmap_b, const GemmParams& p, int grid,
                             cudaStream_t st) {
  using C = GemmCfg<BN>;
  static bool configured = false;  // attribute is per function, device-agnostic
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  gemm_i8_kernel<BN><<<grid, kGemmThreads, C::SMEM, st>>>(
      *reinterpret_cast<const CUtensorMap*>(tmap_a), *reinterpret_cast<const CUtensorMap*>(tmap_b), p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(int bn, const void* tmap_a, const void* tmap_b, const GemmParams& p,
                        int grid, cudaStream_t st) {
  switch (bn) {
    case 64: return launch_bn<64>(tmap_a, tmap_b, p, grid, st);
    case 128: return launch_bn<128>(tmap_a, tmap_b, p, grid, st);
    case 160: return launch_bn<160>(tmap_a, tmap_b, p, grid, st);
    case 192: return launch_bn<192>(tmap_a, tmap_b, p, grid, st);
    case 256: return launch_bn<256>(tmap_a, tmap_b, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t gemm_smem_bytes(int bn) {
  switch (bn) {
    case 64: return GemmCfg<64>::SMEM;
    case 128: return GemmCfg<128>::SMEM;
    case 160: return GemmCfg<160>::SMEM;
    case 192: return GemmCfg<192>::SMEM;
    case 256: return GemmCfg<256>::SMEM;
    default: return 0;
  }
}

int gemm_threads() { return kGemmThreads; }

}  // namespace hq
