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
//   warps 2..9  the epilogue: two warps per 32-lane quarter of tensor memory,
//               each taking half of the tile's columns.  Per tile a warp
//               stages its columns' s_w, colsum and bias in shared memory;
//               per 32-column chunk it reads the accumulator (tcgen05.ld),
//               applies the epilogue in fp32, writes bf16 to a 64-byte
//               swizzled shared buffer and lets a TMA tensor store write the
//               32 x 32 box to Y (clipped at the tensor's edges).
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
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemLimit = 227 * 1024;
constexpr float kAccMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kAccMagicBits = 0x4B400000;

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int HC = BN / 2;  // columns per epilogue warp
  // per epilogue warp: 2 KB output staging (1024-aligned) + params [3][HC]
  static constexpr int EPI_STAGE_BYTES = 2048;
  static constexpr int EPI_PARAM_BYTES = 3 * HC * 4;
  static constexpr int EPI_BYTES = kEpiWarps * (EPI_STAGE_BYTES + EPI_PARAM_BYTES);
  static constexpr int CTL_BYTES = 256;
  static constexpr int STAGES_RAW = (kSmemLimit - 1024 - EPI_BYTES - CTL_BYTES - 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  // instruction descriptor: D s32 (bits 4-5 = 2), A and B signed int8 (bits
  // 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at 24-28.
  static constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) |
                                    (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static constexpr size_t SMEM = size_t(STAGES) * STAGE_BYTES + EPI_BYTES + CTL_BYTES + 1024;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "two 32-column-aligned halves");
  static_assert(B_BYTES % 1024 == 0, "stage bases must stay 1024-byte aligned");
  static_assert(STAGES >= 2, "shared memory budget");
  static_assert(SMEM <= size_t(kSmemLimit), "shared memory budget");
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + size_t(C::STAGES) * C::A_BYTES;
  uint8_t* epi_stage = sB + size_t(C::STAGES) * C::B_BYTES;  // 1024-aligned, [8][2 KB]
  float* epi_param = reinterpret_cast<float*>(epi_stage + kEpiWarps * C::EPI_STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_stage + C::EPI_BYTES);
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
      mbar_init(&tempty[a], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
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
    const int ew = warp - 2;         // 0 .. 7
    const int quarter = warp & 3;    // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = ew >> 2;        // columns [half*HC, half*HC + HC) of the tile
    uint8_t* stg = epi_stage + ew * C::EPI_STAGE_BYTES;
    float* prm = epi_param + ew * (3 * C::HC);
    const int swz = (lane >> 1) & 3;  // 64-byte swizzle of this thread's row
    int acc_iter = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++acc_iter) {
      const int acc = acc_iter & 1;
      const uint32_t acc_phase = (acc_iter >> 1) & 1;
      const int m_idx = tile % p.num_m_tiles;
      const int n_idx = tile / p.num_m_tiles;
      const int col_base = n_idx * BN + half * C::HC;
      // this warp's columns: scale, colsum, bias (coalesced, before the wait)
      for (int c = lane; c < C::HC; c += 32) {
        const int gc = col_base + c;
        const bool in = gc < p.N;
        prm[c] = in ? p.w_scale[gc] : 0.0f;
        prm[C::HC + c] = (in && p.a_mean) ? p.colsum[gc] : 0.0f;
        prm[2 * C::HC + c] = (in && p.bias) ? p.bias[gc] : 0.0f;
      }
      const int row0 = m_idx * BM + quarter * 32;
      const int64_t row = int64_t(row0) + lane;
      const bool row_ok = row < p.T;
      float sx = 0.0f, mt = 0.0f;
      if (row_ok) {
        sx = p.a_scale_per_row ? p.a_scale[row] : p.a_scale[0];
        mt = p.a_mean ? p.a_mean[row] : 0.0f;
      }
      __syncwarp();
      const bool got = !(*abort_flag) && mbar_wait(&tfull[acc], acc_phase, wc);
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + uint32_t(acc * BN + half * C::HC) +
                             (uint32_t(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < C::HC / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + uint32_t(c * 32), r);
        tmem_wait_ld();
        const int col0 = col_base + c * 32;
        const float* pw = prm + c * 32;
        uint32_t packed[16];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 sw = *reinterpret_cast<const float4*>(pw + 4 * g);
          const float4 cs = *reinterpret_cast<const float4*>(pw + C::HC + 4 * g);
          const float4 bb = *reinterpret_cast<const float4*>(pw + 2 * C::HC + 4 * g);
          f2 a01, a23;
          if (p.small_acc) {
            // |acc| < 2^22: acc + 1.5*2^23 is exact in fp32, so subtracting the
            // magic constant recovers float(acc) without the conversion unit
            const f2 mg = pk(kAccMagic, kAccMagic);
            a01 = sub2(pk(__int_as_float(int(r[4 * g + 0]) + kAccMagicBits),
                          __int_as_float(int(r[4 * g + 1]) + kAccMagicBits)), mg);
            a23 = sub2(pk(__int_as_float(int(r[4 * g + 2]) + kAccMagicBits),
                          __int_as_float(int(r[4 * g + 3]) + kAccMagicBits)), mg);
          } else {
            a01 = pk(__int2float_rn(int(r[4 * g + 0])), __int2float_rn(int(r[4 * g + 1])));
            a23 = pk(__int2float_rn(int(r[4 * g + 2])), __int2float_rn(int(r[4 * g + 3])));
          }
          const f2 sx2 = pk(sx, sx), mt2 = pk(mt, mt);
          // y = acc * (s_x * s_w) + (b + m * colsum)
          const f2 y01 = fma2(a01, mul2(sx2, pk(sw.x, sw.y)), fma2(mt2, pk(cs.x, cs.y), pk(bb.x, bb.y)));
          const f2 y23 = fma2(a23, mul2(sx2, pk(sw.z, sw.w)), fma2(mt2, pk(cs.z, cs.w), pk(bb.z, bb.w)));
          packed[2 * g] = pack_bf16x2(y01.x, y01.y);
          packed[2 * g + 1] = pack_bf16x2(y23.x, y23.y);
        }
        // the previous chunk's TMA store must have finished reading the buffer
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          *reinterpret_cast<uint4*>(stg + lane * 64 + ((q ^ swz) << 4)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && col0 < p.N && row0 < p.T) {
          tma_store_2d(&tmY, stg, col0, row0);
          bulk_commit_group();
        }
        if (p.acc_debug && row_ok) {
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (lane == 0) bulk_wait_group<0>();  // all of this warp's stores are complete
    __syncwarp();
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
static cudaError_t launch_bn(const void* tmap_a, const void* tmap_b, const void* tmap_y,
                             const GemmParams& p, int grid, cudaStream_t st) {
  using C = GemmCfg<BN>;
  static bool configured = false;  // attribute is per function, device-agnostic
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  gemm_i8_kernel<BN><<<grid, kGemmThreads, C::SMEM, st>>>(
      *reinterpret_cast<const CUtensorMap*>(tmap_a), *reinterpret_cast<const CUtensorMap*>(tmap_b),
      *reinterpret_cast<const CUtensorMap*>(tmap_y), p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(int bn, const void* tmap_a, const void* tmap_b, const void* tmap_y,
                        const GemmParams& p, int grid, cudaStream_t st) {
  switch (bn) {
    case 64: return launch_bn<64>(tmap_a, tmap_b, tmap_y, p, grid, st);
    case 128: return launch_bn<128>(tmap_a, tmap_b, tmap_y, p, grid, st);
    case 192: return launch_bn<192>(tmap_a, tmap_b, tmap_y, p, grid, st);
    case 256: return launch_bn<256>(tmap_a, tmap_b, tmap_y, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t gemm_smem_bytes(int bn) {
  switch (bn) {
    case 64: return GemmCfg<64>::SMEM;
    case 128: return GemmCfg<128>::SMEM;
    case 192: return GemmCfg<192>::SMEM;
    case 256: return GemmCfg<256>::SMEM;
    default: return 0;
  }
}

int gemm_threads() { return kGemmThreads; }

}  // namespace hq
