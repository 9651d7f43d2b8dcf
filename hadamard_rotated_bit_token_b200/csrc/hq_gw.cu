// hq_gw.cu -- the group-wise 4-bit form with a 16-bit low-rank branch
// ("Data-free 4-bit quantization for diffusion transformers", section
// "Hadamard rotation: the int4 improvement", steps 1-7), in the [N,K]
// orientation (y[t,n] = sum_k W[n,k] X[t,k] + b[n]):
//
//   smoothing  x^ = X diag(sigma^-1),  W^ = W diag(sigma)
//   low rank   l1 = bf16(L1 diag(sigma^-1)) [r,K],  l2 = bf16(L2) [N,r],
//              R  = (W - l2 l1) diag(sigma)          (W^ = l2 l1 diag(sigma) + R)
//   rotation   one H_64 block per group of 64 channels: R H and x^ H
//   quantizers one scale per (row, group): s = max|.| / q, codes = rne(. / s)
//   output     y = sum_j s_x[t,j] s_w[n,j] (codes_x . codes_w)_j + l2 (l1 X) + b
//
// Codes are stored one per byte as fp8 e4m3 holding the integer code
// exactly (every integer of magnitude <= 16 is an e4m3 value), so the tensor
// cores multiply them with tcgen05 kind::f8f6f4 into fp32 accumulators.  One
// group's products sum to at most 64 * 7 * 7 = 3136 in magnitude, an integer
// that fp32 holds exactly: every group's partial sum is exact, as with int32.
//
// Kernels:
//   gw_factor_kernel   l1 and l2 in bf16 (offline);
//   gw_weight_kernel   R, R H_64 per group, the weight group quantizer
//                      (offline; one warp per (row, group), two channels per
//                      lane, the transform over lanes by shuffles);
//   gw_act_kernel      the activation side in one pass over X: a producer
//                      warp streams 128-token x 64-channel bf16 tiles of X
//                      (and the matching 64 columns of l1) into a ring of
//                      shared-memory stages; one thread issues tcgen05
//                      kind::f16 MMAs that accumulate u = X l1^T (128 x r,
//                      fp32) in tensor memory from the same tiles; eight
//                      quantizer warps, one token per lane and one group per
//                      stage, apply sigma^-1, the 64-point fast Walsh-Hadamard
//                      transform in registers, the group max and the codes;
//                      at the end u leaves tensor memory as bf16 (a small
//                      batch may split each block's groups over two CTAs,
//                      whose parts of u the last to finish adds);
//   gw_gemm_kernel     the output: per output tile (128 x 256) and group j,
//                      two kind::f8f6f4 MMAs (K = 64) into one of two fp32
//                      accumulators in tensor memory, and sixteen epilogue
//                      warps that add s_x[t,j] s_w[n,j] times each finished
//                      accumulator into registers while the tensor cores fill
//                      the other; the low-rank term is one more step of two
//                      kind::f16 MMAs (u x l2^T) added with scale 1; the bias
//                      and the bf16 store close the tile.
// Every wait is bounded; a timeout records HQ_ERR_TIMEOUT in the device error
// word and the CTA waits for the copies it started before it exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "hq_device.cuh"
#include "hq_kernels.h"
#include "hq_quant_common.cuh"

namespace hq {

namespace {

constexpr int kGroup = 64;         // channels per group = order of the H block
constexpr int kTokRows = 128;      // tokens per activation tile (MMA M)
constexpr int kXTileBytes = kTokRows * kGroup * 2;  // bf16, one 128-byte row per token
constexpr int kGwQuantWarps = 8;   // two teams of four (one warp per 32-token quarter)
constexpr int kGwActThreads = 64 + 32 * kGwQuantWarps;
// GEMM shape: output tile width, epilogue warps (a multiple of 4: each
// 32-lane quarter of tensor memory gets kGwEpiWarps / 4 of them), columns
// per tensor-memory load, and the register cap that lets the CTA launch
// (the busiest sub-partition runs ceil(warps / 4) warps out of 16384
// registers).
#ifndef HQ_GW_BN
#define HQ_GW_BN 256
#endif
#ifndef HQ_GW_EPI_WARPS
#define HQ_GW_EPI_WARPS 16
#endif
#ifndef HQ_GW_LD_COLS
#define HQ_GW_LD_COLS 8
#endif
#ifndef HQ_GW_MAXNREG
#define HQ_GW_MAXNREG 96
#endif
constexpr int kGwBN = HQ_GW_BN;
constexpr int kGwEpiWarps = HQ_GW_EPI_WARPS;
constexpr int kGwEpiCols = kGwBN * 4 / kGwEpiWarps;  // output columns per epilogue warp
constexpr int kGwEpiChunks = kGwEpiCols / 32;
constexpr int kGwLdCols = HQ_GW_LD_COLS;
static_assert(kGwEpiWarps % 4 == 0 && kGwEpiCols % 32 == 0 && kGwEpiCols % kGwLdCols == 0,
              "whole 32-column chunks per epilogue warp");
// accumulators in tensor memory (each kGwBN fp32 columns of 512): the MMA
// issuer runs up to kGwNB - 1 groups ahead of the slowest epilogue warp
constexpr int kGwNB = 512 / kGwBN > 4 ? 4 : 512 / kGwBN;
static_assert(kGwNB >= 2, "at least two accumulators in tensor memory");
constexpr int kGwGemmThreads = 64 + 32 * kGwEpiWarps;
constexpr int kGwSmemLimit = 227 * 1024;
constexpr int kGwStageBox = 2048;  // one 32 x 32 bf16 output box

// GEMM stage: A codes 128 x 64 bytes and B codes kGwBN x 64 bytes (both
// 64-byte swizzle), then the group's 128 activation scales and kGwBN weight
// scales (the epilogue reads them here: shared-memory broadcast reads cost
// far less than the same reads from L1); a low-rank step puts u (128 x 32
// bf16) and l2 (kGwBN x 32 bf16) in the A and B slots.
constexpr int kGwA = kTokRows * 64;
constexpr int kGwB = kGwBN * 64;
constexpr int kGwSA = kTokRows * 4;
constexpr int kGwSW = kGwBN * 4;
constexpr int kGwStageTx = kGwA + kGwB + kGwSA + kGwSW;
constexpr int kGwStageBytes = (kGwStageTx + 1023) / 1024 * 1024;
constexpr int kGwCtl = 512;
constexpr int kGwFixed = kGwEpiWarps * kGwStageBox + kGwCtl + 1024;
constexpr int kGwStagesRaw = (kGwSmemLimit - kGwFixed) / kGwStageBytes;
constexpr int kGwStages = kGwStagesRaw > 8 ? 8 : kGwStagesRaw;
constexpr size_t kGwGemmSmem = size_t(kGwStages) * kGwStageBytes + kGwFixed;
static_assert(kGwStages >= 3, "shared-memory budget of the group-wise GEMM");
static_assert(kGwGemmSmem <= size_t(kGwSmemLimit), "shared-memory budget");

// Instruction descriptors (D fp32 at bits 4-5 = 1; A / B formats at bits
// 7-9 / 10-12; both operands K-major; N >> 3 at bits 17-22, M >> 4 at 24-28):
// kind::f8f6f4 with e4m3 operands (format 0), kind::f16 with bf16 (format 1).
__host__ __device__ constexpr uint32_t e4m3_idesc(int m, int n) {
  return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
__host__ __device__ constexpr uint32_t bf16_idesc(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// Shared-memory matrix descriptors of K-major tiles written by TMA: rows of
// 128 bytes with 128-byte swizzling (8-row atoms of 1024 bytes, layout type
// 2) or rows of 64 bytes with 64-byte swizzling (8-row atoms of 512 bytes,
// layout type 4); leading byte offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr, uint32_t atom_bytes,
                                                uint32_t layout) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;
  d |= uint64_t(atom_bytes >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(layout) << 61;
  return d;
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) { return kmajor_desc(saddr, 1024, 2); }
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) { return kmajor_desc(saddr, 512, 4); }

// D[tmem] (+)= A * B^T with e4m3 operands, fp32 accumulate, one CTA.
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A * B^T with bf16 operands, fp32 accumulate, one CTA.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Two integer-valued floats -> two e4m3 bytes (a in the low byte), exact for
// |value| <= 16.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return uint32_t(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// 32 fp32 values (bit patterns) -> 32 bf16 (round to nearest even) at dst
// (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_u32(uint16_t* dst16, const uint32_t (&v)[32]) {
  uint4* dst = reinterpret_cast<uint4*>(dst16);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * c + 2 * e]),
                                                __uint_as_float(v[8 * c + 2 * e + 1]));
      h[e] = *reinterpret_cast<uint32_t*>(&b2);
    }
    dst[c] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// Tensor-memory columns holding u (rank 32 or 64; allocations are powers of
// two from 32).
__device__ __forceinline__ uint32_t gw_u_cols(int rank) { return rank <= 32 ? 32u : 64u; }

}  // namespace

// 32 lanes x 8, 16, 32 or 64 consecutive 32-bit columns: thread i of the warp
// receives that many columns from col on of tensor-memory lane
// (warp quarter * 32 + i).
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_32x32b_x32(taddr, r);
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld_32x32b_x32(taddr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// ------------------------------------------------------------ weight side
// l1[r,k] = bf16(L1[r,k] * sigma_inv[k]) and l2 = bf16(L2): the product is
// formed in fp64 and rounded once.
__global__ void gw_factor_kernel(const float* __restrict__ L1, const float* __restrict__ L2,
                                 const float* __restrict__ sigma_inv, int rank, int K, int N,
                                 uint16_t* __restrict__ l1s, uint16_t* __restrict__ l2b) {
  const int64_t n1 = int64_t(rank) * K, n2 = int64_t(N) * rank;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n1 + n2;
       i += int64_t(gridDim.x) * blockDim.x) {
    if (i < n1) {
      const double s = sigma_inv ? double(sigma_inv[i % K]) : 1.0;
      const __nv_bfloat16 h = __double2bfloat16(double(L1[i]) * s);
      l1s[i] = *reinterpret_cast<const uint16_t*>(&h);
    } else {
      const __nv_bfloat16 h = __float2bfloat16_rn(L2[i - n1]);
      l2b[i - n1] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

// One warp per (output channel n, group j), lane i holding channels
// 64 j + 2 i and 64 j + 2 i + 1:
//   R = (W - l2 l1) sigma in fp32 (the rank-r product summed in fp32),
//   v = R H~_64 (unnormalized transform: index bit 0 inside the lane, bits
//   1-5 across lanes by shuffles), a = max |v| over the group,
//   codes = rne(v q / a) (one fused multiply-add against 1.5 * 2^23, which
//   rounds half to even), scale = a / (8 q) (H_64 = H~_64 / 8).
// w_scale is [G][N]; bias_f32[n] = bias[n] (or 0).
__global__ void __launch_bounds__(256) gw_weight_kernel(GwWeightParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.K / kGroup;
  const int64_t n = blockIdx.x;
  if (n >= p.N) return;
  extern __shared__ float l2row[];  // this row's l2 values (rank)
  for (int r = threadIdx.x; r < p.rank; r += blockDim.x) l2row[r] = bf16_to_f(p.l2b[n * p.rank + r]);
  if (threadIdx.x == 0) p.bias_f32[n] = p.bias ? bf16_to_f(p.bias[n]) : 0.0f;
  __syncthreads();
  const float q = float(p.q);
  const float mg = qc::kRoundMagic;
  for (int j = warp; j < G; j += blockDim.x >> 5) {
    const int k = j * kGroup + 2 * lane;
    const uint32_t wv = *reinterpret_cast<const uint32_t*>(p.W + n * p.K + k);
    float a0 = qc::bf16lo(wv), a1 = qc::bf16hi(wv);
    float l0 = 0.0f, l1 = 0.0f;
    for (int r = 0; r < p.rank; ++r) {
      const uint32_t fv = *reinterpret_cast<const uint32_t*>(p.l1s + int64_t(r) * p.K + k);
      l0 = fmaf(l2row[r], qc::bf16lo(fv), l0);
      l1 = fmaf(l2row[r], qc::bf16hi(fv), l1);
    }
    a0 -= l0;
    a1 -= l1;
    if (p.sigma_inv) {
      a0 = __fdiv_rn(a0, p.sigma_inv[k]);
      a1 = __fdiv_rn(a1, p.sigma_inv[k + 1]);
    }
    float v0 = a0 + a1, v1 = a0 - a1;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const float sg = (lane & m) ? -1.0f : 1.0f;
      v0 = fmaf(v0, sg, __shfl_xor_sync(0xffffffffu, v0, m));
      v1 = fmaf(v1, sg, __shfl_xor_sync(0xffffffffu, v1, m));
    }
    float a = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
    const float rr = a > 0.0f ? __fdiv_rn(q, a) : 0.0f;
    const float c0 = fmaf(v0, rr, mg) - mg, c1 = fmaf(v1, rr, mg) - mg;
    *reinterpret_cast<uint16_t*>(p.w_codes + n * p.K + k) = uint16_t(e4m3x2(c0, c1));
    if (lane == 0) p.w_scale[int64_t(j) * p.N + n] = __fdiv_rn(a, 8.0f * q);
  }
}

// ---------------------------------------------------------- activation side
namespace {

// Shared-memory layout of gw_act_kernel: `stages` stages of one X tile
// (128 tokens x 64 channels bf16, 128-byte swizzle) and, with a low-rank
// branch, the same 64 columns of l1 (rank rows, 128-byte swizzle); then
// sigma^-1 for every channel (when given), the barriers and the
// tensor-memory slot.
struct GwActSmem {
  uint32_t stage_bytes, x_off, l1_off, sig_off, bar_off, total;
};

__host__ __device__ inline GwActSmem gw_act_layout(int K, int rank, int stages, bool sigma) {
  GwActSmem L;
  L.x_off = 0;
  L.l1_off = kXTileBytes;
  L.stage_bytes = uint32_t(kXTileBytes + rank * 128);  // multiples of 1024 (rank % 32 == 0)
  L.sig_off = uint32_t(stages) * L.stage_bytes;
  L.bar_off = L.sig_off + (sigma ? uint32_t(K) * 4u : 0u);
  L.total = L.bar_off + uint32_t(2 * stages + 2) * 8u + 16u + 1024u;  // + alignment slack
  return L;
}

}  // namespace

size_t gw_act_smem_bytes(int K, int rank, int stages, bool sigma) {
  return gw_act_layout(K, rank, stages, sigma).total;
}

int gw_act_threads() { return kGwActThreads; }

// One CTA per 128 tokens.  Warp 0: producer; warp 1: tensor memory and (one
// thread) the low-rank MMAs; warps 2..9: quantizers.  Quantizer warp w takes
// tokens 32 (w % 4) .. 32 (w % 4) + 31 of the tile -- tensor-memory lane
// quarter w % 4, which its lanes read u from at the end -- and every other
// group (team (w - 2) / 4 takes groups team, team + 2, ...).
__global__ void __launch_bounds__(kGwActThreads, 1)
    gw_act_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmL1,
                  const GwActParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const GwActSmem L = gw_act_layout(p.K, p.rank, p.stages, p.sigma_inv != nullptr);
  float* sig = reinterpret_cast<float*>(smem + L.sig_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* ufull = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ufull + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;  // this CTA adds the parts of u

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl wc{p.err, p.wait_ns};
  const int G = p.K / kGroup;
  // p.split CTAs share a block of 128 tokens, each taking the groups
  // [j0, j1); with a branch each accumulates its part of u, and the one to
  // finish last adds the parts in part order
  const int blk = int(blockIdx.x) / p.split, part = int(blockIdx.x) % p.split;
  const int j0 = G * part / p.split, j1 = G * (part + 1) / p.split;
  const int GL = j1 - j0;
  const int64_t row0 = int64_t(blk) * kTokRows;
  const bool lowrank = p.rank > 0;
  const int team_warps = 4;

  if (p.sigma_inv) {
    for (int k = threadIdx.x; k < p.K; k += blockDim.x) sig[k] = p.sigma_inv[k];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      // the team's four warps, and the MMAs that read the stage's X tile
      mbar_init(&empty[s], team_warps + (lowrank ? 1 : 0));
    }
    mbar_init(ufull, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmX);
    if (lowrank) prefetch_tmap(&tmL1);
  }
  if (warp == 1 && lowrank) {
    tmem_alloc(tmem_slot, gw_u_cols(p.rank));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = lowrank ? *tmem_slot : 0u;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t tx = L.stage_bytes;
      for (int j = j0; j < j1; ++j) {
        if (*abort_flag || !mbar_wait_spin(&empty[stage], phase ^ 1u, wc)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], tx);
        uint8_t* st = smem + size_t(stage) * L.stage_bytes;
        // the fault hook withholds the first tile's copy (its wait times out)
        if (!(p.fault && j == j0))
          tma_load_2d(st + L.x_off, &tmX, j * kGroup, int32_t(row0), &full[stage]);
        if (lowrank) tma_load_2d(st + L.l1_off, &tmL1, j * kGroup, 0, &full[stage]);
        ++issued;
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok || p.fault) {
        // let the copies still in flight land before the CTA can exit
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < p.stages && i < issued; ++i) {
          if (--s < 0) {
            s = p.stages - 1;
            ph ^= 1u;
          }
          (void)mbar_wait(&full[s], ph, wc);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && lowrank) {
      // ---------------------------------------- low-rank down projection
      const uint32_t idesc = bf16_idesc(kTokRows, p.rank);
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; j < GL; ++j) {
        if (*abort_flag || !mbar_wait_spin(&full[stage], phase, wc)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + size_t(stage) * L.stage_bytes);
        const uint64_t adesc = sw128_desc(sb + L.x_off);
        const uint64_t bdesc = sw128_desc(sb + L.l1_off);
#pragma unroll
        for (int k = 0; k < kGroup / 16; ++k)  // 16 bf16 = 32 bytes per MMA along K
          mma_bf16(tmem_base, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), idesc,
                   (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty[stage]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // u is complete once every MMA issued above has completed (also on
      // abort, so that tensor memory is idle before it is released)
      mma_commit(ufull);
    }
  } else {
    // ---------------------------------------------------------- quantizers
    const int ew = warp - 2;
    const int team = ew >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // token within the tile
    const int64_t t = row0 + r;
    const bool row_ok = t < p.T;
    const int swz = r & 7;  // 128-byte swizzle: chunk c of row r at c ^ (r % 8)
    const float q = float(p.q);
    const f2 mg2 = pk(qc::kRoundMagic, qc::kRoundMagic);
    for (int jl = team; jl < GL; jl += 2) {
      const int j = j0 + jl;  // the group; jl its place in this CTA's sequence
      const int stage = jl % p.stages;
      const uint32_t phase = uint32_t(jl / p.stages) & 1u;
      // one lane waits; the warp barrier orders the others behind its acquire
      bool got = true;
      if (lane == 0) got = !(*abort_flag) && mbar_wait_spin(&full[stage], phase, wc);
      __syncwarp();
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        *abort_flag = 1;
        break;
      }
      const uint32_t xrow = smem_u32(smem + size_t(stage) * L.stage_bytes + L.x_off) + r * 128;
      uint4 x[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) x[c] = qc::ld_shared_v4(xrow + ((c ^ swz) << 4));
      f2 w0[16], w1[16];
      qc::unpack32(*reinterpret_cast<const uint4(*)[4]>(&x[0]), w0);
      qc::unpack32(*reinterpret_cast<const uint4(*)[4]>(&x[4]), w1);
      // the stage's X tile is in registers: hand it back.  The reads went
      // through the generic proxy and the next write into the stage is a
      // tensor copy (async proxy), so every thread fences its own reads
      // before the warp's arrive; without the fence, copies were seen
      // overwriting a stage that some lanes were still reading.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (p.sigma_inv) {
        const float4* s4 = reinterpret_cast<const float4*>(sig + j * kGroup);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 a = s4[i], b = s4[8 + i];
          w0[2 * i] = mul2(w0[2 * i], pk(a.x, a.y));
          w0[2 * i + 1] = mul2(w0[2 * i + 1], pk(a.z, a.w));
          w1[2 * i] = mul2(w1[2 * i], pk(b.x, b.y));
          w1[2 * i + 1] = mul2(w1[2 * i + 1], pk(b.z, b.w));
        }
      }
      // index bits 0-4 inside each 32-channel half, bit 5 between the halves
      qc::fwht32<5>(w0, nullptr, lane);
      qc::fwht32<5>(w1, nullptr, lane);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const f2 a = w0[i], b = w1[i];
        w0[i] = add2(a, b);
        w1[i] = sub2(a, b);
      }
      float mx0, mn0, mx1, mn1;
      qc::maxmin32(w0, mx0, mn0);
      qc::maxmin32(w1, mx1, mn1);
      const float a = fmaxf(fmaxf(mx0, mx1), -fminf(mn0, mn1));
      const float rr = a > 0.0f ? __fdiv_rn(q, a) : 0.0f;
      const f2 rr2 = pk(rr, rr);
      uint32_t cw[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const f2 c0 = sub2(fma2(w0[2 * i], rr2, mg2), mg2);
        const f2 c1 = sub2(fma2(w0[2 * i + 1], rr2, mg2), mg2);
        cw[i] = e4m3x2(c0.x, c0.y) | (e4m3x2(c1.x, c1.y) << 16);
        const f2 d0 = sub2(fma2(w1[2 * i], rr2, mg2), mg2);
        const f2 d1 = sub2(fma2(w1[2 * i + 1], rr2, mg2), mg2);
        cw[8 + i] = e4m3x2(d0.x, d0.y) | (e4m3x2(d1.x, d1.y) << 16);
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes + t * p.K + int64_t(j) * kGroup);
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = make_uint4(cw[4 * c], cw[4 * c + 1], cw[4 * c + 2], cw[4 * c + 3]);
        p.scale[int64_t(j) * p.ld + t] = __fdiv_rn(a, 8.0f * q);
      }
    }
    if (lowrank && team == 0) {
      // u = bf16(X l1^T) from tensor memory: lane quarter `quarter`, one
      // token per lane, rank fp32 columns
      const bool got = !(*abort_flag) && mbar_wait(ufull, 0, wc);
      const bool ok = __all_sync(0xffffffffu, got);
      if (!ok) *abort_flag = 1;
      if (p.split == 1) {
        if (ok) {
          tc_fence_after();
          for (int c0 = 0; c0 < p.rank; c0 += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(c0), v);
            tmem_wait_ld();
            if (row_ok) store_u32(p.u + t * p.rank + c0, v);
          }
        }
      } else {
        // this CTA's part of u to its slot of the workspace; the CTA that
        // finishes last (an atomic ticket per block) adds the parts in part
        // order, so the sum does not depend on which CTA that is
        if (ok) {
          tc_fence_after();
          for (int c0 = 0; c0 < p.rank; c0 += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(c0), v);
            tmem_wait_ld();
            if (row_ok) {
              float4* dst = reinterpret_cast<float4*>(p.upart + (int64_t(part) * p.T + t) * p.rank + c0);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                     __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
            }
          }
        }
        __threadfence();
        named_barrier_sync(1, 32 * team_warps);
        if (warp == 2 && lane == 0)
          *last_flag = atomicAdd(&p.counters[blk], 1u) == unsigned(p.split - 1) ? 1 : 0;
        named_barrier_sync(1, 32 * team_warps);
        if (*last_flag && !*abort_flag) {
          __threadfence();
          for (int c0 = 0; c0 < p.rank; c0 += 32) {
            if (!row_ok) break;
            float s[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) s[c] = 0.0f;
            for (int q = 0; q < p.split; ++q) {
              const float4* src =
                  reinterpret_cast<const float4*>(p.upart + (int64_t(q) * p.T + t) * p.rank + c0);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float4 w = __ldcg(src + c);
                s[4 * c] += w.x;
                s[4 * c + 1] += w.y;
                s[4 * c + 2] += w.z;
                s[4 * c + 3] += w.w;
              }
            }
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(s[c]);
            store_u32(p.u + t * p.rank + c0, v);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lowrank) {
    // every MMA has completed once ufull has (waited on here in case the
    // quantizers gave up early)
    (void)mbar_wait(ufull, 0, wc);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, gw_u_cols(p.rank));
  }
}

// ---------------------------------------------------------------- the GEMM
namespace {

__device__ __forceinline__ int gw_tile_m(const GwGemmParams& p, int tile) {
  const int gsize = p.group_m * p.num_n_tiles;
  const int first = (tile / gsize) * p.group_m;
  const int gm = min(p.num_m_tiles - first, p.group_m);
  return first + (tile % gsize) % gm;
}
__device__ __forceinline__ int gw_tile_n(const GwGemmParams& p, int tile) {
  const int gsize = p.group_m * p.num_n_tiles;
  const int first = (tile / gsize) * p.group_m;
  const int gm = min(p.num_m_tiles - first, p.group_m);
  return (tile % gsize) / gm;
}

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace

size_t gw_gemm_smem_bytes() { return kGwGemmSmem; }
int gw_gemm_bn() { return kGwBN; }
int gw_gemm_threads() { return kGwGemmThreads; }

// Persistent: CTA b takes output tiles b, b + grid, ... in grouped order.
// Per tile, `steps` = (rank > 0) + G steps run through the stage ring and
// the two accumulators in order: the low-rank step first (u x l2^T), then
// group j = 0 .. G-1 (codes x codes^T over channels 64 j .. 64 j + 63).
// Warp 0: producer (one thread); warp 1: tensor memory and (one thread) the
// MMAs; warps 2.. 2 + kGwEpiWarps - 1: epilogue, kGwEpiWarps / 4 warps per
// 32-lane quarter of tensor memory, each taking kGwEpiCols of the tile's
// columns, with the running sums in registers (kGwEpiCols / 2 fp32 pairs a
// thread).
__global__ void __maxnreg__(HQ_GW_MAXNREG)
    gw_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSW,
                   const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                   const __grid_constant__ CUtensorMap tmY, const GwGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* epi_stage = smem + size_t(kGwStages) * kGwStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_stage + kGwEpiWarps * kGwStageBox);
  uint64_t* empty = full + kGwStages;
  uint64_t* tfull = empty + kGwStages;  // [kGwNB] accumulator complete
  uint64_t* tempty = tfull + kGwNB;     // [kGwNB] accumulator read by the epilogue
  uint64_t* drain = tempty + kGwNB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl wc{p.err, p.wait_ns};
  const bool lowrank = p.rank > 0;
  const int steps = (lowrank ? 1 : 0) + p.G;
  const int num_tiles = p.num_m_tiles * p.num_n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGwStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kGwEpiWarps);  // the MMAs' commit and every epilogue warp
    }
    for (int a = 0; a < kGwNB; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kGwEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
    prefetch_tmap(&tmSW);
    prefetch_tmap(&tmY);
    if (lowrank) {
      prefetch_tmap(&tmU);
      prefetch_tmap(&tmL2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = gw_tile_m(p, tile) * kTokRows;
        const int n0 = gw_tile_n(p, tile) * kGwBN;
        for (int st = 0; st < steps; ++st) {
          if (*abort_flag || !mbar_wait_spin(&empty[stage], phase ^ 1u, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sb = smem + size_t(stage) * kGwStageBytes;
          if (lowrank && st == 0) {
            mbar_arrive_expect_tx(&full[stage], uint32_t(kGwA + kGwB));
            tma_load_2d(sb, &tmU, 0, m0, &full[stage]);
            tma_load_2d(sb + kGwA, &tmL2, 0, n0, &full[stage]);
          } else {
            const int j = st - (lowrank ? 1 : 0);
            mbar_arrive_expect_tx(&full[stage], uint32_t(kGwStageTx));
            tma_load_2d(sb, &tmA, j * kGroup, m0, &full[stage]);
            tma_load_2d(sb + kGwA, &tmB, j * kGroup, n0, &full[stage]);
            tma_load_2d(sb + kGwA + kGwB, &tmSA, m0, j, &full[stage]);
            tma_load_2d(sb + kGwA + kGwB + kGwSA, &tmSW, n0, j, &full[stage]);
          }
          ++issued;
          if (++stage == kGwStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < kGwStages && i < issued; ++i) {
          if (--s < 0) {
            s = kGwStages - 1;
            ph ^= 1u;
          }
          (void)mbar_wait(&full[s], ph, wc);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int stage = 0, gstep = 0;
      uint32_t phase = 0;
      bool ok = true;
      constexpr uint32_t kIdF8 = e4m3_idesc(kTokRows, kGwBN);
      constexpr uint32_t kIdBf = bf16_idesc(kTokRows, kGwBN);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int st = 0; st < steps; ++st, ++gstep) {
          const int b = gstep % kGwNB;
          const uint32_t bph = uint32_t(gstep / kGwNB) & 1u;
          if (*abort_flag || !mbar_wait_spin(&tempty[b], bph ^ 1u, wc) ||
              !mbar_wait_spin(&full[stage], phase, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + size_t(stage) * kGwStageBytes);
          const uint64_t adesc = sw64_desc(sb);
          const uint64_t bdesc = sw64_desc(sb + kGwA);
          const uint32_t d = tmem_base + uint32_t(b * kGwBN);
          const bool lr = lowrank && st == 0;
#pragma unroll
          for (int k = 0; k < 2; ++k) {  // 32 bytes along K per MMA
            if (lr)
              mma_bf16(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), kIdBf, k ? 1u : 0u);
            else
              mma_e4m3(d, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), kIdF8, k ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          mma_commit(&tfull[b]);
          if (++stage == kGwStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      mma_commit(drain);
      (void)mbar_wait(drain, 0, wc);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int part = ew >> 2;  // columns [part * kGwEpiCols, (part + 1) * kGwEpiCols) of the tile
    const int r = quarter * 32 + lane;
    uint8_t* stg = epi_stage + ew * kGwStageBox;
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t t_warp =
        tmem_base + uint32_t(part * kGwEpiCols) + (uint32_t(quarter * 32) << 16);
    int stage = 0, gstep = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = gw_tile_m(p, tile) * kTokRows;
      const int n0 = gw_tile_n(p, tile) * kGwBN;
      const int c0 = n0 + part * kGwEpiCols;  // this warp's first output column
      f2 acc[kGwEpiCols / 2];
#pragma unroll
      for (int i = 0; i < kGwEpiCols / 2; ++i) acc[i] = pk(0.0f, 0.0f);

      for (int st = 0; st < steps; ++st, ++gstep) {
        const int b = gstep % kGwNB;
        const uint32_t bph = uint32_t(gstep / kGwNB) & 1u;
        // one lane waits (32 lanes spinning on one barrier word serialize in
        // shared memory); the warp barrier orders the others behind its acquire
        bool got = true;
        if (lane == 0)
          got = !(*abort_flag) && mbar_wait_spin(&tfull[b], bph, wc) &&
                mbar_wait_spin(&full[stage], phase, wc);
        __syncwarp();
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_addr = t_warp + uint32_t(b * kGwBN);
        const uint32_t sb = smem_base + uint32_t(stage) * uint32_t(kGwStageBytes);
        // kGwLdCols columns per tensor-memory load; a chunk's weight scales are
        // read from shared memory before its load, so the two latencies
        // overlap (tcgen05.wait::ld waits for every load in flight, which
        // makes the load round trips the step's critical path).  The
        // accumulator goes back to the MMA issuer once its last chunk landed.
        constexpr int LDC = kGwLdCols;
        if (lowrank && st == 0) {
#pragma unroll
          for (int c = 0; c < kGwEpiCols / LDC; ++c) {
            uint32_t v[LDC];
            tmem_ld_cols(t_addr + uint32_t(LDC * c), v);
            tmem_wait_ld();
            if (c == kGwEpiCols / LDC - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[b]);
            }
#pragma unroll
            for (int i = 0; i < LDC / 2; ++i)
              acc[(LDC / 2) * c + i] =
                  add2(acc[(LDC / 2) * c + i],
                       pk(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])));
          }
        } else {
          const float sa = ld_shared_f32(sb + uint32_t(kGwA + kGwB) + uint32_t(r) * 4u);
          const f2 sa2 = pk(sa, sa);
          const uint32_t sw = sb + uint32_t(kGwA + kGwB + kGwSA + part * kGwEpiCols * 4);
#pragma unroll
          for (int c = 0; c < kGwEpiCols / LDC; ++c) {
            float4 w4[LDC / 4];
#pragma unroll
            for (int g = 0; g < LDC / 4; ++g) w4[g] = ld_shared_f4(sw + uint32_t(4 * (LDC * c + 4 * g)));
            uint32_t v[LDC];
            tmem_ld_cols(t_addr + uint32_t(LDC * c), v);
            tmem_wait_ld();
            if (c == kGwEpiCols / LDC - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[b]);
            }
#pragma unroll
            for (int g = 0; g < LDC / 4; ++g) {
              f2& a0 = acc[(LDC / 2) * c + 2 * g];
              f2& a1 = acc[(LDC / 2) * c + 2 * g + 1];
              a0 = fma2(pk(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1])),
                        mul2(sa2, pk(w4[g].x, w4[g].y)), a0);
              a1 = fma2(pk(__uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3])),
                        mul2(sa2, pk(w4[g].z, w4[g].w)), a1);
            }
          }
        }
        // the warp's reads of the stage's scales, each thread's ordered
        // before the next tensor copy into the stage (async proxy) by its
        // proxy fence; one arrive per warp
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == kGwStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      // ------------------------------------------------ bias and the store
      const int64_t row = int64_t(m0) + r;
#pragma unroll
      for (int c = 0; c < kGwEpiChunks; ++c) {
        const int col = c0 + 32 * c;
        f2* y = &acc[16 * c];  // the bias is added in place
        if (p.bias) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            if (col + 4 * g < p.N) {
              const float4 bb = *reinterpret_cast<const float4*>(p.bias + col + 4 * g);
              y[2 * g] = add2(y[2 * g], pk(bb.x, bb.y));
              y[2 * g + 1] = add2(y[2 * g + 1], pk(bb.z, bb.w));
            }
          }
        }
        if (p.out_f32) {
          if (row < p.T) {
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              if (col + 4 * g < p.N)
                *reinterpret_cast<float4*>(p.out_f32 + row * p.N + col + 4 * g) =
                    make_float4(y[2 * g].x, y[2 * g].y, y[2 * g + 1].x, y[2 * g + 1].y);
            }
          }
          continue;
        }
        // one 32 x 32 box through this warp's staging buffer (64-byte rows,
        // 64-byte swizzle: chunk q of row i at q ^ ((i >> 1) & 3))
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        const int swz = (lane >> 1) & 3;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          *reinterpret_cast<uint4*>(stg + lane * 64 + ((qd ^ swz) << 4)) =
              make_uint4(pack_bf16x2_rn(y[4 * qd].x, y[4 * qd].y),
                         pack_bf16x2_rn(y[4 * qd + 1].x, y[4 * qd + 1].y),
                         pack_bf16x2_rn(y[4 * qd + 2].x, y[4 * qd + 2].y),
                         pack_bf16x2_rn(y[4 * qd + 3].x, y[4 * qd + 3].y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && col < p.N && m0 + quarter * 32 < p.T) {
          tma_store_2d(&tmY, stg, col, m0 + quarter * 32);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_gw_factors(const float* L1, const float* L2, const float* sigma_inv, int rank,
                              int K, int N, uint16_t* l1s, uint16_t* l2b, int sms,
                              cudaStream_t st) {
  const int64_t n = int64_t(rank) * K + int64_t(N) * rank;
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  const int grid = int(blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8);
  gw_factor_kernel<<<grid, 256, 0, st>>>(L1, L2, sigma_inv, rank, K, N, l1s, l2b);
  return cudaGetLastError();
}

cudaError_t launch_gw_weights(const GwWeightParams& p, cudaStream_t st) {
  if (p.N == 0) return cudaSuccess;
  gw_weight_kernel<<<p.N, 256, size_t(p.rank) * 4, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gw_act(const void* tmap_x, const void* tmap_l1, const GwActParams& p, int grid,
                          cudaStream_t st) {
  const size_t smem = gw_act_smem_bytes(p.K, p.rank, p.stages, p.sigma_inv != nullptr);
  cudaError_t e = cudaFuncSetAttribute(gw_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  gw_act_kernel<<<grid, kGwActThreads, smem, st>>>(*static_cast<const CUtensorMap*>(tmap_x),
                                                   *static_cast<const CUtensorMap*>(tmap_l1), p);
  return cudaGetLastError();
}

cudaError_t launch_gw_gemm(const void* tmaps, const GwGemmParams& p, int grid, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gw_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kGwGemmSmem));
  if (e != cudaSuccess) return e;
  const CUtensorMap* m = static_cast<const CUtensorMap*>(tmaps);
  gw_gemm_kernel<<<grid, kGwGemmThreads, kGwGemmSmem, st>>>(
      m[0], m[1], m[2], m[3], m[4], m[5], m[6], p);
  return cudaGetLastError();
}

}  // namespace hq
