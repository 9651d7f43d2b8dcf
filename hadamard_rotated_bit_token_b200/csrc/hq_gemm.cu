// hq_gemm.cu -- integer GEMM with the fused HadaNorm epilogue on 5th-generation
// tensor cores (tcgen05, kind::i8, int32 accumulator in tensor memory).
//
//   acc[t,n] = sum_k A[t,k] * B[n,k]                 (HaTQ Sec. IV-B Eq. (14))
//   Y[t,n]   = bf16( s_x[t] * s_w[n] * acc[t,n]      (accumulator scale, HaTQ Eq. (18))
//                    + b[n] + mu_t * colsum[n] )      (b~ = b + mu W~, HadaNorm Eq. (1))
//
// A = activation codes [T,K] int8 (or two 4-bit codes per byte, see PK
// below), B = weight codes [N,K] int8, both K-major.
// Two kernels share one warp layout (320 threads, one CTA per SM; the packed
// form adds warps 10..13):
//   warp 0      one thread issues TMA tensor loads (128-byte swizzle) of the
//               A and B K-slices into a ring of shared-memory stages, and per
//               output tile bulk copies of the tile's columns of s_w, colsum
//               and bias into a two-slot parameter ring;
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma and
//               commits each stage back to the producer and each finished
//               accumulator to the epilogue;
//   warps 2..9  the epilogue: two warps per 32-lane quarter of tensor memory,
//               each taking half of the tile's columns.  A warp reads its
//               columns of the accumulator (tcgen05.ld, up to three 32-column
//               chunks per wait) and hands the accumulator back to the MMA
//               issuer as soon as the last read has landed; then per chunk it
//               applies the epilogue in fp32 (row scale and mean from
//               registers, prefetched one tile ahead; column parameters from
//               the ring), writes bf16 to a 64-byte swizzled shared buffer and
//               lets a TMA tensor store write the 32 x 32 box to Y (clipped at
//               the tensor's edges).
//
// gemm_i8_kernel<BN, LOGO, PK>: one CTA per 128 x BN output tile (BN 64..256).
//   LOGO > 0 selects the weight-only Hadamard epilogue (HaTQ Sec. IV-B
//   Eq. (17)): Y = (s_x s_w acc) H_out + b, the fast Walsh-Hadamard transform
//   over each block of 2^LOGO output columns done in registers after the
//   dequantization (no mean term: that form has no centering).
//   PK: A holds two 4-bit codes per byte.  TMA loads each stage's 128 x
//   64-byte packed tile (64-byte swizzle) next to B; four more warps (warps
//   10..13, one per 32-lane quarter of tensor memory) each read their rows'
//   packed bytes, widen them to int8 (each nibble moved to the high half of
//   its byte: 16 * code, sign included) and store them with tcgen05.st into
//   tensor memory, where the MMA takes its A operand; a third barrier hands
//   the stage to the MMA issuer.  The accumulator is then 16 times the code
//   products' sum, exactly; the epilogue's row scale carries the factor
//   1/16.  No tensor-core kind multiplies 4-bit integers on sm_100a; with A
//   in tensor memory the widened tile never passes through shared memory,
//   whose traffic (tensor loads in, MMA operand reads out) bounds the main
//   loop, so the packed stage costs less shared-memory traffic than an int8
//   one.  A's stages sit in tensor memory after the two accumulators, so
//   packed tiles are at most 192 columns wide.
// gemm_i8_pair_kernel: a cluster of two CTAs per 256 x 256 output tile with
//   the CTA-pair MMA (cta_group::2, M = 256): each CTA loads 128 rows of A and
//   128 rows of B into its own shared memory, so one SM moves half the B
//   bytes per MMA that the single-CTA kernel moves.  Both CTAs' copies
//   complete on the even CTA's stage barrier, whose producer expects the
//   bytes of both; the even CTA issues the MMAs and commits to both CTAs.
// Two accumulators in tensor memory let the epilogue of one tile overlap the
// main loop of the next.  Every wait is bounded; a timeout records
// HQ_ERR_TIMEOUT in the device error word, and the CTA waits for every copy it
// started (or, in the pair kernel, the even CTA for the pair's copies) before
// it exits.
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
constexpr int kConvWarps = 4;  // packed-A converters of the single-CTA kernel (one per lane quarter)
constexpr int kSmemLimit = 227 * 1024;
constexpr int kStageBox = 2048;           // one 32 x 32 bf16 output box
constexpr float kAccMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kAccMagicBits = 0x4B400000;

// instruction descriptor: D s32 (bits 4-5 = 2), A and B signed int8 (bits
// 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at 24-28.
constexpr uint32_t i8_idesc(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

constexpr int tmem_cols_for(int cols) {
  return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}

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

// Output tile `tile` -> (M tile, N tile) in groups of p.group_m M tiles: the
// tiles of a group run N tile by N tile over the group's M tiles, so the CTAs
// working at one time share a few M tiles of A and a few N tiles of B, which
// stay in L2 while the output streams past (plain M-fastest order sweeps all
// of A every round of tiles, and the output evicts it).
__device__ __forceinline__ int tile_m(const GemmParams& p, int tile) {
  const int gsize = p.group_m * p.num_n_tiles;
  const int first = (tile / gsize) * p.group_m;
  const int gm = min(p.num_m_tiles - first, p.group_m);
  return first + (tile % gsize) % gm;
}
__device__ __forceinline__ int tile_n(const GemmParams& p, int tile) {
  const int gsize = p.group_m * p.num_n_tiles;
  const int first = (tile / gsize) * p.group_m;
  const int gm = min(p.num_m_tiles - first, p.group_m);
  return (tile % gsize) / gm;
}

// ------------------------------------------------------- parameter ring
// Slot a holds the columns [n0, n0 + W) of one output tile: s_w at [0, W),
// colsum at [W, 2W), bias at [2W, 3W) (fp32).  An absent vector, and every
// column past N, reads zero or a finite stale value: the ring is zeroed at
// kernel start and absent vectors are never copied.
template <int W>
__device__ __forceinline__ void param_ring_zero(float* ring, int tid, int nthreads) {
  for (int i = tid; i < 2 * 3 * W; i += nthreads) ring[i] = 0.0f;
}

// Producer side: copies the tile's columns [n0, min(n0 + W, N)) into `slot`,
// completion counted on `bar`.
template <int W>
__device__ __forceinline__ void param_ring_load(const GemmParams& p, float* slot, int n0,
                                                uint64_t* bar) {
  const int cols = p.N - n0 < W ? p.N - n0 : W;
  const uint32_t nb = uint32_t(cols) * 4u;  // N % 16 == 0: a multiple of 64 bytes
  const bool cs = p.a_mean != nullptr && p.colsum != nullptr;
  const bool bi = p.bias != nullptr;
  mbar_arrive_expect_tx(bar, nb * (1u + (cs ? 1u : 0u) + (bi ? 1u : 0u)));
  bulk_load(slot, p.w_scale + n0, nb, bar);
  if (cs) bulk_load(slot + W, p.colsum + n0, nb, bar);
  if (bi) bulk_load(slot + 2 * W, p.bias + n0, nb, bar);
}

// ------------------------------------------------------- packed A operand
// One word of eight 4-bit two's-complement codes (element 2j in the low
// nibble of byte j) -> two words of eight int8 values 16 * code, in element
// order: each nibble moved to the high half of its own byte is already the
// sign-extended code times 16, so no sign extension is needed.
__device__ __forceinline__ void widen_i4x8(uint32_t v, uint32_t& lo, uint32_t& hi) {
  const uint32_t ev = (v << 4) & 0xF0F0F0F0u;  // elements 0, 2, 4, 6
  const uint32_t od = v & 0xF0F0F0F0u;         // elements 1, 3, 5, 7
  lo = __byte_perm(ev, od, 0x5140);
  hi = __byte_perm(ev, od, 0x7362);
}

// ------------------------------------------------------------- epilogue
// Per-warp state of the epilogue for one output tile.
struct EpiTile {
  int row0;      // first output row of this warp's 32 rows
  int col_base;  // first output column of this warp's columns
  int64_t row;   // this thread's output row
  bool row_ok;   // row < T
  float sx, mt;  // this row's activation scale and mean
};

// This thread's row scale and mean (zero past T).
__device__ __forceinline__ void load_row_params(const GemmParams& p, int64_t row, float& sx,
                                                float& mt) {
  sx = 0.0f;
  mt = 0.0f;
  if (row < p.T) {
    // packed A enters the MMA as 16 * code, so the accumulator is 16 times
    // the code products' sum; times acc_unit = 1/16 (exact) undoes it
    sx = (p.a_scale_per_row ? p.a_scale[row] : p.a_scale[0]) * p.acc_unit;
    mt = p.a_mean ? p.a_mean[row] : 0.0f;
  }
}

// Raw accumulators of chunk c to acc_debug (bit-exact checks), when asked for.
__device__ __forceinline__ void epi_acc_debug(const GemmParams& p, const uint32_t (&r)[32], int c,
                                              const EpiTile& e) {
  if (p.acc_debug && e.row_ok) {
    const int col0 = e.col_base + c * 32;
    int32_t* arow = p.acc_debug + e.row * p.N;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (col0 + 4 * g < p.N) {
        const int sh = p.acc_shift;  // exact: a packed A's accumulator is a multiple of 16
        *reinterpret_cast<int4*>(arow + col0 + 4 * g) =
            make_int4(int(r[4 * g]) >> sh, int(r[4 * g + 1]) >> sh, int(r[4 * g + 2]) >> sh,
                      int(r[4 * g + 3]) >> sh);
      }
    }
  }
}

// One 32-column chunk c of the warp's columns: accumulators r (this thread's
// row) -> fp32 epilogue -> bf16 pairs in `packed`.  prm points at the warp's
// first column in a parameter slot of width W.
template <int W>
__device__ __forceinline__ void epi_math(const GemmParams& p, const uint32_t (&r)[32], int c,
                                         const EpiTile& e, const float* prm,
                                         uint32_t (&packed)[16]) {
  const float* pw = prm + c * 32;
  const f2 sx2 = pk(e.sx, e.sx), mt2 = pk(e.mt, e.mt);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const float4 sw = *reinterpret_cast<const float4*>(pw + 4 * g);
    const float4 cs = *reinterpret_cast<const float4*>(pw + W + 4 * g);
    const float4 bb = *reinterpret_cast<const float4*>(pw + 2 * W + 4 * g);
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
    // y = acc * (s_x * s_w) + (b + m * colsum)
    const f2 y01 = fma2(a01, mul2(sx2, pk(sw.x, sw.y)), fma2(mt2, pk(cs.x, cs.y), pk(bb.x, bb.y)));
    const f2 y23 = fma2(a23, mul2(sx2, pk(sw.z, sw.w)), fma2(mt2, pk(cs.z, cs.w), pk(bb.z, bb.w)));
    packed[2 * g] = pack_bf16x2(y01.x, y01.y);
    packed[2 * g + 1] = pack_bf16x2(y23.x, y23.y);
  }
  epi_acc_debug(p, r, c, e);
}

// Weight-only Hadamard form, step 1 for chunk c: z = acc * (s_x * s_w) in the
// output Hadamard basis (no mean term: the form has no centering).
template <int W>
__device__ __forceinline__ void epi_dequant(const GemmParams& p, const uint32_t (&r)[32], int c,
                                            const EpiTile& e, const float* prm, f2 (&z)[16]) {
  const float* pw = prm + c * 32;
  const f2 sx2 = pk(e.sx, e.sx);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const float4 sw = *reinterpret_cast<const float4*>(pw + 4 * g);
    f2 a01, a23;
    if (p.small_acc) {
      const f2 mg = pk(kAccMagic, kAccMagic);
      a01 = sub2(pk(__int_as_float(int(r[4 * g + 0]) + kAccMagicBits),
                    __int_as_float(int(r[4 * g + 1]) + kAccMagicBits)), mg);
      a23 = sub2(pk(__int_as_float(int(r[4 * g + 2]) + kAccMagicBits),
                    __int_as_float(int(r[4 * g + 3]) + kAccMagicBits)), mg);
    } else {
      a01 = pk(__int2float_rn(int(r[4 * g + 0])), __int2float_rn(int(r[4 * g + 1])));
      a23 = pk(__int2float_rn(int(r[4 * g + 2])), __int2float_rn(int(r[4 * g + 3])));
    }
    z[2 * g] = mul2(a01, mul2(sx2, pk(sw.x, sw.y)));
    z[2 * g + 1] = mul2(a23, mul2(sx2, pk(sw.z, sw.w)));
  }
  epi_acc_debug(p, r, c, e);
}

// Unnormalized fast Walsh-Hadamard transform over blocks of 2^LOGB (<= 32)
// consecutive columns of a chunk held as 16 column pairs: index bit 0 inside
// each pair, bits 1 .. LOGB-1 between pairs.
template <int LOGB>
__device__ __forceinline__ void fwht_chunk(f2 (&z)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = z[i].x, b = z[i].y;
    z[i] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int bit = 1; bit < LOGB; ++bit) {
    const int hh = 1 << (bit - 1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & hh) == 0) {
        const f2 x = z[i], y = z[i + hh];
        z[i] = add2(x, y);
        z[i + hh] = sub2(x, y);
      }
    }
  }
}

// Weight-only Hadamard form, last step for chunk c: y = z / sqrt(m) + b in
// the original output basis -> bf16 pairs.
template <int W>
__device__ __forceinline__ void epi_finish(const GemmParams& p, const f2 (&z)[16], int c,
                                           const float* prm, uint32_t (&packed)[16]) {
  const float* pw = prm + c * 32;
  const f2 inv2 = pk(p.inv_sqrt_out, p.inv_sqrt_out);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const float4 bb = *reinterpret_cast<const float4*>(pw + 2 * W + 4 * g);
    const f2 y01 = fma2(z[2 * g], inv2, pk(bb.x, bb.y));
    const f2 y23 = fma2(z[2 * g + 1], inv2, pk(bb.z, bb.w));
    packed[2 * g] = pack_bf16x2(y01.x, y01.y);
    packed[2 * g + 1] = pack_bf16x2(y23.x, y23.y);
  }
}

// Chunk c's bf16 values into staging box `buf` (64-byte swizzled rows), then
// one thread stores the 32 x 32 box to Y (clipped at the tensor's edges) as
// its own bulk group.
__device__ __forceinline__ void epi_store_chunk(const GemmParams& p, const CUtensorMap* tmY,
                                                const uint32_t (&packed)[16], int col0, int row0,
                                                uint8_t* buf, int lane) {
  const int swz = (lane >> 1) & 3;  // 64-byte swizzle of this thread's row
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((q ^ swz) << 4)) =
        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && col0 < p.N && row0 < p.T) {
    tma_store_2d(tmY, buf, col0, row0);
    bulk_commit_group();
  }
}

// The warp's HC columns (HC / 32 chunks) of one accumulator at tensor-memory
// address t_addr (lane quarter already encoded), through NBOX staging boxes
// of kStageBox bytes:
//   - the chunks are read from tensor memory in groups of up to three per
//     wait (96 accumulator registers); right after the last group's wait
//     `release_acc` hands the accumulator back to the MMA issuer, so the
//     next main loop into it can start while this tile is still being stored;
//   - per chunk: the epilogue arithmetic, then a wait until the store that
//     last used the chunk's box has read it, then the box and its TMA store;
//   - `release_params` frees the parameter slot after the last chunk's
//     arithmetic.
// LOGO > 0 selects the weight-only Hadamard epilogue with output blocks of
// 2^LOGO columns (4, 5 or 6): dequantize, a fast Walsh-Hadamard transform
// over each block (inside a chunk, and for 64-column blocks one more stage
// between the two chunks of a group), then 1/sqrt(m) and the bias.
template <int HC, int W, int NBOX, int LOGO, int GMAX, class RelAcc, class RelPrm>
__device__ __forceinline__ void epi_tile(const GemmParams& p, const CUtensorMap* tmY,
                                         uint32_t t_addr, const EpiTile& e, const float* prm,
                                         uint8_t* stg, int lane, RelAcc release_acc,
                                         RelPrm release_params) {
  constexpr int NCH = HC / 32;
  constexpr int G0 = NCH <= 3 ? NCH : 2;
  constexpr int G = G0 <= GMAX ? G0 : (NCH % 2 == 0 && GMAX >= 2 ? 2 : 1);
  static_assert(NCH % G == 0, "whole groups of chunks");
  static_assert(LOGO == 0 || (LOGO >= 4 && LOGO <= 5) || (LOGO == 6 && G % 2 == 0),
                "output blocks of 16 or 32 columns, or 64 over chunk pairs");
#pragma unroll
  for (int c0 = 0; c0 < NCH; c0 += G) {
    uint32_t r[G][32];
#pragma unroll
    for (int c = 0; c < G; ++c) tmem_ld_32x32b_x32(t_addr + uint32_t((c0 + c) * 32), r[c]);
    tmem_wait_ld();
    if (c0 + G == NCH) release_acc();
    if constexpr (LOGO == 0) {
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const int ch = c0 + c;
        uint32_t packed[16];
        epi_math<W>(p, r[c], ch, e, prm, packed);
        if (ch == NCH - 1) release_params();
        if (lane == 0) bulk_wait_group_read<NBOX - 1>();
        __syncwarp();
        epi_store_chunk(p, tmY, packed, e.col_base + ch * 32, e.row0,
                        stg + (ch % NBOX) * kStageBox, lane);
      }
    } else {
      f2 z[G][16];
#pragma unroll
      for (int c = 0; c < G; ++c) {
        epi_dequant<W>(p, r[c], c0 + c, e, prm, z[c]);
        fwht_chunk<(LOGO < 5 ? LOGO : 5)>(z[c]);
      }
      if constexpr (LOGO == 6) {
        // index bit 5: between the two 32-column chunks of each pair
#pragma unroll
        for (int c = 0; c < G; c += 2) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const f2 x = z[c][i], y = z[c + 1][i];
            z[c][i] = add2(x, y);
            z[c + 1][i] = sub2(x, y);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const int ch = c0 + c;
        uint32_t packed[16];
        epi_finish<W>(p, z[c], ch, prm, packed);
        if (ch == NCH - 1) release_params();
        if (lane == 0) bulk_wait_group_read<NBOX - 1>();
        __syncwarp();
        epi_store_chunk(p, tmY, packed, e.col_base + ch * 32, e.row0,
                        stg + (ch % NBOX) * kStageBox, lane);
      }
    }
  }
}

}  // namespace

// ------------------------------------------------------- single-CTA kernel
template <int BN, bool PK>
struct GemmCfg {
  static constexpr int A_BYTES = PK ? 0 : BM * BK;      // A's shared stage (PK: in tensor memory)
  static constexpr int B_BYTES = BN * BK;
  static constexpr int P_BYTES = PK ? BM * BK / 2 : 0;  // packed A as loaded (64-byte swizzle)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + P_BYTES;
  static constexpr uint32_t STAGE_TX = uint32_t(STAGE_BYTES);  // bytes the tensor loads bring
  static constexpr int THREADS = kGemmThreads + (PK ? 32 * kConvWarps : 0);
  static constexpr int NBAR_STAGE = PK ? 3 : 2;  // full, empty (, converted)
  static constexpr int HC = BN / 2;  // columns per epilogue warp
  // accumulator chunks read per tensor-memory wait: at most 3; one for packed
  // 192-column tiles, whose 448 threads leave 128 registers a thread
  static constexpr int EPI_GMAX = (PK && BN == 192) ? 1 : 3;
  static constexpr int NBOX = 1;  // output staging boxes per epilogue warp
  static constexpr int EPI_STAGE_BYTES = NBOX * kStageBox;
  static constexpr int RING_BYTES = 2 * 3 * BN * 4;
  static constexpr int CTL_BYTES = 256;
  static constexpr int FIXED = kEpiWarps * EPI_STAGE_BYTES + RING_BYTES + CTL_BYTES + 1024;
  static constexpr int STAGES_RAW = (kSmemLimit - FIXED) / STAGE_BYTES;
  // PK: A's stages (32 columns each) follow the two accumulators in the 512
  // columns of tensor memory; the barrier block holds 7 stages of 3 barriers
  static constexpr int TMEM_STAGE_CAP = PK ? (512 - 2 * BN) / 32 : 8;
  static constexpr int STAGE_CAP = PK ? (TMEM_STAGE_CAP < 7 ? TMEM_STAGE_CAP : 7) : 8;
  static constexpr int STAGES = STAGES_RAW > STAGE_CAP ? STAGE_CAP : STAGES_RAW;
  static constexpr int A_COL0 = 2 * BN;  // first tensor-memory column of A's stages (PK)
  static constexpr int TMEM_COLS = tmem_cols_for(2 * BN + (PK ? 32 * STAGES : 0));
  static constexpr uint32_t IDESC = i8_idesc(BM, BN);
  static constexpr size_t SMEM = size_t(STAGES) * STAGE_BYTES + FIXED;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "two 32-column-aligned halves");
  static_assert(B_BYTES % 1024 == 0, "stage bases must stay 1024-byte aligned");
  static_assert(STAGES >= 2, "shared / tensor memory budget");
  static_assert(!PK || 2 * BN + 32 * STAGES <= 512, "tensor memory budget");
  static_assert(8 * NBAR_STAGE * STAGES + 80 <= CTL_BYTES, "barrier block");
  static_assert(SMEM <= size_t(kSmemLimit), "shared memory budget");
};

template <int BN, int LOGO, bool PK>
__global__ void __launch_bounds__(GemmCfg<BN, PK>::THREADS, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using C = GemmCfg<BN, PK>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + size_t(C::STAGES) * C::A_BYTES;
  uint8_t* sP = sB + size_t(C::STAGES) * C::B_BYTES;  // packed A (PK only)
  uint8_t* epi_stage = sP + size_t(C::STAGES) * C::P_BYTES;  // 1024-aligned
  float* ring = reinterpret_cast<float*>(epi_stage + kEpiWarps * C::EPI_STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(ring) + C::RING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* conv = empty + C::STAGES;    // (PK) stage s's A widened into tensor memory
  uint64_t* tfull = conv + (PK ? C::STAGES : 0);  // [2] accumulator complete
  uint64_t* tempty = tfull + 2;          // [2] accumulator drained by the epilogue
  uint64_t* pfull = tempty + 2;          // [2] parameter slot loaded
  uint64_t* pempty = pfull + 2;          // [2] parameter slot read by the epilogue
  uint64_t* drain = pempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtl wc{p.err, p.wait_ns};

  param_ring_zero<BN>(ring, threadIdx.x, C::THREADS);
  fence_proxy_async_smem();  // the zeros precede the ring's bulk copies
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      if (PK) mbar_init(&conv[s], kConvWarps);  // one arrival per converter warp
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);  // one arrival per epilogue warp
      mbar_init(&pfull[a], 1);
      mbar_init(&pempty[a], kEpiWarps);
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
      int issued = 0, tiles_issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_idx = tile_m(p, tile);
        const int n_idx = tile_n(p, tile);
        const int a = tiles_issued & 1;
        if (*abort_flag || !mbar_wait(&pempty[a], ((tiles_issued >> 1) & 1) ^ 1u, wc)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        param_ring_load<BN>(p, ring + a * 3 * BN, n_idx * BN, &pfull[a]);
        ++tiles_issued;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(&empty[stage], phase ^ 1u, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_TX);
          if constexpr (PK)  // K bytes of packed A per stage: BK / 2 (a multiple of 16)
            tma_load_2d(sP + size_t(stage) * C::P_BYTES, &tmA, kb * (BK / 2), m_idx * BM,
                        &full[stage]);
          else
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
        // let the copies still in flight land before the CTA can exit
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < C::STAGES && i < issued; ++i) {
          if (--s < 0) {
            s = C::STAGES - 1;
            ph ^= 1u;
          }
          (void)mbar_wait(&full[s], ph, wc);
        }
        for (int j = tiles_issued > 2 ? tiles_issued - 2 : 0; j < tiles_issued; ++j)
          (void)mbar_wait(&pfull[j & 1], uint32_t(j >> 1) & 1u, wc);
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
          // B landed (full) and, for packed A, the converters stored A (conv)
          if (*abort_flag || !mbar_wait(&full[stage], phase, wc) ||
              (PK && !mbar_wait(&conv[stage], phase, wc))) {
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
            if constexpr (PK)  // A in tensor memory: 8 columns of four codes per 32 bytes
              mma_i8_tmem_a(d_tmem, tmem_base + uint32_t(C::A_COL0 + 32 * stage + 8 * k),
                            bdesc + uint64_t(2 * k), C::IDESC, (kb > 0 || k > 0) ? 1u : 0u);
            else
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
  } else if (warp < 2 + kEpiWarps) {
    // ----------------------------------------------------------- epilogue
    const int ew = warp - 2;         // 0 .. 7
    const int quarter = warp & 3;    // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = ew >> 2;        // columns [half*HC, half*HC + HC) of the tile
    uint8_t* stg = epi_stage + ew * C::EPI_STAGE_BYTES;
    int acc_iter = 0;
    float sx_next = 0.0f, mt_next = 0.0f;
    if (int(blockIdx.x) < num_tiles)
      load_row_params(p, int64_t(tile_m(p, int(blockIdx.x))) * BM + quarter * 32 + lane,
                      sx_next, mt_next);
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++acc_iter) {
      const int acc = acc_iter & 1;
      const uint32_t acc_phase = (acc_iter >> 1) & 1;
      const int m_idx = tile_m(p, tile);
      const int n_idx = tile_n(p, tile);
      EpiTile e;
      e.row0 = m_idx * BM + quarter * 32;
      e.col_base = n_idx * BN + half * C::HC;
      e.row = int64_t(e.row0) + lane;
      e.row_ok = e.row < p.T;
      e.sx = sx_next;
      e.mt = mt_next;
      const int next = tile + int(gridDim.x);
      if (next < num_tiles)  // next tile's row parameters, in flight during this one
        load_row_params(p, int64_t(tile_m(p, next)) * BM + quarter * 32 + lane, sx_next,
                        mt_next);
      const bool got = !(*abort_flag) && mbar_wait(&tfull[acc], acc_phase, wc) &&
                       mbar_wait(&pfull[acc], acc_phase, wc);
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_addr = tmem_base + uint32_t(acc * BN + half * C::HC) +
                              (uint32_t(quarter * 32) << 16);
      epi_tile<C::HC, BN, C::NBOX, LOGO, C::EPI_GMAX>(
          p, &tmY, t_addr, e, ring + acc * 3 * BN + half * C::HC, stg, lane,
          [&] {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
          },
          [&] {
            // the parameter reads (generic proxy), each thread's ordered
            // before the next bulk copy into the slot by its proxy fence
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[acc]);
          });
    }
    if (lane == 0) bulk_wait_group<0>();  // all of this warp's stores are complete
    __syncwarp();
  } else if constexpr (PK) {
    // ------------------------------------------------- packed-A converters
    // Lane i of converter warp w owns row r = 32 (w % 4) + i of every A tile,
    // which is tensor-memory lane r.  Per stage it reads the row's 64 packed
    // bytes (four 16-byte chunks; with the 64-byte swizzle chunk c of row r
    // sits at chunk c ^ ((r >> 1) & 3), so the 8 rows of a quarter-warp read
    // 8 distinct bank groups), widens them to 128 int8 values and stores
    // them as 32 columns of four values each at A's stage in tensor memory.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int swz = (r >> 1) & 3;
    const uint32_t t_row = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(C::A_COL0);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        // the stage's packed tile has landed, and the MMAs that read its
        // previous A from tensor memory have completed
        const bool got = !(*abort_flag) && mbar_wait(&full[stage], phase, wc) &&
                         mbar_wait(&empty[stage], phase ^ 1u, wc);
        if (!__all_sync(0xffffffffu, got)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* src = sP + size_t(stage) * C::P_BYTES + r * 64;
        uint32_t a[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + ((c ^ swz) << 4));
          widen_i4x8(v.x, a[8 * c + 0], a[8 * c + 1]);
          widen_i4x8(v.y, a[8 * c + 2], a[8 * c + 3]);
          widen_i4x8(v.z, a[8 * c + 4], a[8 * c + 5]);
          widen_i4x8(v.w, a[8 * c + 6], a[8 * c + 7]);
        }
        tmem_st_32x32b_x32(t_row + uint32_t(32 * stage), a);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------- CTA-pair kernel
struct PairCfg {
  static constexpr int BN = 256;          // output columns per pair tile (N of each MMA)
  static constexpr int BM_PAIR = 2 * BM;  // output rows per pair tile (M of each MMA)
  static constexpr int B_ROWS = BN / 2;   // rows of B each CTA holds
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
  static constexpr int HC = BN / 2;  // columns per epilogue warp
  static constexpr int NBOX = 2;  // output staging boxes per epilogue warp
  static constexpr int EPI_STAGE_BYTES = NBOX * kStageBox;
  static constexpr int RING_BYTES = 2 * 3 * BN * 4;
  static constexpr int CTL_BYTES = 512;
  static constexpr int FIXED = kEpiWarps * EPI_STAGE_BYTES + RING_BYTES + CTL_BYTES + 1024;
  static constexpr int STAGES_RAW = (kSmemLimit - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int TMEM_COLS = tmem_cols_for(2 * BN);
  static constexpr uint32_t IDESC = i8_idesc(BM_PAIR, BN);
  static constexpr size_t SMEM = size_t(STAGES) * STAGE_BYTES + FIXED;
  static_assert(B_BYTES % 1024 == 0, "stage bases must stay 1024-byte aligned");
  static_assert(STAGES >= 2, "shared memory budget");
  static_assert(16 * STAGES + 96 <= CTL_BYTES, "barrier block");
  static_assert(SMEM <= size_t(kSmemLimit), "shared memory budget");
};

// Clusters of two CTAs; CTA rank r of a cluster owns rows [128 r, 128 r + 128)
// of every 256-row pair tile (its A rows and its half of the accumulator) and
// B rows [128 r, 128 r + 128) of the tile's 256 columns.  Barriers, all in
// each CTA's own shared memory (those marked "rank 0" used only there):
//   full[s]    (rank 0) stage s of both CTAs landed: rank 0's producer
//              expects the bytes of both and both CTAs' copies count on it;
//   empty[s]   the MMAs have read stage s (pair commit to both CTAs);
//   tfull[a]   accumulator a is complete (pair commit to both CTAs);
//   tempty[a]  (rank 0) the 16 epilogue warps of the pair have read
//              accumulator a (remote arrivals);
//   pfull[a], pempty[a]   this CTA's parameter slot a loaded / read;
//   drain      every MMA issued has completed (pair commit to both CTAs).
// At exit each producer posts the number of stages it loaded to rank 0,
// whose producer then waits until every copy of either CTA has landed: it
// supplies the missing arrival or cancels the missing bytes of a stage that
// only one CTA loaded (after a bounded wait gave up).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + size_t(C::STAGES) * C::A_BYTES;
  uint8_t* epi_stage = sB + size_t(C::STAGES) * C::B_BYTES;  // 1024-aligned
  float* ring = reinterpret_cast<float*>(epi_stage + kEpiWarps * C::EPI_STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(ring) + C::RING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* pfull = tempty + 2;
  uint64_t* pempty = pfull + 2;
  uint64_t* drain = pempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* issued_by = tmem_slot + 2;  // [2], rank 0: stages each CTA loaded

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const WaitCtl wc{p.err, p.wait_ns};

  param_ring_zero<C::BN>(ring, threadIdx.x, kGemmThreads);
  fence_proxy_async_smem();  // the zeros precede the ring's bulk copies
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);
      mbar_init(&pfull[a], 1);
      mbar_init(&pempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    issued_by[0] = issued_by[1] = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.num_m_tiles * p.num_n_tiles;
  const int cluster_id = int(blockIdx.x >> 1);
  const int num_clusters = int(gridDim.x >> 1);
  const int KB = (p.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      const uint32_t full0 = mapa_shared(full, 0);  // rank 0's full[0]
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0, tiles_issued = 0;
      bool ok = true;
      for (int tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
        const int m_idx = tile_m(p, tile);
        const int n_idx = tile_n(p, tile);
        const int a_row = m_idx * C::BM_PAIR + int(rank) * BM;
        const int b_row = n_idx * C::BN + int(rank) * C::B_ROWS;
        const int a = tiles_issued & 1;
        if (*abort_flag || !mbar_wait(&pempty[a], ((tiles_issued >> 1) & 1) ^ 1u, wc)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        param_ring_load<C::BN>(p, ring + a * 3 * C::BN, n_idx * C::BN, &pfull[a]);
        ++tiles_issued;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait<true>(&empty[stage], phase ^ 1u, wc)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const uint32_t bar = full0 + uint32_t(stage) * 8u;
          tma_load_2d_pair(sA + size_t(stage) * C::A_BYTES, &tmA, kb * BK, a_row, bar);
          tma_load_2d_pair(sB + size_t(stage) * C::B_BYTES, &tmB, kb * BK, b_row, bar);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int j = tiles_issued > 2 ? tiles_issued - 2 : 0; j < tiles_issued; ++j)
          (void)mbar_wait(&pfull[j & 1], uint32_t(j >> 1) & 1u, wc);
      }
      st_shared_cluster_u32(mapa_shared(&issued_by[rank], 0), uint32_t(issued));
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (rank 0)
      int stage = 0;
      uint32_t phase = 0;
      int acc_iter = 0;
      bool ok = true;
      const uint32_t a_base = smem_u32(sA);
      const uint32_t b_base = smem_u32(sB);
      for (int tile = cluster_id; tile < num_tiles && ok; tile += num_clusters, ++acc_iter) {
        const int acc = acc_iter & 1;
        const uint32_t acc_phase = (acc_iter >> 1) & 1;
        if (*abort_flag || !mbar_wait<true>(&tempty[acc], acc_phase ^ 1u, wc)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * C::BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait<true>(&full[stage], phase, wc)) {
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
            mma_i8_pair(d_tmem, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), C::IDESC,
                        (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], 0x3);
      }
      // every issued MMA completes before either CTA releases its shared
      // memory or tensor memory
      mma_commit_pair(drain, 0x3);
      (void)mbar_wait<true>(drain, 0, wc);
    } else if (lane == 0) {
      (void)mbar_wait<true>(drain, 0, wc);  // rank 1: the pair's last commit has landed
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int ew = warp - 2;         // 0 .. 7
    const int quarter = warp & 3;    // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = ew >> 2;        // columns [half*HC, half*HC + HC) of the tile
    uint8_t* stg = epi_stage + ew * C::EPI_STAGE_BYTES;
    const uint32_t tempty0 = mapa_shared(tempty, 0);
    const int row_off = int(rank) * BM + quarter * 32 + lane;
    int acc_iter = 0;
    float sx_next = 0.0f, mt_next = 0.0f;
    if (cluster_id < num_tiles)
      load_row_params(p, int64_t(tile_m(p, cluster_id)) * C::BM_PAIR + row_off, sx_next,
                      mt_next);
    for (int tile = cluster_id; tile < num_tiles; tile += num_clusters, ++acc_iter) {
      const int acc = acc_iter & 1;
      const uint32_t acc_phase = (acc_iter >> 1) & 1;
      const int m_idx = tile_m(p, tile);
      const int n_idx = tile_n(p, tile);
      EpiTile e;
      e.row0 = m_idx * C::BM_PAIR + int(rank) * BM + quarter * 32;
      e.col_base = n_idx * C::BN + half * C::HC;
      e.row = int64_t(e.row0) + lane;
      e.row_ok = e.row < p.T;
      e.sx = sx_next;
      e.mt = mt_next;
      const int next = tile + num_clusters;
      if (next < num_tiles)  // next tile's row parameters, in flight during this one
        load_row_params(p, int64_t(tile_m(p, next)) * C::BM_PAIR + row_off, sx_next,
                        mt_next);
      const bool got = !(*abort_flag) && mbar_wait<true>(&tfull[acc], acc_phase, wc) &&
                       mbar_wait(&pfull[acc], acc_phase, wc);
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_addr = tmem_base + uint32_t(acc * C::BN + half * C::HC) +
                              (uint32_t(quarter * 32) << 16);
      epi_tile<C::HC, C::BN, C::NBOX, 0, 3>(
          p, &tmY, t_addr, e, ring + acc * 3 * C::BN + half * C::HC, stg, lane,
          [&] {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(tempty0 + uint32_t(acc) * 8u);
          },
          [&] {
            // the parameter reads (generic proxy), each thread's ordered
            // before the next bulk copy into the slot by its proxy fence
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[acc]);
          });
    }
    if (lane == 0) bulk_wait_group<0>();  // all of this warp's stores are complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both producers have posted their stage counts
  if (rank == 0 && threadIdx.x == 0) {
    // every stage copy of either CTA lands before either CTA can exit
    const int L = int(issued_by[0]), P = int(issued_by[1]);
    const int hi = L > P ? L : P;
    for (int s = 0; s < C::STAGES && s < hi; ++s) {
      const int i = s + ((hi - 1 - s) / C::STAGES) * C::STAGES;  // last copy into stage s
      const bool by0 = i < L, by1 = i < P;
      if (by0 && !by1) mbar_complete_tx(&full[s], C::STAGE_BYTES);
      if (by1 && !by0) mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
      (void)mbar_wait<true>(&full[s], uint32_t(i / C::STAGES) & 1u, wc);
    }
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------- tensor-core ceiling
// The dense int8 rate of this device, measured: the GEMMs' main loop with
// nothing but the MMAs.  Each CTA zeroes STAGES operand stages laid out
// exactly as the GEMMs' (A 128 x 128 bytes, B 256 x 128 bytes per stage,
// 128-byte swizzle), then one thread issues k_blocks x 4 MMAs of 128 x 256 x
// 32 (kind::i8) into one tensor-memory accumulator, cycling through the
// stages, commits and waits.  No loads, no epilogue: an upper bound for the
// single-CTA GEMM.  The CTA-pair form (clusters of two, cta_group::2, M =
// 256, N = 256, each CTA holding half of A and half of B) bounds the pair
// GEMM.  The operands are zeros, so the accumulator ends at zero.
struct CeilCfg {
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = 256 * BK;  // single CTA: 256 rows; pair: 128 of them used
  static constexpr size_t SMEM = size_t(STAGES) * (A_BYTES + B_BYTES) + 1024 + 64;
};

template <bool PAIR>
__global__ void __launch_bounds__(128, 1) mma_ceiling_kernel(int64_t k_blocks, unsigned int* err,
                                                             unsigned long long wait_ns) {
  using C = CeilCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + size_t(C::STAGES) * C::A_BYTES;
  uint64_t* drain = reinterpret_cast<uint64_t*>(sB + size_t(C::STAGES) * C::B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5;
  const WaitCtl wc{err, wait_ns};
  uint4* z = reinterpret_cast<uint4*>(smem);
  const int n16 = C::STAGES * (C::A_BYTES + C::B_BYTES) / 16;
  for (int i = threadIdx.x; i < n16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();  // the zeros precede the tensor cores' operand reads
  if (threadIdx.x == 0) {
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, 256);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 256);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t d_tmem = *tmem_slot;
  const bool issuer = threadIdx.x == 0 && (!PAIR || cluster_ctarank() == 0);
  if (issuer) {
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    constexpr uint32_t idesc = PAIR ? i8_idesc(2 * BM, 256) : i8_idesc(BM, 256);
    for (int64_t kb = 0; kb < k_blocks; ++kb) {
      const int s = int(kb % C::STAGES);
      const uint64_t adesc = sw128_kmajor_desc(a_base + uint32_t(s) * C::A_BYTES);
      const uint64_t bdesc = sw128_kmajor_desc(b_base + uint32_t(s) * C::B_BYTES);
#pragma unroll
      for (int k = 0; k < BK / 32; ++k) {
        const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
        if constexpr (PAIR)
          mma_i8_pair(d_tmem, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), idesc, accum);
        else
          mma_i8(d_tmem, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), idesc, accum);
      }
    }
    if constexpr (PAIR)
      mma_commit_pair(drain, 0x3);
    else
      mma_commit(drain);
  }
  if (threadIdx.x == 0) (void)mbar_wait<PAIR>(drain, 0, wc);  // every MMA has completed
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(d_tmem, 256);
    else
      tmem_dealloc(d_tmem, 256);
  }
}

cudaError_t launch_mma_ceiling(bool pair, int64_t k_blocks, int ctas, unsigned int* err,
                               unsigned long long wait_ns, cudaStream_t st) {
  static bool configured[2] = {false, false};
  const void* fn = pair ? (const void*)mma_ceiling_kernel<true> : (const void*)mma_ceiling_kernel<false>;
  if (!configured[pair ? 1 : 0]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(CeilCfg::SMEM));
    if (e != cudaSuccess) return e;
    configured[pair ? 1 : 0] = true;
  }
  if (pair) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(ctas));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = CeilCfg::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, mma_ceiling_kernel<true>, k_blocks, err, wait_ns);
  }
  mma_ceiling_kernel<false><<<ctas, 128, CeilCfg::SMEM, st>>>(k_blocks, err, wait_ns);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ launch
template <int BN, int LOGO, bool PK>
static cudaError_t launch_bn(const void* tmap_a, const void* tmap_b, const void* tmap_y,
                             const GemmParams& p, int grid, cudaStream_t st) {
  using C = GemmCfg<BN, PK>;
  static bool configured = false;  // attribute is per function, device-agnostic
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<BN, LOGO, PK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  gemm_i8_kernel<BN, LOGO, PK><<<grid, C::THREADS, C::SMEM, st>>>(
      *reinterpret_cast<const CUtensorMap*>(tmap_a), *reinterpret_cast<const CUtensorMap*>(tmap_b),
      *reinterpret_cast<const CUtensorMap*>(tmap_y), p);
  return cudaGetLastError();
}

template <int LOGO, bool PK>
static cudaError_t launch_logo(int bn, const void* tmap_a, const void* tmap_b,
                               const void* tmap_y, const GemmParams& p, int grid, cudaStream_t st) {
  switch (bn) {
    case 128: return launch_bn<128, LOGO, PK>(tmap_a, tmap_b, tmap_y, p, grid, st);
    case 256:  // packed A's stages leave no tensor memory for 256-column tiles
      if constexpr (!PK) return launch_bn<256, LOGO, PK>(tmap_a, tmap_b, tmap_y, p, grid, st);
      return cudaErrorInvalidValue;
    default:
      if constexpr (LOGO <= 5) {
        if (bn == 64) return launch_bn<64, LOGO, PK>(tmap_a, tmap_b, tmap_y, p, grid, st);
        if (bn == 192) return launch_bn<192, LOGO, PK>(tmap_a, tmap_b, tmap_y, p, grid, st);
      }
      return cudaErrorInvalidValue;
  }
}

template <bool PK>
static cudaError_t launch_pk(int bn, int logo, const void* tmap_a, const void* tmap_b,
                             const void* tmap_y, const GemmParams& p, int grid, cudaStream_t st) {
  switch (logo) {
    case 0: return launch_logo<0, PK>(bn, tmap_a, tmap_b, tmap_y, p, grid, st);
    case 4: return launch_logo<4, PK>(bn, tmap_a, tmap_b, tmap_y, p, grid, st);
    case 5: return launch_logo<5, PK>(bn, tmap_a, tmap_b, tmap_y, p, grid, st);
    case 6: return launch_logo<6, PK>(bn, tmap_a, tmap_b, tmap_y, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(int bn, int logo, bool packed_a, const void* tmap_a, const void* tmap_b,
                        const void* tmap_y, const GemmParams& p, int grid, cudaStream_t st) {
  return packed_a ? launch_pk<true>(bn, logo, tmap_a, tmap_b, tmap_y, p, grid, st)
                  : launch_pk<false>(bn, logo, tmap_a, tmap_b, tmap_y, p, grid, st);
}

static cudaError_t configure_pair() {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(PairCfg::SMEM));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return cudaSuccess;
}

cudaError_t gemm_pair_max_clusters(int* clusters) {
  cudaError_t e = configure_pair();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(sms & ~1));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = PairCfg::SMEM;
  return cudaOccupancyMaxActiveClusters(clusters, gemm_i8_pair_kernel, &cfg);
}

cudaError_t launch_gemm_pair(const void* tmap_a, const void* tmap_b, const void* tmap_y,
                             const GemmParams& p, int clusters, cudaStream_t st) {
  cudaError_t e = configure_pair();
  if (e != cudaSuccess) return e;
  gemm_i8_pair_kernel<<<2 * clusters, kGemmThreads, PairCfg::SMEM, st>>>(
      *reinterpret_cast<const CUtensorMap*>(tmap_a), *reinterpret_cast<const CUtensorMap*>(tmap_b),
      *reinterpret_cast<const CUtensorMap*>(tmap_y), p);
  return cudaGetLastError();
}

template <bool PK>
static size_t smem_of(int bn) {
  switch (bn) {
    case 64: return GemmCfg<64, PK>::SMEM;
    case 128: return GemmCfg<128, PK>::SMEM;
    case 192: return GemmCfg<192, PK>::SMEM;
    case 256:
      if constexpr (!PK) return GemmCfg<256, PK>::SMEM;
      return 0;
    default: return 0;
  }
}

size_t gemm_smem_bytes(int bn, bool packed_a) {
  return packed_a ? smem_of<true>(bn) : smem_of<false>(bn);
}

size_t gemm_pair_smem_bytes() { return PairCfg::SMEM; }
int gemm_pair_stages() { return PairCfg::STAGES; }

int gemm_threads(bool packed_a) { return kGemmThreads + (packed_a ? 32 * kConvWarps : 0); }

}  // namespace hq
