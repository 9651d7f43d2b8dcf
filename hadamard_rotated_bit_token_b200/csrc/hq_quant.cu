// hq_quant.cu -- fused row quantizer for the Hadamard-domain linear layer.
//
// One kernel serves both sides of the HadaNorm identity (HadaNorm review,
// "What carries the argument", Eq. (1)):
//   activations:  Y = X diag(sigma^-1),  Z = Y H,  V = Z - mu_t,  per-token
//                 (or per-tensor) symmetric quantization of V;
//   weights:      Y = W diag(sigma),     W~ = Y H, per-row (output channel)
//                 symmetric quantization of W~ and its row sum (the mu W~ term
//                 of b~).
// H is block diagonal with Sylvester blocks of order n = 2^LOGN ("Data-free
// 4-bit quantization for diffusion transformers", "Hadamard rotation", step 7;
// HaTQ supplement Eq. (34)).  The transform is an unnormalized fast
// Walsh-Hadamard transform (additions and subtractions only, HaTQ Sec. IV-D);
// the 1/sqrt(n) normalization is folded into the reported scale and mean
// (HQ-DM summary 2.1, HaTQ supplement VII-C), which leaves the codes
// unchanged because they depend only on V / max|V|.
//
// Quantizer: HaTQ Sec. III-A Eq. (3), q = 2^(b-1) - 1, s = max|V| / q,
// code = rne(V / s), computed as rne(V * (q / max|V|)) with one fused
// multiply-add against 1.5 * 2^23, which rounds half to even and leaves the
// code in the low byte of the result's bit pattern.
//
// Row mean: sum_k Z_hat[b,k] = n * Y[b,0] for each block b (every column of
// H~ but the first sums to zero), so mu_hat = (n / K) * sum_b Y[b,0]; this
// identity (HaTQ Eq. (23) read column-wise) gives the exact mean of the
// rotated row from the first channel of each block, summed in block order.
//
// Work decomposition (persistent CTAs over tiles of R rows; every thread
// owns one 32-channel slice of one row of each tile, the same slice of every
// tile):
//   load     four coalesced 16-byte loads straight into registers, issued one
//            tile ahead of the tile being processed (no shared-memory stage);
//   rotate   bf16 -> fp32, times the channel multiplier, butterflies on the 5
//            in-register index bits, then the remaining bits across the n/32
//            threads of a block: warp shuffles for n <= 128; for n >= 256 a
//            shared-memory transpose among up to 8 lanes swaps index bits
//            with in-register ones and shuffles take bits 8 and up;
//   stats    the row's max / min by a warp reduction over the lanes of the
//            row (redux.sync) and one shared-memory atomic per warp segment;
//            the segment that completes the row (a per-row arrival counter)
//            computes the row's mean, scale and reciprocal once, publishes
//            them and releases the row's barrier;
//   quantize codes packed 4 per word and stored, one per byte, or two per
//            byte (4-bit two's-complement nibbles, element 2j in the low
//            nibble) when the caller asks for packed codes.
// No CTA-wide barrier in the loop: warps wait only for the rows they hold.
// With n = 1 (no rotation) the transform is skipped and the codes are formed
// by a correctly rounded division (see the quantize step).
//
// Also here: the offline column reductions for sigma, and the weight side of
// the weight-only Hadamard form (wh_weights_kernel: W rotated along the
// output channels, quantized per row, in fp64).
// Arithmetic on pairs of lanes uses Blackwell's packed fp32x2 instructions.
#include <cuda.h>

#include <cmath>

#include "hq_device.cuh"
#include "hq_kernels.h"

namespace hq {

namespace {

constexpr int kQuantThreads = 320;          // up to 10 warps, all workers
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Order-preserving map of floats onto unsigned integers (for max / min of
// floats by integer reductions and atomics).
__device__ __forceinline__ uint32_t ord_f32(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Streaming 16-byte load of data read once (not kept in L1).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Shared-memory layout of one CTA (byte offsets from a 16-byte aligned base).
struct QuantSmem {
  uint32_t mult, xbuf, pmax, pmin, cnt, res, y0, rowbar, flags, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }
__host__ __device__ inline int padded_blocks(int B) { return (B + 3) & ~3; }

// R rows per tile, K channels, B blocks per row, `nwarps` warps.  The row
// statistics are double-buffered by tile parity.
__host__ __device__ inline QuantSmem quant_smem_layout(int R, int K, int B, int nwarps, bool xpose) {
  QuantSmem L;
  uint32_t off = 0;
  L.mult = off;  // channel multipliers, chunk-major [8][S] float4 (S = ceil(K / 32))
  off += 128u * uint32_t((K + 31) / 32);
  L.xbuf = off;  // per-warp transpose buffers
  off += xpose ? 4096u * nwarps : 0u;
  L.pmax = off;
  off += 4u * 2 * R;
  L.pmin = off;
  off += 4u * 2 * R;
  L.cnt = off;
  off += 4u * 2 * R;
  off = align_up(off, 8);
  L.res = off;  // [2][R] (mean, reciprocal scale)
  off += 8u * 2 * R;
  off = align_up(off, 16);
  L.y0 = off;  // [2][R][padded B] first channel of every block
  off += 4u * 2 * R * padded_blocks(B);
  off = align_up(off, 8);
  L.flags = off;  // [0] abort, [1] CTA max (mode 1)
  off += 16;
  L.total = off;
  return L;
}

}  // namespace

size_t quant_smem_bytes(int R, int K, int B, int nwarps, bool xpose) {
  return quant_smem_layout(R, K, B, nwarps, xpose).total;
}

// MODE 0: per-row dynamic scale (activations per token, or weights per row)
// MODE 1: per-tensor pass 1: only the tensor-wide max |V| (into tensor_max)
// MODE 2: per-tensor pass 2: scale from tensor_max
// MODE 3: per-tensor static scale from static_scale[0] (real units)
// CM: 0 no centering, 1 the row mean removed after the rotation, 2 removed
// before it (the HQ_CENTER_* values).
template <int LOGN, int MODE, int CM>
__global__ void __launch_bounds__(kQuantThreads, 2) quant_rows_kernel(const QuantParams p) {
  constexpr bool CENTER = (CM == 1);
  constexpr bool PRE = (CM == 2);
  constexpr int N = 1 << LOGN;
  constexpr int LREG = LOGN < 5 ? LOGN : 5;        // index bits inside a thread's slice
  constexpr int LOG_TT = LOGN > 5 ? LOGN - 5 : 0;  // index bits across threads
  constexpr int TT = 1 << LOG_TT;                  // threads per Hadamard block
  // Cross-thread bits: for n <= 128 (at most two) all by warp shuffles; for
  // larger blocks the lowest LX of them by a shared-memory transpose among
  // G = 2^LX lanes (swapping them with in-register bits 5-LX..4), the rest
  // by warp shuffles (measured: shuffles win at two cross-thread bits, the
  // transpose at three and more).
  constexpr int LX = LOGN <= 7 ? 0 : (LOG_TT < 3 ? LOG_TT : 3);
  constexpr int G = 1 << LX;                       // lanes per transpose group = groups per thread
  constexpr int GS = 32 / G;                       // elements per group
  constexpr int GP = GS / 2;                       // f32x2 pairs per group
  constexpr int CH = GS / 4;                       // 16-byte chunks per group
  constexpr bool XPOSE = LX > 0;
  constexpr int NSHFL = LOG_TT - LX;
  constexpr int BPT = N >= 32 ? 1 : 32 / N;        // blocks per thread slice (n < 32)
  constexpr bool kClamp = (MODE >= 2);
  constexpr bool kQuantize = (MODE != 1);

  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.S;  // 32-channel slices per row
  const int R = p.R;  // rows per tile
  const int K = p.K;
  // blocks whose first channels are kept (none for n = 1: no rotation, no
  // centering, no row sums)
  const int B = LOGN == 0 ? 0 : K >> LOGN;
  const int BP = padded_blocks(B);
  const int64_t T = p.T;
  const int64_t ntiles = (T + R - 1) / R;
  const QuantSmem L = quant_smem_layout(R, K, B, int(blockDim.x) >> 5, XPOSE);
  float4* msm = reinterpret_cast<float4*>(smem + L.mult);
  uint32_t* pmax = reinterpret_cast<uint32_t*>(smem + L.pmax);
  uint32_t* pmin = reinterpret_cast<uint32_t*>(smem + L.pmin);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + L.cnt);
  float2* res = reinterpret_cast<float2*>(smem + L.res);
  float* y0buf = reinterpret_cast<float*>(smem + L.y0);
  uint64_t* rowbar = reinterpret_cast<uint64_t*>(smem + L.rowbar);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flags);
  const WaitCtl wc{p.err, p.wait_ns};
  const bool has_mult = p.mult != nullptr;
  const bool need_sum = LOGN > 0 && (CM != 0 || p.rowsum != nullptr);
  // the rows' block sums (first rotated channel of each block) instead of
  // their blocks' first input channels
  const bool block_sums = LOGN > 0 && (PRE || (p.rowsum != nullptr && p.rowsum_pre));

  const bool active = tid < R * S;
  const int row0 = active ? tid / S : 0;  // this thread's row of every tile
  const int slice = active ? tid - row0 * S : 0;
  const int member = slice & (TT - 1);
  const int blk = slice >> LOG_TT;        // block of the row (n >= 32)
  // K a multiple of 16 but not of 32 (n = 16 or 1): the row's last slice
  // holds 16 channels; its upper half is padding, kept out of every
  // statistic and never stored
  const bool half = (K & 31) != 0 && slice == S - 1;

  // first tile's slice in flight while the CTA sets up
  const uint16_t* xcol = p.X + slice * 32;
  uint4 nxt[4] = {};
  auto load_slice = [&](int64_t tile) {
    const int64_t row = tile * R + row0;
    if (active && row < T) {
      const uint4* src = reinterpret_cast<const uint4*>(xcol + row * K);
#pragma unroll
      for (int c = 0; c < 4; ++c) nxt[c] = (half && c >= 2) ? make_uint4(0, 0, 0, 0) : ld_stream(src + c);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) nxt[c] = make_uint4(0, 0, 0, 0);
    }
  };
  if (int64_t(blockIdx.x) < ntiles) load_slice(blockIdx.x);

  if (tid == 0) {
    for (int r = 0; r < R; ++r) mbar_init(&rowbar[r], 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_mbarrier_init();
  }
  for (int i = tid; i < 2 * R; i += blockDim.x) {
    pmax[i] = 0u;
    pmin[i] = 0xFFFFFFFFu;
    cnt[i] = 0u;
  }
  for (int i = tid; i < 2 * R * BP; i += blockDim.x) y0buf[i] = 0.0f;  // padding stays zero
  if (has_mult) {
    // chunk-major copy: thread `slice` reads chunk c at msm[c * S + slice], so
    // consecutive slices hit consecutive 16-byte words
    for (int i = tid; i < 8 * S; i += blockDim.x) {
      const int c = i / S, sl = i - c * S;
      if (sl * 32 + 4 * c >= K) {  // past the row's end (a half slice): unused
        msm[i] = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        continue;
      }
      float4 m4 = *reinterpret_cast<const float4*>(p.mult + sl * 32 + 4 * c);
      if (p.invert_mult) {
        m4.x = 1.0f / m4.x;
        m4.y = 1.0f / m4.y;
        m4.z = 1.0f / m4.z;
        m4.w = 1.0f / m4.w;
      }
      msm[i] = m4;
    }
  }
  __syncthreads();

  // lanes of this warp that hold slices of this thread's row
  const int wbase = warp * 32;
  const int seg_lo = max(row0 * S, wbase) - wbase;
  const int seg_hi = min(min(row0 * S + S, R * S), wbase + 32) - wbase;
  const int seg_len = seg_hi - seg_lo;
  const unsigned segmask = seg_len >= 32 ? 0xFFFFFFFFu : (((1u << seg_len) - 1u) << seg_lo);
  const bool seg_leader = active && lane == seg_lo;

  const int tl = lane & (G - 1);        // lane within the transpose group
  const int sub = lane >> LX;           // transpose group within the warp
  uint8_t* xb = smem + L.xbuf + warp * 4096 + sub * (G * 128);
  const int csw = sub & (CH - 1);       // chunk swizzle of this transpose group

  float r_tensor = 0.0f;
  // n = 1 (no rotation): the code is rne(V * num / den) with a correctly
  // rounded division -- num = q and den = max |V| for dynamic scales, num = 1
  // and den = s for a static one -- so a bf16 value lying exactly on a
  // rounding tie (common without a rotation) is rounded half to even, as the
  // quantizer's definition asks; den_tensor is the per-tensor den
  float den_tensor = 0.0f;
  if (MODE == 2) {
    const float a = __uint_as_float(*p.tensor_max);
    den_tensor = a;
    r_tensor = a > 0.0f ? __fdiv_rn(float(p.q), a) : 0.0f;
    if (blockIdx.x == 0 && tid == 0 && p.scale) p.scale[0] = (a / float(p.q)) * p.inv_sqrt_n;
  } else if (MODE == 3) {
    const float s = p.static_scale[0];
    den_tensor = s * p.sqrt_n;
    r_tensor = s > 0.0f ? __fdiv_rn(1.0f, s * p.sqrt_n) : 0.0f;
  }
  const float n_over_k = float(N) / float(K);
  const float inv_k = 1.0f / float(K);
  const float qf = float(p.q);
  const float s_unit = p.inv_sqrt_n / qf;

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int pb = it & 1;  // statistics buffer of this tile
    const int sr = pb * R + row0;
    f2 w[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      w[4 * c + 0] = pk(bf16lo(nxt[c].x), bf16hi(nxt[c].x));
      w[4 * c + 1] = pk(bf16lo(nxt[c].y), bf16hi(nxt[c].y));
      w[4 * c + 2] = pk(bf16lo(nxt[c].z), bf16hi(nxt[c].z));
      w[4 * c + 3] = pk(bf16lo(nxt[c].w), bf16hi(nxt[c].w));
    }
    if (tile + gridDim.x < ntiles) load_slice(tile + gridDim.x);  // one tile ahead

    if (has_mult) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 m4 = msm[i * S + slice];
        w[2 * i] = mul2(w[2 * i], pk(m4.x, m4.y));
        w[2 * i + 1] = mul2(w[2 * i + 1], pk(m4.z, m4.w));
      }
    }
    // first channel of each block (Y[b,0]) for the row mean / row sum
    if (need_sum && !block_sums && active && member == 0) {
      float* yrow = y0buf + sr * BP;
#pragma unroll
      for (int b = 0; b < BPT; ++b)
        if (blk * BPT + b < B) yrow[blk * BPT + b] = w[(b * N) >> 1].x;
    }
    // index bit 0: the two halves of a pair (n = 1: no rotation)
    if (LOGN >= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = w[i].x, b = w[i].y;
        w[i] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
      }
    }
    // index bits 1 .. LREG-1: between pairs
#pragma unroll
    for (int bit = 1; bit < LREG; ++bit) {
      const int hh = 1 << (bit - 1);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & hh) == 0) {
          const f2 x = w[i], y = w[i + hh];
          w[i] = add2(x, y);
          w[i + hh] = sub2(x, y);
        }
      }
    }
    if (XPOSE) {
      // swap index bits 5..4+LX (lanes of a G-lane group) with bits
      // 5-LX..4 (register groups of GS elements); slots XOR-swizzled by
      // lane, chunks by group, so 16-byte accesses do not conflict
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const f2 a = w[g * GP + 2 * c], b = w[g * GP + 2 * c + 1];
          *reinterpret_cast<float4*>(xb + (tl * G + (g ^ tl)) * (GS * 4) + ((c ^ csw) << 4)) =
              make_float4(a.x, a.y, b.x, b.y);
        }
      }
      __syncwarp();
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const float4 v = *reinterpret_cast<const float4*>(xb + (g * G + (tl ^ g)) * (GS * 4) +
                                                            ((c ^ csw) << 4));
          w[g * GP + 2 * c] = pk(v.x, v.y);
          w[g * GP + 2 * c + 1] = pk(v.z, v.w);
        }
      }
      __syncwarp();
      // index bits 5..4+LX are now the register-group bits
#pragma unroll
      for (int k = 0; k < LX; ++k) {
        const int hh = GP << k;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if ((i & hh) == 0) {
            const f2 x = w[i], y = w[i + hh];
            w[i] = add2(x, y);
            w[i + hh] = sub2(x, y);
          }
        }
      }
    }
    // remaining index bits (5+LX and up) across lanes
#pragma unroll
    for (int j = 0; j < NSHFL; ++j) {
      const int mask = 1 << (LX + j);
      const float sg = (lane & mask) ? -1.0f : 1.0f;
      const f2 sg2 = pk(sg, sg);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const f2 o = pk(__shfl_xor_sync(0xffffffffu, w[i].x, mask),
                        __shfl_xor_sync(0xffffffffu, w[i].y, mask));
        w[i] = fma2(w[i], sg2, o);
      }
    }

    // each block's first rotated channel is its block sum sum_j Y[b,j]; the
    // row needs them when centering before the rotation (they are the only
    // channels it moves) and for the weights' pre-rotation correction
    float first[BPT];
    if (block_sums && member == 0) {
#pragma unroll
      for (int b = 0; b < BPT; ++b) {
        first[b] = w[(b * N) >> 1].x;
        if (active && blk * BPT + b < B) y0buf[sr * BP + blk * BPT + b] = first[b];
        // left out of this slice's max / min (channel 1 of block 0 stands in)
        if (PRE) w[(b * N) >> 1].x = w[0].y;
      }
    }

    // a half slice's padding repeats a real value (channels 2 and 3, never a
    // block's first channel), so it leaves the max and min unchanged
    if (half) {
#pragma unroll
      for (int i = 8; i < 16; ++i) w[i] = w[1];
    }
    // row max / min: reduce over this warp's lanes of the row, one atomic per
    // warp segment; the segment that completes the row finalizes it
    float mx = max3(w[0].x, w[0].y, w[1].x);
    float mn = min3(w[0].x, w[0].y, w[1].x);
    mx = fmaxf(mx, w[1].y);
    mn = fminf(mn, w[1].y);
#pragma unroll
    for (int i = 2; i < 16; ++i) {
      mx = max3(mx, w[i].x, w[i].y);
      mn = min3(mn, w[i].x, w[i].y);
    }
    if (PRE && member == 0) {
#pragma unroll
      for (int b = 0; b < BPT; ++b) w[(b * N) >> 1].x = first[b];
    }
    __syncwarp();  // this warp's first-channel stores precede its leaders' arrivals
    bool ok = true;
    if (active) {
      const uint32_t umx = __reduce_max_sync(segmask, ord_f32(mx));
      const uint32_t umn = __reduce_min_sync(segmask, ord_f32(mn));
      if (seg_leader) {
        atomicMax(&pmax[sr], umx);
        atomicMin(&pmin[sr], umn);
        __threadfence_block();
        const uint32_t before = atomicAdd(&cnt[sr], uint32_t(seg_len));
        if (before + uint32_t(seg_len) == uint32_t(S)) {
          // last segment of the row: every slice's max, min and first
          // channels are in shared memory
          __threadfence_block();
          const int64_t row = tile * R + row0;
          float rsum = 0.0f;
          if (need_sum) {
            // block order; the padding past B holds zeros, which leave the sum unchanged
            const float4* y4 = reinterpret_cast<const float4*>(y0buf + sr * BP);
            for (int b4 = 0; b4 < (B + 3) / 4; ++b4) {
              const float4 v = y4[b4];
              rsum = __fadd_rn(__fadd_rn(__fadd_rn(__fadd_rn(rsum, v.x), v.y), v.z), v.w);
            }
          }
          // CM 1: m_hat = mean of the rotated row, subtracted everywhere.
          // CM 2: mu = rsum / K (the blocks' sums add up to the row's sum);
          // the rotated row changes only at each block's first channel, by
          // -n mu (unnormalized transform), which m_hat then holds.
          const float mu = PRE ? rsum * inv_k : 0.0f;
          const float m_hat = CENTER ? n_over_k * rsum : (PRE ? float(N) * mu : 0.0f);
          float rmx = unord_f32(pmax[sr]);
          float rmn = unord_f32(pmin[sr]);
          if (PRE) {
            const float* yrow = y0buf + sr * BP;
            for (int b = 0; b < B; ++b) {
              const float v = __fsub_rn(yrow[b], m_hat);
              rmx = fmaxf(rmx, v);
              rmn = fminf(rmn, v);
            }
          }
          const float a_hat = PRE ? fmaxf(rmx, -rmn)
                                  : fmaxf(__fsub_rn(rmx, m_hat), __fsub_rn(m_hat, rmn));
          float r_rec = r_tensor;
          // q / a_hat to within 2 ulp: moves a code only when V * q / a_hat
          // lies within a few ulp of a rounding boundary
          if (MODE == 0) r_rec = a_hat > 0.0f ? __fdividef(qf, a_hat) : 0.0f;
          // n = 1 keeps the row's max itself, the divisor of its exact path
          res[sr] = make_float2(m_hat, LOGN == 0 ? a_hat : r_rec);
          pmax[sr] = 0u;  // ready for tile it + 2
          pmin[sr] = 0xFFFFFFFFu;
          cnt[sr] = 0u;
          if (row < T) {
            if (MODE == 0) p.scale[row] = a_hat * s_unit;  // a_hat / (q sqrt(n))
            if (MODE == 1)
              atomicMax(reinterpret_cast<unsigned*>(const_cast<int*>(&flags[1])),
                        __float_as_uint(a_hat));
            if (kQuantize && p.mean) p.mean[row] = PRE ? mu : m_hat * p.inv_sqrt_n;
            // sum_k sigma_k W[n,k] = the blocks' sums, or
            // sum_k W~[n,k] = sqrt(n) * sum_b Y[b,0]
            if (p.rowsum) p.rowsum[row] = p.rowsum_pre ? rsum : rsum * p.sqrt_n;
          }
          // test hook: the first row of this CTA's first tile is never released
          if (!(p.fault_withhold_row && it == 0 && row0 == 0)) mbar_arrive(&rowbar[row0]);
        }
      }
      ok = mbar_wait(&rowbar[row0], uint32_t(it & 1), wc);
    }
    if (!__all_sync(0xffffffffu, ok && !flags[0])) {  // warp-uniform exit
      flags[0] = 1;
      break;
    }
    if (!active) continue;

    const int64_t row = tile * R + row0;
    if (!kQuantize || row >= T) continue;
    const float2 st = res[sr];
    if (PRE && member == 0) {
#pragma unroll
      for (int b = 0; b < BPT; ++b) w[(b * N) >> 1].x = __fsub_rn(w[(b * N) >> 1].x, st.x);
    }
    const float mshift = PRE ? 0.0f : st.x;
    const f2 mh2 = pk(mshift, mshift), rr2 = pk(st.y, st.y), mg2 = pk(kRoundMagic, kRoundMagic);
    // n = 1: numerator factor and divisor of the exact path
    const float num = MODE == 3 ? 1.0f : qf;
    const float den = MODE == 0 ? st.y : den_tensor;
    uint32_t words[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      uint32_t b[4];
      if (LOGN == 0) {
        // codes as int32 + the magic's bit pattern, like the fused path
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float v = (u & 1) ? w[2 * g + (u >> 1)].y : w[2 * g + (u >> 1)].x;
          const int c = den > 0.0f ? __float2int_rn(__fdiv_rn(__fmul_rn(v, num), den)) : 0;
          b[u] = uint32_t(c) + kRoundMagicBits;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const f2 t = fma2(sub2(w[2 * g + u], mh2), rr2, mg2);
          b[2 * u] = __float_as_uint(t.x);
          b[2 * u + 1] = __float_as_uint(t.y);
        }
      }
      if (kClamp) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int c = int(b[u] - kRoundMagicBits);
          b[u] = uint32_t(max(-p.q, min(p.q, c)));
        }
      }
      words[g] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                             0x5410);
    }
    if (p.packed) {
      // two codes per byte, element 2j of the row in the low nibble of byte
      // j: t keeps (c0 | c1 << 4) in byte 0 and (c2 | c3 << 4) in byte 2 of
      // each word of four codes
      uint32_t t[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) t[g] = (words[g] & 0x0F0F0F0Fu) | ((words[g] >> 4) & 0xF0F0F0F0u);
      uint8_t* prow = reinterpret_cast<uint8_t*>(p.codes) + row * (K / 2);
      if constexpr (!XPOSE) {
        if (half)
          *reinterpret_cast<uint2*>(prow + slice * 16) =
              make_uint2(__byte_perm(t[0], t[1], 0x6420), __byte_perm(t[2], t[3], 0x6420));
        else
          *reinterpret_cast<uint4*>(prow + slice * 16) =
              make_uint4(__byte_perm(t[0], t[1], 0x6420), __byte_perm(t[2], t[3], 0x6420),
                         __byte_perm(t[4], t[5], 0x6420), __byte_perm(t[6], t[7], 0x6420));
      } else {
        static_assert(GS == 4, "four codes (two bytes) per register group");
        uint8_t* base = prow + (blk * N + GS * tl + (32 * G) * (member >> LX)) / 2;
#pragma unroll
        for (int g = 0; g < G; ++g)
          *reinterpret_cast<uint16_t*>(base + 16 * g) = uint16_t(__byte_perm(t[g], 0u, 0x0020));
      }
      continue;
    }
    int8_t* crow = p.codes + row * K;
    if (!XPOSE) {
      uint4* dst = reinterpret_cast<uint4*>(crow + slice * 32);
      dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
      if (!half) dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    } else {
      // register group g: index bits 5..4+LX = g, bits 5-LX..4 = tl, bits
      // 5+LX.. = member >> LX; GS consecutive codes per group
      int8_t* base = crow + blk * N + GS * tl + (32 * G) * (member >> LX);
      constexpr int WPG = GS / 4;  // words per group
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (WPG == 4) {
          *reinterpret_cast<uint4*>(base + 32 * g) =
              make_uint4(words[4 * g], words[4 * g + 1], words[4 * g + 2], words[4 * g + 3]);
        } else if (WPG == 2) {
          *reinterpret_cast<uint2*>(base + 32 * g) = make_uint2(words[2 * g], words[2 * g + 1]);
        } else {
          *reinterpret_cast<uint32_t*>(base + 32 * g) = words[g];
        }
      }
    }
  }

  __syncthreads();
  if (MODE == 1 && tid == 0 && !flags[0]) atomicMax(p.tensor_max, unsigned(flags[1]));
}

// ---------------------------------------------------------------- dispatch
template <int MODE, int CM>
static const void* pick_by_logn(int logn) {
  switch (logn) {
    case 0:  // n = 1, no rotation: only without centering
      if constexpr (CM == 0) return (const void*)quant_rows_kernel<0, MODE, 0>;
      return nullptr;
    case 4: return (const void*)quant_rows_kernel<4, MODE, CM>;
    case 5: return (const void*)quant_rows_kernel<5, MODE, CM>;
    case 6: return (const void*)quant_rows_kernel<6, MODE, CM>;
    case 7: return (const void*)quant_rows_kernel<7, MODE, CM>;
    case 8: return (const void*)quant_rows_kernel<8, MODE, CM>;
    case 9: return (const void*)quant_rows_kernel<9, MODE, CM>;
    case 10: return (const void*)quant_rows_kernel<10, MODE, CM>;
    default: return nullptr;
  }
}

template <int MODE>
static const void* pick_by_center(int logn, int center) {
  switch (center) {
    case 0: return pick_by_logn<MODE, 0>(logn);
    case 1: return pick_by_logn<MODE, 1>(logn);
    case 2: return pick_by_logn<MODE, 2>(logn);
    default: return nullptr;
  }
}

const void* quant_kernel_ptr(int logn, int mode, int center) {
  switch (mode) {
    case 0: return pick_by_center<0>(logn, center);
    case 1: return pick_by_center<1>(logn, center);
    case 2: return pick_by_center<2>(logn, center);
    case 3: return pick_by_center<3>(logn, center);
    default: return nullptr;
  }
}

int quant_max_threads() { return kQuantThreads; }

// ------------------------------------------------- calibration reductions
// out[k] = max(out[k], max_r |M[r,k]|) for a bf16 matrix M[rows, K]; out holds
// non-negative floats, so their bit patterns order like unsigned integers.
__global__ void __launch_bounds__(256) col_absmax_kernel(const uint16_t* __restrict__ M,
                                                         int64_t rows, int K,
                                                         float* __restrict__ out,
                                                         int rows_per_block) {
  const int groups = K / 8;
  const int g = blockIdx.x * 32 + threadIdx.x;
  const int64_t r_begin = int64_t(blockIdx.y) * rows_per_block;
  int64_t r_end = r_begin + rows_per_block;
  if (r_end > rows) r_end = rows;
  float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (g < groups) {
    for (int64_t r = r_begin + threadIdx.y; r < r_end; r += blockDim.y) {
      const uint4 w = *reinterpret_cast<const uint4*>(M + r * K + g * 8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        m[2 * u] = fmaxf(m[2 * u], fabsf(bf16lo(ws[u])));
        m[2 * u + 1] = fmaxf(m[2 * u + 1], fabsf(bf16hi(ws[u])));
      }
    }
  }
  __shared__ float red[8][32][9];
#pragma unroll
  for (int u = 0; u < 8; ++u) red[threadIdx.y][threadIdx.x][u] = m[u];
  __syncthreads();
  if (threadIdx.y == 0 && g < groups) {
    for (int y = 1; y < blockDim.y; ++y)
#pragma unroll
      for (int u = 0; u < 8; ++u) m[u] = fmaxf(m[u], red[y][threadIdx.x][u]);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      atomicMax(reinterpret_cast<unsigned*>(out + g * 8 + u), __float_as_uint(m[u]));
  }
}

// sigma_inv[k] = amax_w[k]^(1-alpha) / amax_x[k]^alpha  (1 / sigma of HadaNorm
// Eq. (3)); on entry sigma_inv holds amax_w.  sigma = 1 when a maximum is 0.
__global__ void sigma_inv_kernel(const float* __restrict__ act_absmax, float* __restrict__ sigma_inv,
                                 int K, float alpha) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float aw = sigma_inv[k];
  const float ax = act_absmax[k];
  float r = 1.0f;
  if (ax > 0.0f && aw > 0.0f) {
    float num, den;
    if (alpha == 0.5f) {
      num = sqrtf(aw);
      den = sqrtf(ax);
    } else {
      num = powf(aw, 1.0f - alpha);
      den = powf(ax, alpha);
    }
    r = num / den;
  }
  sigma_inv[k] = r;
}

__global__ void fill_kernel(float* __restrict__ p, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ in, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = __uint_as_float(uint32_t(in[i]) << 16);
}

// ------------------------------------------- weight-only Hadamard weights
// Weight side of the weight-only Hadamard form (HaTQ Sec. IV-B, Eq. (15)-
// (17)): Wbar = H_out W diag(sigma), the rows of W rotated along the output
// channels in blocks of M = 2^LOGO (unnormalized fast Walsh-Hadamard
// transform over the M rows of a block, then times 1/sqrt(M)), quantized per
// row.  The codes depend only on Wbar / max|Wbar| = S / max|S| with S the
// unnormalized sums, so they are formed from S: offline (once per layer),
// in fp64, where sums of bf16 values are exact, so rne(S q / max|S|) with a
// correctly rounded division decides a value lying exactly on a rounding tie
// half to even (such ties are common: S is a sum of bf16 values).  Without a
// rotation along K the activations keep their outlier channels, which
// multiply any weight code flip into whole output columns.  One CTA per block of M rows; thread j takes columns j,
// j + blockDim, ...; pass 1 collects each row's max |Wbar| (shared-memory
// atomics on the bits of non-negative doubles), pass 2 recomputes the same
// values and writes the codes.
template <int LOGO>
__global__ void __launch_bounds__(256) wh_weights_kernel(const uint16_t* __restrict__ W,
                                                         const float* __restrict__ sigma_inv,
                                                         int K, int q, double inv_sqrt_m,
                                                         int8_t* __restrict__ codes,
                                                         float* __restrict__ w_scale) {
  constexpr int M = 1 << LOGO;
  __shared__ unsigned long long rmax[M];  // bits of each row's max |S| (non-negative)
  const int64_t r0 = int64_t(blockIdx.x) * M;
  for (int i = threadIdx.x; i < M; i += blockDim.x) rmax[i] = 0ull;
  __syncthreads();
  // column k of the block: sigma_k W[r0 + j, k] rotated over j, unnormalized (fp64)
  auto column = [&](int k, double (&v)[M]) {
    // sigma = 1 / sigma_inv in fp32, as the activation side divides by it
    const double sg = sigma_inv ? double(1.0f / sigma_inv[k]) : 1.0;
#pragma unroll
    for (int j = 0; j < M; ++j) v[j] = double(bf16lo(uint32_t(W[(r0 + j) * K + k]))) * sg;
#pragma unroll
    for (int h = 1; h < M; h <<= 1) {
#pragma unroll
      for (int i = 0; i < M; ++i) {
        if ((i & h) == 0) {
          const double a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
      }
    }
  };
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    double v[M];
    column(k, v);
#pragma unroll
    for (int j = 0; j < M; ++j)
      if (v[j] != 0.0) atomicMax(&rmax[j], (unsigned long long)__double_as_longlong(fabs(v[j])));
  }
  __syncthreads();
  const double qd = double(q);
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    double v[M];
    column(k, v);
#pragma unroll
    for (int j = 0; j < M; ++j) {
      const double a = __longlong_as_double((long long)rmax[j]);
      const int c = a > 0.0 ? __double2int_rn((v[j] * qd) / a) : 0;  // round half to even
      codes[(r0 + j) * K + k] = int8_t(max(-q, min(q, c)));
    }
  }
  for (int j = threadIdx.x; j < M; j += blockDim.x)
    w_scale[r0 + j] = float((__longlong_as_double((long long)rmax[j]) * inv_sqrt_m) / qd);
}

cudaError_t launch_wh_weights(const uint16_t* W, const float* sigma_inv, int K, int N, int m,
                              int q, int8_t* codes, float* w_scale, cudaStream_t st) {
  const double inv = 1.0 / std::sqrt(double(m));
  const dim3 grid(unsigned(N / m));
  const int threads = K < 256 ? ((K + 31) / 32) * 32 : 256;
  switch (m) {
    case 16:
      wh_weights_kernel<4><<<grid, threads, 0, st>>>(W, sigma_inv, K, q, inv, codes, w_scale);
      break;
    case 32:
      wh_weights_kernel<5><<<grid, threads, 0, st>>>(W, sigma_inv, K, q, inv, codes, w_scale);
      break;
    case 64:
      wh_weights_kernel<6><<<grid, threads, 0, st>>>(W, sigma_inv, K, q, inv, codes, w_scale);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_col_absmax(const uint16_t* M, int64_t rows, int K, float* out, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int groups = K / 8;
  const int rows_per_block = 512;
  dim3 block(32, 8);
  const int64_t gy = (rows + rows_per_block - 1) / rows_per_block;
  if (gy > 65535) {
    // fold very tall matrices into several launches
    for (int64_t r0 = 0; r0 < rows; r0 += int64_t(65535) * rows_per_block) {
      const int64_t rr = (rows - r0) < int64_t(65535) * rows_per_block ? (rows - r0)
                                                                       : int64_t(65535) * rows_per_block;
      cudaError_t e = launch_col_absmax(M + r0 * K, rr, K, out, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  dim3 grid((groups + 31) / 32, unsigned(gy));
  col_absmax_kernel<<<grid, block, 0, st>>>(M, rows, K, out, rows_per_block);
  return cudaGetLastError();
}

cudaError_t launch_sigma_inv(const float* act_absmax, float* sigma_inv, int K, float alpha,
                             cudaStream_t st) {
  sigma_inv_kernel<<<(K + 255) / 256, 256, 0, st>>>(act_absmax, sigma_inv, K, alpha);
  return cudaGetLastError();
}

cudaError_t launch_fill(float* p, int n, float v, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  fill_kernel<<<(n + 255) / 256, 256, 0, st>>>(p, n, v);
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f32(const uint16_t* in, float* out, int n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  bf16_to_f32_kernel<<<(n + 255) / 256, 256, 0, st>>>(in, out, n);
  return cudaGetLastError();
}

}  // namespace hq
