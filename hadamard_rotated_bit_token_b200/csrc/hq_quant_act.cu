// hq_quant_act.cu -- the activation quantizer of the layer (HadaNorm review,
// "What carries the argument", Eq. (1)): per row t of X,
//   Y = X diag(sigma^-1);  Z = Y H (block FWHT, hq_quant_common.cuh);
//   centring after H:  m_t = mean_k Z[t,k], V = Z - m_t;
//   centring before H: m_t = mean_k Y[t,k], V = (Y - m_t) H (only each
//                      block's first rotated channel moves, by -n m_t);
//   s_t = max_k |V| / q (per token; or one scale per tensor), codes =
//   clamp(rne(V / s_t), +-q) (HaTQ Sec. III-A Eq. (3)).
// The mean after H comes from the blocks' first input channels: every column
// of H~ but the first sums to zero, so sum_k Z_hat[b,k] = n Y[b,0] and
// m_hat = (n / K) sum_b Y[b,0] (HaTQ Eq. (23) read column-wise), summed in
// block order.
//
// Both kernels are fed the same way: one producer warp streams tiles of rows
// into a ring of shared-memory stages with tensor copies, several tiles
// ahead of the consumer warps.  The copies see X as a [T * K/32, 32] bf16
// matrix of 64-byte rows (one row per 32-channel slice) with the 64-byte
// swizzle: slice q's 16-byte chunk c lands at chunk c ^ ((q >> 1) & 3), so
// the eight slices a quarter-warp reads hit eight different bank groups.
// They differ in how a row is spread over the consumers:
//   quant_wrow_kernel  a warp owns whole rows: SPL slices per lane when the
//                      row has 32 * SPL slices (K = 1024 * SPL), or several
//                      rows of S <= 32 slices each.  The row's statistics
//                      are warp reductions; no thread waits for another warp.
//   quant_seg_kernel   any K: consumer c owns slice c % S of row c / S of
//                      the tile, so rows span several warps ("segments").
//                      Each segment reduces its part of the row's max / min
//                      in the warp and its first lane writes them to the
//                      row's slot; one hardware named barrier per tile among
//                      the consumer warps, then every thread combines its
//                      row's slots in segment order.
#include <cuda.h>

#include <cmath>

#include "hq_kernels.h"
#include "hq_quant_common.cuh"

namespace hq {

using namespace qc;

namespace {

// ------------------------------------------------------------ shared parts
#ifndef HQ_SEG_CTAS
#define HQ_SEG_CTAS 2
#endif
#ifndef HQ_SEG_CONSUMERS
#define HQ_SEG_CONSUMERS 256
#endif
constexpr int kSegConsumers = HQ_SEG_CONSUMERS;  // segment kernel: 8 consumer warps, 2 CTAs per SM
constexpr int kSegThreads = kSegConsumers + 32;
// rows of more than 256 slices (K above 8192): up to 480 consumers, one CTA
// per SM
constexpr int kSegConsumersBig = 480;
constexpr int kSegThreadsBig = kSegConsumersBig + 32;
constexpr int kSegCtas = HQ_SEG_CTAS;

// Shared-memory layout (byte offsets from a 1024-aligned base): the ring of
// stages first, then the channel multipliers, the per-warp transpose
// buffers, the row statistics, the barriers and flags.
struct ActSmem {
  uint32_t stage_bytes, park, mult, xbuf, slots, y0, full, empty, stat, flags, total;
};

// rows: rows per tile; ncw: consumer warps; slot_f4: float4 slots (segment
// kernel); y0_floats: floats of mean terms; park_bytes: parked transformed
// slices (segment kernel); stat_bars: tile-statistics barriers.
__host__ __device__ inline ActSmem act_smem_layout(int rows, int S, int K, int stages, int ncw,
                                                   uint32_t xbuf_per_warp, int slot_f4,
                                                   int y0_floats, uint32_t park_bytes = 0,
                                                   int stat_bars = 0) {
  ActSmem L;
  L.stage_bytes = align_up(uint32_t(rows * S * 64), 1024u);
  uint32_t off = uint32_t(stages) * L.stage_bytes;
  L.park = off;  // 1024-aligned
  off += park_bytes;
  L.mult = off;  // chunk-major [8][S] float4
  off += 4u * K;
  L.xbuf = off;
  off += xbuf_per_warp * ncw;
  off = align_up(off, 16);
  L.slots = off;
  off += 16u * slot_f4;
  L.y0 = off;
  off += 4u * y0_floats;
  off = align_up(off, 8);
  L.full = off;
  off += 8u * stages;
  L.empty = off;
  off += 8u * stages;
  L.stat = off;
  off += 8u * stat_bars;
  L.flags = off;  // [1] CTA max (mode 1), [2 + tile parity] consumers stop
  off += 16;
  L.total = off + 1024;  // room to align the dynamic base
  return L;
}

// One CTA's set-up: barriers (full: one arrival + bytes; empty: one arrival
// per consumer warp), flags, the channel multipliers.
__device__ __forceinline__ void act_setup(const QuantParams& p, uint8_t* smem, const ActSmem& L,
                                          int ncw, const CUtensorMap* tmX) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flags);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(ncw));  // one arrive per consumer warp
    }
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    flags[3] = 0;
    fence_mbarrier_init();
    prefetch_tmap(tmX);
  }
  if (p.mult) {
    float4* msm = reinterpret_cast<float4*>(smem + L.mult);
    for (int i = tid; i < 8 * p.S; i += blockDim.x) {
      const int c = i / p.S, sl = i - c * p.S;
      float4 m4 = *reinterpret_cast<const float4*>(p.mult + sl * 32 + 4 * c);
      if (p.invert_mult) {  // the weight side multiplies by sigma = 1 / sigma_inv
        m4.x = 1.0f / m4.x;
        m4.y = 1.0f / m4.y;
        m4.z = 1.0f / m4.z;
        m4.w = 1.0f / m4.w;
      }
      msm[i] = m4;
    }
  }
}

// The producer (one thread): tile after tile of `rows` rows into the ring,
// each stage as p.boxes tensor copies of p.box_rows slice rows.  Before
// returning it waits until every copy it issued has landed.
__device__ __forceinline__ void act_produce(const QuantParams& p, uint8_t* smem, const ActSmem& L,
                                            const CUtensorMap* tmX, int rows, int64_t ntiles,
                                            const WaitCtl& wc) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);
  const int NS = p.stages;
  const uint32_t bytes = uint32_t(rows * p.S * 64);
  int used = 0, s = 0;  // ring positions used
  uint32_t ph = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    if (!mbar_wait(&empty[s], ph ^ 1u, wc)) break;
    // test hook: the first tile's copy is never issued, so the consumers'
    // bounded wait for it gives up
    if (!(p.fault_withhold_row && used == 0)) {
      mbar_arrive_expect_tx(&full[s], bytes);
      uint8_t* dst = smem + size_t(s) * L.stage_bytes;
      const int32_t y0 = int32_t(tile * rows * p.S);
      for (int b = 0; b < p.boxes; ++b)
        tma_load_2d(dst + size_t(b) * p.box_rows * 64, tmX, 0, y0 + b * p.box_rows, &full[s]);
    }
    ++used;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  for (int i = used > NS ? used - NS : 0; i < used; ++i)
    if (!(p.fault_withhold_row && i == 0))
      (void)mbar_wait(&full[i % NS], uint32_t(i / NS) & 1u, wc);
}

// The four 16-byte chunks of slice row q of a stage (64-byte swizzle).
__device__ __forceinline__ void load_slice(uint32_t stage_addr, int q, uint4 (&x)[4]) {
  const uint32_t a = stage_addr + uint32_t(q) * 64u;
  const int swz = (q >> 1) & 3;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) x[ch] = ld_shared_v4(a + uint32_t((ch ^ swz) << 4));
}

// The per-tensor scales of modes 2 (dynamic, second pass) and 3 (static):
// the reciprocal applied to the unnormalized values.
template <int MODE>
__device__ __forceinline__ float tensor_reciprocal(const QuantParams& p, bool writer) {
  if (MODE == 2) {
    const float a = __uint_as_float(*p.tensor_max);
    if (writer && p.scale) p.scale[0] = (a / float(p.q)) * p.inv_sqrt_n;
    return a > 0.0f ? __fdiv_rn(float(p.q), a) : 0.0f;
  }
  if (MODE == 3) {
    const float s0 = p.static_scale[0];
    return s0 > 0.0f ? __fdiv_rn(1.0f, s0 * p.sqrt_n) : 0.0f;
  }
  return 0.0f;
}

}  // namespace

// ------------------------------------------------------- warp-row kernel
// Consumer warps own whole rows.  SPL >= 1: one row per warp and tile, lane l
// holding slices l, l + 32, ..., l + 32 (SPL - 1) (K = 1024 SPL); SPL == 0:
// p.rpw rows of S <= 32 slices per warp and tile, lane l holding slice
// l % S of the warp's row l / S.  A tile is p.R rows (one per warp, or p.rpw
// per warp).  A warp that gives up on a wait stops by itself: no thread
// waits for another warp.
template <int SPL>
struct WRowCfg {
  static constexpr int NW = SPL <= 1 ? 8 : (SPL == 2 ? 6 : 4);  // consumer warps
  static constexpr int THREADS = 32 * (NW + 1);
  // registers a thread: two CTAs per SM, at most 16384 per SM sub-partition
  static constexpr int REGS = SPL <= 1 ? 96 : (SPL == 2 ? 128 : 168);
};

template <int LOGN, int MODE, int CM, int SPL>
__global__ void __maxnreg__(WRowCfg<SPL>::REGS)
    quant_wrow_kernel(const __grid_constant__ CUtensorMap tmX, const QuantParams p) {
  using F = Fwht<LOGN>;
  constexpr bool CENTER = (CM == 1);
  constexpr bool PRE = (CM == 2);
  constexpr int NSL = SPL == 0 ? 1 : SPL;  // slices per lane
  constexpr bool kClamp = (MODE >= 2);
  constexpr bool kQuantize = (MODE != 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.S, K = p.K, RT = p.R;
  const int RPW = SPL == 0 ? p.rpw : 1;
  const int ncw = int(blockDim.x >> 5) - 1;
  const int B = K >> LOGN;
  const int BP = padded_blocks(B);
  const int64_t T = p.T;
  const int64_t ntiles = (T + RT - 1) / RT;
  const ActSmem L = act_smem_layout(RT, S, K, p.stages, ncw, F::XBUF_BYTES, 0, ncw * RPW * BP);
  const float4* msm = reinterpret_cast<const float4*>(smem + L.mult);
  float* y0buf = reinterpret_cast<float*>(smem + L.y0);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flags);
  const WaitCtl wc{p.err, p.wait_ns};

  // which per-block terms the row needs: the mean after H and the weights'
  // rotated row sum take the blocks' first input channels, the mean before H
  // and the weights' pre-rotation sum the blocks' sums
  const bool y0_terms = CENTER || (p.rowsum != nullptr && !p.rowsum_pre);
  const bool sum_terms = PRE || (p.rowsum != nullptr && p.rowsum_pre);
  act_setup(p, smem, L, ncw, &tmX);
  for (int i = threadIdx.x; i < ncw * RPW * BP; i += blockDim.x) y0buf[i] = 0.0f;  // padding
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) act_produce(p, smem, L, &tmX, RT, ntiles, wc);
  } else {
    const int cw = warp - 1;
    // this lane's row of the warp and its (first) slice
    int r_in_w = 0, slice0 = lane;
    bool active = true;
    unsigned segmask = 0xFFFFFFFFu;
    if (SPL == 0) {
      r_in_w = lane / S;
      slice0 = lane - r_in_w * S;
      active = r_in_w < RPW;
      if (!active) {
        r_in_w = 0;
        slice0 = 0;
      }
      const int lo = r_in_w * S;
      segmask = !active ? 0u : (S >= 32 ? 0xFFFFFFFFu : (((1u << S) - 1u) << lo));
    }
    const int rloc = cw * RPW + r_in_w;  // row inside the tile
    float* y0row = y0buf + rloc * BP;
    uint8_t* xb = smem + L.xbuf + cw * F::XBUF_BYTES;
    const float r_tensor = tensor_reciprocal<MODE>(p, blockIdx.x == 0 && warp == 1 && lane == 0);
    const int cb = p.packed ? K / 2 : K;  // code bytes per row
    int s = 0;
    uint32_t ph = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      // one lane waits (32 lanes spinning on one barrier word serialize in
      // shared memory); the warp barrier orders the others behind its acquire
      bool got = true;
      if (lane == 0) got = mbar_wait_spin(&full[s], ph, wc);
      __syncwarp();
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      const uint32_t st_addr = smem_u32(smem) + uint32_t(s) * L.stage_bytes;
      f2 w[NSL][16];
      float mx = -INFINITY, mn = INFINITY, fmx = -INFINITY, fmn = INFINITY;
      float first[NSL][F::BPT];
      // one slice at a time: load, transform, statistics (pin32 keeps the
      // next slice's loads behind this slice's work)
#pragma unroll
      for (int j = 0; j < NSL; ++j) {
        const int slice = slice0 + 32 * j;
        const int member = slice & (F::TT - 1);
        const int blk = slice >> F::LOG_TT;
        {
          uint4 x[4] = {};
          if (active) load_slice(st_addr, rloc * S + slice, x);
          unpack32(x, w[j]);
        }
        if (p.mult) scale32(w[j], msm, S, slice);
        // the mean's (or the row sum's) terms, one per block: the blocks'
        // first input channels (their rotated row sums are n times these)
        if (y0_terms && active && member == 0) {
#pragma unroll
          for (int b = 0; b < F::BPT; ++b) y0row[blk * F::BPT + b] = w[j][first_pair<LOGN>(b)].x;
        }
        fwht32<LOGN>(w[j], xb, lane);
        // or the blocks' rotated first channels, the block sums; centring
        // before H moves only these channels, so they stay out of the max /
        // min here and enter them after the shift
        if (sum_terms && member == 0) {
#pragma unroll
          for (int b = 0; b < F::BPT; ++b) {
            first[j][b] = w[j][first_pair<LOGN>(b)].x;
            if (active) y0row[blk * F::BPT + b] = first[j][b];
            if (PRE) {
              fmx = fmaxf(fmx, first[j][b]);
              fmn = fminf(fmn, first[j][b]);
              w[j][first_pair<LOGN>(b)].x = w[j][0].y;  // channel 1 of block 0 stands in
            }
          }
        }
        float a, c;
        maxmin32(w[j], a, c);
        mx = fmaxf(mx, a);
        mn = fminf(mn, c);
        if (PRE && member == 0) {
#pragma unroll
          for (int b = 0; b < F::BPT; ++b) w[j][first_pair<LOGN>(b)].x = first[j][b];
        }
        if (NSL > 1) pin32(w[j]);
      }
      // every lane has the tile's slices in registers before the stage goes
      // back; the loads went through the generic proxy, so each thread's proxy
      // fence orders them before the producer's next tensor copy into the
      // stage; the mean's terms are in shared memory
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
      }
      float rmx = -INFINITY, rmn = INFINITY, rfx = -INFINITY, rfn = INFINITY, rsum = 0.0f;
      if (active) {
        rmx = unord_f32(__reduce_max_sync(segmask, ord_f32(mx)));
        rmn = unord_f32(__reduce_min_sync(segmask, ord_f32(mn)));
        if (PRE) {
          rfx = unord_f32(__reduce_max_sync(segmask, ord_f32(fmx)));
          rfn = unord_f32(__reduce_min_sync(segmask, ord_f32(fmn)));
        }
        if (y0_terms || sum_terms) {  // in block order: independent of the tiling
          const float4* y4 = reinterpret_cast<const float4*>(y0row);
          for (int b4 = 0; b4 < BP / 4; ++b4) {
            const float4 v = y4[b4];
            rsum = __fadd_rn(__fadd_rn(__fadd_rn(__fadd_rn(rsum, v.x), v.y), v.z), v.w);
          }
        }
      }
      __syncwarp();  // the sums are read before the next tile overwrites them
      const float mu = PRE ? rsum * p.inv_k : 0.0f;
      const float m_hat = CENTER ? p.n_over_k * rsum : (PRE ? float(F::N) * mu : 0.0f);
      if (PRE) {
        rmx = fmaxf(rmx, __fsub_rn(rfx, m_hat));
        rmn = fminf(rmn, __fsub_rn(rfn, m_hat));
      }
      const float a_hat = PRE ? fmaxf(rmx, -rmn)
                              : fmaxf(__fsub_rn(rmx, m_hat), __fsub_rn(m_hat, rmn));
      const int64_t row = tile * RT + rloc;
      const bool row_ok = active && row < T;
      if (row_ok && slice0 == 0) {
        if (MODE == 0) p.scale[row] = a_hat * p.s_unit;  // a_hat / (q sqrt(n))
        if (MODE == 1)
          atomicMax(reinterpret_cast<unsigned*>(const_cast<int*>(&flags[1])), __float_as_uint(a_hat));
        if (kQuantize && p.mean) p.mean[row] = PRE ? mu : m_hat * p.inv_sqrt_n;
        // weights: sum_k sigma_k W[n,k] (the blocks' sums) or sum_k W~[n,k] =
        // sqrt(n) sum_b Y[b,0]
        if (p.rowsum) p.rowsum[row] = p.rowsum_pre ? rsum : rsum * p.sqrt_n;
      }
      if (!kQuantize || !row_ok) continue;
      // q / a_hat to within 2 ulp: moves a code only when V q / a_hat lies
      // within a few ulp of a rounding boundary
      const float rr = MODE == 0 ? (a_hat > 0.0f ? __fdividef(float(p.q), a_hat) : 0.0f) : r_tensor;
      int8_t* crow = p.codes + row * cb;
#pragma unroll
      for (int j = 0; j < NSL; ++j) {
        const int slice = slice0 + 32 * j;
        if (PRE && (slice & (F::TT - 1)) == 0) {
#pragma unroll
          for (int b = 0; b < F::BPT; ++b)
            w[j][first_pair<LOGN>(b)].x = __fsub_rn(w[j][first_pair<LOGN>(b)].x, m_hat);
        }
        uint32_t words[8];
        quant32<CM == 1, kClamp>(w[j], m_hat, rr, p.q, words);
        store32<LOGN>(words, crow + code_offset<LOGN>(slice, lane, p.packed), p.packed != 0);
      }
    }
  }
  __syncthreads();
  if (MODE == 1 && threadIdx.x == 0) atomicMax(p.tensor_max, unsigned(flags[1]));
}

// ------------------------------------------------------------ segment kernel
// Any K: consumer c owns slice c % S of row c / S of every tile (p.R rows).
template <int LOGN, int MODE, int CM, bool BIG>
__global__ void __launch_bounds__(BIG ? kSegThreadsBig : kSegThreads, BIG ? 1 : kSegCtas)
    quant_seg_kernel(const __grid_constant__ CUtensorMap tmX, const QuantParams p) {
  using F = Fwht<LOGN>;
  constexpr bool CENTER = (CM == 1);
  constexpr bool PRE = (CM == 2);
  constexpr bool kClamp = (MODE >= 2);
  constexpr bool kQuantize = (MODE != 1);
  constexpr int SLOT_W = PRE ? 2 : 1;  // float4 slots per segment

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.S, R = p.R, K = p.K, MSEG = p.max_seg;
  const int RS = R * S;
  const int ncw = int(blockDim.x >> 5) - 1;
  const int B = K >> LOGN;
  const int BP = padded_blocks(B);
  const int64_t T = p.T;
  const int64_t ntiles = (T + R - 1) / R;
  const ActSmem L = act_smem_layout(R, S, K, p.stages, ncw, F::XBUF_BYTES, 2 * R * MSEG * SLOT_W,
                                    2 * R * BP);
  const float4* msm = reinterpret_cast<const float4*>(smem + L.mult);
  float4* slots = reinterpret_cast<float4*>(smem + L.slots);
  float* y0buf = reinterpret_cast<float*>(smem + L.y0);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flags);
  const WaitCtl wc{p.err, p.wait_ns};

  const bool y0_terms = CENTER || (p.rowsum != nullptr && !p.rowsum_pre);
  const bool sum_terms = PRE || (p.rowsum != nullptr && p.rowsum_pre);
  act_setup(p, smem, L, ncw, &tmX);
  // neutral statistics in every slot: the slots past a row's last segment
  // are never written and combine as no-ops; the mean terms' padding is zero
  for (int i = tid; i < 2 * R * MSEG * SLOT_W; i += blockDim.x)
    slots[i] = make_float4(-INFINITY, INFINITY, 0.0f, 0.0f);
  for (int i = tid; i < 2 * R * BP; i += blockDim.x) y0buf[i] = 0.0f;
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) act_produce(p, smem, L, &tmX, R, ntiles, wc);
  } else {
    const int c = tid - 32;  // consumer index = slice row of the stage
    const int cw = warp - 1;
    const bool active = c < RS;
    const int row0 = active ? c / S : 0;  // this thread's row of every tile
    const int slice = active ? c - row0 * S : 0;
    const int member = slice & (F::TT - 1);
    const int blk = slice >> F::LOG_TT;
    // this warp's segment of the row: lanes [seg_lo, seg_hi)
    const int wbase = cw * 32;
    const int seg_lo = max(row0 * S, wbase) - wbase;
    const int seg_hi = min(min(row0 * S + S, RS), wbase + 32) - wbase;
    const int seg_len = seg_hi - seg_lo;
    const unsigned segmask = !active ? 0u
                             : seg_len >= 32 ? 0xFFFFFFFFu : (((1u << seg_len) - 1u) << seg_lo);
    const bool seg_leader = active && lane == seg_lo;
    float4* my_slots = slots + size_t(row0) * MSEG * SLOT_W;  // tile parity 0
    const int my_seg = cw - (row0 * S) / 32;
    const int slot_stride = R * MSEG * SLOT_W;                 // to tile parity 1
    uint8_t* xb = smem + L.xbuf + cw * F::XBUF_BYTES;
    const float r_tensor = tensor_reciprocal<MODE>(p, blockIdx.x == 0 && c == 0);
    const int cb = p.packed ? K / 2 : K;
    const int code_off = code_offset<LOGN>(slice, lane, p.packed);

    int s = 0;
    uint32_t ph = 0;
    for (int64_t tile = blockIdx.x, it = 0; tile < ntiles; tile += gridDim.x, ++it) {
      const int pb = int(it & 1);
      // a wait that gives up is recorded and acted on by every consumer warp
      // together after the tile barrier below, so no warp is ever left
      // waiting there (the flag of a tile parity is read only after that
      // tile's barrier and written only before it)
      // one lane waits; the warp barrier orders the others behind its acquire
      if (lane == 0 && !mbar_wait_spin(&full[s], ph, wc)) flags[2 + pb] = 1;
      __syncwarp();
      uint4 x[4] = {};
      if (active) load_slice(smem_u32(smem) + uint32_t(s) * L.stage_bytes, c, x);
      f2 w[16];
      unpack32(x, w);
      // the loads went through the generic proxy: each thread's proxy fence
      // orders them before the producer's next tensor copy into the stage
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
      }
      if (p.mult) scale32(w, msm, S, slice);
      float* y0row = y0buf + (pb * R + row0) * BP + blk * F::BPT;
      if (y0_terms && active && member == 0) {
#pragma unroll
        for (int b = 0; b < F::BPT; ++b) y0row[b] = w[first_pair<LOGN>(b)].x;
      }
      fwht32<LOGN>(w, xb, lane);
      float first[F::BPT];
      float fmx = -INFINITY, fmn = INFINITY;
      if (sum_terms && member == 0) {
#pragma unroll
        for (int b = 0; b < F::BPT; ++b) {
          first[b] = w[first_pair<LOGN>(b)].x;
          if (active) y0row[b] = first[b];
          if (PRE) {
            fmx = fmaxf(fmx, first[b]);
            fmn = fminf(fmn, first[b]);
            w[first_pair<LOGN>(b)].x = w[0].y;  // channel 1 of block 0 stands in
          }
        }
      }
      float mx, mn;
      maxmin32(w, mx, mn);
      if (PRE && member == 0) {
#pragma unroll
        for (int b = 0; b < F::BPT; ++b) w[first_pair<LOGN>(b)].x = first[b];
      }
      __syncwarp();
      float4* sl = my_slots + pb * slot_stride;
      if (active) {
        const uint32_t umx = __reduce_max_sync(segmask, ord_f32(mx));
        const uint32_t umn = __reduce_min_sync(segmask, ord_f32(mn));
        uint32_t ufx = 0u, ufn = 0xFFFFFFFFu;
        if (PRE) {
          ufx = __reduce_max_sync(segmask, ord_f32(fmx));
          ufn = __reduce_min_sync(segmask, ord_f32(fmn));
        }
        if (seg_leader) {
          sl[my_seg * SLOT_W] = make_float4(unord_f32(umx), unord_f32(umn), 0.0f, 0.0f);
          if (PRE) sl[my_seg * SLOT_W + 1] = make_float4(unord_f32(ufx), unord_f32(ufn), 0.0f, 0.0f);
        }
      }
      // every segment of every row of the tile has published its partials
      __syncwarp();
      named_barrier_sync(1, ncw * 32);
      if (flags[2 + pb]) break;
      // the row's statistics from its segments' slots, in segment order
      float rmx = -INFINITY, rmn = INFINITY, rsum = 0.0f, rfx = -INFINITY, rfn = INFINITY;
      for (int k = 0; k < MSEG; ++k) {
        const float4 v = sl[k * SLOT_W];
        rmx = fmaxf(rmx, v.x);
        rmn = fminf(rmn, v.y);
        if (PRE) {
          const float4 f = sl[k * SLOT_W + 1];
          rfx = fmaxf(rfx, f.x);
          rfn = fminf(rfn, f.y);
        }
      }
      // the mean's terms in block order (independent of the tiling)
      if (y0_terms || sum_terms) {
        const float4* y4 = reinterpret_cast<const float4*>(y0buf + (pb * R + row0) * BP);
        for (int b4 = 0; b4 < BP / 4; ++b4) {
          const float4 v = y4[b4];
          rsum = __fadd_rn(__fadd_rn(__fadd_rn(__fadd_rn(rsum, v.x), v.y), v.z), v.w);
        }
      }
      const float mu = PRE ? rsum * p.inv_k : 0.0f;
      const float m_hat = CENTER ? p.n_over_k * rsum : (PRE ? float(F::N) * mu : 0.0f);
      if (PRE) {
        rmx = fmaxf(rmx, __fsub_rn(rfx, m_hat));
        rmn = fminf(rmn, __fsub_rn(rfn, m_hat));
      }
      const float a_hat = PRE ? fmaxf(rmx, -rmn)
                              : fmaxf(__fsub_rn(rmx, m_hat), __fsub_rn(m_hat, rmn));
      const int64_t row = tile * R + row0;
      const bool row_ok = active && row < T;
      if (row_ok && slice == 0) {
        if (MODE == 0) p.scale[row] = a_hat * p.s_unit;
        if (MODE == 1)
          atomicMax(reinterpret_cast<unsigned*>(const_cast<int*>(&flags[1])), __float_as_uint(a_hat));
        if (kQuantize && p.mean) p.mean[row] = PRE ? mu : m_hat * p.inv_sqrt_n;
        if (p.rowsum) p.rowsum[row] = p.rowsum_pre ? rsum : rsum * p.sqrt_n;
      }
      if (!kQuantize || !row_ok) continue;
      const float rr = MODE == 0 ? (a_hat > 0.0f ? __fdividef(float(p.q), a_hat) : 0.0f) : r_tensor;
      if (PRE && member == 0) {
#pragma unroll
        for (int b = 0; b < F::BPT; ++b)
          w[first_pair<LOGN>(b)].x = __fsub_rn(w[first_pair<LOGN>(b)].x, m_hat);
      }
      uint32_t words[8];
      quant32<CM == 1, kClamp>(w, m_hat, rr, p.q, words);
      store32<LOGN>(words, p.codes + row * cb + code_off, p.packed != 0);
    }
  }
  __syncthreads();
  if (MODE == 1 && tid == 0 && !flags[2] && !flags[3])
    atomicMax(p.tensor_max, unsigned(flags[1]));
}

// ---------------------------------------------------------------- dispatch
// The warp-row kernels for SPL 2, 3 and 4 are instantiated in their own
// translation units (hq_quant_act_spl{2,3,4}.cu include this file with
// HQ_ACT_PART set), so the instantiations compile in parallel.
#ifndef HQ_ACT_PART
#define HQ_ACT_PART 0
#endif

template <int MODE, int CM, int SPL>
static const void* wrow_by_logn(int logn) {
  switch (logn) {
    case 4: return (const void*)quant_wrow_kernel<4, MODE, CM, SPL>;
    case 5: return (const void*)quant_wrow_kernel<5, MODE, CM, SPL>;
    case 6: return (const void*)quant_wrow_kernel<6, MODE, CM, SPL>;
    case 7: return (const void*)quant_wrow_kernel<7, MODE, CM, SPL>;
    case 8: return (const void*)quant_wrow_kernel<8, MODE, CM, SPL>;
    case 9: return (const void*)quant_wrow_kernel<9, MODE, CM, SPL>;
    case 10: return (const void*)quant_wrow_kernel<10, MODE, CM, SPL>;
    default: return nullptr;
  }
}

template <int SPL>
static const void* wrow_ptr(int logn, int mode, int center) {
  switch (mode * 3 + center) {
    case 0: return wrow_by_logn<0, 0, SPL>(logn);
    case 1: return wrow_by_logn<0, 1, SPL>(logn);
    case 2: return wrow_by_logn<0, 2, SPL>(logn);
    case 3: return wrow_by_logn<1, 0, SPL>(logn);
    case 4: return wrow_by_logn<1, 1, SPL>(logn);
    case 5: return wrow_by_logn<1, 2, SPL>(logn);
    case 6: return wrow_by_logn<2, 0, SPL>(logn);
    case 7: return wrow_by_logn<2, 1, SPL>(logn);
    case 8: return wrow_by_logn<2, 2, SPL>(logn);
    case 9: return wrow_by_logn<3, 0, SPL>(logn);
    case 10: return wrow_by_logn<3, 1, SPL>(logn);
    case 11: return wrow_by_logn<3, 2, SPL>(logn);
    default: return nullptr;
  }
}

template <int MODE, int CM, bool BIG>
static const void* seg_by_logn(int logn) {
  switch (logn) {
    case 4: return (const void*)quant_seg_kernel<4, MODE, CM, BIG>;
    case 5: return (const void*)quant_seg_kernel<5, MODE, CM, BIG>;
    case 6: return (const void*)quant_seg_kernel<6, MODE, CM, BIG>;
    case 7: return (const void*)quant_seg_kernel<7, MODE, CM, BIG>;
    case 8: return (const void*)quant_seg_kernel<8, MODE, CM, BIG>;
    case 9: return (const void*)quant_seg_kernel<9, MODE, CM, BIG>;
    case 10: return (const void*)quant_seg_kernel<10, MODE, CM, BIG>;
    default: return nullptr;
  }
}

template <bool BIG>
static const void* seg_ptr(int logn, int mode, int center) {
  switch (mode * 3 + center) {
    case 0: return seg_by_logn<0, 0, BIG>(logn);
    case 1: return seg_by_logn<0, 1, BIG>(logn);
    case 2: return seg_by_logn<0, 2, BIG>(logn);
    case 3: return seg_by_logn<1, 0, BIG>(logn);
    case 4: return seg_by_logn<1, 1, BIG>(logn);
    case 5: return seg_by_logn<1, 2, BIG>(logn);
    case 6: return seg_by_logn<2, 0, BIG>(logn);
    case 7: return seg_by_logn<2, 1, BIG>(logn);
    case 8: return seg_by_logn<2, 2, BIG>(logn);
    case 9: return seg_by_logn<3, 0, BIG>(logn);
    case 10: return seg_by_logn<3, 1, BIG>(logn);
    case 11: return seg_by_logn<3, 2, BIG>(logn);
    default: return nullptr;
  }
}

#if HQ_ACT_PART == 5
const void* quant_seg_big_ptr(int logn, int mode, int center) { return seg_ptr<true>(logn, mode, center); }
#elif HQ_ACT_PART == 2
const void* quant_wrow_ptr_spl2(int logn, int mode, int center) { return wrow_ptr<2>(logn, mode, center); }
#elif HQ_ACT_PART == 3
const void* quant_wrow_ptr_spl3(int logn, int mode, int center) { return wrow_ptr<3>(logn, mode, center); }
#elif HQ_ACT_PART == 4
const void* quant_wrow_ptr_spl4(int logn, int mode, int center) { return wrow_ptr<4>(logn, mode, center); }
#else
const void* quant_wrow_ptr_spl2(int logn, int mode, int center);
const void* quant_wrow_ptr_spl3(int logn, int mode, int center);
const void* quant_wrow_ptr_spl4(int logn, int mode, int center);
const void* quant_seg_big_ptr(int logn, int mode, int center);

const void* quant_seg_kernel_ptr(int logn, int mode, int center, bool big) {
  return big ? quant_seg_big_ptr(logn, mode, center) : seg_ptr<false>(logn, mode, center);
}


const void* quant_wrow_kernel_ptr(int logn, int mode, int center, int spl) {
  switch (spl) {
    case 0: return wrow_ptr<0>(logn, mode, center);
    case 1: return wrow_ptr<1>(logn, mode, center);
    case 2: return quant_wrow_ptr_spl2(logn, mode, center);
    case 3: return quant_wrow_ptr_spl3(logn, mode, center);
    case 4: return quant_wrow_ptr_spl4(logn, mode, center);
    default: return nullptr;
  }
}

int quant_seg_max_consumers(bool big) { return big ? kSegConsumersBig : kSegConsumers; }

int quant_wrow_warps(int spl) {
  switch (spl) {
    case 0: return WRowCfg<0>::NW;
    case 1: return WRowCfg<1>::NW;
    case 2: return WRowCfg<2>::NW;
    case 3: return WRowCfg<3>::NW;
    case 4: return WRowCfg<4>::NW;
    default: return 0;
  }
}

int quant_seg_ctas_per_sm(bool big) { return big ? 1 : kSegCtas; }

size_t quant_seg_smem_bytes(int R, int S, int K, int n, int stages, int max_seg, bool pre) {
  const int ncw = (R * S + 31) / 32;
  const uint32_t xb = n >= (1 << HQ_XPOSE_MIN_LOGN) && n >= 64 ? 4096u : 0u;
  return act_smem_layout(R, S, K, stages, ncw, xb, 2 * R * max_seg * (pre ? 2 : 1),
                         2 * R * padded_blocks(K / n)).total;
}

size_t quant_wrow_smem_bytes(int rows, int S, int K, int n, int stages, int ncw, int rpw) {
  const uint32_t xb = n >= (1 << HQ_XPOSE_MIN_LOGN) && n >= 64 ? 4096u : 0u;
  return act_smem_layout(rows, S, K, stages, ncw, xb, 0, ncw * rpw * padded_blocks(K / n)).total;
}
#endif

}  // namespace hq
