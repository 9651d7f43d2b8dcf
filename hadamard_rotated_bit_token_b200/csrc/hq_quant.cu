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
// multiply-add against 1.5 * 2^23, which rounds half to even.
//
// Row mean: sum_k Z_hat[b,k] = n * Y[b,0] for each block b (the columns of
// H~ sum to zero except the first), so mu_hat = (n / K) * sum_b Y[b, 0]; this
// identity (HaTQ Eq. (23) read column-wise) gives the exact mean of the
// rotated row without a second reduction over Z.
//
// Data path per CTA (persistent over row tiles of R rows):
//   TMA bulk copy of the contiguous tile (R*K bf16) into a ring of shared
//   memory stages -> each thread takes a 32-channel slice of one row ->
//   bf16 -> fp32, times the channel multiplier -> butterflies on the 5
//   in-register index bits -> butterflies on the remaining bits across the
//   n/32 threads of the block (warp shuffles) -> per-block max / min ->
//   barrier -> one warp per row reduces the blocks, computes mean and scale ->
//   barrier -> codes, packed 4 per word, 32 bytes per thread, coalesced.
#include "hq_device.cuh"
#include "hq_kernels.h"

namespace hq {

namespace {

constexpr int kMaxQuantThreads = 384;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

struct __align__(16) RowPart {
  float mx, mn, y0, pad;
};

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

}  // namespace

// MODE 0: per-row dynamic scale (activations per token, or weights per row)
// MODE 1: per-tensor pass 1: only the tensor-wide max |V| (into tensor_max)
// MODE 2: per-tensor pass 2: scale from tensor_max
// MODE 3: per-tensor static scale from static_scale[0] (real units)
template <int LOGN, int MODE, bool CENTER>
__global__ void __launch_bounds__(kMaxQuantThreads, 1) quant_rows_kernel(const QuantParams p) {
  constexpr int N = 1 << LOGN;
  constexpr int LREG = LOGN < 5 ? LOGN : 5;      // in-register butterfly bits
  constexpr int TT = N >= 32 ? N / 32 : 1;        // threads per Hadamard block
  constexpr int LOG_TT = LOGN > 5 ? LOGN - 5 : 0;
  constexpr int BPT = N >= 32 ? 1 : 32 / N;       // blocks per thread slice
  constexpr bool kClamp = (MODE >= 2);

  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int S = p.S;
  const int R = p.R;
  const int K = p.K;
  const int E = S / TT;                            // block partials per row
  const int active = R * S;
  const bool is_worker = tid < active;
  const int row_in_tile = is_worker ? tid / S : 0;
  const int slice = is_worker ? tid - row_in_tile * S : 0;
  const int team_idx = slice / TT;
  const int member = slice - team_idx * TT;

  // shared layout
  const uint32_t tile_bytes = p.tile_bytes;
  uint8_t* stages = smem;
  size_t off = size_t(p.nstage) * tile_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  off = (off + 8u * p.nstage + 15u) & ~size_t(15);
  RowPart* part = reinterpret_cast<RowPart*>(smem + off);      // 16-byte aligned
  off += sizeof(RowPart) * size_t(R) * E;
  float2* rowstat = reinterpret_cast<float2*>(smem + off);
  off += sizeof(float2) * size_t(R);
  int* flags = reinterpret_cast<int*>(smem + off);  // [0] abort, [1] cta max bits

  const int64_t T = p.T;
  const int64_t ntiles = (T + R - 1) / R;

  if (tid == 0) {
    for (int s = 0; s < p.nstage; ++s) mbar_init(&full[s], 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  auto issue = [&](int64_t tile, int s) {
    const int64_t r0 = tile * R;
    const int64_t rows = (T - r0) < R ? (T - r0) : R;
    const uint32_t bytes = uint32_t(rows) * uint32_t(K) * 2u;
    mbar_arrive_expect_tx(&full[s], bytes);
    bulk_load(stages + size_t(s) * tile_bytes, p.X + r0 * K, bytes, &full[s]);
  };

  const WaitCtl wc{p.err, p.wait_ns};
  const bool skip_first = (MODE == 0 || MODE == 2) && p.fault_skip_load;
  if (tid == 0) {
    int64_t t = blockIdx.x;
    for (int s = 0; s < p.nstage && t < ntiles; ++s, t += gridDim.x) {
      if (s == 0 && skip_first) continue;  // test hook: this stage never completes
      issue(t, s);
    }
  }

  // per-channel multipliers for this thread's 32 channels (fixed across tiles)
  float mult[32];
  const bool has_mult = p.mult != nullptr;
  if (has_mult) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      float4 m4 = *reinterpret_cast<const float4*>(p.mult + slice * 32 + i);
      if (p.invert_mult) {
        mult[i] = 1.0f / m4.x;
        mult[i + 1] = 1.0f / m4.y;
        mult[i + 2] = 1.0f / m4.z;
        mult[i + 3] = 1.0f / m4.w;
      } else {
        mult[i] = m4.x;
        mult[i + 1] = m4.y;
        mult[i + 2] = m4.z;
        mult[i + 3] = m4.w;
      }
    }
  }

  // tensor-wide reciprocal scale for the per-tensor quantize passes
  float r_tensor = 0.0f;
  if (MODE == 2) {
    const float a = __uint_as_float(*p.tensor_max);
    r_tensor = a > 0.0f ? float(p.q) / a : 0.0f;
    if (blockIdx.x == 0 && tid == 0 && p.scale) p.scale[0] = (a / float(p.q)) * p.inv_sqrt_n;
  } else if (MODE == 3) {
    const float s = p.static_scale[0];
    r_tensor = s > 0.0f ? 1.0f / (s * p.sqrt_n) : 0.0f;
  }

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int s = it % p.nstage;
    const uint32_t parity = (it / p.nstage) & 1;
    if (!mbar_wait(&full[s], parity, wc)) flags[0] = 1;

    const int64_t row = tile * R + row_in_tile;
    const bool valid = is_worker && row < T;

    float v[32];
    float y0 = 0.0f;
    if (is_worker) {
      const uint4* src = reinterpret_cast<const uint4*>(stages + size_t(s) * tile_bytes +
                                                        (size_t(row_in_tile) * K + slice * 32) * 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 w = src[c];
        v[8 * c + 0] = bf16lo(w.x);
        v[8 * c + 1] = bf16hi(w.x);
        v[8 * c + 2] = bf16lo(w.y);
        v[8 * c + 3] = bf16hi(w.y);
        v[8 * c + 4] = bf16lo(w.z);
        v[8 * c + 5] = bf16hi(w.z);
        v[8 * c + 6] = bf16lo(w.w);
        v[8 * c + 7] = bf16hi(w.w);
      }
      if (has_mult) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], mult[i]);
      }
      // first channel of each block, for the row mean / row sum
      if (member == 0) {
#pragma unroll
        for (int b = 0; b < BPT; ++b) y0 += v[b * (32 / BPT)];
      }
      // butterflies on the in-register index bits (natural Sylvester order)
#pragma unroll
      for (int h = 1; h < (1 << LREG); h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if ((i & h) == 0) {
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
          }
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.0f;
    }
    // butterflies across the n/32 threads of a block (element bit 5 + j is
    // lane bit j); all lanes of the warp take part
#pragma unroll
    for (int j = 0; j < LOG_TT; ++j) {
      const float sgn = ((lane >> j) & 1) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], 1 << j);
        v[i] = __fmaf_rn(v[i], sgn, o);
      }
    }
    // per-thread max / min, reduced over the block's threads
    float mx = max3(v[0], v[1], v[2]);
    float mn = min3(v[0], v[1], v[2]);
#pragma unroll
    for (int i = 3; i < 31; i += 2) {
      mx = max3(mx, v[i], v[i + 1]);
      mn = min3(mn, v[i], v[i + 1]);
    }
    mx = fmaxf(mx, v[31]);
    mn = fminf(mn, v[31]);
#pragma unroll
    for (int j = 0; j < LOG_TT; ++j) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1 << j));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1 << j));
    }
    if (is_worker && member == 0) {
      RowPart rp;
      rp.mx = mx;
      rp.mn = mn;
      rp.y0 = y0;
      rp.pad = 0.0f;
      part[row_in_tile * E + team_idx] = rp;
    }
    __syncthreads();  // partials complete; the stage has been consumed

    if (flags[0]) break;
    if (tid == 0) {
      const int64_t nt = tile + int64_t(p.nstage) * gridDim.x;
      if (nt < ntiles) issue(nt, s);
    }

    // one warp per row: reduce the block partials, derive mean and scale
    for (int rr = warp; rr < R; rr += nwarps) {
      float rmx = -INFINITY, rmn = INFINITY, rsum = 0.0f;
      for (int e = lane; e < E; e += 32) {
        const RowPart q = part[rr * E + e];
        rmx = fmaxf(rmx, q.mx);
        rmn = fminf(rmn, q.mn);
        rsum += q.y0;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        rmx = fmaxf(rmx, __shfl_xor_sync(0xffffffffu, rmx, o));
        rmn = fminf(rmn, __shfl_xor_sync(0xffffffffu, rmn, o));
        rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
      }
      const int64_t grow = tile * R + rr;
      if (lane == 0 && grow < T) {
        const float m_hat = CENTER ? (float(N) / float(K)) * rsum : 0.0f;
        const float a_hat = fmaxf(__fsub_rn(rmx, m_hat), __fsub_rn(m_hat, rmn));
        float r_rec;
        if (MODE == 0) {
          r_rec = a_hat > 0.0f ? float(p.q) / a_hat : 0.0f;
          p.scale[grow] = (a_hat / float(p.q)) * p.inv_sqrt_n;
        } else if (MODE == 1) {
          atomicMax(reinterpret_cast<unsigned*>(&flags[1]), __float_as_uint(a_hat));
          r_rec = 0.0f;
        } else {
          r_rec = r_tensor;
        }
        if (MODE != 1 && p.mean) p.mean[grow] = m_hat * p.inv_sqrt_n;
        if (p.rowsum) p.rowsum[grow] = rsum * p.sqrt_n;  // sqrt(n) * sum_b Y[b,0]
        rowstat[rr] = make_float2(m_hat, r_rec);
      }
    }
    __syncthreads();

    if (MODE != 1 && valid) {
      const float2 st = rowstat[row_in_tile];
      const float m_hat = st.x, rr = st.y;
      uint32_t words[8];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float d = __fsub_rn(v[4 * w + u], m_hat);
          const float t = __fmaf_rn(d, rr, kRoundMagic);
          int c = int(__float_as_uint(t) - kRoundMagicBits);
          if (kClamp) c = max(-p.q, min(p.q, c));
          b[u] = uint32_t(c);
        }
        words[w] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                               0x5410);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.codes + row * K + slice * 32);
      dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
      dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    }
  }

  if (flags[0]) {
    // abort: let any bulk copies this CTA issued land before the CTA exits
    if (tid == 0) {
      int it2 = it;
      for (int64_t t = int64_t(blockIdx.x) + int64_t(it) * gridDim.x; t < ntiles && it2 < it + p.nstage;
           t += gridDim.x, ++it2) {
        const int s = it2 % p.nstage;
        if (!(it2 == 0 && skip_first)) (void)mbar_wait(&full[s], (it2 / p.nstage) & 1, wc);
      }
    }
    __syncthreads();
    return;
  }
  if (MODE == 1 && tid == 0) atomicMax(p.tensor_max, unsigned(flags[1]));
}

// ---------------------------------------------------------------- dispatch
template <int MODE, bool CENTER>
static const void* pick_by_logn(int logn) {
  switch (logn) {
    case 4: return (const void*)quant_rows_kernel<4, MODE, CENTER>;
    case 5: return (const void*)quant_rows_kernel<5, MODE, CENTER>;
    case 6: return (const void*)quant_rows_kernel<6, MODE, CENTER>;
    case 7: return (const void*)quant_rows_kernel<7, MODE, CENTER>;
    case 8: return (const void*)quant_rows_kernel<8, MODE, CENTER>;
    case 9: return (const void*)quant_rows_kernel<9, MODE, CENTER>;
    case 10: return (const void*)quant_rows_kernel<10, MODE, CENTER>;
    default: return nullptr;
  }
}

const void* quant_kernel_ptr(int logn, int mode, bool center) {
  switch (mode) {
    case 0: return center ? pick_by_logn<0, true>(logn) : pick_by_logn<0, false>(logn);
    case 1: return center ? pick_by_logn<1, true>(logn) : pick_by_logn<1, false>(logn);
    case 2: return center ? pick_by_logn<2, true>(logn) : pick_by_logn<2, false>(logn);
    case 3: return center ? pick_by_logn<3, true>(logn) : pick_by_logn<3, false>(logn);
    default: return nullptr;
  }
}

int quant_max_threads() { return kMaxQuantThreads; }

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
