// hq_api.cu -- host side of the C ABI declared in include/hq.h: argument
// checks, launch configuration, tensor-map encoding, and the device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/hq.h"
#include "../../include/hq_gw.h"
#include "hq_kernels.h"

namespace hq {

// The device error word (one per device that loads the library).
__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kVersion = 10400;  // 1.4.0: the group-wise form (include/hq_gw.h)
constexpr int kMaxHostChunks = 64;  // row chunks of hq_forward_host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  unsigned int* err = nullptr;
  bool quant_attr_set[11][4][3] = {};  // [log2 n][mode][centering]
  bool qact_attr_set[7][11][4][3] = {};  // [kernel][log2 n][mode][centering] attributes set
  int pair_clusters = -1;  // co-resident clusters of the CTA-pair GEMM (-1: not queried)
  // hq_forward_host's upload and download streams (created on first use)
  cudaStream_t up = nullptr, down = nullptr;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;
unsigned long long g_wait_ns = 0;  // 0 -> default
int g_fault = 0;
int g_gemm_variant = 0;  // HQ_GEMM_AUTO

unsigned long long wait_ns() { return g_wait_ns ? g_wait_ns : 2000000000ull; }

hq_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return HQ_ERR_CUDA;
    d.cc_major = prop.major;
    d.cc_minor = prop.minor;
    d.sm_count = prop.multiProcessorCount;
    if (prop.major != 10) return HQ_ERR_DEVICE;  // sm_100a code only
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return HQ_ERR_CUDA;
    d.err = static_cast<unsigned int*>(addr);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return HQ_ERR_DEVICE;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return HQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int ilog2_exact(int n) {
  if (n <= 0 || (n & (n - 1)) != 0) return -1;
  int l = 0;
  while ((1 << l) < n) ++l;
  return l;
}

// Shape rules shared by the quantizer entry points (K side only).
hq_status check_k_side(const hq_layer_desc* d) {
  const int logn = ilog2_exact(d->had_order);
  if (d->K <= 0 || d->had_order <= 0) return HQ_ERR_INVALID_ARGUMENT;
  if (logn != 0 && (logn < 4 || logn > 10)) return HQ_ERR_UNSUPPORTED;
  // K: whole blocks, whole 16-channel groups; at most 15360 with a rotation
  // (the segment kernel's 480 slices a row), 10240 without one (the row
  // kernel's 320 slices)
  if (d->K % d->had_order != 0 || d->K % 16 != 0) return HQ_ERR_UNSUPPORTED;
  if (d->K > (logn == 0 ? 10240 : 15360)) return HQ_ERR_UNSUPPORTED;
  if (d->code_format != HQ_CODES_I8 && d->code_format != HQ_CODES_I4_PACKED)
    return HQ_ERR_UNSUPPORTED;
  // two codes per byte hold 3- and 4-bit activation codes only, in rows of
  // whole 16-byte units
  if (d->code_format == HQ_CODES_I4_PACKED &&
      ((d->a_bits != 3 && d->a_bits != 4) || d->K % 32 != 0))
    return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

// Bytes per row of activation codes: K, or K / 2 when packed.
int64_t code_row_bytes(const hq_layer_desc* d) {
  return d->code_format == HQ_CODES_I4_PACKED ? d->K / 2 : d->K;
}

// The output side: out_order 0 or 1 is the double-Hadamard form; 16, 32 or
// 64 the weight-only Hadamard form, which leaves K unrotated and has no
// centering.
hq_status check_out_side(const hq_layer_desc* d) {
  if (d->out_order < 0) return HQ_ERR_INVALID_ARGUMENT;
  if (d->out_order <= 1) return HQ_OK;
  if (d->out_order != 16 && d->out_order != 32 && d->out_order != 64) return HQ_ERR_UNSUPPORTED;
  if (d->had_order != 1 || d->centering != HQ_CENTER_NONE) return HQ_ERR_UNSUPPORTED;
  if (d->N % d->out_order != 0) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

hq_status check_desc(const hq_layer_desc* d) {
  if (d == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  if (d->N <= 0) return HQ_ERR_INVALID_ARGUMENT;
  if (d->act_gran < HQ_PER_TOKEN || d->act_gran > HQ_PER_TENSOR_STATIC) return HQ_ERR_INVALID_ARGUMENT;
  if (d->centering < HQ_CENTER_NONE || d->centering > HQ_CENTER_TOKEN_MEAN_PRE)
    return HQ_ERR_INVALID_ARGUMENT;
  hq_status s = check_k_side(d);
  if (s != HQ_OK) return s;
  if (d->N % 16 != 0) return HQ_ERR_UNSUPPORTED;
  s = check_out_side(d);
  if (s != HQ_OK) return s;
  if (d->had_order == 1 && d->centering != HQ_CENTER_NONE) return HQ_ERR_UNSUPPORTED;
  if (d->a_bits != 3 && d->a_bits != 4 && d->a_bits != 8) return HQ_ERR_UNSUPPORTED;
  if (d->w_bits != 4 && d->w_bits != 8) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

// The last failure behind an HQ_ERR_CUDA (hq_debug_last_cuda_error): a
// runtime error code, or 100000 + a driver result code from tensor-map
// encoding.
int g_last_cuda_error = 0;

hq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return HQ_OK;
  g_last_cuda_error = int(e);
  return HQ_ERR_CUDA;
}

hq_status from_cu(CUresult r) {
  if (r == CUDA_SUCCESS) return HQ_OK;
  g_last_cuda_error = 100000 + int(r);
  return HQ_ERR_CUDA;
}

constexpr int kQuantCtasPerSm = 2;  // quantizer CTAs per SM (its launch bounds)
#ifndef HQ_GROUP_M
#define HQ_GROUP_M 8
#endif
constexpr int kGroupM = HQ_GROUP_M;  // M tiles per group of the GEMM's tile order

// Rows per tile R and threads per CTA (one thread per 32-channel slice of
// each row, whole warps).  The kernel is issue-bound, so an SM's time is
// about (tiles it runs) x (threads of its CTAs): the cost of R is the tile
// rounds of the persistent grid (`slots` CTAs at most, `per_sm` per SM) times
// the CTAs the busiest SM holds times the threads per CTA, idle lanes
// included.  Among the shapes within 3 % of the lowest cost the one with the
// most threads per CTA wins (more loads in flight).  Measured on B200: for
// K = 1152, T = 8192 this picks R = 7 (1171 tiles over 296 CTAs, a nearly
// full last round) over R = 8 (1024 tiles), 15.2 -> 14.4 us; for K = 3072,
// T = 16384 the 2 % cheaper R = 2 made the step slower than R = 3.
void quant_shape(int K, int64_t T, int sms, int per_sm, int* R_out, int* nt_out) {
  const int S = (K + 31) / 32;  // the last slice may hold 16 channels
  const int maxT = quant_max_threads();
  const int64_t slots = int64_t(sms) * per_sm;
  auto cost_of = [&](int R, int nt) {
    const int64_t tiles = (T + R - 1) / R;
    const int64_t grid = tiles < slots ? tiles : slots;
    const int64_t rounds = (tiles + grid - 1) / grid;
    const int64_t ctas_per_sm = (grid + sms - 1) / sms;
    return double(rounds) * double(ctas_per_sm) * nt;
  };
  double lowest = 1e300;
  for (int R = 1; R * S <= maxT; ++R) {
    const int nt = ((R * S + 31) / 32) * 32;
    const double c = cost_of(R, nt);
    if (c < lowest) lowest = c;
  }
  int bestR = 1, bestNT = 0;
  for (int R = 1; R * S <= maxT; ++R) {
    const int nt = ((R * S + 31) / 32) * 32;
    if (cost_of(R, nt) <= lowest * 1.03 && nt > bestNT) {
      bestR = R;
      bestNT = nt;
    }
  }
  if (bestNT == 0) bestNT = ((S + 31) / 32) * 32;  // S > maxT cannot occur (K <= 10240)
  *R_out = bestR;
  *nt_out = bestNT;
}

struct QuantLaunch {
  QuantParams p;
  int threads;
  size_t smem;
  int grid;
  int logn;
};

hq_status make_quant_launch(const DeviceState* dev, int K, int n, int64_t T, const uint16_t* X,
                            QuantLaunch* out) {
  QuantLaunch& L = *out;
  std::memset(&L.p, 0, sizeof(L.p));
  const int per_sm = kQuantCtasPerSm;
  int R, nt;
  quant_shape(K, T > 0 ? T : 1, dev->sm_count, per_sm, &R, &nt);
  const int logn = ilog2_exact(n);
  const bool xpose = logn >= 8;  // shared-memory transposes for n >= 256
  L.p.X = X;
  L.p.T = T;
  L.p.K = K;
  L.p.S = (K + 31) / 32;
  L.p.R = R;
  L.p.inv_sqrt_n = float(1.0 / std::sqrt(double(n)));
  L.p.sqrt_n = float(std::sqrt(double(n)));
  L.p.err = dev->err;
  L.p.wait_ns = wait_ns();
  L.threads = nt;
  L.logn = logn;
  L.smem = quant_smem_bytes(R, K, n == 1 ? 0 : K / n, nt / 32, xpose);
  const int64_t ntiles = (T + R - 1) / R;
  const int64_t slots = int64_t(dev->sm_count) * per_sm;
  L.grid = int(ntiles < slots ? ntiles : slots);
  return HQ_OK;
}

hq_status run_quant(DeviceState* dev, QuantLaunch& L, int mode, int center, cudaStream_t st) {
  const int logn = L.logn;
  const void* fn = quant_kernel_ptr(logn, mode, center);
  if (fn == nullptr) return HQ_ERR_UNSUPPORTED;
  if (L.p.T <= 0) return HQ_OK;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    bool& set = dev->quant_attr_set[logn][mode][center];
    if (!set) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024) !=
          cudaSuccess)
        return HQ_ERR_CUDA;
      set = true;
    }
  }
  void* args[] = {&L.p};
  return from_cuda(cudaLaunchKernel(fn, dim3(L.grid), dim3(L.threads), args, L.smem, st));
}

// ---------------------------------------------------------------------------
// The TMA-fed activation quantizers (had_order >= 16).

// CTAs of the warp-row kernel per SM, and the shared memory each may use
constexpr int kQActCtasPerSm = 2;
constexpr size_t kQActSmemPerCta = size_t(228 / kQActCtasPerSm - 1) * 1024;
size_t seg_smem_per_cta(bool big) { return size_t(228 / quant_seg_ctas_per_sm(big) - 1) * 1024; }

// Rows of the [T*S, 32] view per tensor copy for a stage of RS rows: the
// whole stage when it fits one box (at most 256 rows), else the largest
// multiple of 8 rows that divides RS (so every copy starts on a 512-byte
// boundary, where the 64-byte swizzle pattern starts over); 0 if none.
int qact_box_rows(int RS) {
  if (RS <= 256) return RS;
  for (int br = 256; br >= 8; br -= 8)
    if (RS % br == 0) return br;
  return 0;
}

// Warp segments the longest row of a segment-kernel tile spans.
int qact_max_seg(int R, int S) {
  int m = 1;
  for (int r = 0; r < R; ++r) {
    const int n = (r * S + S - 1) / 32 - (r * S) / 32 + 1;
    if (n > m) m = n;
  }
  return m;
}

// How hq_quantize_act runs for K channels, blocks of n and T tokens.
struct ActPlan {
  bool wrow;     // the warp-row kernel (else the segment kernel)
  bool big;      // segment kernel: the large-row variant
  int spl;       // warp-row: slices a lane (0: several rows per warp)
  int rpw;       // warp-row: rows per warp
  int rows;      // rows per tile
  int threads;   // per CTA (producer warp included)
  int stages;    // ring stages
  int max_seg;   // segment kernel: segments a row spans
  size_t smem;   // dynamic shared memory per CTA
};

// Ring stages that fit beside `fixed` bytes in `budget` (at most 6, at least
// 2; 0 if not).
int qact_stages(size_t fixed, int rows, int S, size_t budget = kQActSmemPerCta) {
  const size_t stage = (size_t(rows) * S * 64 + 1023) / 1024 * 1024;
  if (fixed + 2 * stage > budget) return 0;
  const size_t st = (budget - fixed) / stage;
  return int(st > 6 ? 6 : st);
}

// Warp-row kernel when every row fits a warp (K = 1024 spl, spl <= 4, or
// K < 1024); otherwise the segment kernel.  Its variants (two CTAs of up to
// 256 consumers an SM, or one of up to 480) and rows per tile are chosen by
// the fewest tile rounds first: the kernel is latency-bound, and a round is
// one tile's chain of copy, transform, row combine and store in every CTA.
// Among equal rounds, the issue-bound cost (tile rounds x CTAs on the busiest
// SM x threads per CTA; the most threads within 3 % of the lowest), and the
// two-CTA variant.  On the DiT fc2 shape (K = 4608: one row of 144 slices
// fills 144 of 256 consumers) three-row tiles of the one-CTA variant take
// 19 rounds instead of 28: 49.8 us against 56.5 us on B200.
bool qact_plan(int K, int n, int centering, int64_t T, int sms, ActPlan* out) {
  ActPlan& P = *out;
  if (K % 32 != 0 || n < 16) return false;  // whole 32-channel slices, a rotation
  const int S = K / 32;
  const bool pre = centering == HQ_CENTER_TOKEN_MEAN_PRE;
  if ((S % 32 == 0 && S / 32 <= 4) || S < 32) {
    P.wrow = true;
    P.big = false;
    P.spl = S < 32 ? 0 : S / 32;
    P.rpw = S < 32 ? 32 / S : 1;
    const int nw = quant_wrow_warps(P.spl);
    P.rows = nw * P.rpw;
    P.threads = 32 * (nw + 1);
    P.max_seg = 1;
    if (qact_box_rows(P.rows * S) == 0) return false;
    P.stages = qact_stages(quant_wrow_smem_bytes(P.rows, S, K, n, 0, nw, P.rpw), P.rows, S);
    if (P.stages < 2) return false;
    P.smem = quant_wrow_smem_bytes(P.rows, S, K, n, P.stages, nw, P.rpw);
    return true;
  }
  P.wrow = false;
  P.spl = 0;
  P.rpw = 0;
  struct Choice {
    int R = 0, nt = 0, stages = 0;
    int64_t rounds = 0;
  };
  // the best tile shape of one variant, or R = 0 if none fits
  auto best_of = [&](bool big) {
    const int maxC = quant_seg_max_consumers(big);
    const int64_t slots = int64_t(sms) * quant_seg_ctas_per_sm(big);
    auto stages_for = [&](int R) {
      if (qact_box_rows(R * S) == 0) return 0;
      return qact_stages(quant_seg_smem_bytes(R, S, K, n, 0, qact_max_seg(R, S), pre), R, S,
                         seg_smem_per_cta(big));
    };
    auto rounds_of = [&](int R) {
      const int64_t tiles = (T + R - 1) / R;
      const int64_t grid = tiles < slots ? tiles : slots;
      return (tiles + grid - 1) / grid;
    };
    auto cost_of = [&](int R, int nt) {
      const int64_t tiles = (T + R - 1) / R;
      const int64_t grid = tiles < slots ? tiles : slots;
      const int64_t ctas_per_sm = (grid + sms - 1) / sms;
      return double(rounds_of(R)) * double(ctas_per_sm) * nt;
    };
    int64_t fewest = INT64_MAX;
    for (int R = 1; R * S <= maxC; ++R)
      if (stages_for(R) >= 2 && rounds_of(R) < fewest) fewest = rounds_of(R);
    double lowest = 1e300;
    for (int R = 1; R * S <= maxC; ++R) {
      if (stages_for(R) < 2 || rounds_of(R) != fewest) continue;
      const double c = cost_of(R, ((R * S + 31) / 32) * 32);
      if (c < lowest) lowest = c;
    }
    Choice c;
    for (int R = 1; R * S <= maxC; ++R) {
      if (stages_for(R) < 2 || rounds_of(R) != fewest) continue;
      const int nt = ((R * S + 31) / 32) * 32;
      if (cost_of(R, nt) <= lowest * 1.03 && nt > c.nt) {
        c.R = R;
        c.nt = nt;
        c.stages = stages_for(R);
        c.rounds = fewest;
      }
    }
    return c;
  };
  Choice two;  // rows longer than 256 slices only fit the one-CTA variant
  if (S <= quant_seg_max_consumers(false)) two = best_of(false);
  const Choice one = best_of(true);
  P.big = two.R == 0 || (one.R != 0 && one.rounds < two.rounds);
  const Choice& ch = P.big ? one : two;
  if (ch.R == 0) return false;
  P.rows = ch.R;
  P.threads = ch.nt + 32;
  P.max_seg = qact_max_seg(ch.R, S);
  P.stages = ch.stages;
  P.smem = quant_seg_smem_bytes(ch.R, S, K, n, P.stages, P.max_seg, pre);
  return true;
}

// ---------------------------------------------------------------------------
// Tensor-map cache.  A tensor map is a pure function of its parameters (base
// address, extents, box, layout), so maps are kept in a small table keyed by
// them and reused by later calls on the same buffers and shapes, instead of
// being encoded on the host on every call.  Round-robin replacement; guarded
// by g_mutex.
struct TmapKey {
  int kind;  // which encoder
  const void* base;
  int64_t rows;
  int64_t cols;
  int box;
  bool operator==(const TmapKey& o) const {
    return kind == o.kind && base == o.base && rows == o.rows && cols == o.cols && box == o.box;
  }
};
constexpr int kTmapCacheSize = 64;
struct TmapCache {
  TmapKey key[kTmapCacheSize];
  CUtensorMap map[kTmapCacheSize];
  bool used[kTmapCacheSize] = {};
  int next = 0;
};
TmapCache g_tmaps;
unsigned long long g_tmap_hits = 0, g_tmap_misses = 0;

template <class Encode>
hq_status cached_tmap(const TmapKey& k, CUtensorMap* out, Encode encode) {
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int i = 0; i < kTmapCacheSize; ++i) {
      if (g_tmaps.used[i] && g_tmaps.key[i] == k) {
        *out = g_tmaps.map[i];
        ++g_tmap_hits;
        return HQ_OK;
      }
    }
  }
  hq_status s = encode(out);
  if (s != HQ_OK) return s;
  std::lock_guard<std::mutex> lock(g_mutex);
  const int i = g_tmaps.next;
  g_tmaps.next = (i + 1) % kTmapCacheSize;
  g_tmaps.key[i] = k;
  g_tmaps.map[i] = *out;
  g_tmaps.used[i] = true;
  ++g_tmap_misses;
  return HQ_OK;
}

hq_status encode_act_view_raw(CUtensorMap* m, const void* X, int64_t T, int K, int box_rows) {
  const int S = K / 32;
  cuuint64_t dims[2] = {32u, cuuint64_t(T) * cuuint64_t(S)};
  cuuint64_t strides[1] = {64u};
  cuuint32_t box[2] = {32u, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return from_cu(r);
}

struct QActLaunch {
  QuantParams p;
  CUtensorMap tmap;
  ActPlan plan;
  int grid;
  int logn;
};

hq_status make_quant_act_launch(const DeviceState* dev, const hq_layer_desc* d, int64_t T,
                                const uint16_t* X, QActLaunch* out, int centering) {
  QActLaunch& L = *out;
  std::memset(&L.p, 0, sizeof(L.p));
  const int K = d->K, n = d->had_order;
  if (!qact_plan(K, n, centering, T > 0 ? T : 1, dev->sm_count, &L.plan))
    return HQ_ERR_UNSUPPORTED;
  const ActPlan& P = L.plan;
  const int S = K / 32;
  if (T * int64_t(S) + int64_t(P.rows) * S >= (int64_t(1) << 31)) return HQ_ERR_UNSUPPORTED;
  L.logn = ilog2_exact(n);
  L.p.X = X;
  L.p.T = T;
  L.p.K = K;
  L.p.S = S;
  L.p.R = P.rows;
  L.p.rpw = P.rpw;
  L.p.inv_sqrt_n = float(1.0 / std::sqrt(double(n)));
  L.p.sqrt_n = float(std::sqrt(double(n)));
  L.p.err = dev->err;
  L.p.wait_ns = wait_ns();
  L.p.stages = P.stages;
  L.p.box_rows = qact_box_rows(P.rows * S);
  L.p.boxes = P.rows * S / L.p.box_rows;
  L.p.max_seg = P.max_seg;
  L.p.n_over_k = float(n) / float(K);
  L.p.inv_k = 1.0f / float(K);
  const int64_t ntiles = (T + P.rows - 1) / P.rows;
  const int64_t slots =
      int64_t(dev->sm_count) * (P.wrow ? kQActCtasPerSm : quant_seg_ctas_per_sm(P.big));
  L.grid = int(ntiles < slots ? ntiles : slots);
  const int box_rows = L.p.box_rows;
  return cached_tmap(TmapKey{4, X, T, K, box_rows}, &L.tmap, [&](CUtensorMap* o) {
    return encode_act_view_raw(o, X, T, K, box_rows);
  });
}

hq_status run_quant_act(DeviceState* dev, QActLaunch& L, int mode, int center, cudaStream_t st) {
  const int logn = L.logn;
  const ActPlan& P = L.plan;
  const void* fn = P.wrow ? quant_wrow_kernel_ptr(logn, mode, center, P.spl)
                          : quant_seg_kernel_ptr(logn, mode, center, P.big);
  if (fn == nullptr) return HQ_ERR_UNSUPPORTED;
  if (L.p.T <= 0) return HQ_OK;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    const int slot = P.wrow ? 1 + P.spl : (P.big ? 6 : 0);
    bool& set = dev->qact_attr_set[slot][logn][mode][center];
    if (!set) {
      // kQActCtasPerSm CTAs of up to kQActSmemPerCta each: the largest
      // shared-memory carveout
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(P.wrow ? kQActSmemPerCta : seg_smem_per_cta(P.big))) !=
              cudaSuccess ||
          cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
        return HQ_ERR_CUDA;
      set = true;
    }
  }
  void* args[] = {&L.tmap, &L.p};
  return from_cuda(cudaLaunchKernel(fn, dim3(L.grid), dim3(P.threads), args, P.smem, st));
}

// hq_quantize_act with a Hadamard rotation along K: the TMA-fed kernel.
hq_status quantize_act_tma(DeviceState* dev, const hq_layer_desc* desc, const uint16_t* X,
                           int64_t T, const float* sigma_inv, int8_t* a_codes, float* a_scale,
                           float* a_mean, void* workspace, cudaStream_t st) {
  QActLaunch L;
  hq_status s = make_quant_act_launch(dev, desc, T, X, &L, desc->centering);
  if (s != HQ_OK) return s;
  L.p.mult = sigma_inv;
  L.p.invert_mult = 0;
  L.p.codes = a_codes;
  L.p.scale = a_scale;
  L.p.mean = a_mean;
  L.p.q = (1 << (desc->a_bits - 1)) - 1;
  L.p.s_unit = L.p.inv_sqrt_n / float(L.p.q);
  L.p.packed = desc->code_format == HQ_CODES_I4_PACKED ? 1 : 0;
  L.p.fault_withhold_row = g_fault == HQ_FAULT_QUANT_WITHHOLD_ROW ? 1 : 0;
  const int center = desc->centering;
  if (desc->act_gran == HQ_PER_TOKEN) return run_quant_act(dev, L, 0, center, st);
  if (desc->act_gran == HQ_PER_TENSOR_STATIC) {
    L.p.static_scale = a_scale;
    L.p.scale = nullptr;
    return run_quant_act(dev, L, 3, center, st);
  }
  // dynamic per tensor: pass 1 finds max |V| over the tensor, pass 2 quantizes
  L.p.tensor_max = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(workspace, 0, 16, st) != cudaSuccess) return HQ_ERR_CUDA;
  QActLaunch L1 = L;
  L1.p.codes = nullptr;
  L1.p.mean = nullptr;
  L1.p.fault_withhold_row = 0;
  s = run_quant_act(dev, L1, 1, center, st);
  if (s != HQ_OK) return s;
  return run_quant_act(dev, L, 2, center, st);
}

hq_status encode_kmajor_i8_raw(CUtensorMap* m, const void* base, int64_t rows, int K,
                               int box_rows) {
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K)};
  cuuint32_t box[2] = {128u, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return from_cu(r);
}

// Packed activation codes [T, K/2] bytes: box {64 bytes (one K block of 128
// codes), 128 rows}, 64-byte swizzle (the GEMM's converters read one row per
// lane without bank conflicts and widen it themselves).
hq_status encode_packed_a_raw(CUtensorMap* m, const void* base, int64_t rows, int K) {
  cuuint64_t dims[2] = {cuuint64_t(K / 2), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K / 2)};
  cuuint32_t box[2] = {64u, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return from_cu(r);
}

hq_status encode_out_bf16_raw(CUtensorMap* m, const void* base, int64_t rows, int N) {
  cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(N) * 2u};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return from_cu(r);
}

hq_status encode_kmajor_i8(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
  return cached_tmap(TmapKey{1, base, rows, K, box_rows}, m, [&](CUtensorMap* o) {
    return encode_kmajor_i8_raw(o, base, rows, K, box_rows);
  });
}
hq_status encode_packed_a(CUtensorMap* m, const void* base, int64_t rows, int K) {
  return cached_tmap(TmapKey{2, base, rows, K, 0}, m,
                     [&](CUtensorMap* o) { return encode_packed_a_raw(o, base, rows, K); });
}
hq_status encode_out_bf16(CUtensorMap* m, const void* base, int64_t rows, int N) {
  return cached_tmap(TmapKey{3, base, rows, N, 0}, m,
                     [&](CUtensorMap* o) { return encode_out_bf16_raw(o, base, rows, N); });
}

// GEMM kernel choice.  Both kernels are persistent with one CTA per SM, so a
// launch takes about (tile rounds) x (time of one tile).  Measured on B200:
// one 128 x n x 32 i8 MMA takes about 126 + n/16 cycles for n <= 256 --
// nearly flat in n, so wide tiles win -- and the single-CTA main loop runs
// about 15% behind that rate (operand loads).  The epilogue's traffic through
// shared memory costs roughly 2000 cycles per 32-column chunk of each
// epilogue warp (fitted to tile-width sweeps of several layer shapes).  The CTA pair halves the B bytes per
// MMA but its 256 x 256 tiles carry twice the epilogue per CTA; it pays off
// only for long main loops over wide N.
struct GemmChoice {
  bool pair;
  int bn;  // single-CTA tile width
};

GemmChoice choose_gemm(int64_t T, int N, int K, int sms, int pair_clusters, int variant,
                       int logo, bool packed) {
  static const int cands[] = {256, 192, 128, 64};
  const int64_t mt = (T + 127) / 128;
  const int64_t kb = (K + 127) / 128;
  int best_bn = 128;
  double best_cost = 1e300;
  for (int bn : cands) {
    // 64-column output blocks of the weight-only form need 64 columns per epilogue warp
    if (logo == 6 && bn % 128 != 0) continue;
    // packed codes keep A's stages in tensor memory beside the accumulators
    if (packed && bn > 192) continue;
    const int64_t tiles = mt * ((N + bn - 1) / bn);
    const int64_t rounds = (tiles + sms - 1) / sms;
    const double tile = double(kb) * 4.0 * (126.0 + bn / 16.0) * 1.15 + 2000.0 * (bn / 64);
    const double cost = double(rounds) * tile;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_bn = bn;
    }
  }
  // the weight-only Hadamard epilogue and packed codes run in the
  // single-CTA kernel only
  if (variant == HQ_GEMM_SINGLE_CTA || pair_clusters <= 0 || logo > 0 || packed)
    return {false, best_bn};
  if (variant == HQ_GEMM_CTA_PAIR) return {true, 256};
  // automatic: the pair for long main loops (>= 20 K blocks) over N in whole
  // 256-column tiles, when it needs no more tile rounds than the best single
  const int64_t ptiles = ((T + 255) / 256) * ((N + 255) / 256);
  const int64_t prounds = (ptiles + pair_clusters - 1) / pair_clusters;
  const int64_t srounds = (mt * ((N + best_bn - 1) / best_bn) + sms - 1) / sms;
  const bool pair = kb >= 20 && N % 256 == 0 && prounds <= srounds;
  return {pair, best_bn};
}

// Argument checks of hq_quantize_act (description, pointers, alignment);
// T == 0 passes without looking at the pointers.
hq_status check_quant_args(const hq_layer_desc* desc, const uint16_t* X, int64_t T,
                           const float* sigma_inv, const int8_t* a_codes, const float* a_scale,
                           const float* a_mean, const void* workspace, size_t workspace_bytes) {
  hq_status s = check_desc(desc);
  if (s != HQ_OK) return s;
  if (T < 0) return HQ_ERR_INVALID_ARGUMENT;
  if (T == 0) return HQ_OK;  // nothing to read or write: pointers may be null
  if (X == nullptr || a_codes == nullptr || a_scale == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  const bool dyn = desc->act_gran == HQ_PER_TENSOR_DYNAMIC;
  if (dyn && (workspace == nullptr || workspace_bytes < 16)) return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(X) || !aligned16(a_codes) || !aligned4(a_scale) || (a_mean && !aligned4(a_mean)) ||
      (sigma_inv && !aligned16(sigma_inv)) || (dyn && !aligned16(workspace)))
    return HQ_ERR_MISALIGNED;
  return HQ_OK;
}

// Argument checks of hq_linear (shape, pointers, alignment); T == 0 passes
// without looking at the pointers.
hq_status check_linear_args(const hq_layer_desc* desc, int64_t T, const int8_t* a_codes,
                            const float* a_scale, const float* a_mean, const int8_t* w_codes,
                            const float* w_scale, const float* colsum, const float* bias_f32,
                            const uint16_t* Y, const int32_t* acc_debug) {
  if (desc == nullptr || T < 0) return HQ_ERR_INVALID_ARGUMENT;
  if (desc->K <= 0 || desc->N <= 0) return HQ_ERR_INVALID_ARGUMENT;
  if (desc->act_gran < HQ_PER_TOKEN || desc->act_gran > HQ_PER_TENSOR_STATIC)
    return HQ_ERR_INVALID_ARGUMENT;
  if (desc->K % 16 != 0 || desc->N % 16 != 0) return HQ_ERR_UNSUPPORTED;
  if (desc->a_bits < 2 || desc->a_bits > 8 || desc->w_bits < 2 || desc->w_bits > 8)
    return HQ_ERR_UNSUPPORTED;
  if (desc->code_format != HQ_CODES_I8 && desc->code_format != HQ_CODES_I4_PACKED)
    return HQ_ERR_UNSUPPORTED;
  // packed: codes of at most 4 bits, and rows of K / 2 bytes in whole 16-byte units
  if (desc->code_format == HQ_CODES_I4_PACKED && (desc->a_bits > 4 || desc->K % 32 != 0))
    return HQ_ERR_UNSUPPORTED;
  if (desc->out_order < 0) return HQ_ERR_INVALID_ARGUMENT;
  if (desc->out_order > 1) {
    if (desc->out_order != 16 && desc->out_order != 32 && desc->out_order != 64)
      return HQ_ERR_UNSUPPORTED;
    if (desc->N % desc->out_order != 0) return HQ_ERR_UNSUPPORTED;
    if (a_mean != nullptr) return HQ_ERR_INVALID_ARGUMENT;  // the form has no centering
  }
  if (T == 0) return HQ_OK;  // nothing to read or write: pointers may be null
  if (a_codes == nullptr || a_scale == nullptr || w_codes == nullptr || w_scale == nullptr ||
      Y == nullptr)
    return HQ_ERR_INVALID_ARGUMENT;
  if (a_mean != nullptr && colsum == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(a_codes) || !aligned16(w_codes) || !aligned16(Y) || !aligned16(w_scale) ||
      (colsum && !aligned16(colsum)) || (bias_f32 && !aligned16(bias_f32)) || !aligned4(a_scale) ||
      (a_mean && !aligned4(a_mean)) || (acc_debug && !aligned16(acc_debug)))
    return HQ_ERR_MISALIGNED;
  return HQ_OK;
}


// ---------------------------------------------------------------------------
// Group-wise form: tensor maps and shape rules.
hq_status check_gw_desc(const hq_gw_desc* d) {
  if (d == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  if (d->K <= 0 || d->N <= 0 || d->group <= 0 || d->rank < 0) return HQ_ERR_INVALID_ARGUMENT;
  if (d->group != 64 || d->K % 64 != 0 || d->K > 16384 || d->N % 16 != 0) return HQ_ERR_UNSUPPORTED;
  if (d->rank != 0 && d->rank != 32) return HQ_ERR_UNSUPPORTED;
  if (d->a_bits < 2 || d->a_bits > 4 || d->w_bits < 2 || d->w_bits > 4) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

int64_t gw_ld(int64_t cols) { return (cols + 3) / 4 * 4; }

// codes [rows, K] bytes, box {64, box_rows}, 64-byte swizzle
hq_status encode_gw_codes(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
  return cached_tmap(TmapKey{10, base, rows, K, box_rows}, m, [&](CUtensorMap* o) {
    cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(K)};
    cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(o, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return from_cu(r);
  });
}

// bf16 [rows, K], box {64, box_rows}, 128-byte swizzle (X tiles, l1 tiles)
hq_status encode_gw_bf16_k64(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
  return cached_tmap(TmapKey{11, base, rows, K, box_rows}, m, [&](CUtensorMap* o) {
    cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(K) * 2u};
    cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return from_cu(r);
  });
}

// fp32 [G][gw_ld(cols)] (cols valid per row), box {box, 1}, no swizzle
hq_status encode_gw_scales(CUtensorMap* m, const void* base, int G, int64_t cols, int box) {
  return cached_tmap(TmapKey{12, base, G, cols, box}, m, [&](CUtensorMap* o) {
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(G)};
    cuuint64_t strides[1] = {cuuint64_t(gw_ld(cols)) * 4u};
    cuuint32_t box2[2] = {cuuint32_t(box), 1u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims,
                          strides, box2, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return from_cu(r);
  });
}

// bf16 [rows, rank] (rank 32: 64-byte rows), box {rank, box_rows}, 64-byte swizzle
hq_status encode_gw_rank(CUtensorMap* m, const void* base, int64_t rows, int rank, int box_rows) {
  return cached_tmap(TmapKey{13, base, rows, rank, box_rows}, m, [&](CUtensorMap* o) {
    cuuint64_t dims[2] = {cuuint64_t(rank), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(rank) * 2u};
    cuuint32_t box[2] = {cuuint32_t(rank), cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return from_cu(r);
  });
}

hq_status gw_linear_impl(const hq_gw_desc* d, int64_t T, const uint8_t* a_codes,
                         const float* a_scale, const uint16_t* u, const uint8_t* w_codes,
                         const float* w_scale, const uint16_t* l2b, const float* bias_f32,
                         uint16_t* Y, float* Y32, hq_stream_t stream) {
  hq_status s = check_gw_desc(d);
  if (s != HQ_OK) return s;
  if (T < 0) return HQ_ERR_INVALID_ARGUMENT;
  if ((Y == nullptr && Y32 == nullptr) || a_codes == nullptr || a_scale == nullptr ||
      w_codes == nullptr || w_scale == nullptr || (d->rank > 0 && (u == nullptr || l2b == nullptr)))
    return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(a_codes) || !aligned16(a_scale) || !aligned16(w_codes) || !aligned16(w_scale) ||
      (bias_f32 && !aligned16(bias_f32)) || (Y && !aligned16(Y)) || (Y32 && !aligned16(Y32)) ||
      (d->rank > 0 && (!aligned16(u) || !aligned16(l2b))))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceState* dev;
  s = device_state(&dev);
  if (s != HQ_OK) return s;
  const int K = d->K, N = d->N, G = K / 64;
  CUtensorMap maps[7];
  if ((s = encode_gw_codes(&maps[0], a_codes, T, K, 128)) != HQ_OK) return s;
  const int bn = gw_gemm_bn();
  if ((s = encode_gw_codes(&maps[1], w_codes, N, K, bn)) != HQ_OK) return s;
  if ((s = encode_gw_scales(&maps[2], a_scale, G, T, 128)) != HQ_OK) return s;
  if ((s = encode_gw_scales(&maps[3], w_scale, G, N, bn)) != HQ_OK) return s;
  if (d->rank > 0) {
    if ((s = encode_gw_rank(&maps[4], u, T, d->rank, 128)) != HQ_OK) return s;
    if ((s = encode_gw_rank(&maps[5], l2b, N, d->rank, bn)) != HQ_OK) return s;
  } else {
    maps[4] = maps[0];  // not read without the branch
    maps[5] = maps[0];
  }
  if (Y) {
    if ((s = encode_out_bf16(&maps[6], Y, T, N)) != HQ_OK) return s;
  } else {
    maps[6] = maps[0];  // not written: the fp32 sums go to Y32
  }
  GwGemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.bias = bias_f32;
  p.out_f32 = Y32;
  p.T = T;
  p.N = N;
  p.K = K;
  p.G = G;
  p.rank = d->rank;
  if (gw_ld(T) >= (int64_t(1) << 31)) return HQ_ERR_UNSUPPORTED;
  p.num_m_tiles = int((T + 127) / 128);
  p.num_n_tiles = (N + bn - 1) / bn;
  p.group_m = 8;
  p.err = dev->err;
  p.wait_ns = wait_ns();
  const int64_t tiles = int64_t(p.num_m_tiles) * p.num_n_tiles;
  if (tiles >= (int64_t(1) << 31)) return HQ_ERR_UNSUPPORTED;
  const int grid = int(tiles < dev->sm_count ? tiles : dev->sm_count);
  return from_cuda(launch_gw_gemm(maps, p, grid, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace
}  // namespace hq

using namespace hq;

extern "C" {

const char* hq_status_string(hq_status s) {
  switch (s) {
    case HQ_OK: return "HQ_OK";
    case HQ_ERR_INVALID_ARGUMENT: return "HQ_ERR_INVALID_ARGUMENT";
    case HQ_ERR_UNSUPPORTED: return "HQ_ERR_UNSUPPORTED";
    case HQ_ERR_MISALIGNED: return "HQ_ERR_MISALIGNED";
    case HQ_ERR_CUDA: return "HQ_ERR_CUDA";
    case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT";
    case HQ_ERR_DEVICE: return "HQ_ERR_DEVICE";
    default: return "HQ_ERR_UNKNOWN";
  }
}

int hq_version(void) { return kVersion; }

hq_status hq_calib_act_absmax(const hq_layer_desc* desc, const uint16_t* X, int64_t T,
                              float* absmax, hq_stream_t stream) {
  if (desc == nullptr || T < 0 || desc->K <= 0) return HQ_ERR_INVALID_ARGUMENT;
  if (desc->K % 8 != 0) return HQ_ERR_UNSUPPORTED;
  if (T == 0) return HQ_OK;
  if (X == nullptr || absmax == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(X) || !aligned4(absmax)) return HQ_ERR_MISALIGNED;
  DeviceState* dev;
  hq_status s = device_state(&dev);
  if (s != HQ_OK) return s;
  return from_cuda(launch_col_absmax(X, T, desc->K, absmax, reinterpret_cast<cudaStream_t>(stream)));
}

hq_status hq_prepare_weights(const hq_layer_desc* desc, const uint16_t* W, const uint16_t* bias,
                             const float* act_absmax, float alpha, int8_t* w_codes, float* w_scale,
                             float* colsum, float* sigma_inv, float* bias_f32, hq_stream_t stream) {
  hq_status s = check_desc(desc);
  if (s != HQ_OK) return s;
  if (W == nullptr || w_codes == nullptr || w_scale == nullptr || colsum == nullptr ||
      sigma_inv == nullptr || bias_f32 == nullptr)
    return HQ_ERR_INVALID_ARGUMENT;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(W) || !aligned16(w_codes) || !aligned16(sigma_inv) || !aligned4(w_scale) ||
      !aligned4(colsum) || !aligned4(bias_f32) || (bias && !aligned4(bias)) ||
      (act_absmax && !aligned4(act_absmax)))
    return HQ_ERR_MISALIGNED;
  DeviceState* dev;
  s = device_state(&dev);
  if (s != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int K = desc->K, N = desc->N;
  // sigma^-1 (HadaNorm review Eq. (3)); sigma_inv first holds max_n |W[n,k]|
  if (act_absmax) {
    if (cudaMemsetAsync(sigma_inv, 0, sizeof(float) * size_t(K), st) != cudaSuccess)
      return HQ_ERR_CUDA;
    s = from_cuda(launch_col_absmax(W, N, K, sigma_inv, st));
    if (s != HQ_OK) return s;
    s = from_cuda(launch_sigma_inv(act_absmax, sigma_inv, K, alpha, st));
  } else {
    s = from_cuda(launch_fill(sigma_inv, K, 1.0f, st));
  }
  if (s != HQ_OK) return s;
  const int qw = (1 << (desc->w_bits - 1)) - 1;
  if (desc->out_order > 1) {
    // weight-only Hadamard form: Wbar = H_out W diag(sigma) quantized per row;
    // no centering, so no correction vector
    s = from_cuda(launch_wh_weights(W, act_absmax ? sigma_inv : nullptr, K, N, desc->out_order,
                                    qw, w_codes, w_scale, st));
    if (s == HQ_OK) s = from_cuda(launch_fill(colsum, N, 0.0f, st));
    if (s != HQ_OK) return s;
    if (bias) return from_cuda(launch_bf16_to_f32(bias, bias_f32, N, st));
    return from_cuda(launch_fill(bias_f32, N, 0.0f, st));
  }
  // W~ rows: multiply by sigma (= 1 / sigma_inv), rotate, quantize per row,
  // and record each row's sum (colsum of W~ in the pages' orientation); with
  // had_order 1 (no rotation, no centering) no sum is needed.  Rows of whole
  // 32-channel slices take the TMA-fed kernels, the others the row kernel.
  ActPlan wap;
  if (desc->had_order >= 16 && qact_plan(K, desc->had_order, HQ_CENTER_NONE, N, dev->sm_count, &wap)) {
    QActLaunch AL;
    s = make_quant_act_launch(dev, desc, N, W, &AL, HQ_CENTER_NONE);
    if (s != HQ_OK) return s;
    AL.p.mult = act_absmax ? sigma_inv : nullptr;
    AL.p.invert_mult = 1;
    AL.p.codes = w_codes;
    AL.p.scale = w_scale;
    AL.p.mean = nullptr;
    AL.p.rowsum = colsum;
    AL.p.rowsum_pre = desc->centering == HQ_CENTER_TOKEN_MEAN_PRE ? 1 : 0;
    AL.p.q = qw;
    AL.p.s_unit = AL.p.inv_sqrt_n / float(qw);
    s = run_quant_act(dev, AL, 0, HQ_CENTER_NONE, st);
    if (s != HQ_OK) return s;
    if (bias) return from_cuda(launch_bf16_to_f32(bias, bias_f32, N, st));
    return from_cuda(launch_fill(bias_f32, N, 0.0f, st));
  }
  QuantLaunch L;
  s = make_quant_launch(dev, K, desc->had_order, N, W, &L);
  if (s != HQ_OK) return s;
  L.p.X = W;
  L.p.mult = act_absmax ? sigma_inv : nullptr;
  L.p.invert_mult = 1;
  L.p.codes = w_codes;
  L.p.scale = w_scale;
  L.p.mean = nullptr;
  L.p.rowsum = desc->had_order > 1 ? colsum : nullptr;
  L.p.rowsum_pre = desc->centering == HQ_CENTER_TOKEN_MEAN_PRE ? 1 : 0;
  L.p.q = qw;
  s = run_quant(dev, L, 0, 0, st);
  if (s == HQ_OK && desc->had_order == 1) s = from_cuda(launch_fill(colsum, N, 0.0f, st));
  if (s != HQ_OK) return s;
  if (bias) return from_cuda(launch_bf16_to_f32(bias, bias_f32, N, st));
  return from_cuda(launch_fill(bias_f32, N, 0.0f, st));
}

size_t hq_quantize_act_workspace_bytes(const hq_layer_desc* desc, int64_t T) {
  (void)T;
  if (desc == nullptr) return 0;
  return desc->act_gran == HQ_PER_TENSOR_DYNAMIC ? 16 : 0;
}

hq_status hq_quantize_act(const hq_layer_desc* desc, const uint16_t* X, int64_t T,
                          const float* sigma_inv, int8_t* a_codes, float* a_scale, float* a_mean,
                          void* workspace, size_t workspace_bytes, hq_stream_t stream) {
  hq_status s = check_quant_args(desc, X, T, sigma_inv, a_codes, a_scale, a_mean, workspace,
                                 workspace_bytes);
  if (s != HQ_OK || T == 0) return s;
  DeviceState* dev;
  s = device_state(&dev);
  if (s != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // rotated activations: the TMA-fed kernels, whenever a tile of them fits
  // (every K up to 8192); otherwise, and without a rotation, the row kernel
  ActPlan ap;
  if (desc->had_order >= 16 &&
      qact_plan(desc->K, desc->had_order, desc->centering, T, dev->sm_count, &ap))
    return quantize_act_tma(dev, desc, X, T, sigma_inv, a_codes, a_scale, a_mean, workspace, st);
  QuantLaunch L;
  s = make_quant_launch(dev, desc->K, desc->had_order, T, X, &L);
  if (s != HQ_OK) return s;
  L.p.X = X;
  L.p.mult = sigma_inv;
  L.p.invert_mult = 0;
  L.p.codes = a_codes;
  L.p.scale = a_scale;
  L.p.mean = a_mean;
  L.p.rowsum = nullptr;
  L.p.q = (1 << (desc->a_bits - 1)) - 1;
  L.p.packed = desc->code_format == HQ_CODES_I4_PACKED ? 1 : 0;
  L.p.fault_withhold_row = g_fault == HQ_FAULT_QUANT_WITHHOLD_ROW ? 1 : 0;
  const int center = desc->centering;  // HQ_CENTER_* = the kernel's centering mode
  if (desc->act_gran == HQ_PER_TOKEN) return run_quant(dev, L, 0, center, st);
  if (desc->act_gran == HQ_PER_TENSOR_STATIC) {
    L.p.static_scale = a_scale;
    L.p.scale = nullptr;
    return run_quant(dev, L, 3, center, st);
  }
  // dynamic per tensor: pass 1 finds max |V| over the tensor, pass 2 quantizes
  L.p.tensor_max = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(workspace, 0, 16, st) != cudaSuccess) return HQ_ERR_CUDA;
  QuantLaunch L1 = L;
  L1.p.codes = nullptr;
  L1.p.mean = nullptr;
  L1.p.fault_withhold_row = 0;
  s = run_quant(dev, L1, 1, center, st);
  if (s != HQ_OK) return s;
  return run_quant(dev, L, 2, center, st);
}

hq_status hq_linear(const hq_layer_desc* desc, int64_t T, const int8_t* a_codes,
                    const float* a_scale, const float* a_mean, const int8_t* w_codes,
                    const float* w_scale, const float* colsum, const float* bias_f32, uint16_t* Y,
                    int32_t* acc_debug, hq_stream_t stream) {
  hq_status s = check_linear_args(desc, T, a_codes, a_scale, a_mean, w_codes, w_scale, colsum,
                                  bias_f32, Y, acc_debug);
  if (s != HQ_OK || T == 0) return s;
  DeviceState* dev;
  s = device_state(&dev);
  if (s != HQ_OK) return s;
  const int K = desc->K, N = desc->N;
  if (dev->pair_clusters < 0) {
    int c = 0;
    if (gemm_pair_max_clusters(&c) != cudaSuccess) {
      (void)cudaGetLastError();
      c = 0;
    }
    dev->pair_clusters = c;
  }
  int variant;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    variant = g_gemm_variant;
  }
  // weight-only Hadamard form: output blocks of m = out_order columns
  const int m = desc->out_order > 1 ? desc->out_order : 1;
  const int logo = ilog2_exact(m);
  const bool packed = desc->code_format == HQ_CODES_I4_PACKED;
  if (variant == HQ_GEMM_CTA_PAIR && dev->pair_clusters <= 0 && logo == 0) return HQ_ERR_UNSUPPORTED;
  const GemmChoice gc =
      choose_gemm(T, N, K, dev->sm_count, dev->pair_clusters, variant, logo, packed);
  const int bn = gc.pair ? 256 : gc.bn;
  CUtensorMap ta, tb, ty;
  s = packed ? encode_packed_a(&ta, a_codes, T, K) : encode_kmajor_i8(&ta, a_codes, T, K, 128);
  if (s != HQ_OK) return s;
  s = encode_kmajor_i8(&tb, w_codes, N, K, gc.pair ? 128 : bn);
  if (s != HQ_OK) return s;
  s = encode_out_bf16(&ty, Y, T, N);
  if (s != HQ_OK) return s;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.a_scale = a_scale;
  p.a_scale_per_row = desc->act_gran == HQ_PER_TOKEN ? 1 : 0;
  {
    // |acc| <= 2^(a_bits-1) * 2^(w_bits-1) * K for codes within their declared
    // widths, 16 times that for packed codes (widened to 16 * code)
    const double bound = std::ldexp(1.0, desc->a_bits - 1) * std::ldexp(1.0, desc->w_bits - 1) *
                         K * (packed ? 16.0 : 1.0);
    p.small_acc = bound < 4194304.0 ? 1 : 0;
  }
  p.acc_unit = packed ? 0.0625f : 1.0f;
  p.acc_shift = packed ? 4 : 0;
  p.a_mean = a_mean;
  p.w_scale = w_scale;
  p.colsum = colsum;
  p.bias = bias_f32;
  p.Y = Y;
  p.acc_debug = acc_debug;
  p.T = T;
  p.N = N;
  p.K = K;
  p.inv_sqrt_out = float(1.0 / std::sqrt(double(m)));
  p.err = dev->err;
  p.wait_ns = wait_ns();
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // tile order: groups of kGroupM M tiles (shared A and B tiles stay in L2)
  p.group_m = kGroupM;
  if (gc.pair) {
    p.num_m_tiles = int((T + 255) / 256);
    p.num_n_tiles = (N + 255) / 256;
    const int64_t tiles = int64_t(p.num_m_tiles) * p.num_n_tiles;
    const int clusters = int(tiles < dev->pair_clusters ? tiles : dev->pair_clusters);
    return from_cuda(launch_gemm_pair(&ta, &tb, &ty, p, clusters, st));
  }
  p.num_m_tiles = int((T + 127) / 128);
  p.num_n_tiles = (N + bn - 1) / bn;
  const int64_t tiles = int64_t(p.num_m_tiles) * p.num_n_tiles;
  const int grid = int(tiles < dev->sm_count ? tiles : dev->sm_count);
  return from_cuda(launch_gemm(bn, logo, packed, &ta, &tb, &ty, p, grid, st));
}

hq_status hq_forward_host(const hq_layer_desc* desc, const uint16_t* X_host, int64_t T,
                          uint16_t* X_dev, const float* sigma_inv, int8_t* a_codes,
                          float* a_scale, float* a_mean, void* workspace, size_t workspace_bytes,
                          const int8_t* w_codes, const float* w_scale, const float* colsum,
                          const float* bias_f32, uint16_t* Y_dev, uint16_t* Y_host, int chunks,
                          hq_stream_t stream) {
  hq_status s = check_quant_args(desc, X_dev, T, sigma_inv, a_codes, a_scale, a_mean, workspace,
                                 workspace_bytes);
  if (s != HQ_OK) return s;
  const float* mean_in = desc->centering != HQ_CENTER_NONE ? a_mean : nullptr;
  s = check_linear_args(desc, T, a_codes, a_scale, mean_in, w_codes, w_scale, colsum, bias_f32,
                        Y_dev, nullptr);
  if (s != HQ_OK) return s;
  if (chunks < 1 || chunks > kMaxHostChunks) return HQ_ERR_INVALID_ARGUMENT;
  if (T == 0) return HQ_OK;
  if (X_host == nullptr || Y_host == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  DeviceState* dev;
  s = device_state(&dev);
  if (s != HQ_OK) return s;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (dev->up == nullptr) {
      cudaStream_t up = nullptr, down = nullptr;
      if (cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess) return HQ_ERR_CUDA;
      if (cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) != cudaSuccess) {
        (void)cudaStreamDestroy(up);
        return HQ_ERR_CUDA;
      }
      dev->up = up;
      dev->down = down;
    }
  }
  const int K = desc->K, N = desc->N;
  const int64_t cb = code_row_bytes(desc);  // bytes per row of a_codes
  const bool per_row = desc->act_gran == HQ_PER_TOKEN;
  // a tensor-wide dynamic scale needs every row before any code: one chunk
  if (desc->act_gran == HQ_PER_TENSOR_DYNAMIC) chunks = 1;
  // chunk boundaries: multiples of 128 rows (the GEMM's tile), at most `chunks` of them
  int64_t step = ((T + chunks - 1) / chunks + 127) / 128 * 128;
  const int nc = int((T + step - 1) / step);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // this call's events, destroyed once their waits are enqueued (CUDA
  // releases them when the work completes)
  cudaEvent_t ev[2 * kMaxHostChunks + 2] = {};
  const int nev = 2 * nc + 2;
  auto release = [&]() {
    for (int e = 0; e < nev; ++e)
      if (ev[e]) (void)cudaEventDestroy(ev[e]);
  };
  for (int e = 0; e < nev; ++e) {
    if (cudaEventCreateWithFlags(&ev[e], cudaEventDisableTiming) != cudaSuccess) {
      release();
      return HQ_ERR_CUDA;
    }
  }
  cudaEvent_t ev_fork = ev[0], ev_join = ev[1], *ev_in = ev + 2, *ev_done = ev + 2 + nc;
  auto fail = [&](hq_status code) {
    // join what was started, so that nothing outlives the call's ordering on `stream`
    (void)cudaEventRecord(ev_join, dev->down);
    (void)cudaStreamWaitEvent(st, ev_join, 0);
    (void)cudaEventRecord(ev_join, dev->up);
    (void)cudaStreamWaitEvent(st, ev_join, 0);
    release();
    return code;
  };
  // fork: both copy streams start after the work already on `stream`
  if (cudaEventRecord(ev_fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(dev->up, ev_fork, 0) != cudaSuccess ||
      cudaStreamWaitEvent(dev->down, ev_fork, 0) != cudaSuccess)
    return fail(HQ_ERR_CUDA);
  // uploads of every chunk, back to back on the upload stream
  for (int c = 0; c < nc; ++c) {
    const int64_t lo = c * step, rows = (T - lo) < step ? (T - lo) : step;
    if (cudaMemcpyAsync(X_dev + lo * K, X_host + lo * K, size_t(rows) * K * 2,
                        cudaMemcpyHostToDevice, dev->up) != cudaSuccess ||
        cudaEventRecord(ev_in[c], dev->up) != cudaSuccess)
      return fail(HQ_ERR_CUDA);
  }
  // each chunk's layer on `stream` once its upload has landed, and its
  // download on the download stream once its output is ready
  for (int c = 0; c < nc; ++c) {
    const int64_t lo = c * step, rows = (T - lo) < step ? (T - lo) : step;
    if (cudaStreamWaitEvent(st, ev_in[c], 0) != cudaSuccess) return fail(HQ_ERR_CUDA);
    const bool whole = nc == 1;
    s = hq_quantize_act(desc, X_dev + lo * K, rows, sigma_inv, a_codes + lo * cb,
                        (per_row && !whole) ? a_scale + lo : a_scale,
                        a_mean ? a_mean + lo : nullptr, workspace, workspace_bytes, stream);
    if (s == HQ_OK)
      s = hq_linear(desc, rows, a_codes + lo * cb, (per_row && !whole) ? a_scale + lo : a_scale,
                    mean_in ? mean_in + lo : nullptr, w_codes, w_scale, colsum, bias_f32,
                    Y_dev + lo * N, nullptr, stream);
    if (s != HQ_OK) return fail(s);
    if (cudaEventRecord(ev_done[c], st) != cudaSuccess ||
        cudaStreamWaitEvent(dev->down, ev_done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(Y_host + lo * N, Y_dev + lo * N, size_t(rows) * N * 2,
                        cudaMemcpyDeviceToHost, dev->down) != cudaSuccess)
      return fail(HQ_ERR_CUDA);
  }
  // join: `stream` continues after the last download
  if (cudaEventRecord(ev_join, dev->down) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev_join, 0) != cudaSuccess)
    return fail(HQ_ERR_CUDA);
  release();
  return HQ_OK;
}

hq_status hq_check_device_error(hq_stream_t stream) {
  DeviceState* dev;
  hq_status s = device_state(&dev);
  if (s != HQ_OK) return s;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HQ_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpy(&word, dev->err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HQ_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpy(dev->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return HQ_ERR_CUDA;
    return static_cast<hq_status>(word);
  }
  return HQ_OK;
}

hq_status hq_debug_set_wait_limit(uint64_t nanoseconds) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_wait_ns = nanoseconds;
  return HQ_OK;
}

hq_status hq_debug_set_gemm_variant(int variant) {
  if (variant != HQ_GEMM_AUTO && variant != HQ_GEMM_SINGLE_CTA && variant != HQ_GEMM_CTA_PAIR)
    return HQ_ERR_INVALID_ARGUMENT;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_gemm_variant = variant;
  return HQ_OK;
}

hq_status hq_debug_plan(const hq_layer_desc* desc, int64_t T, int sms, int pair_clusters,
                        int32_t* quant_rows, int32_t* quant_threads, int32_t* gemm_pair,
                        int32_t* gemm_bn) {
  hq_status s = check_desc(desc);
  if (s != HQ_OK) return s;
  if (T < 1 || sms < 1 || pair_clusters < 0) return HQ_ERR_INVALID_ARGUMENT;
  int R, nt;
  ActPlan ap;
  if (desc->had_order >= 16 && qact_plan(desc->K, desc->had_order, desc->centering, T, sms, &ap)) {
    R = ap.rows;  // the TMA-fed kernels
    nt = ap.threads;
  } else {
    quant_shape(desc->K, T, sms, kQuantCtasPerSm, &R, &nt);
  }
  const int logo = ilog2_exact(desc->out_order > 1 ? desc->out_order : 1);
  const GemmChoice gc = choose_gemm(T, desc->N, desc->K, sms, pair_clusters, HQ_GEMM_AUTO, logo,
                                    desc->code_format == HQ_CODES_I4_PACKED);
  if (quant_rows) *quant_rows = R;
  if (quant_threads) *quant_threads = nt;
  if (gemm_pair) *gemm_pair = gc.pair ? 1 : 0;
  if (gemm_bn) *gemm_bn = gc.pair ? 256 : gc.bn;
  return HQ_OK;
}

hq_status hq_debug_mma_ceiling(int pair, int64_t k_blocks, int32_t* ctas, hq_stream_t stream) {
  if ((pair != 0 && pair != 1) || k_blocks < 1 || k_blocks > (int64_t(1) << 24) || ctas == nullptr)
    return HQ_ERR_INVALID_ARGUMENT;
  DeviceState* dev;
  hq_status s = device_state(&dev);
  if (s != HQ_OK) return s;
  int n = dev->sm_count;
  if (pair) {
    if (dev->pair_clusters < 0) {
      int c = 0;
      if (gemm_pair_max_clusters(&c) != cudaSuccess) {
        (void)cudaGetLastError();
        c = 0;
      }
      dev->pair_clusters = c;
    }
    if (dev->pair_clusters <= 0) return HQ_ERR_UNSUPPORTED;
    n = 2 * dev->pair_clusters;
  }
  *ctas = n;
  return from_cuda(launch_mma_ceiling(pair != 0, k_blocks, n, dev->err, wait_ns(),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

hq_status hq_debug_tmap_cache(uint64_t* hits, uint64_t* misses) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (hits) *hits = g_tmap_hits;
  if (misses) *misses = g_tmap_misses;
  return HQ_OK;
}

hq_status hq_debug_inject_fault(int kind) {
  if (kind != HQ_FAULT_NONE && kind != HQ_FAULT_QUANT_WITHHOLD_ROW) return HQ_ERR_INVALID_ARGUMENT;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_fault = kind;
  return HQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of hq_quantize_act.
//
// Some callers cannot allocate device memory at the point where they quantize:
// a runtime whose device memory is fixed when the model is loaded (embedded or
// safety-certified deployments), a host callback or plugin that has no
// allocator handle, or code running where an allocation would synchronize or
// is forbidden.  hq_quantize_act needs a small workspace for the per-tensor
// dynamic scale; this variant takes it from a fixed array that the library
// holds in device memory instead of from the caller.
//
// The array lives for as long as the library is loaded, on every device that
// loads it (kNoAllocScratchBytes per device).  Its device address is looked up
// once per device, on the first call made with that device current; make that
// first call before any stream capture.  All calls share the one array and it
// keeps the previous call's contents: the quantizer clears the bytes it uses
// at the start of every call, and two calls whose kernels overlap on the GPU
// (different streams without ordering between them) race on it.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[hq::kMaxDevices] = {};
}  // namespace

extern "C" hq_status hq_quantize_act_noalloc(const hq_layer_desc* desc, const uint16_t* X,
                                              int64_t T, const float* sigma_inv, int8_t* a_codes,
                                              float* a_scale, float* a_mean, hq_stream_t stream) {
  if (desc == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  const size_t need = hq_quantize_act_workspace_bytes(desc, T);
  if (need > kNoAllocScratchBytes) return HQ_ERR_UNSUPPORTED;  // beyond the fixed array
  void* ws = nullptr;
  if (need > 0 && T > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
    if (dev < 0 || dev >= hq::kMaxDevices) return HQ_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return HQ_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
    }
    ws = g_noalloc_ptr[dev];
  }
  return hq_quantize_act(desc, X, T, sigma_inv, a_codes, a_scale, a_mean, ws,
                         ws ? kNoAllocScratchBytes : 0, stream);
}

// ---------------------------------------------------------------------------
// Group-wise form (include/hq_gw.h).
using namespace hq;

extern "C" {

int64_t hq_gw_scale_ld(int64_t T) { return T < 0 ? 0 : gw_ld(T); }

int hq_debug_last_cuda_error(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  const int e = g_last_cuda_error;
  g_last_cuda_error = 0;
  return e;
}

hq_status hq_gw_sigma_inv(const hq_gw_desc* desc, const uint16_t* W, const float* act_absmax,
                          float alpha, float* sigma_inv, hq_stream_t stream) {
  hq_status s = check_gw_desc(desc);
  if (s != HQ_OK) return s;
  if (W == nullptr || sigma_inv == nullptr || !(alpha >= 0.0f && alpha <= 1.0f))
    return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(W) || !aligned16(sigma_inv) || (act_absmax && !aligned16(act_absmax)))
    return HQ_ERR_MISALIGNED;
  DeviceState* dev;
  if ((s = device_state(&dev)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (act_absmax == nullptr) return from_cuda(launch_fill(sigma_inv, desc->K, 1.0f, st));
  // sigma_inv first holds max_n |W[n,k]| (the column maxima accumulate into it)
  s = from_cuda(cudaMemsetAsync(sigma_inv, 0, sizeof(float) * size_t(desc->K), st));
  if (s != HQ_OK) return s;
  s = from_cuda(launch_col_absmax(W, desc->N, desc->K, sigma_inv, st));
  if (s != HQ_OK) return s;
  return from_cuda(launch_sigma_inv(act_absmax, sigma_inv, desc->K, alpha, st));
}

hq_status hq_gw_prepare_weights(const hq_gw_desc* desc, const uint16_t* W, const uint16_t* bias,
                                const float* sigma_inv, const float* L1, const float* L2,
                                uint8_t* w_codes, float* w_scale, uint16_t* l1s, uint16_t* l2b,
                                float* bias_f32, hq_stream_t stream) {
  hq_status s = check_gw_desc(desc);
  if (s != HQ_OK) return s;
  const int rank = desc->rank;
  if (W == nullptr || w_codes == nullptr || w_scale == nullptr || bias_f32 == nullptr ||
      (rank > 0 && (L1 == nullptr || L2 == nullptr || l1s == nullptr || l2b == nullptr)))
    return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(W) || !aligned16(w_codes) || !aligned16(w_scale) || !aligned16(bias_f32) ||
      (sigma_inv && !aligned16(sigma_inv)) || (bias && !aligned4(bias)) ||
      (rank > 0 && (!aligned16(L1) || !aligned16(L2) || !aligned16(l1s) || !aligned16(l2b))))
    return HQ_ERR_MISALIGNED;
  DeviceState* dev;
  if ((s = device_state(&dev)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rank > 0) {
    s = from_cuda(launch_gw_factors(L1, L2, sigma_inv, rank, desc->K, desc->N, l1s, l2b,
                                    dev->sm_count, st));
    if (s != HQ_OK) return s;
  }
  GwWeightParams p;
  p.W = W;
  p.bias = bias;
  p.sigma_inv = sigma_inv;
  p.l1s = rank > 0 ? l1s : nullptr;
  p.l2b = rank > 0 ? l2b : nullptr;
  p.w_codes = w_codes;
  p.w_scale = w_scale;
  p.bias_f32 = bias_f32;
  p.K = desc->K;
  p.N = desc->N;
  p.rank = rank;
  p.q = (1 << (desc->w_bits - 1)) - 1;
  return from_cuda(launch_gw_weights(p, st));
}

size_t hq_gw_quantize_act_workspace_bytes(const hq_gw_desc* desc, int64_t T) {
  if (check_gw_desc(desc) != HQ_OK || T <= 0 || desc->rank == 0) return 0;
  const int64_t blocks = (T + 127) / 128;
  // two fp32 parts of u per token, then one ticket per 128-token block
  return size_t(2 * T * desc->rank * 4 + (blocks * 4 + 15) / 16 * 16);
}

hq_status hq_gw_quantize_act(const hq_gw_desc* desc, const uint16_t* X, int64_t T,
                             const float* sigma_inv, const uint16_t* l1s, uint8_t* a_codes,
                             float* a_scale, uint16_t* u, void* workspace, size_t workspace_bytes,
                             hq_stream_t stream) {
  hq_status s = check_gw_desc(desc);
  if (s != HQ_OK) return s;
  const int rank = desc->rank;
  if (T < 0 || X == nullptr || a_codes == nullptr || a_scale == nullptr ||
      (rank > 0 && (l1s == nullptr || u == nullptr)))
    return HQ_ERR_INVALID_ARGUMENT;
  if (!aligned16(X) || !aligned16(a_codes) || !aligned16(a_scale) ||
      (sigma_inv && !aligned16(sigma_inv)) || (rank > 0 && (!aligned16(l1s) || !aligned16(u))) ||
      (workspace && !aligned16(workspace)))
    return HQ_ERR_MISALIGNED;
  if (T == 0) return HQ_OK;
  DeviceState* dev;
  if ((s = device_state(&dev)) != HQ_OK) return s;
  const int K = desc->K;
  CUtensorMap tx, tl;
  if ((s = encode_gw_bf16_k64(&tx, X, T, K, 128)) != HQ_OK) return s;
  if (rank > 0) {
    if ((s = encode_gw_bf16_k64(&tl, l1s, rank, K, rank)) != HQ_OK) return s;
  } else {
    tl = tx;  // not read without the branch
  }
  GwActParams p;
  std::memset(&p, 0, sizeof(p));
  p.sigma_inv = sigma_inv;
  p.codes = a_codes;
  p.scale = a_scale;
  p.u = rank > 0 ? u : nullptr;
  p.T = T;
  p.K = K;
  p.ld = int(gw_ld(T));
  p.rank = rank;
  p.q = (1 << (desc->a_bits - 1)) - 1;
  p.fault = g_fault == HQ_FAULT_QUANT_WITHHOLD_ROW ? 1 : 0;
  p.err = dev->err;
  p.wait_ns = wait_ns();
  if (gw_ld(T) >= (int64_t(1) << 31)) return HQ_ERR_UNSUPPORTED;
  // as many stages (up to 8) as fit beside sigma^-1
  int stages = 8;
  while (stages > 2 && gw_act_smem_bytes(K, rank, stages, sigma_inv != nullptr) > 227u * 1024u)
    --stages;
  p.stages = stages;
  const int64_t blocks = (T + 127) / 128;
  if (blocks >= (int64_t(1) << 30)) return HQ_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Blocks that fill less than half the GPU are split: two CTAs per block,
  // each taking half of the groups (the branch's parts of u go through the
  // workspace, so without one a block stays whole).
  p.split = 1;
  const size_t need = hq_gw_quantize_act_workspace_bytes(desc, T);
  if (2 * blocks <= dev->sm_count && K / 64 >= 2 &&
      (rank == 0 || (workspace != nullptr && workspace_bytes >= need))) {
    p.split = 2;
    if (rank > 0) {
      p.upart = static_cast<float*>(workspace);
      p.counters = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) +
                                                   size_t(2 * T * rank * 4));
      s = from_cuda(cudaMemsetAsync(p.counters, 0, size_t(blocks) * 4, st));
      if (s != HQ_OK) return s;
    }
  }
  return from_cuda(launch_gw_act(&tx, &tl, p, int(blocks * p.split), st));
}

hq_status hq_gw_linear(const hq_gw_desc* desc, int64_t T, const uint8_t* a_codes,
                       const float* a_scale, const uint16_t* u, const uint8_t* w_codes,
                       const float* w_scale, const uint16_t* l2b, const float* bias_f32,
                       uint16_t* Y, hq_stream_t stream) {
  if (Y == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  return gw_linear_impl(desc, T, a_codes, a_scale, u, w_codes, w_scale, l2b, bias_f32, Y, nullptr,
                        stream);
}

hq_status hq_gw_debug_linear_f32(const hq_gw_desc* desc, int64_t T, const uint8_t* a_codes,
                                 const float* a_scale, const uint16_t* u, const uint8_t* w_codes,
                                 const float* w_scale, const uint16_t* l2b, const float* bias_f32,
                                 float* Y32, hq_stream_t stream) {
  if (Y32 == nullptr) return HQ_ERR_INVALID_ARGUMENT;
  return gw_linear_impl(desc, T, a_codes, a_scale, u, w_codes, w_scale, l2b, bias_f32, nullptr,
                        Y32, stream);
}

}  // extern "C"
