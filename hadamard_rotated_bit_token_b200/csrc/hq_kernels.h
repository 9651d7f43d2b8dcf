// hq_kernels.h -- kernel parameter blocks and launch helpers shared between
// the kernels (.cu) and the host-side C ABI (hq_api.cu).  Internal header.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace hq {

struct QuantParams {
  const uint16_t* X;          // [T,K] bf16 rows to transform
  const float* mult;          // [K] channel multiplier (sigma^-1 or sigma), or null
  int invert_mult;            // 1: use 1/mult[k] as the multiplier
  int8_t* codes;              // [T,K] int8 codes, or [T,K/2] bytes when packed
  int packed;                 // 1: two codes per byte (element 2j in the low nibble)
  float* scale;               // [T] per-row scales, or [1] for per-tensor modes
  float* mean;                // [T] per-row mean of the rotated row (real units), or null
  float* rowsum;              // [T] per-row correction sum (see rowsum_pre), or null
  int rowsum_pre;             // rowsum = sum_k Y[t,k] (1) or the rotated row's sum (0)
  unsigned int* tensor_max;   // per-tensor: bits of max |V_hat| (unnormalized)
  const float* static_scale;  // per-tensor static scale (real units)
  int64_t T;
  int K;
  int S;                      // 32-channel slices per row (K / 32)
  int R;                      // rows per tile (one thread per slice of each row)
  int q;                      // 2^(bits-1) - 1
  float inv_sqrt_n;           // 1 / sqrt(n), fp32
  float sqrt_n;               // sqrt(n), fp32
  int fault_withhold_row;     // test hook: never release the first row of the first tile
  unsigned int* err;          // device error word
  unsigned long long wait_ns; // bounded-wait limit
  // TMA-fed activation kernels only (hq_quant_act.cu)
  int stages;                 // shared-memory ring stages of R rows each
  int box_rows;               // rows of the [T*K/32, 32] view per tensor copy (S or S/2)
  int boxes;                  // tensor copies per stage (R * S / box_rows)
  int max_seg;                // warp segments a row can span (slots per row)
  int rpw;                    // warp-row kernel with S < 32: rows per warp
  float n_over_k;             // n / K (the rotated row's mean from its blocks' first channels)
  float inv_k;                // 1 / K
  float s_unit;               // 1 / (q sqrt(n)): reported scale per unit of max |V_hat|
};

// Returns the kernel entry for log2(n) in [4,10] (or 0: n = 1, no rotation,
// centering 0 only), mode in [0,3], centering in [0,2] (the HQ_CENTER_*
// values), or NULL; the kernel
// takes (QuantParams p) and runs R * S active threads per CTA (rounded up to
// whole warps, at most quant_max_threads()).
const void* quant_kernel_ptr(int logn, int mode, int center);
int quant_max_threads();

// Dynamic shared memory of one quantizer CTA: R rows per tile, K channels,
// B blocks per row, `nwarps` warps, transposes for n >= 256.
size_t quant_smem_bytes(int R, int K, int B, int nwarps, bool xpose);

// The TMA-fed activation quantizers (hq_quant_act.cu): one producer warp
// streams tiles of rows into a ring of shared-memory stages through a tensor
// map over X viewed as [T*K/32, 32] bf16 (64-byte rows, 64-byte swizzle, box
// {32, box_rows}); each kernel takes (const CUtensorMap tmX, QuantParams p).
// log2(n) in [4, 10], mode in [0, 3], centering in [0, 2].
//   segment kernel: any K (a multiple of 32); R * S consumer threads, one per
//     32-channel slice of each of the tile's R rows, 32 more for the producer.
//   warp-row kernel: warps own whole rows; spl = K / 1024 in [1, 4] slices a
//     lane and one row per warp, or spl = 0 for S = K/32 < 32: p.rpw rows
//     of S lanes each per warp; quant_wrow_warps(spl) consumer warps.
//   big: the segment kernel for rows of more than 256 slices (up to 480
//     consumers, one CTA per SM).
// Both kernels also serve the weight side (p.invert_mult: multiply by
// 1 / p.mult; p.rowsum: the row's correction sum).
const void* quant_seg_kernel_ptr(int logn, int mode, int center, bool big);
const void* quant_wrow_kernel_ptr(int logn, int mode, int center, int spl);
int quant_seg_max_consumers(bool big);
int quant_seg_ctas_per_sm(bool big);
int quant_wrow_warps(int spl);
// Dynamic shared memory of one CTA (n = Hadamard order; rows per tile).
size_t quant_seg_smem_bytes(int R, int S, int K, int n, int stages, int max_seg, bool pre);
size_t quant_wrow_smem_bytes(int rows, int S, int K, int n, int stages, int ncw, int rpw);

struct GemmParams {
  const float* a_scale;   // [T] or [1]
  int a_scale_per_row;    // 1: a_scale[t]; 0: a_scale[0]
  int small_acc;          // 1: every |acc| < 2^22 (from the declared code widths and K)
  const float* a_mean;    // [T] or null
  const float* w_scale;   // [N]
  const float* colsum;    // [N] or null
  const float* bias;      // [N] or null
  uint16_t* Y;            // [T,N] bf16
  int32_t* acc_debug;     // [T,N] or null
  int64_t T;
  int N;
  int K;
  int num_m_tiles;
  int num_n_tiles;
  int group_m;                // M tiles per group of the tile order (>= 1)
  float inv_sqrt_out;         // 1/sqrt(m) of the output-side transform (weight-only form)
  float acc_unit;             // accumulator units per code product: 1, or 1/16 when A is packed
  int acc_shift;              // acc_debug = raw accumulator >> acc_shift (0, or 4 when packed)
  unsigned int* err;          // device error word
  unsigned long long wait_ns; // bounded-wait limit
};

// Launches the tcgen05 GEMM for N tile width bn (64, 128, 192 or 256) and
// output-side transform log2(m) = logo (0: none; 4 or 5 with any bn; 6 with
// bn 128 or 256).  tmap_a / tmap_b / tmap_y point to host CUtensorMap
// objects (copied into the launch): A [T,K] and B [N,K] int8 with box
// {128, 128 | bn} and 128-byte swizzle; Y [T,N] bf16 with box {32, 32} and
// 64-byte swizzle.  packed_a: A holds two 4-bit codes per byte, [T,K/2]
// bytes with box {64, 128} and 64-byte swizzle; the kernel widens each tile
// to int8 (16 * code) in tensor memory, so the caller passes acc_unit =
// 1/16 and acc_shift = 4; bn 64, 128 or 192 (128 with logo 6).
cudaError_t launch_gemm(int bn, int logo, bool packed_a, const void* tmap_a, const void* tmap_b,
                        const void* tmap_y, const GemmParams& p, int grid, cudaStream_t st);
size_t gemm_smem_bytes(int bn, bool packed_a);
int gemm_threads(bool packed_a);

// The CTA-pair GEMM: clusters of two CTAs, each cluster computing 256 x 256
// output tiles (GemmParams.num_m_tiles / num_n_tiles count pair tiles).
// tmap_a / tmap_b: box {128, 128} like launch_gemm; tmap_y as above.
// `clusters` must not exceed gemm_pair_max_clusters() (co-resident clusters
// of the current device), since the kernel is persistent.
cudaError_t launch_gemm_pair(const void* tmap_a, const void* tmap_b, const void* tmap_y,
                             const GemmParams& p, int clusters, cudaStream_t st);
cudaError_t gemm_pair_max_clusters(int* clusters);
size_t gemm_pair_smem_bytes();
int gemm_pair_stages();

// MMA-only loop (the int8 tensor-core ceiling): `ctas` CTAs (an even number
// of them in clusters of two when pair), each issuing k_blocks x 4 MMAs of
// 128 x 256 x 32 (pair: 256 x 256 x 32 per cluster, half per CTA).
cudaError_t launch_mma_ceiling(bool pair, int64_t k_blocks, int ctas, unsigned int* err,
                               unsigned long long wait_ns, cudaStream_t st);

cudaError_t launch_col_absmax(const uint16_t* M, int64_t rows, int K, float* out, cudaStream_t st);
cudaError_t launch_sigma_inv(const float* act_absmax, float* sigma_inv, int K, float alpha,
                             cudaStream_t st);
cudaError_t launch_fill(float* p, int n, float v, cudaStream_t st);
cudaError_t launch_bf16_to_f32(const uint16_t* in, float* out, int n, cudaStream_t st);
// Weight-only Hadamard form, weight side: codes [N,K] and w_scale [N] of
// Wbar = H_out W diag(sigma) (blocks of m in {16, 32, 64} rows; N % m == 0);
// sigma_inv NULL means sigma = 1.
cudaError_t launch_wh_weights(const uint16_t* W, const float* sigma_inv, int K, int N, int m,
                              int q, int8_t* codes, float* w_scale, cudaStream_t st);

// ---------------------------------------------------------------------------
// Group-wise form (64-channel groups, fp8 e4m3 bytes holding integer codes,
// rank-32 16-bit low-rank branch): hq_gw.cu.
struct GwWeightParams {
  const uint16_t* W;        // [N,K] bf16
  const uint16_t* bias;     // [N] bf16 or null
  const float* sigma_inv;   // [K] or null
  const uint16_t* l1s;      // [rank,K] bf16 (already rounded)
  const uint16_t* l2b;      // [N,rank] bf16
  uint8_t* w_codes;         // [N,K] e4m3
  float* w_scale;           // [K/64][N]
  float* bias_f32;          // [N]
  int K, N, rank, q;
};

struct GwActParams {
  const float* sigma_inv;   // [K] or null
  uint8_t* codes;           // [T,K] e4m3
  float* scale;             // [K/64][ld]
  uint16_t* u;              // [T,rank] bf16 (rank > 0)
  float* upart;             // [split][T][rank] fp32 partial u (split > 1, rank > 0)
  unsigned int* counters;   // [blocks] zeroed before the launch (split > 1, rank > 0)
  int64_t T;
  int K, ld, rank, q, stages;
  int split;                // CTAs per 128-token block (1 or 2), each taking a range of groups
  int fault;                // withhold the first tile's copy (timeout path)
  unsigned int* err;
  unsigned long long wait_ns;
};

struct GwGemmParams {
  const float* bias;        // [N] or null
  float* out_f32;           // [T,N] fp32 instead of the bf16 store, or null
  int64_t T;
  int N, K, G, rank;
  int num_m_tiles, num_n_tiles, group_m;
  unsigned int* err;
  unsigned long long wait_ns;
};

// l1s = bf16(L1 diag(sigma_inv)) [rank,K], l2b = bf16(L2) [N,rank].
cudaError_t launch_gw_factors(const float* L1, const float* L2, const float* sigma_inv, int rank,
                              int K, int N, uint16_t* l1s, uint16_t* l2b, int sms, cudaStream_t st);
// R = (W - l2 l1) sigma, R H_64 per group, codes and scales; one CTA per row.
cudaError_t launch_gw_weights(const GwWeightParams& p, cudaStream_t st);
// split CTAs per 128 tokens (grid = blocks * split).  tmap_x: X [T,K] bf16,
// box {64, 128}, 128-byte swizzle; tmap_l1: l1s [rank,K] bf16, box
// {64, rank}, 128-byte swizzle.
cudaError_t launch_gw_act(const void* tmap_x, const void* tmap_l1, const GwActParams& p, int grid,
                          cudaStream_t st);
size_t gw_act_smem_bytes(int K, int rank, int stages, bool sigma);
int gw_act_threads();
// tmaps: 7 CUtensorMap in order A codes [T,K] u8 box {64,128} and B codes
// [N,K] u8 box {64,bn} (64-byte swizzle); s_x [G][ld] f32 box {128,1}; s_w
// [G][N] f32 box {bn,1}; u [T,32] bf16 box {32,128} and l2 [N,32] bf16
// box {32,bn} (64-byte swizzle); Y [T,N] bf16 box {32,32} (64-byte swizzle);
// bn = gw_gemm_bn().
cudaError_t launch_gw_gemm(const void* tmaps, const GwGemmParams& p, int grid, cudaStream_t st);
size_t gw_gemm_smem_bytes();
int gw_gemm_threads();
int gw_gemm_bn();  // output tile width (the B, s_w and l2 boxes have this many rows)

}  // namespace hq
