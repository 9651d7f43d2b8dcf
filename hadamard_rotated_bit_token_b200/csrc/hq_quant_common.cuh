// hq_quant_common.cuh -- device building blocks of the activation quantizers:
// one thread's 32-channel slice of a row through
//   bf16 -> fp32, times sigma^-1, block fast Walsh-Hadamard transform,
//   symmetric round-half-even codes, and the code stores,
// shared by the kernels that differ only in how rows are spread over threads
// and how a row's statistics are combined (hq_quant_act.cu).
//
// The transform is the unnormalized FWHT over blocks of n = 2^LOGN channels
// (H = diag(H~_n, ...), HaTQ supplement Eq. (34); "Data-free 4-bit
// quantization for diffusion transformers", "Hadamard rotation", step 7):
// additions and subtractions only (HaTQ Sec. IV-D), with 1/sqrt(n) folded
// into the reported scale and mean, which leaves the codes unchanged because
// they depend only on V / max|V|.  The codes follow HaTQ Sec. III-A Eq. (3):
// code = rne(V * q / max|V|), taken with one fused multiply-add against
// 1.5 * 2^23, which rounds half to even and leaves the code in the low byte.
//
// Index bits of an element inside its block: bits 0-4 are the element's
// place in the thread's slice (register bits); bits 5 .. LOGN-1 select the
// slice among the TT = n/32 slices of the block and equal the low bits of the
// thread's lane (a block's slices sit in TT consecutive, aligned lanes).
// The cross-thread bits go through warp shuffles for n <= 128 (at most two
// bits); for n >= 256 the first three through one shared-memory transpose
// among G = 2^LX lanes and the rest (n = 512, 1024) through shuffles.
#pragma once

#include <cstdint>

#include "hq_device.cuh"

#ifndef HQ_XPOSE_MIN_LOGN
#define HQ_XPOSE_MIN_LOGN 8
#endif

namespace hq {
namespace qc {

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

// Order-preserving map of floats onto unsigned integers (max / min of floats
// by integer warp reductions).
__device__ __forceinline__ uint32_t ord_f32(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }
__host__ __device__ inline int padded_blocks(int B) { return (B + 3) & ~3; }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Shape of the transform of one 32-channel slice for blocks of 2^LOGN.
template <int LOGN>
struct Fwht {
  static constexpr int N = 1 << LOGN;
  static constexpr int LREG = LOGN < 5 ? LOGN : 5;        // index bits inside the slice
  static constexpr int LOG_TT = LOGN > 5 ? LOGN - 5 : 0;  // index bits across lanes
  static constexpr int TT = 1 << LOG_TT;                  // slices (lanes) per block
  // transposed bits: from n = 2^HQ_XPOSE_MIN_LOGN on (shuffles below)
  static constexpr int LX = LOGN < HQ_XPOSE_MIN_LOGN ? 0 : (LOG_TT < 3 ? LOG_TT : 3);
  static constexpr int G = 1 << LX;       // lanes per transpose group
  static constexpr int GS = 32 / G;       // elements per register group
  static constexpr int GP = GS / 2;       // fp32 pairs per register group
  static constexpr int CH = GS / 4;       // 16-byte chunks per register group
  static constexpr bool XPOSE = LX > 0;
  static constexpr int NSHFL = LOG_TT - LX;
  static constexpr int BPT = N >= 32 ? 1 : 32 / N;  // blocks per slice (n < 32)
  static constexpr uint32_t XBUF_BYTES = XPOSE ? 4096u : 0u;  // transpose buffer per warp
};

// 32 bf16 values (four 16-byte chunks) -> 16 fp32 pairs in channel order.
__device__ __forceinline__ void unpack32(const uint4 (&x)[4], f2 (&w)[16]) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    w[4 * ch + 0] = pk(bf16lo(x[ch].x), bf16hi(x[ch].x));
    w[4 * ch + 1] = pk(bf16lo(x[ch].y), bf16hi(x[ch].y));
    w[4 * ch + 2] = pk(bf16lo(x[ch].z), bf16hi(x[ch].z));
    w[4 * ch + 3] = pk(bf16lo(x[ch].w), bf16hi(x[ch].w));
  }
}

// Times the channel multipliers of slice `slice` (chunk-major [8][S] float4).
__device__ __forceinline__ void scale32(f2 (&w)[16], const float4* msm, int S, int slice) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 m4 = msm[i * S + slice];
    w[2 * i] = mul2(w[2 * i], pk(m4.x, m4.y));
    w[2 * i + 1] = mul2(w[2 * i + 1], pk(m4.z, m4.w));
  }
}

// Unnormalized FWHT of every block the slice belongs to.  xb: this warp's
// transpose buffer (Fwht<LOGN>::XBUF_BYTES); every lane of the warp calls.
template <int LOGN>
__device__ __forceinline__ void fwht32(f2 (&w)[16], uint8_t* xb_warp, int lane) {
  using F = Fwht<LOGN>;
  // index bit 0 inside pairs
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = w[i].x, b = w[i].y;
    w[i] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  // bits 1 .. LREG-1 between pairs
#pragma unroll
  for (int bit = 1; bit < F::LREG; ++bit) {
    const int hh = 1 << (bit - 1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & hh) == 0) {
        const f2 u = w[i], v = w[i + hh];
        w[i] = add2(u, v);
        w[i + hh] = sub2(u, v);
      }
    }
  }
  if constexpr (F::XPOSE) {
    // swap index bits 5 .. 4+LX (lanes of a G-lane group) with bits
    // 5-LX .. 4 (register groups of GS elements); slots XOR-swizzled by lane,
    // chunks by group, so the 16-byte accesses do not conflict
    constexpr int G = F::G, GS = F::GS, GP = F::GP, CH = F::CH, LX = F::LX;
    const int tl = lane & (G - 1);
    const int sub = lane >> LX;
    uint8_t* xb = xb_warp + sub * (G * 128);
    const int csw = sub & (CH - 1);
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int ch = 0; ch < CH; ++ch) {
        const f2 a = w[g * GP + 2 * ch], b = w[g * GP + 2 * ch + 1];
        *reinterpret_cast<float4*>(xb + (tl * G + (g ^ tl)) * (GS * 4) + ((ch ^ csw) << 4)) =
            make_float4(a.x, a.y, b.x, b.y);
      }
    }
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int ch = 0; ch < CH; ++ch) {
        const float4 v = *reinterpret_cast<const float4*>(xb + (g * G + (tl ^ g)) * (GS * 4) +
                                                          ((ch ^ csw) << 4));
        w[g * GP + 2 * ch] = pk(v.x, v.y);
        w[g * GP + 2 * ch + 1] = pk(v.z, v.w);
      }
    }
    __syncwarp();
    // index bits 5 .. 4+LX are now the register-group bits
#pragma unroll
    for (int k = 0; k < LX; ++k) {
      const int hh = GP << k;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & hh) == 0) {
          const f2 u = w[i], v = w[i + hh];
          w[i] = add2(u, v);
          w[i + hh] = sub2(u, v);
        }
      }
    }
  }
  // remaining index bits (5+LX and up) across lanes
#pragma unroll
  for (int j = 0; j < F::NSHFL; ++j) {
    const int mask = 1 << (F::LX + j);
    const float sg = (lane & mask) ? -1.0f : 1.0f;
    const f2 sg2 = pk(sg, sg);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const f2 o = pk(__shfl_xor_sync(0xffffffffu, w[i].x, mask),
                      __shfl_xor_sync(0xffffffffu, w[i].y, mask));
      w[i] = fma2(w[i], sg2, o);
    }
  }
}

// Pins the slice's 32 values: an empty volatile asm that reads and writes
// them, so later volatile asm (the next slice's shared-memory loads) cannot
// be hoisted above the work that produced them.  Keeps one slice's
// transform in flight at a time, which bounds register use when a thread
// holds several slices.
__device__ __forceinline__ void pin32(f2 (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    asm volatile(""
                 : "+f"(w[i].x), "+f"(w[i].y), "+f"(w[i + 1].x), "+f"(w[i + 1].y),
                   "+f"(w[i + 2].x), "+f"(w[i + 2].y), "+f"(w[i + 3].x), "+f"(w[i + 3].y));
  }
}

// Register index of block b's first channel in a slice whose member index is
// 0 (n >= 32: one block, index 0; n < 32: BPT blocks of the slice).
template <int LOGN>
__device__ __forceinline__ constexpr int first_pair(int b) {
  return (b * Fwht<LOGN>::N) >> 1;
}

// max / min of the 32 values in four independent chains.
__device__ __forceinline__ void maxmin32(const f2 (&w)[16], float& mx, float& mn) {
  float mxa[4], mna[4];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    mxa[q4] = fmaxf(w[4 * q4].x, w[4 * q4].y);
    mna[q4] = fminf(w[4 * q4].x, w[4 * q4].y);
#pragma unroll
    for (int i = 4 * q4 + 1; i < 4 * q4 + 4; ++i) {
      mxa[q4] = max3(mxa[q4], w[i].x, w[i].y);
      mna[q4] = min3(mna[q4], w[i].x, w[i].y);
    }
  }
  mx = fmaxf(max3(mxa[0], mxa[1], mxa[2]), mxa[3]);
  mn = fminf(min3(mna[0], mna[1], mna[2]), mna[3]);
}

// Codes of (w - shift) * rr, one byte each, four per word in channel order
// of the registers; CLAMP: limited to [-q, q].
template <bool SHIFT, bool CLAMP>
__device__ __forceinline__ void quant32(const f2 (&w)[16], float shift, float rr, int q,
                                        uint32_t (&words)[8]) {
  const f2 sh2 = pk(shift, shift), rr2 = pk(rr, rr), mg2 = pk(kRoundMagic, kRoundMagic);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    uint32_t b[4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const f2 t = fma2(SHIFT ? sub2(w[2 * g + u], sh2) : w[2 * g + u], rr2, mg2);
      b[2 * u] = __float_as_uint(t.x);
      b[2 * u + 1] = __float_as_uint(t.y);
    }
    if (CLAMP) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int cv = int(b[u] - kRoundMagicBits);
        b[u] = uint32_t(max(-q, min(q, cv)));
      }
    }
    words[g] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                           0x5410);
  }
}

// Byte offset, inside the row's codes, of the first code this thread stores
// for its slice (packed: two codes per byte).
template <int LOGN>
__device__ __forceinline__ int code_offset(int slice, int lane, bool packed) {
  using F = Fwht<LOGN>;
  if constexpr (!F::XPOSE) {
    return packed ? slice * 16 : slice * 32;
  } else {
    // register group g: index bits 5..4+LX = g, bits 5-LX..4 = the lane in
    // its transpose group, bits 5+LX.. = the slice's remaining member bits
    const int blk = slice >> F::LOG_TT;
    const int member = slice & (F::TT - 1);
    const int e = blk * F::N + F::GS * (lane & (F::G - 1)) + (32 * F::G) * (member >> F::LX);
    return packed ? e / 2 : e;
  }
}

// Stores the slice's codes (words from quant32) at dst = row codes +
// code_offset(); packed: two codes per byte, element 2j in the low nibble.
template <int LOGN>
__device__ __forceinline__ void store32(const uint32_t (&words)[8], int8_t* dst, bool packed) {
  using F = Fwht<LOGN>;
  constexpr int G = F::G, GS = F::GS;
  constexpr int WPG = GS / 4;  // words per register group
  if (packed) {
    uint32_t t2[8];  // (c0 | c1 << 4) in byte 0 and (c2 | c3 << 4) in byte 2
#pragma unroll
    for (int g = 0; g < 8; ++g) t2[g] = (words[g] & 0x0F0F0F0Fu) | ((words[g] >> 4) & 0xF0F0F0F0u);
    if constexpr (!F::XPOSE) {
      *reinterpret_cast<uint4*>(dst) =
          make_uint4(__byte_perm(t2[0], t2[1], 0x6420), __byte_perm(t2[2], t2[3], 0x6420),
                     __byte_perm(t2[4], t2[5], 0x6420), __byte_perm(t2[6], t2[7], 0x6420));
    } else {
      // register group g: GS consecutive codes, GS / 2 bytes at 16 g
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (WPG == 4) {
          *reinterpret_cast<uint2*>(dst + 16 * g) =
              make_uint2(__byte_perm(t2[4 * g], t2[4 * g + 1], 0x6420),
                         __byte_perm(t2[4 * g + 2], t2[4 * g + 3], 0x6420));
        } else if (WPG == 2) {
          *reinterpret_cast<uint32_t*>(dst + 16 * g) = __byte_perm(t2[2 * g], t2[2 * g + 1], 0x6420);
        } else {
          *reinterpret_cast<uint16_t*>(dst + 16 * g) = uint16_t(__byte_perm(t2[g], 0u, 0x0020));
        }
      }
    }
    return;
  }
  if constexpr (!F::XPOSE) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    d4[0] = make_uint4(words[0], words[1], words[2], words[3]);
    d4[1] = make_uint4(words[4], words[5], words[6], words[7]);
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (WPG == 4) {
        *reinterpret_cast<uint4*>(dst + 32 * g) =
            make_uint4(words[4 * g], words[4 * g + 1], words[4 * g + 2], words[4 * g + 3]);
      } else if (WPG == 2) {
        *reinterpret_cast<uint2*>(dst + 32 * g) = make_uint2(words[2 * g], words[2 * g + 1]);
      } else {
        *reinterpret_cast<uint32_t*>(dst + 32 * g) = words[g];
      }
    }
  }
}

}  // namespace qc
}  // namespace hq
