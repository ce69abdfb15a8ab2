// Device building blocks for the Hadamard rotation + quantization kernels.
//
// The rotation of a block of b = 2^k elements by the Sylvester matrix
// ("Rotation Transform", AutoRound docs, section 1.5: H -> [[H, H], [H, -H]])
// factors over the k index bits: H_b = H_2 (x) ... (x) H_2.  Applying H_2 along
// one index bit is one butterfly stage (u, v) -> (u + v, u - v); the stages
// commute, so any bit can be processed whenever it is held inside one
// thread's registers.  All arithmetic is IEEE fp32 round-to-nearest-even.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace hadq {

// *_BLOCKED: MXFP4 / NVFP4 whose scales are written in the tiled layout that
// block-scaled tensor-core GEMMs read (blocked_scale_offset).
enum OutMode : int {
  OUT_F32 = 0, OUT_BF16 = 1, OUT_INT4 = 2, OUT_MXFP4 = 3, OUT_NVFP4 = 4, OUT_CODEBOOK = 5,
  OUT_MXFP4_BLOCKED = 6, OUT_NVFP4_BLOCKED = 7
};

// Random Hadamard signs ("Rotation Transform", section 1.5: H @ diag(+/-1) /
// sqrt(N), the signs persisted as int8).  AFTER: output column j of every
// block is multiplied by s_j (R = H diag(s)); BEFORE: input column j is
// (R = diag(s) H, the transpose and inverse).  s has one int8 per block
// column; a negative entry is -1.
enum SignSide : int { SIGNS_NONE = 0, SIGNS_BEFORE = 1, SIGNS_AFTER = 2 };

struct Signs {
  const int8_t* s;   // b entries, device memory, 16-byte aligned; unused for SIGNS_NONE
  int side;
};

// 1 if block column `col` is negated.
__device__ __forceinline__ uint32_t neg_bit(const int8_t* __restrict__ s, int col) {
  return s[col] < 0 ? 1u : 0u;
}

// The sign bits (bit 7) of the four int8 in w, as bits 0..3: after masking,
// one multiply moves bits 7, 15, 23, 31 to 21, 22, 23, 24 without carries.
__device__ __forceinline__ uint32_t sign_nibble(uint32_t w) {
  return (((w >> 7) & 0x01010101u) * 0x00204081u >> 21) & 0xFu;
}

// Bit k set when s[c0 + k] < 0, for k < 32 (c0 a multiple of 16).
__device__ __forceinline__ uint32_t sign_bits32(const int8_t* __restrict__ s, int c0) {
  const uint4 a = *reinterpret_cast<const uint4*>(s + c0);
  const uint4 b = *reinterpret_cast<const uint4*>(s + c0 + 16);
  return sign_nibble(a.x) | sign_nibble(a.y) << 4 | sign_nibble(a.z) << 8 | sign_nibble(a.w) << 12 |
         sign_nibble(b.x) << 16 | sign_nibble(b.y) << 20 | sign_nibble(b.z) << 24 | sign_nibble(b.w) << 28;
}

// Bit k set when s[c0 + k] < 0, for k < W, W in {2, 4, 8, 16} (c0 a multiple of W).
template <int W>
__device__ __forceinline__ uint32_t sign_bits_small(const int8_t* __restrict__ s, int c0) {
  if constexpr (W == 16) {
    const uint4 a = *reinterpret_cast<const uint4*>(s + c0);
    return sign_nibble(a.x) | sign_nibble(a.y) << 4 | sign_nibble(a.z) << 8 | sign_nibble(a.w) << 12;
  } else if constexpr (W == 8) {
    const uint2 a = *reinterpret_cast<const uint2*>(s + c0);
    return sign_nibble(a.x) | sign_nibble(a.y) << 4;
  } else if constexpr (W == 4) {
    return sign_nibble(*reinterpret_cast<const uint32_t*>(s + c0));
  } else {
    static_assert(W == 2, "2, 4, 8 or 16 signs");
    return sign_nibble(*reinterpret_cast<const uint16_t*>(s + c0)) & 3u;
  }
}

// Register bit order of a mask under the quad permutation reg<true>: bits 1
// and 2 of every nibble swap places.
__device__ __forceinline__ uint32_t perm_quad_bits(uint32_t m) {
  return (m & 0x99999999u) | ((m & 0x22222222u) << 1) | ((m & 0x44444444u) >> 1);
}

// 1.5 * 2^23: adding it to |v| < 2^22 leaves round-half-even(v) in the low
// mantissa bits (fp32 addition rounds to the nearest representable value, and
// the spacing at this magnitude is exactly 1).
constexpr float kRoundMagic = 12582912.0f;
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// ------------------------------------------------------------ launch control

// Programmatic dependent launch: wait until the previous grid in the stream
// has completed and its writes are visible (a no-op without the launch
// attribute), then let the next grid start scheduling its CTAs.  Called
// before the first global memory access of every kernel.
__device__ __forceinline__ void grid_dependency_sync() {
  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();
}

// Hint the TMA unit to stage [p, p + bytes) into L2 (16-byte aligned address,
// size a multiple of 16, range inside the tensor).  Uses no SM resources.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- butterflies

__device__ __forceinline__ void bfly1(float& a, float& b) {
  const float s = __fadd_rn(a, b);
  const float d = __fsub_rn(a, b);
  a = s;
  b = d;
}

// Two butterflies at once with the sm_100 packed fp32 add/sub: (a0, b0) and (a1, b1).
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 pa, pb, ps, pd;\n\t"
      "mov.b64 pa, {%0, %1};\n\t"
      "mov.b64 pb, {%2, %3};\n\t"
      "add.rn.f32x2 ps, pa, pb;\n\t"
      "sub.rn.f32x2 pd, pa, pb;\n\t"
      "mov.b64 {%0, %1}, ps;\n\t"
      "mov.b64 {%2, %3}, pd;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// H_2 along register-index bit K of an N-element register array.  Bit 0 pairs
// the two halves of a packed register pair, so it uses scalar adds; every
// other bit uses packed f32x2 adds.
template <int N, int K>
__device__ __forceinline__ void fwht_stage(float (&v)[N]) {
  static_assert((2 << K) <= N, "stage bit out of range");
  constexpr int D = 1 << K;
  if constexpr (K == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 2) bfly1(v[i], v[i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 2)
      if ((i & D) == 0) bfly2(v[i], v[i + 1], v[i + D], v[i + D + 1]);
  }
}

// Stages for register-index bits [LO, HI).
template <int N, int LO, int HI>
__device__ __forceinline__ void fwht_bits(float (&v)[N]) {
  if constexpr (LO < HI) {
    fwht_stage<N, LO>(v);
    fwht_bits<N, LO + 1, HI>(v);
  }
}

// Stages for the low `nbits` register-index bits (runtime count, uniform per launch):
// the block-diagonal rotation of b = 2^nbits inside an N-element segment.
template <int N, int K = 0>
__device__ __forceinline__ void fwht_low(float (&v)[N], int nbits) {
  if constexpr ((2 << K) <= N) {
    if (K < nbits) fwht_stage<N, K>(v);
    fwht_low<N, K + 1>(v, nbits);
  }
}

// --------------------------------------------------------------- loads/stores

// bf16 pair -> two fp32 (exact): the low half moved up by a byte permute, the
// high half masked; both stay off the fp32 pipe.
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(__byte_perm(w, 0u, 0x1044));
  hi = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ldg_stream(const uint2* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ldg_stream(const uint32_t* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// 32 bytes (one whole sector) in one 256-bit load; p must be 32-byte aligned.
__device__ __forceinline__ void ldg_stream32(const void* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

// NE contiguous input elements starting at element index e -> dst[0..NE).
// A thread's run is far from its neighbours' (a segment or a team chunk), so
// a 16-byte load uses half of each 32-byte sector it fetches and the next
// load fetches the sector again (L1 is bypassed); with WIDE, runs of 32 bytes
// or more therefore load whole sectors with 256-bit loads when the run is
// 32-byte aligned (the API promises 16), and 16-byte loads otherwise.
template <bool IN_BF16, int NE, bool WIDE = true>
__device__ __forceinline__ void load_elems(const void* __restrict__ x, int64_t e, float* dst) {
  if constexpr (IN_BF16) {
    const uint16_t* p = static_cast<const uint16_t*>(x) + e;
    if constexpr (WIDE && NE % 16 == 0) {
      if ((reinterpret_cast<uintptr_t>(p) & 31) == 0) {
#pragma unroll
        for (int i = 0; i < NE / 16; ++i) {
          uint4 w, u;
          ldg_stream32(p + 16 * i, w, u);
          unpack_bf16x2(w.x, dst[16 * i + 0], dst[16 * i + 1]);
          unpack_bf16x2(w.y, dst[16 * i + 2], dst[16 * i + 3]);
          unpack_bf16x2(w.z, dst[16 * i + 4], dst[16 * i + 5]);
          unpack_bf16x2(w.w, dst[16 * i + 6], dst[16 * i + 7]);
          unpack_bf16x2(u.x, dst[16 * i + 8], dst[16 * i + 9]);
          unpack_bf16x2(u.y, dst[16 * i + 10], dst[16 * i + 11]);
          unpack_bf16x2(u.z, dst[16 * i + 12], dst[16 * i + 13]);
          unpack_bf16x2(u.w, dst[16 * i + 14], dst[16 * i + 15]);
        }
        return;
      }
    }
    if constexpr (NE % 8 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 8; ++i) {
        const uint4 w = ldg_stream(reinterpret_cast<const uint4*>(p) + i);
        unpack_bf16x2(w.x, dst[8 * i + 0], dst[8 * i + 1]);
        unpack_bf16x2(w.y, dst[8 * i + 2], dst[8 * i + 3]);
        unpack_bf16x2(w.z, dst[8 * i + 4], dst[8 * i + 5]);
        unpack_bf16x2(w.w, dst[8 * i + 6], dst[8 * i + 7]);
      }
    } else if constexpr (NE == 4) {
      const uint2 w = ldg_stream(reinterpret_cast<const uint2*>(p));
      unpack_bf16x2(w.x, dst[0], dst[1]);
      unpack_bf16x2(w.y, dst[2], dst[3]);
    } else {
      static_assert(NE == 2, "unsupported bf16 chunk");
      const uint32_t w = ldg_stream(reinterpret_cast<const uint32_t*>(p));
      unpack_bf16x2(w, dst[0], dst[1]);
    }
  } else {
    const float* p = static_cast<const float*>(x) + e;
    if constexpr (WIDE && NE % 8 == 0) {
      if ((reinterpret_cast<uintptr_t>(p) & 31) == 0) {
#pragma unroll
        for (int i = 0; i < NE / 8; ++i) {
          uint4 w, u;
          ldg_stream32(p + 8 * i, w, u);
          dst[8 * i + 0] = __uint_as_float(w.x);
          dst[8 * i + 1] = __uint_as_float(w.y);
          dst[8 * i + 2] = __uint_as_float(w.z);
          dst[8 * i + 3] = __uint_as_float(w.w);
          dst[8 * i + 4] = __uint_as_float(u.x);
          dst[8 * i + 5] = __uint_as_float(u.y);
          dst[8 * i + 6] = __uint_as_float(u.z);
          dst[8 * i + 7] = __uint_as_float(u.w);
        }
        return;
      }
    }
    if constexpr (NE % 4 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 4; ++i) {
        const uint4 w = ldg_stream(reinterpret_cast<const uint4*>(p) + i);
        dst[4 * i + 0] = __uint_as_float(w.x);
        dst[4 * i + 1] = __uint_as_float(w.y);
        dst[4 * i + 2] = __uint_as_float(w.z);
        dst[4 * i + 3] = __uint_as_float(w.w);
      }
    } else {
      static_assert(NE == 2, "unsupported fp32 chunk");
      const uint2 w = ldg_stream(reinterpret_cast<const uint2*>(p));
      dst[0] = __uint_as_float(w.x);
      dst[1] = __uint_as_float(w.y);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

// ----------------------------------------------------------- register orders
// A thread's register array holds its elements either in element order or,
// after the team transpose, with the two low element-index bits swapped inside
// every quad (registers 4q..4q+3 = elements 4q, 4q+2, 4q+1, 4q+3), which lets
// the element-bit-0 butterfly use packed f32x2 adds.  reg<PERM>(e) maps an
// element index to its register (the swap is its own inverse).

template <bool PERM>
__host__ __device__ constexpr int reg(int e) {
  return PERM ? ((e & ~3) | ((e & 1) << 1) | ((e >> 1) & 1)) : e;
}

// Flip the sign of register i where bit i of the mask (word i / 32) is set.
// Each thread's mask is fixed for a whole launch: a thread always holds the
// same block columns in the same registers.  The mask words pass through an
// opaque move first, so the per-element sign words are formed here, at each
// use, instead of being hoisted out of the caller's loop (N live registers).
template <int N>
__device__ __forceinline__ void apply_signs(float (&v)[N], const uint32_t (&m_in)[(N + 31) / 32]) {
  uint32_t m[(N + 31) / 32];
#pragma unroll
  for (int w = 0; w < (N + 31) / 32; ++w) asm volatile("mov.b32 %0, %1;" : "=r"(m[w]) : "r"(m_in[w]));
#pragma unroll
  for (int i = 0; i < N; ++i)
    v[i] = __uint_as_float(__float_as_uint(v[i]) ^ ((m[i >> 5] << (31 - (i & 31))) & 0x80000000u));
}

// ------------------------------------------------------------------ quantizers

// max(|a|, |b|, |c|) in one instruction (the three-input max with absolute
// inputs of sm_100).
__device__ __forceinline__ float max3abs(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Absmax of registers [lo, lo + cnt) (cnt a multiple of 4; order does not
// matter): two independent chains that each take two new registers per
// three-input max, then one max of the two.
template <int N>
__device__ __forceinline__ float absmax_regs(const float (&v)[N], int lo, int cnt) {
  float ma = v[lo], mb = v[lo + 1];     // raw: every max below takes absolute values
#pragma unroll
  for (int i = 2; i < cnt; i += 4) {
    ma = max3abs(ma, v[lo + i], v[lo + i + 1]);
    if (i + 2 < cnt) mb = max3abs(mb, v[lo + i + 2], v[lo + i + 3]);
  }
  return max3abs(ma, mb, mb);
}

// Eight int4 codes rne(v * rn) of elements e0..e0+7 (register order PERM), as
// two's-complement nibbles, element i in bits [4i, 4i + 4).  Valid when every
// |v * rn| < 7.5 (no clamp needed): each product is rounded once onto the
// integer grid by a fused multiply-add with 1.5*2^23 + 8, leaving q + 8 in
// 1..15 in the low bits; the eight words are combined by shift-add (Horner),
// the constant high parts removed, and the offset-8 nibbles turned into
// two's complement by flipping their top bits.
template <bool PERM, int N>
__device__ __forceinline__ uint32_t pack_int4x8(const float (&v)[N], int e0, float rn) {
  constexpr float kM = kRoundMagic + 8.0f;
  const float2 r2 = make_float2(rn, rn), m2 = make_float2(kM, kM);
  uint32_t t[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __ffma2_rn(make_float2(v[reg<PERM>(e0 + i)], v[reg<PERM>(e0 + i + 1)]), r2, m2);
    t[i] = __float_as_uint(p.x);
    t[i + 1] = __float_as_uint(p.y);
  }
  // Low byte of t[i] + (t[i+1] << 4) is the offset nibble pair: t[i] & 0xFF is
  // 8 + q (no borrow), and the magic part of t[i+1] shifted by 4 has a zero
  // low byte.  Gather the four low bytes, then flip the nibbles' top bits.
  const uint32_t p0 = t[0] + (t[1] << 4), p1 = t[2] + (t[3] << 4);
  const uint32_t p2 = t[4] + (t[5] << 4), p3 = t[6] + (t[7] << 4);
  const uint32_t w = __byte_perm(__byte_perm(p0, p1, 0x0040), __byte_perm(p2, p3, 0x0040), 0x5410);
  return w ^ 0x88888888u;
}

// The same with an explicit clamp to [-7, 7] (subnormal, zero or huge scales).
template <bool PERM, int N>
__device__ __forceinline__ uint32_t pack_int4x8_clamped(const float (&v)[N], int e0, float rn) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float q = fminf(fmaxf(v[reg<PERM>(e0 + i)] * rn, -7.0f), 7.0f);
    const uint32_t b = __float_as_uint(__fadd_rn(q, kRoundMagic + 8.0f)) - (kRoundMagicBits + 8u);
    w |= (b & 0xFu) << (4 * i);
  }
  return w;
}

// Four int8 codes rne(v * rn), element i in byte i (|v * rn| < 127.5).
template <bool PERM, int N>
__device__ __forceinline__ uint32_t pack_int8x4(const float (&v)[N], int e0, float rn) {
  const float2 r2 = make_float2(rn, rn), m2 = make_float2(kRoundMagic, kRoundMagic);
  const float2 p0 = __ffma2_rn(make_float2(v[reg<PERM>(e0)], v[reg<PERM>(e0 + 1)]), r2, m2);
  const float2 p1 = __ffma2_rn(make_float2(v[reg<PERM>(e0 + 2)], v[reg<PERM>(e0 + 3)]), r2, m2);
  const uint32_t lo = __byte_perm(__float_as_uint(p0.x), __float_as_uint(p0.y), 0x5140);
  const uint32_t hi = __byte_perm(__float_as_uint(p1.x), __float_as_uint(p1.y), 0x5140);
  return __byte_perm(lo, hi, 0x5410);
}

// Eight E2M1 codes (round to nearest even, saturating at +/-6, sign in bit 3)
// of v * f, element i in bits [4i, 4i + 4).  The product is formed as
// v * f + 0, which turns a zero of either sign into +0, so an exact zero
// codes as 0 (only a negative nonzero value sets the sign bit).
template <bool PERM, int N>
__device__ __forceinline__ uint32_t pack_e2m1x8(const float (&v)[N], int e0, float f) {
  const float2 f2 = make_float2(f, f), z2 = make_float2(0.f, 0.f);
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __ffma2_rn(make_float2(v[reg<PERM>(e0 + i)], v[reg<PERM>(e0 + i + 1)]), f2, z2);
    a[i] = p.x;
    a[i + 1] = p.y;
  }
  uint32_t w;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(w)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  return w;
}

// Scale arithmetic.  The int4 and NVFP4 scales are m * fp32(1/7) and
// m * fp32(1/6) (within 1.5 ulp of m / 7, m / 6) before their rounding to
// fp16 / E4M3: the rounded scale can differ from the rounding of the exact
// quotient only within 2^-23 (relative) of a rounding midpoint of the scale
// format, where either neighbour is a valid scale.  The int8 scale, stored in
// fp32, is the correctly rounded quotient m / 127.  The factor that takes an
// unnormalised rotated value z to code units is the correctly rounded
// quotient norm / s of the stored scale, so an int code is the single
// rounding of the exact product z * (norm / s) onto the integer grid: it can
// differ from the exactly rounded y / s only through the fp32 rotation's own
// error and the factor's half-ulp (at most 4.5e-7 of a code unit at
// |y / s| = 7.5).
constexpr float kInv7 = 1.0f / 7.0f;
constexpr float kInv6 = 1.0f / 6.0f;
__device__ __forceinline__ float int4_scale_f32(float m) { return m * kInv7; }
__device__ __forceinline__ float int8_scale(float m) { return __fdiv_rn(m, 127.0f); }
__device__ __forceinline__ float nvfp4_scale_f32(float m) { return m * kInv6; }
__device__ __forceinline__ float code_factor(float norm, float s) { return __fdiv_rn(norm, s); }

// 32 output bytes at p: one 256-bit store (full 32-byte sectors) when p is
// 32-byte aligned, else two 128-bit stores.  A thread's run of outputs is
// contiguous while the runs of the lanes of a warp are not, so 16-byte stores
// would fill every sector in two halves.
__device__ __forceinline__ void store32(void* p, const uint4& a, const uint4& b) {
  if ((reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
  } else {
    reinterpret_cast<uint4*>(p)[0] = a;
    reinterpret_cast<uint4*>(p)[1] = b;
  }
}

// --------------------------------------------------------------- epilogues
// Each epilogue owns N consecutive rotated-but-unnormalised values z of one
// row (register order PERM), starting at flattened element index e0;
// y = z * norm is the rotation.

// Rotation output (fp32 or bf16).
template <bool PERM, int N, bool OUT_IS_BF16>
__device__ __forceinline__ void store_rotated(const float (&v)[N], float norm, void* __restrict__ out, int64_t e0) {
  if constexpr (OUT_IS_BF16) {
    uint16_t* o = static_cast<uint16_t*>(out) + e0;
    static_assert(N % 8 == 0, "bf16 chunk must hold whole 16-byte stores");
    auto chunk = [&](int i) {
      uint4 w;
      w.x = pack_bf16x2(v[reg<PERM>(8 * i + 0)] * norm, v[reg<PERM>(8 * i + 1)] * norm);
      w.y = pack_bf16x2(v[reg<PERM>(8 * i + 2)] * norm, v[reg<PERM>(8 * i + 3)] * norm);
      w.z = pack_bf16x2(v[reg<PERM>(8 * i + 4)] * norm, v[reg<PERM>(8 * i + 5)] * norm);
      w.w = pack_bf16x2(v[reg<PERM>(8 * i + 6)] * norm, v[reg<PERM>(8 * i + 7)] * norm);
      return w;
    };
    if constexpr (N % 16 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; i += 2) store32(o + 8 * i, chunk(i), chunk(i + 1));
    } else {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) reinterpret_cast<uint4*>(o)[i] = chunk(i);
    }
  } else {
    float* o = static_cast<float*>(out) + e0;
    static_assert(N % 4 == 0, "fp32 chunk must hold whole float4s");
    auto chunk = [&](int i) {
      return make_uint4(__float_as_uint(v[reg<PERM>(4 * i)] * norm), __float_as_uint(v[reg<PERM>(4 * i + 1)] * norm),
                        __float_as_uint(v[reg<PERM>(4 * i + 2)] * norm), __float_as_uint(v[reg<PERM>(4 * i + 3)] * norm));
    };
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 4; i += 2) store32(o + 4 * i, chunk(i), chunk(i + 1));
    } else {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) reinterpret_cast<uint4*>(o)[i] = chunk(i);
    }
  }
}

// Symmetric int4, group in {32, 64, 128} with group | N: scale fp16(m / 7).
template <bool PERM, int N>
__device__ __forceinline__ void store_int4(const float (&v)[N], float norm, int group, uint8_t* __restrict__ codes,
                                           __half* __restrict__ scales, int64_t e0) {
  static_assert(N % 32 == 0, "int4 groups need 32-element sub-blocks");
  constexpr int NS = N / 32;
  float m32[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) m32[j] = absmax_regs(v, 32 * j, 32);   // a 32-block is closed under reg<>
  const int spg = group >> 5;  // 32-element sub-blocks per group: 1, 2 or 4
  uint4 prev = make_uint4(0u, 0u, 0u, 0u);   // codes of sub-block j - 1, stored with those of j
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    float mz = m32[j];
    if constexpr (NS >= 2) {
      if (spg >= 2) mz = fmaxf(mz, m32[j ^ 1]);
    }
    if constexpr (NS >= 4) {
      if (spg >= 4) mz = fmaxf(mz, fmaxf(m32[j ^ 2], m32[j ^ 3]));
    }
    const float m = mz * norm;                         // absmax of y (rounding is monotone)
    const __half s16 = __float2half_rn(int4_scale_f32(m));
    const float s = __half2float(s16);
    const float rn = (s > 0.f && s <= 65504.f) ? code_factor(norm, s) : 0.f;   // zero / inf scale -> zero codes
    uint4 w;
    if (mz * rn < 7.25f) {        // normal scale: every |v * rn| <= 7.0035, no clamp
      w.x = pack_int4x8<PERM>(v, 32 * j + 0, rn);
      w.y = pack_int4x8<PERM>(v, 32 * j + 8, rn);
      w.z = pack_int4x8<PERM>(v, 32 * j + 16, rn);
      w.w = pack_int4x8<PERM>(v, 32 * j + 24, rn);
    } else {
      w.x = pack_int4x8_clamped<PERM>(v, 32 * j + 0, rn);
      w.y = pack_int4x8_clamped<PERM>(v, 32 * j + 8, rn);
      w.z = pack_int4x8_clamped<PERM>(v, 32 * j + 16, rn);
      w.w = pack_int4x8_clamped<PERM>(v, 32 * j + 24, rn);
    }
    if constexpr (NS == 1) {
      reinterpret_cast<uint4*>(codes + (e0 >> 1))[0] = w;
    } else if (j & 1) {
      store32(codes + ((e0 + 32 * (j - 1)) >> 1), prev, w);
    } else {
      prev = w;
    }
    if ((j & (spg - 1)) == 0) scales[(e0 + 32 * j) >> (__ffs(group) - 1)] = s16;   // group is a power of 2
  }
}

// Symmetric int4 codes of 32 consecutive outputs whose group (32, 64 or 128
// elements, group-aligned) has the absmax mz of the unnormalised values,
// joined by the caller; the arithmetic of store_int4.  The thread whose e0 is
// the group's first element stores the scale.
__device__ __forceinline__ void store_int4_piece32(const float (&v)[32], float norm, float mz, int group,
                                                   uint8_t* __restrict__ codes, __half* __restrict__ scales,
                                                   int64_t e0) {
  const float m = mz * norm;
  const __half s16 = __float2half_rn(int4_scale_f32(m));
  const float s = __half2float(s16);
  const float rn = (s > 0.f && s <= 65504.f) ? code_factor(norm, s) : 0.f;
  uint4 w;
  if (mz * rn < 7.25f) {
    w = make_uint4(pack_int4x8<false>(v, 0, rn), pack_int4x8<false>(v, 8, rn), pack_int4x8<false>(v, 16, rn),
                   pack_int4x8<false>(v, 24, rn));
  } else {
    w = make_uint4(pack_int4x8_clamped<false>(v, 0, rn), pack_int4x8_clamped<false>(v, 8, rn),
                   pack_int4x8_clamped<false>(v, 16, rn), pack_int4x8_clamped<false>(v, 24, rn));
  }
  reinterpret_cast<uint4*>(codes + (e0 >> 1))[0] = w;
  if ((e0 & (group - 1)) == 0) scales[e0 >> (__ffs(group) - 1)] = s16;
}

// Symmetric int4 with group 128 for a thread holding 64 consecutive outputs
// (a group-aligned half when e0 % 128 == 0, the other half in lane ^ 1): the
// group absmax is exchanged with that lane.  Every lane of the warp must call
// it; ok = false computes and stores nothing.
template <bool PERM>
__device__ __forceinline__ void store_int4_pair(const float (&v)[64], float norm, uint8_t* __restrict__ codes,
                                                __half* __restrict__ scales, int64_t e0, bool ok) {
  float mz = fmaxf(absmax_regs(v, 0, 32), absmax_regs(v, 32, 32));
  mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 1));
  const float m = mz * norm;
  const __half s16 = __float2half_rn(int4_scale_f32(m));
  const float s = __half2float(s16);
  const float rn = (s > 0.f && s <= 65504.f) ? code_factor(norm, s) : 0.f;
  uint4 w0, w1;
  if (mz * rn < 7.25f) {
    w0 = make_uint4(pack_int4x8<PERM>(v, 0, rn), pack_int4x8<PERM>(v, 8, rn), pack_int4x8<PERM>(v, 16, rn),
                    pack_int4x8<PERM>(v, 24, rn));
    w1 = make_uint4(pack_int4x8<PERM>(v, 32, rn), pack_int4x8<PERM>(v, 40, rn), pack_int4x8<PERM>(v, 48, rn),
                    pack_int4x8<PERM>(v, 56, rn));
  } else {
    w0 = make_uint4(pack_int4x8_clamped<PERM>(v, 0, rn), pack_int4x8_clamped<PERM>(v, 8, rn),
                    pack_int4x8_clamped<PERM>(v, 16, rn), pack_int4x8_clamped<PERM>(v, 24, rn));
    w1 = make_uint4(pack_int4x8_clamped<PERM>(v, 32, rn), pack_int4x8_clamped<PERM>(v, 40, rn),
                    pack_int4x8_clamped<PERM>(v, 48, rn), pack_int4x8_clamped<PERM>(v, 56, rn));
  }
  if (ok) {
    store32(codes + (e0 >> 1), w0, w1);
    if ((e0 & 127) == 0) scales[e0 >> 7] = s16;
  }
}

// Symmetric int4 for a thread holding N consecutive outputs (register order
// natural), group in {32, 64, 128}.  A group larger than N spans group / N
// (2 or 4) consecutive lanes, group-aligned: its absmax is exchanged with
// shuffles, so every lane of the warp must call this; ok = false computes and
// stores nothing.
template <int N>
__device__ __forceinline__ void store_int4_lanes(const float (&v)[N], float norm, int group,
                                                 uint8_t* __restrict__ codes, __half* __restrict__ scales,
                                                 int64_t e0, bool ok) {
  static_assert(N % 32 == 0 && N <= 128, "32..128 outputs per thread");
  if (group <= N) {
    if (ok) store_int4<false, N>(v, norm, group, codes, scales, e0);
    return;
  }
  float mz = absmax_regs(v, 0, N);
  mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 1));
  if (group >= 4 * N) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 2));
  const float m = mz * norm;
  const __half s16 = __float2half_rn(int4_scale_f32(m));
  const float s = __half2float(s16);
  const float rn = (s > 0.f && s <= 65504.f) ? code_factor(norm, s) : 0.f;
  const bool plain = mz * rn < 7.25f;
  uint4 prev = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int j = 0; j < N / 32; ++j) {
    uint4 w;
    if (plain) {
      w = make_uint4(pack_int4x8<false>(v, 32 * j, rn), pack_int4x8<false>(v, 32 * j + 8, rn),
                     pack_int4x8<false>(v, 32 * j + 16, rn), pack_int4x8<false>(v, 32 * j + 24, rn));
    } else {
      w = make_uint4(pack_int4x8_clamped<false>(v, 32 * j, rn), pack_int4x8_clamped<false>(v, 32 * j + 8, rn),
                     pack_int4x8_clamped<false>(v, 32 * j + 16, rn), pack_int4x8_clamped<false>(v, 32 * j + 24, rn));
    }
    if (ok) {
      if constexpr (N == 32) {
        reinterpret_cast<uint4*>(codes + (e0 >> 1))[0] = w;
      } else if (j & 1) {
        store32(codes + ((e0 + 32 * (j - 1)) >> 1), prev, w);
      }
    }
    prev = w;
  }
  if (ok && (e0 & (group - 1)) == 0) scales[e0 >> (__ffs(group) - 1)] = s16;   // the group's first lane
}

// Offset of scale k (row-major index over rows x 2^LOG_C scale columns) in
// the tiled scale layout of block-scaled tensor-core GEMMs (the "1D block
// scaling factors" layout of NVIDIA's cuBLAS documentation): 128-row x
// 4-column tiles of 512 bytes, row-block major; inside a tile, scale (r, c)
// at (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.  LOG_C = 0: row-major (k).
template <int LOG_C>
__device__ __forceinline__ int64_t scale_offset(int64_t k) {
  if constexpr (LOG_C == 0) {
    return k;
  } else {
    static_assert(LOG_C >= 2, "whole 4-column tiles");
    const int64_t r = k >> LOG_C;
    const int c = static_cast<int>(k & ((int64_t(1) << LOG_C) - 1));
    return (((r >> 7) << (LOG_C - 2)) + (c >> 2)) * 512 + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
  }
}

// The same tiled offset for a run-time number of scale columns per row
// (a multiple of 4): scale k = row * cols + column.  One 32-bit division per
// call; callers use it once per thread and chunk.
struct TiledScales {
  int64_t r;   // row of the first scale of the chunk
  int c;       // its column
  int cols;    // scale columns per row
  __device__ __forceinline__ TiledScales(int64_t k, int cols_) : cols(cols_) {
    // k < 2^32: a scale per 16 elements or more, and fewer than 2^36 elements
    // of 2 bytes or more fit any device memory
    const uint32_t q = static_cast<uint32_t>(k) / static_cast<uint32_t>(cols_);
    r = q;
    c = static_cast<int>(static_cast<uint32_t>(k) - q * static_cast<uint32_t>(cols_));
  }
  // Offset of scale k + j, j small enough to stay in the row.
  __device__ __forceinline__ int64_t operator()(int j) const {
    const int cj = c + j;
    return ((r >> 7) * (cols >> 2) + (cj >> 2)) * 512 + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (cj & 3);
  }
};

// MXFP4: per 32 elements an E8M0 exponent e = clamp(floor(log2 m) - 2, -127, 127).
// LOG_C: the scale layout (scale_offset); tiled_cols > 0: the tiled layout
// with that many scale columns per row (TiledScales).
template <bool PERM, int N, int LOG_C = 0>
__device__ __forceinline__ void store_mxfp4(const float (&v)[N], float norm, uint8_t* __restrict__ codes,
                                            uint8_t* __restrict__ scales, int64_t e0, int tiled_cols = 0) {
  static_assert(N % 32 == 0, "MX groups are 32 elements");
  uint4 prev = make_uint4(0u, 0u, 0u, 0u);   // codes of sub-block j - 1, stored with those of j
#pragma unroll
  for (int j = 0; j < N / 32; ++j) {
    const float m = absmax_regs(v, 32 * j, 32) * norm;
    // floor(log2 m) is the unbiased exponent field for normal m; zero and
    // subnormal m (and anything below 2^-125) clamp to e = -127, byte 0.
    const int ebits = static_cast<int>((__float_as_uint(m) >> 23) & 0xFF);
    const int byte = max(ebits - 2, 0);               // e + 127
    const int e = byte - 127;                         // in [-127, 126]
    const float f = norm * __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // norm * 2^-e, exact
    uint4 w;
    w.x = pack_e2m1x8<PERM>(v, 32 * j + 0, f);
    w.y = pack_e2m1x8<PERM>(v, 32 * j + 8, f);
    w.z = pack_e2m1x8<PERM>(v, 32 * j + 16, f);
    w.w = pack_e2m1x8<PERM>(v, 32 * j + 24, f);
    if constexpr (N == 32) {
      reinterpret_cast<uint4*>(codes + (e0 >> 1))[0] = w;
    } else if (j & 1) {
      store32(codes + ((e0 + 32 * (j - 1)) >> 1), prev, w);
    } else {
      prev = w;
    }
    if (tiled_cols > 0) scales[TiledScales(e0 >> 5, tiled_cols)(j)] = static_cast<uint8_t>(byte);
    else scales[scale_offset<LOG_C>((e0 >> 5) + j)] = static_cast<uint8_t>(byte);
  }
}

// FP8 E4M3 bytes of two non-negative values (round half to even, saturating
// at 448): `hi` in bits 8..15, `lo` in bits 0..7.
__device__ __forceinline__ uint16_t e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// The values of two E4M3 bytes (exact in fp16): .x from bits 0..7, .y from 8..15.
__device__ __forceinline__ float2 e4m3x2_values(uint16_t b) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
  return make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu))),
                     __half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16))));
}

// NVFP4: per 16 elements an E4M3 scale s = e4m3(m / 6) of the block absmax m
// of v = z * nq (nq = the rotation's 1/sqrt(b) divided by the per-tensor
// scale) and E2M1 codes of v / s; s == 0 gives codes 0.  Pairs of blocks
// store 16 code bytes and 2 scale bytes at once.
template <bool PERM, int N, int LOG_C = 0>
__device__ __forceinline__ void store_nvfp4(const float (&v)[N], float nq, uint8_t* __restrict__ codes,
                                            uint8_t* __restrict__ scales, int64_t e0, int tiled_cols = 0) {
  static_assert(N % 16 == 0, "NVFP4 blocks are 16 elements");
  if constexpr (N == 16) {
    const float m = absmax_regs(v, 0, 16) * nq;
    const uint16_t b = e4m3x2(0.f, nvfp4_scale_f32(m));
    const float s = e4m3x2_values(b).x;
    const float f = s > 0.f ? code_factor(nq, s) : 0.f;
    reinterpret_cast<uint2*>(codes + (e0 >> 1))[0] = make_uint2(pack_e2m1x8<PERM>(v, 0, f), pack_e2m1x8<PERM>(v, 8, f));
    if (tiled_cols > 0) scales[TiledScales(e0 >> 4, tiled_cols)(0)] = static_cast<uint8_t>(b & 0xFFu);
    else scales[scale_offset<LOG_C>(e0 >> 4)] = static_cast<uint8_t>(b & 0xFFu);
  } else {
    static_assert(N % 32 == 0, "NVFP4 chunks above 16 elements come in pairs of blocks");
    uint4 prev = make_uint4(0u, 0u, 0u, 0u);   // codes of blocks 2j - 2, 2j - 1, stored with those of 2j, 2j + 1
#pragma unroll
    for (int j = 0; j < N / 32; ++j) {
      const float m0 = absmax_regs(v, 32 * j, 16) * nq;
      const float m1 = absmax_regs(v, 32 * j + 16, 16) * nq;
      const uint16_t b = e4m3x2(nvfp4_scale_f32(m1), nvfp4_scale_f32(m0));
      const float2 s = e4m3x2_values(b);
      const float f0 = s.x > 0.f ? code_factor(nq, s.x) : 0.f;
      const float f1 = s.y > 0.f ? code_factor(nq, s.y) : 0.f;
      const uint4 w = make_uint4(pack_e2m1x8<PERM>(v, 32 * j, f0), pack_e2m1x8<PERM>(v, 32 * j + 8, f0),
                                 pack_e2m1x8<PERM>(v, 32 * j + 16, f1), pack_e2m1x8<PERM>(v, 32 * j + 24, f1));
      if constexpr (N == 32) {
        reinterpret_cast<uint4*>(codes + (e0 >> 1))[0] = w;
      } else if (j & 1) {
        store32(codes + ((e0 + 32 * (j - 1)) >> 1), prev, w);
      } else {
        prev = w;
      }
      // Scales 2i, 2i + 1 are neighbours in either layout (tile columns pair up).
      const int64_t off = tiled_cols > 0 ? TiledScales(e0 >> 4, tiled_cols)(2 * j)
                                         : scale_offset<LOG_C>((e0 + 32 * j) >> 4);
      reinterpret_cast<uint16_t*>(scales + off)[0] = b;
    }
  }
}

// Symmetric int8 with a per-row scale s = fp32(m / 127) (m = the row absmax of y).
template <bool PERM, int N>
__device__ __forceinline__ void store_int8(const float (&v)[N], float norm, float m, int8_t* __restrict__ codes,
                                           int64_t e0) {
  static_assert(N % 8 == 0, "int8 chunk must hold whole 8-byte stores");
  const float s = int8_scale(m);
  const bool tiny = s > 0.f && s < 1.0e-36f;   // norm / s may be inexact or overflow: divide per element
  const float rn = (s >= 1.0e-36f && s <= 3.0e38f) ? code_factor(norm, s) : 0.f;
  if (!tiny) {                   // normal scale: every |v * rn| < 127.5, no clamp; zero scale: zero codes
    if constexpr (N % 32 == 0) {
      auto chunk = [&](int i) {
        return make_uint4(pack_int8x4<PERM>(v, 16 * i, rn), pack_int8x4<PERM>(v, 16 * i + 4, rn),
                          pack_int8x4<PERM>(v, 16 * i + 8, rn), pack_int8x4<PERM>(v, 16 * i + 12, rn));
      };
#pragma unroll
      for (int i = 0; i < N / 16; i += 2) store32(codes + e0 + 16 * i, chunk(i), chunk(i + 1));
    } else if constexpr (N % 16 == 0) {
      uint4* o = reinterpret_cast<uint4*>(codes + e0);
#pragma unroll
      for (int i = 0; i < N / 16; ++i)
        o[i] = make_uint4(pack_int8x4<PERM>(v, 16 * i, rn), pack_int8x4<PERM>(v, 16 * i + 4, rn),
                          pack_int8x4<PERM>(v, 16 * i + 8, rn), pack_int8x4<PERM>(v, 16 * i + 12, rn));
    } else {
      uint2* o = reinterpret_cast<uint2*>(codes + e0);
#pragma unroll
      for (int i = 0; i < N / 8; ++i)
        o[i] = make_uint2(pack_int8x4<PERM>(v, 8 * i, rn), pack_int8x4<PERM>(v, 8 * i + 4, rn));
    }
  } else {
    // Tiny scale: norm / s may be inexact or overflow -- divide per element, clamp.
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      uint32_t w = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float q = fminf(fmaxf(__fdiv_rn(v[reg<PERM>(4 * i + k)] * norm, s), -127.f), 127.f);
        w |= ((__float_as_uint(__fadd_rn(q, kRoundMagic)) - kRoundMagicBits) & 0xFFu) << (8 * k);
      }
      reinterpret_cast<uint32_t*>(codes + e0)[i] = w;
    }
  }
}

// Max over the CTA (blockDim.x a multiple of 32, every thread participating).
__device__ __forceinline__ float cta_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  v = lane < nw ? red[lane] : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  __syncthreads();
  return v;
}

}  // namespace hadq
