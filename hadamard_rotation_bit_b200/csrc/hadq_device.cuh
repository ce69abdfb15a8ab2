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

enum OutMode : int { OUT_F32 = 0, OUT_BF16 = 1, OUT_INT4 = 2, OUT_MXFP4 = 3 };

// 1.5 * 2^23: adding it to |v| < 2^22 leaves round-half-even(v) in the low
// mantissa bits (fp32 addition rounds to the nearest representable value, and
// the spacing at this magnitude is exactly 1).
constexpr float kRoundMagic = 12582912.0f;
constexpr int kRoundMagicBits = 0x4B400000;

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

// H_2 along register-index bit K of an N-element register array.
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

__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
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

// NE contiguous input elements starting at element index e -> dst[0..NE).
template <bool IN_BF16, int NE>
__device__ __forceinline__ void load_elems(const void* __restrict__ x, int64_t e, float* dst) {
  if constexpr (IN_BF16) {
    const uint16_t* p = static_cast<const uint16_t*>(x) + e;
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

// ------------------------------------------------------------------ quantizers

// Eight int4 codes clamp(rne(v * rn), -7, 7) as two's-complement nibbles,
// element i in bits [4i, 4i + 4).  The product is rounded once onto the
// integer grid by the fused multiply-add with the magic constant (+8 keeps
// the offset code in 1..15 so the clamp is an integer min/max).
__device__ __forceinline__ uint32_t pack_int4x8(const float* v, float rn) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int b = __float_as_int(__fmaf_rn(v[i], rn, kRoundMagic + 8.0f));
    b = min(max(b, kRoundMagicBits + 1), kRoundMagicBits + 15);
    w |= static_cast<uint32_t>((b - (kRoundMagicBits + 8)) & 0xF) << (4 * i);
  }
  return w;
}

// Four int8 codes clamp(rne(v * rn), -127, 127), element i in byte i.
__device__ __forceinline__ uint32_t pack_int8x4(const float* v, float rn) {
  int b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    b[i] = __float_as_int(__fmaf_rn(v[i], rn, kRoundMagic));
    b[i] = min(max(b[i], kRoundMagicBits - 127), kRoundMagicBits + 127);
  }
  const uint32_t lo = __byte_perm(b[0], b[1], 0x5140);
  const uint32_t hi = __byte_perm(b[2], b[3], 0x5140);
  return __byte_perm(lo, hi, 0x5410);
}

// Eight E2M1 codes (round to nearest even, saturating at +/-6, sign in bit 3)
// of v * f, element i in bits [4i, 4i + 4).
__device__ __forceinline__ uint32_t pack_e2m1x8(const float* v, float f) {
  const float a0 = v[0] * f, a1 = v[1] * f, a2 = v[2] * f, a3 = v[3] * f;
  const float a4 = v[4] * f, a5 = v[5] * f, a6 = v[6] * f, a7 = v[7] * f;
  uint32_t w;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(w)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return w;
}

template <int N>
__device__ __forceinline__ float absmax32(const float (&v)[N], int j) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[32 * j + i]));
  return m;
}

// --------------------------------------------------------------- epilogues
// Each epilogue owns N consecutive rotated-but-unnormalised values z of one
// row, starting at flattened element index e0; y = z * norm is the rotation.

// Rotation output (fp32 or bf16).
template <int N, bool OUT_IS_BF16>
__device__ __forceinline__ void store_rotated(const float (&v)[N], float norm, void* __restrict__ out, int64_t e0) {
  if constexpr (OUT_IS_BF16) {
    uint16_t* o = static_cast<uint16_t*>(out) + e0;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * i + 0] * norm, v[8 * i + 1] * norm);
        w.y = pack_bf16x2(v[8 * i + 2] * norm, v[8 * i + 3] * norm);
        w.z = pack_bf16x2(v[8 * i + 4] * norm, v[8 * i + 5] * norm);
        w.w = pack_bf16x2(v[8 * i + 6] * norm, v[8 * i + 7] * norm);
        reinterpret_cast<uint4*>(o)[i] = w;
      }
    } else {
      static_assert(N % 2 == 0, "odd bf16 chunk");
#pragma unroll
      for (int i = 0; i < N / 2; ++i) reinterpret_cast<uint32_t*>(o)[i] = pack_bf16x2(v[2 * i] * norm, v[2 * i + 1] * norm);
    }
  } else {
    float* o = static_cast<float*>(out) + e0;
    static_assert(N % 4 == 0, "fp32 chunk must hold whole float4s");
#pragma unroll
    for (int i = 0; i < N / 4; ++i)
      reinterpret_cast<float4*>(o)[i] =
          make_float4(v[4 * i] * norm, v[4 * i + 1] * norm, v[4 * i + 2] * norm, v[4 * i + 3] * norm);
  }
}

// Symmetric int4, group in {32, 64, 128} with group | N: scale fp16(m / 7).
template <int N>
__device__ __forceinline__ void store_int4(const float (&v)[N], float norm, int group, uint8_t* __restrict__ codes,
                                           __half* __restrict__ scales, int64_t e0) {
  static_assert(N % 32 == 0, "int4 groups need 32-element sub-blocks");
  constexpr int NS = N / 32;
  float m32[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) m32[j] = absmax32(v, j);
  const int spg = group >> 5;  // 32-element sub-blocks per group: 1, 2 or 4
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
    const __half s16 = __float2half_rn(__fdiv_rn(m, 7.0f));
    const float s = __half2float(s16);
    const float r = (s > 0.f && s <= 65504.f) ? __frcp_rn(s) : 0.f;   // zero / inf scale -> zero codes
    const float rn = r * norm;
    uint4 w;
    w.x = pack_int4x8(&v[32 * j + 0], rn);
    w.y = pack_int4x8(&v[32 * j + 8], rn);
    w.z = pack_int4x8(&v[32 * j + 16], rn);
    w.w = pack_int4x8(&v[32 * j + 24], rn);
    reinterpret_cast<uint4*>(codes + ((e0 + 32 * j) >> 1))[0] = w;
    if ((j & (spg - 1)) == 0) scales[(e0 + 32 * j) / group] = s16;
  }
}

// MXFP4: per 32 elements an E8M0 exponent e = clamp(floor(log2 m) - 2, -127, 127).
template <int N>
__device__ __forceinline__ void store_mxfp4(const float (&v)[N], float norm, uint8_t* __restrict__ codes,
                                            uint8_t* __restrict__ scales, int64_t e0) {
  static_assert(N % 32 == 0, "MX groups are 32 elements");
#pragma unroll
  for (int j = 0; j < N / 32; ++j) {
    const float m = absmax32(v, j) * norm;
    // floor(log2 m) is the unbiased exponent field for normal m; zero and
    // subnormal m (and anything below 2^-125) clamp to e = -127, byte 0.
    const int ebits = static_cast<int>((__float_as_uint(m) >> 23) & 0xFF);
    const int byte = max(ebits - 2, 0);               // e + 127
    const int e = byte - 127;                         // in [-127, 126]
    const float f = norm * __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // norm * 2^-e, exact
    uint4 w;
    w.x = pack_e2m1x8(&v[32 * j + 0], f);
    w.y = pack_e2m1x8(&v[32 * j + 8], f);
    w.z = pack_e2m1x8(&v[32 * j + 16], f);
    w.w = pack_e2m1x8(&v[32 * j + 24], f);
    reinterpret_cast<uint4*>(codes + ((e0 + 32 * j) >> 1))[0] = w;
    scales[(e0 >> 5) + j] = static_cast<uint8_t>(byte);
  }
}

// Symmetric int8 with a per-row scale s = fp32(m / 127) (m = the row absmax of y).
template <int N>
__device__ __forceinline__ void store_int8(const float (&v)[N], float norm, float m, int8_t* __restrict__ codes,
                                           int64_t e0) {
  static_assert(N % 8 == 0, "int8 chunk must hold whole 8-byte stores");
  const float s = __fdiv_rn(m, 127.0f);
  const float r = (s > 0.f && s <= 3.0e38f) ? __frcp_rn(s) : 0.f;
  if (r <= 1.0e30f) {
    const float rn = r * norm;
    if constexpr (N % 16 == 0) {
      uint4* o = reinterpret_cast<uint4*>(codes + e0);
#pragma unroll
      for (int i = 0; i < N / 16; ++i) {
        uint4 w;
        w.x = pack_int8x4(&v[16 * i + 0], rn);
        w.y = pack_int8x4(&v[16 * i + 4], rn);
        w.z = pack_int8x4(&v[16 * i + 8], rn);
        w.w = pack_int8x4(&v[16 * i + 12], rn);
        o[i] = w;
      }
    } else {
      uint2* o = reinterpret_cast<uint2*>(codes + e0);
#pragma unroll
      for (int i = 0; i < N / 8; ++i) o[i] = make_uint2(pack_int8x4(&v[8 * i], rn), pack_int8x4(&v[8 * i + 4], rn));
    }
  } else {
    // Scale so small that its reciprocal overflows: divide element by element.
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      float q[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) q[k] = fminf(fmaxf(__fdiv_rn(v[4 * i + k] * norm, s), -127.f), 127.f);
      reinterpret_cast<uint32_t*>(codes + e0)[i] = pack_int8x4(q, 1.0f);
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
