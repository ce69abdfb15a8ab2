// Rotation + quantization kernels (sm_100a).
//
// Two data layouts cover every block size b = 2^k of the block-diagonal
// rotation ("Rotation Transform", AutoRound docs, sections 1.2 / 2.1; b = n is
// the full rotation of section 1.5):
//
//  * segment kernels (b <= 128): a thread owns S = min(128, 2^v2(n))
//    consecutive elements of a row (S >= b, b | S), runs the log2(b) butterfly
//    stages on the low index bits in registers, and writes its S outputs.
//    One thread per segment, no cross-thread traffic.
//  * team kernels (256 <= b <= 8192): a team of T = b / 128 threads owns one
//    block.  Index bits: e = [hi: t bits | mid: t bits | vec: 7 - t bits],
//    t = log2 T.  Phase 1: each thread loads, for every hi value, one
//    contiguous chunk of 2^(7-t) elements (the team reads 128 contiguous
//    elements per hi value) and runs the 7 stages of its register bits
//    (vec + hi).  A transpose through shared memory (fp32, XOR-swizzled in
//    16-byte quads so both sides are bank-conflict free for t >= 3) hands
//    every thread the 128 consecutive elements with hi = its team index.
//    Phase 2 runs the remaining t stages (mid bits); the thread then holds a
//    whole run of 128 consecutive outputs for the quantizer.
//
// The per-token int8 format needs the whole row before any code is written,
// so it has row kernels: one CTA per row, the same two layouts inside, and a
// CTA-wide absmax reduction before the epilogue.
//
// The normalisation 1/sqrt(b) is never applied element by element on the
// quantized paths: it is folded into the group absmax (fp32 rounding is
// monotone, so max|fl(z * c)| = fl(max|z| * c)) and into the reciprocal
// scale.  For even log2(b) it is an exact power of 2.
#pragma once

#include "hadq_device.cuh"

namespace hadq {

constexpr int kThreads = 128;

// ----------------------------------------------------------- segment kernels

template <int LOGS, bool IN_BF16, int MODE>
__global__ void __launch_bounds__(kThreads)
segment_kernel(const void* __restrict__ x, int64_t segs, int nbits, float norm, int group,
               void* __restrict__ out0, void* __restrict__ out1) {
  constexpr int S = 1 << LOGS;
  float v[S];
  for (int64_t s = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; s < segs;
       s += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t e0 = s << LOGS;
    load_elems<IN_BF16, S>(x, e0, v);
    fwht_low<S>(v, nbits);
    if constexpr (MODE == OUT_F32) {
      store_rotated<S, false>(v, norm, out0, e0);
    } else if constexpr (MODE == OUT_BF16) {
      store_rotated<S, true>(v, norm, out0, e0);
    } else if constexpr (MODE == OUT_INT4) {
      store_int4<S>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
    } else {
      store_mxfp4<S>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
    }
  }
}

// Per-token int8, b <= 128: one CTA per row, blockDim = n / S rounded up to 32 (<= 256).
template <int LOGS, bool IN_BF16>
__global__ void __launch_bounds__(256)
segment_row_int8_kernel(const void* __restrict__ x, int64_t rows, int64_t n, int nbits, float norm,
                        int8_t* __restrict__ codes, float* __restrict__ scales) {
  constexpr int S = 1 << LOGS;
  __shared__ float red[32];
  const int segs_row = static_cast<int>(n >> LOGS);
  const bool active = static_cast<int>(threadIdx.x) < segs_row;
  float v[S];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t e0 = r * n + (static_cast<int64_t>(threadIdx.x) << LOGS);
    if (active) {
      load_elems<IN_BF16, S>(x, e0, v);
      fwht_low<S>(v, nbits);
    } else {
#pragma unroll
      for (int i = 0; i < S; ++i) v[i] = 0.f;
    }
    float mz = 0.f;
#pragma unroll
    for (int i = 0; i < S; ++i) mz = fmaxf(mz, fabsf(v[i]));
    const float m = cta_max(mz, red) * norm;
    if (active) store_int8<S>(v, norm, m, codes, e0);
    if (threadIdx.x == 0) scales[r] = __fdiv_rn(m, 127.0f);
  }
}

// --------------------------------------------------------------- team kernels

template <int LOGB>
struct TeamShape {
  static constexpr int t = LOGB - 7;          // log2(threads per team)
  static constexpr int T = 1 << t;            // threads per team
  static constexpr int V = 7 - t;             // vec bits per phase-1 chunk
  static constexpr int CE = 1 << V;           // elements per phase-1 chunk
  static constexpr int B = 1 << LOGB;
  static_assert(LOGB >= 8 && LOGB <= 13, "team kernels cover 256..8192");
};

template <int T>
__device__ __forceinline__ void team_sync() {
  if constexpr (T <= 32) {
    __syncwarp();
  } else {
    __syncthreads();
  }
}

// Rotate one block of 2^LOGB elements (element base `base`) by a team; on
// return v[0..128) holds the unnormalised outputs base + tau*128 + [0, 128).
// `rows` points at this team's T x 128-float shared buffer; `grow` is the
// team's first row in the CTA buffer (the swizzle key).
template <int LOGB, bool IN_BF16>
__device__ __forceinline__ void team_rotate(const void* __restrict__ x, int64_t base, bool valid, int tau,
                                            float* __restrict__ rows, int grow, float (&v)[128]) {
  using Sh = TeamShape<LOGB>;
  if (valid) {
#pragma unroll
    for (int h = 0; h < Sh::T; ++h) load_elems<IN_BF16, Sh::CE>(x, base + h * 128 + tau * Sh::CE, &v[h * Sh::CE]);
  } else {
#pragma unroll
    for (int i = 0; i < 128; ++i) v[i] = 0.f;
  }
  // Phase 1: register bits = vec (element bits 0..V-1) and hi (element bits 7..).
  fwht_bits<128, 0, 7>(v);
  // Transpose: row h of the team buffer holds elements h*128 + [0, 128).
#pragma unroll
  for (int h = 0; h < Sh::T; ++h) {
    const int g = grow + h;
    float* rowp = rows + h * 128;
    if constexpr (Sh::CE >= 4) {
#pragma unroll
      for (int k = 0; k < Sh::CE / 4; ++k) {
        const int q = tau * (Sh::CE / 4) + k;
        reinterpret_cast<float4*>(rowp)[q ^ (g & 31)] =
            make_float4(v[h * Sh::CE + 4 * k], v[h * Sh::CE + 4 * k + 1], v[h * Sh::CE + 4 * k + 2],
                        v[h * Sh::CE + 4 * k + 3]);
      }
    } else {
      const int q = tau >> 1;
      reinterpret_cast<float2*>(rowp)[((q ^ (g & 31)) << 1) + (tau & 1)] = make_float2(v[h * 2], v[h * 2 + 1]);
    }
  }
  team_sync<Sh::T>();
  {
    const int g = grow + tau;
    const float4* rowp = reinterpret_cast<const float4*>(rows + tau * 128);
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const float4 f = rowp[q ^ (g & 31)];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  team_sync<Sh::T>();
  // Phase 2: the mid bits (element bits V..6).
  fwht_bits<128, Sh::V, 7>(v);
}

template <int LOGB, bool IN_BF16, int MODE>
__global__ void __launch_bounds__(kThreads)
team_kernel(const void* __restrict__ x, int64_t units, float norm, int group, void* __restrict__ out0,
            void* __restrict__ out1) {
  using Sh = TeamShape<LOGB>;
  constexpr int TEAMS = kThreads / Sh::T;
  extern __shared__ float4 smem_f4[];
  float* buf = reinterpret_cast<float*>(smem_f4);
  const int team = threadIdx.x >> Sh::t;
  const int tau = threadIdx.x & (Sh::T - 1);
  float* rows = buf + team * Sh::T * 128;
  float v[128];
  for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * TEAMS; u0 < units;
       u0 += static_cast<int64_t>(gridDim.x) * TEAMS) {
    const int64_t u = u0 + team;
    const bool valid = u < units;
    const int64_t base = u << LOGB;
    team_rotate<LOGB, IN_BF16>(x, base, valid, tau, rows, team * Sh::T, v);
    if (valid) {
      const int64_t e0 = base + tau * 128;
      if constexpr (MODE == OUT_F32) {
        store_rotated<128, false>(v, norm, out0, e0);
      } else if constexpr (MODE == OUT_BF16) {
        store_rotated<128, true>(v, norm, out0, e0);
      } else if constexpr (MODE == OUT_INT4) {
        store_int4<128>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
      } else {
        store_mxfp4<128>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
      }
    }
  }
}

// Per-token int8, b >= 256: one CTA per row of n elements (n / b teams).
// blockDim = n / 128 rounded up to 32; dynamic shared memory = n floats.
template <int LOGB, bool IN_BF16>
__global__ void __launch_bounds__(256)
team_row_int8_kernel(const void* __restrict__ x, int64_t rows, int64_t n, float norm, int8_t* __restrict__ codes,
                     float* __restrict__ scales) {
  using Sh = TeamShape<LOGB>;
  extern __shared__ float4 smem_f4[];
  float* buf = reinterpret_cast<float*>(smem_f4);
  __shared__ float red[32];
  const int nthreads = static_cast<int>(n >> 7);
  const bool active = static_cast<int>(threadIdx.x) < nthreads;
  const int team = threadIdx.x >> Sh::t;
  const int tau = threadIdx.x & (Sh::T - 1);
  float* team_rows = buf + (active ? team * Sh::T * 128 : 0);
  float v[128];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t base = r * n + (static_cast<int64_t>(team) << LOGB);
    if (active) {
      team_rotate<LOGB, IN_BF16>(x, base, true, tau, team_rows, team * Sh::T, v);
    } else {
      // Idle threads still take part in every barrier of team_rotate.
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
      team_sync<Sh::T>();
      team_sync<Sh::T>();
    }
    float mz = 0.f;
#pragma unroll
    for (int i = 0; i < 128; ++i) mz = fmaxf(mz, fabsf(v[i]));
    const float m = cta_max(mz, red) * norm;
    if (active) store_int8<128>(v, norm, m, codes, base + tau * 128);
    if (threadIdx.x == 0) scales[r] = __fdiv_rn(m, 127.0f);
  }
}

}  // namespace hadq
