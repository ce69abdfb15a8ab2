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
//  * team kernels (256 <= b <= 8192): a team of T = b / P threads owns one
//    block, P = 2^p values per thread (P = 64 for b <= 2048, 128 above).
//    Index bits: e = [hi: t bits | mid: t bits | vec: p - t bits], t = log2 T.
//    Phase 1: each thread loads, for every hi value, one contiguous chunk of
//    2^(p-t) elements (the team reads P contiguous elements per hi value) and
//    runs the stages of its register bits (vec + hi).  A transpose through
//    shared memory (fp32 rows of P + 4 pad floats: conflict-free on both
//    sides for P = 128 and t >= 5, immediate offsets) hands every thread the P
//    consecutive elements with hi = its team index.  Phase 2 runs the
//    remaining stages (mid bits); the thread then holds a whole run of P
//    consecutive outputs for the quantizer (an int4 group of 128 at P = 64
//    spans a thread and its neighbour lane: one shuffle of the absmax).  When
//    the chunk holds at least 4 elements, the transpose stores every quad as
//    (e0, e2, e1, e3), so the element-bit-0 stage runs in phase 2 on packed
//    f32x2 pairs instead of as scalar adds in phase 1.  P = 64 halves the
//    registers of the short blocks, so more warps per SM hide the loads.
//
// The per-token int8 format needs the whole row before any code is written,
// so it has row kernels: one CTA per row, the same two layouts inside, and a
// CTA-wide absmax reduction before the epilogue.
//
// The normalisation 1/sqrt(b) is never applied element by element on the
// quantized paths: it is folded into the group absmax (fp32 rounding is
// monotone, so max|fl(z * c)| = fl(max|z| * c)) and into the reciprocal
// scale.  For even log2(b) it is an exact power of 2.
//
// Every kernel starts with the programmatic-dependent-launch handshake (see
// grid_dependency_sync) and prefetches its next unit of input into L2 while it
// computes the current one.
//
// Random Hadamard signs (Signs, SIGNS_BEFORE / SIGNS_AFTER) are compiled in
// only for SG = true (the deterministic kernels carry no trace of them): a
// thread always owns the same block columns in the same registers, so it
// reads its signs once into a bit mask and flips the loaded values (before)
// or the rotated values (after) with one XOR of the sign bit each.
#pragma once

#include "hadq_device.cuh"

namespace hadq {

constexpr int kThreads = 128;
constexpr int kRowFloats = 132;   // per-token team rows: 128 floats + one quad of padding

// log2 of the values per team thread for block 2^logb, and the team kernel's
// dynamic shared memory (one transpose row of P + 4 floats per thread).
__host__ __device__ constexpr int team_logp(int logb) { return logb <= 11 ? 6 : 7; }
__host__ __device__ constexpr int team_smem_bytes(int logb) { return kThreads * ((1 << team_logp(logb)) + 4) * 4; }

// ----------------------------------------------------------- segment kernels

// Segments of 64 bytes or more load whole sectors (256-bit loads: block 32
// bf16 -> MXFP4 0.904 -> 0.953 of HBM, block 128 fp32 -> int4 0.585 -> 0.811);
// 32-byte segments keep two 16-byte loads, which measured faster there
// (block 16 bf16 -> NVFP4 0.929, against 0.852 with one 256-bit load).
template <bool IN_BF16, int S>
constexpr bool kWideRun = S * (IN_BF16 ? 2 : 4) >= 64;

// A segment of S elements starts on a block boundary (b = 2^nbits divides S),
// so register i holds block column i mod b in every segment.
template <int S>
__device__ __forceinline__ void segment_sign_mask(const Signs& sg, int nbits, uint32_t (&sm)[(S + 31) / 32]) {
#pragma unroll
  for (int w = 0; w < (S + 31) / 32; ++w) sm[w] = 0u;
  if (sg.side == SIGNS_NONE) return;
  const int b = 1 << nbits;
  if (b >= 32) {
#pragma unroll
    for (int w = 0; w < (S + 31) / 32; ++w) sm[w] = sign_bits32(sg.s, (32 * w) & (b - 1));
  } else {
    uint32_t p = 0;                      // the b signs, repeated every b bits
    for (int i = 0; i < b; ++i) p |= neg_bit(sg.s, i) << i;
    for (int k = b; k < 32; k <<= 1) p |= p << k;
#pragma unroll
    for (int w = 0; w < (S + 31) / 32; ++w) sm[w] = p;
  }
}

// FULL: b == S, all LOGS stages unconditionally; otherwise the low nbits stages.
// An int4 group may span 2 or 4 consecutive segments (S >= 32, group <= 128):
// their threads are consecutive lanes, so the group absmax is one or two
// shuffles.  The grid loop is therefore warp-uniform: every lane runs every
// iteration (past the last segment with zeros, storing nothing), so that all
// lanes take part in the shuffles.
template <int LOGS, bool IN_BF16, int MODE, bool FULL, bool SG>
__global__ void __launch_bounds__(kThreads)
segment_kernel(const void* __restrict__ x, int64_t segs, int nbits, float norm, int group,
               void* __restrict__ out0, void* __restrict__ out1, Signs sg) {
  constexpr int S = 1 << LOGS;
  constexpr uint32_t kSegBytes = S * (IN_BF16 ? 2 : 4);
  grid_dependency_sync();
  uint32_t sm[(S + 31) / 32];
  if constexpr (SG) segment_sign_mask<S>(sg, nbits, sm);
  float v[S];
  const int lane = threadIdx.x & 31;
  for (int64_t s0 = static_cast<int64_t>(blockIdx.x) * kThreads; s0 < segs;
       s0 += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t s = s0 + threadIdx.x;
    const bool valid = s < segs;
    if constexpr (MODE != OUT_INT4) {
      if (!valid) break;   // no cross-lane work: the lanes past the end may leave
    }
    if (lane == 0 && valid) {   // the warp's next 32 segments are contiguous
      const int64_t nxt = s + static_cast<int64_t>(gridDim.x) * kThreads;
      if (nxt < segs) {
        const int64_t cnt = segs - nxt < 32 ? segs - nxt : 32;
        prefetch_l2(static_cast<const char*>(x) + nxt * kSegBytes, static_cast<uint32_t>(cnt) * kSegBytes);
      }
    }
    const int64_t e0 = s << LOGS;
    if (valid) {
      load_elems<IN_BF16, S, kWideRun<IN_BF16, S>>(x, e0, v);
    } else {
#pragma unroll
      for (int i = 0; i < S; ++i) v[i] = 0.f;
    }
    if constexpr (SG) {
      if (sg.side == SIGNS_BEFORE) apply_signs<S>(v, sm);
    }
    if constexpr (FULL) {
      fwht_bits<S, 0, LOGS>(v);
    } else {
      fwht_low<S>(v, nbits);
    }
    if constexpr (SG) {
      if (sg.side == SIGNS_AFTER) apply_signs<S>(v, sm);
    }
    if constexpr (MODE == OUT_F32) {
      store_rotated<false, S, false>(v, norm, out0, e0);
    } else if constexpr (MODE == OUT_BF16) {
      store_rotated<false, S, true>(v, norm, out0, e0);
    } else if constexpr (MODE == OUT_INT4) {
      store_int4_lanes<S>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0, valid);
    } else if constexpr (MODE == OUT_NVFP4) {
      store_nvfp4<false, S>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
    } else {
      store_mxfp4<false, S>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
    }
  }
}

// Per-token int8, b <= 128: one CTA per row, blockDim = n / S rounded up to 32 (<= 256).
template <int LOGS, bool IN_BF16, bool FULL, bool SG>
__global__ void __launch_bounds__(256)
segment_row_int8_kernel(const void* __restrict__ x, int64_t rows, int64_t n, int nbits, float norm,
                        int8_t* __restrict__ codes, float* __restrict__ scales, Signs sg) {
  constexpr int S = 1 << LOGS;
  grid_dependency_sync();
  uint32_t sm[(S + 31) / 32];
  if constexpr (SG) segment_sign_mask<S>(sg, nbits, sm);
  __shared__ float red[32];
  const int segs_row = static_cast<int>(n >> LOGS);
  const bool active = static_cast<int>(threadIdx.x) < segs_row;
  const int64_t row_bytes = n * (IN_BF16 ? 2 : 4);
  float v[S];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    if (threadIdx.x == 0 && r + gridDim.x < rows)
      prefetch_l2(static_cast<const char*>(x) + (r + gridDim.x) * row_bytes, static_cast<uint32_t>(row_bytes));
    const int64_t e0 = r * n + (static_cast<int64_t>(threadIdx.x) << LOGS);
    if (active) {
      load_elems<IN_BF16, S, kWideRun<IN_BF16, S>>(x, e0, v);
      if constexpr (SG) {
        if (sg.side == SIGNS_BEFORE) apply_signs<S>(v, sm);
      }
      if constexpr (FULL) {
        fwht_bits<S, 0, LOGS>(v);
      } else {
        fwht_low<S>(v, nbits);
      }
      if constexpr (SG) {
        if (sg.side == SIGNS_AFTER) apply_signs<S>(v, sm);
      }
    } else {
#pragma unroll
      for (int i = 0; i < S; ++i) v[i] = 0.f;
    }
    const float m = cta_max(absmax_regs(v, 0, S), red) * norm;
    if (active) store_int8<false, S>(v, norm, m, codes, e0);
    if (threadIdx.x == 0) scales[r] = int8_scale(m);
  }
}

// --------------------------------------------------------------- team kernels

template <int LOGB, int LOGP = team_logp(LOGB)>
struct TeamShape {
  static constexpr int P = 1 << LOGP;         // values per thread
  static constexpr int t = LOGB - LOGP;       // log2(threads per team)
  static constexpr int T = 1 << t;            // threads per team
  static constexpr int V = LOGP - t;          // vec bits per phase-1 chunk
  static constexpr int CE = 1 << V;           // elements per phase-1 chunk
  static constexpr int B = 1 << LOGB;
  static constexpr int ROW = P + 4;           // transpose row (floats), one quad of padding
  static constexpr int W = P / 32;            // sign-mask words
  static constexpr bool PERM = V >= 2;        // quads transposed as (e0, e2, e1, e3)
  static constexpr int C4 = CE / 4;           // quads per phase-1 chunk (0: float2 chunks)
  // Quad q of a transpose row is stored at swz(q).  Team thread tau writes
  // its chunk into quads tau * C4 + k of every row and reads back all quads of
  // row tau; the XOR (an involution inside the row) spreads the writes of the
  // 8 lanes a 128-byte wavefront serves over 8 distinct 16-byte bank groups
  // where the plain layout repeats them: C4 = 4 (b = 256: the 4 threads of a
  // team 16 quads apart, two teams 68 quads apart) and C4 = 2 (b = 512: 8
  // threads 2 quads apart).  The reads stay conflict-free (row stride 17 quads).
  static __device__ __forceinline__ int swz(int q) {
    if constexpr (C4 == 4) return q ^ ((q >> 2) & 3);
    if constexpr (C4 == 2) return q ^ ((q >> 3) & 1);
    return q;
  }
  static_assert(LOGB >= 8 && LOGB <= 13 && t >= 1 && V >= 1, "team kernels cover 256..8192");
};

template <int T>
__device__ __forceinline__ void team_sync() {
  if constexpr (T <= 32) {
    __syncwarp();
  } else {
    __syncthreads();
  }
}

// Sign mask of team thread tau.  BEFORE: phase-1 register h * CE + j holds
// block column h * P + tau * CE + j.  AFTER: register i holds output column
// tau * P + reg<PERM>(i).
template <int LOGB, int LOGP>
__device__ __forceinline__ void team_sign_mask(const Signs& sg, int tau, uint32_t (&sm)[TeamShape<LOGB, LOGP>::W]) {
  using Sh = TeamShape<LOGB, LOGP>;
#pragma unroll
  for (int w = 0; w < Sh::W; ++w) sm[w] = 0u;
  if (sg.side == SIGNS_AFTER) {
#pragma unroll
    for (int w = 0; w < Sh::W; ++w) {
      const uint32_t m = sign_bits32(sg.s, tau * Sh::P + 32 * w);
      sm[w] = Sh::PERM ? perm_quad_bits(m) : m;
    }
  } else if (sg.side == SIGNS_BEFORE) {
    if constexpr (Sh::CE >= 32) {
#pragma unroll
      for (int w = 0; w < Sh::W; ++w) {   // register 32 w + k = column (32 w / CE) * P + tau * CE + (32 w) % CE + k
        const int i = 32 * w;
        sm[w] = sign_bits32(sg.s, (i / Sh::CE) * Sh::P + tau * Sh::CE + (i % Sh::CE));
      }
    } else {
#pragma unroll
      for (int h = 0; h < Sh::T; ++h)   // registers h * CE + [0, CE) = columns h * P + tau * CE + [0, CE)
        sm[(h * Sh::CE) >> 5] |= sign_bits_small<Sh::CE>(sg.s, h * Sh::P + tau * Sh::CE) << ((h * Sh::CE) & 31);
    }
  }
}

// Rotate one block of 2^LOGB elements (element base `base`) by a team; on
// return v[0..P) holds the unnormalised outputs base + tau*P + [0, P) in
// register order TeamShape<LOGB, LOGP>::PERM.  `rows` is this team's T x ROW
// shared buffer.  With SG and `before`, the loaded values are first
// multiplied by the signs in `sm` (team_sign_mask, BEFORE layout).
template <int LOGB, int LOGP, bool IN_BF16, bool SG>
__device__ __forceinline__ void team_rotate(const void* __restrict__ x, int64_t base, bool valid, int tau,
                                            float* __restrict__ rows, float (&v)[1 << LOGP], bool before,
                                            const uint32_t (&sm)[TeamShape<LOGB, LOGP>::W]) {
  using Sh = TeamShape<LOGB, LOGP>;
  constexpr int P = Sh::P;
  if (valid) {
#pragma unroll
    for (int h = 0; h < Sh::T; ++h) load_elems<IN_BF16, Sh::CE>(x, base + h * P + tau * Sh::CE, &v[h * Sh::CE]);
    if constexpr (SG) {
      if (before) apply_signs<P>(v, sm);
    }
  } else {
#pragma unroll
    for (int i = 0; i < P; ++i) v[i] = 0.f;
  }
  // Phase 1: register index h * CE + j (j = element bits 0..V-1, h = element bits LOGB-t..).
  if constexpr (Sh::PERM) {
    fwht_bits<P, 1, LOGP>(v);          // element bit 0 waits for phase 2
  } else {
    fwht_bits<P, 0, LOGP>(v);
  }
  // Transpose: buffer row h holds elements h*P + [0, P).
#pragma unroll
  for (int h = 0; h < Sh::T; ++h) {
    float* rowp = rows + h * Sh::ROW;
    if constexpr (Sh::CE >= 4) {
#pragma unroll
      for (int k = 0; k < Sh::CE / 4; ++k) {
        const float* s = &v[h * Sh::CE + 4 * k];
        reinterpret_cast<float4*>(rowp)[Sh::swz(tau * (Sh::CE / 4) + k)] =
            Sh::PERM ? make_float4(s[0], s[2], s[1], s[3]) : make_float4(s[0], s[1], s[2], s[3]);
      }
    } else {
      reinterpret_cast<float2*>(rowp)[tau] = make_float2(v[h * 2], v[h * 2 + 1]);
    }
  }
  team_sync<Sh::T>();
  {
    const float4* rowp = reinterpret_cast<const float4*>(rows + tau * Sh::ROW);
#pragma unroll
    for (int q = 0; q < P / 4; ++q) {
      const float4 f = rowp[Sh::swz(q)];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  team_sync<Sh::T>();
  // Phase 2: the mid bits (element bits V..LOGP-1), and element bit 0 (register bit 1 under PERM).
  if constexpr (Sh::PERM) fwht_stage<P, 1>(v);
  fwht_bits<P, Sh::V, LOGP>(v);
}

template <int LOGB, bool IN_BF16, int MODE, bool SG>
__global__ void __launch_bounds__(kThreads, team_logp(LOGB) == 6 ? 4 : 3)
team_kernel(const void* __restrict__ x, int64_t units, float norm, int group, void* __restrict__ out0,
            void* __restrict__ out1, Signs sg) {
  constexpr int LOGP = team_logp(LOGB);
  using Sh = TeamShape<LOGB, LOGP>;
  constexpr int P = Sh::P;
  constexpr int TEAMS = kThreads / Sh::T;
  constexpr uint32_t kUnitBytes = Sh::B * (IN_BF16 ? 2 : 4);
  grid_dependency_sync();
  extern __shared__ float4 smem_f4[];
  float* buf = reinterpret_cast<float*>(smem_f4);
  const int team = threadIdx.x >> Sh::t;
  const int tau = threadIdx.x & (Sh::T - 1);
  float* rows = buf + team * Sh::T * Sh::ROW;
  uint32_t sm[Sh::W];
  if constexpr (SG) team_sign_mask<LOGB, LOGP>(sg, tau, sm);
  float v[P];
  for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * TEAMS; u0 < units;
       u0 += static_cast<int64_t>(gridDim.x) * TEAMS) {
    const int64_t u = u0 + team;
    if (tau == 0) {
      const int64_t nxt = u + static_cast<int64_t>(gridDim.x) * TEAMS;
      if (nxt < units) prefetch_l2(static_cast<const char*>(x) + nxt * kUnitBytes, kUnitBytes);
    }
    const bool valid = u < units;
    const int64_t base = u << LOGB;
    team_rotate<LOGB, LOGP, IN_BF16, SG>(x, base, valid, tau, rows, v, sg.side == SIGNS_BEFORE, sm);
    if constexpr (SG) {
      if (sg.side == SIGNS_AFTER) apply_signs<P>(v, sm);
    }
    const int64_t e0 = base + tau * P;
    if constexpr (MODE == OUT_INT4 && P < 128) {
      // A group of 128 spans this thread and lane ^ 1: every lane joins the
      // shuffle (invalid teams hold zeros and store nothing).
      if (group > P) {
        store_int4_pair<Sh::PERM>(v, norm, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0, valid);
      } else if (valid) {
        store_int4<Sh::PERM, P>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
      }
    } else if (valid) {
      if constexpr (MODE == OUT_F32) {
        store_rotated<Sh::PERM, P, false>(v, norm, out0, e0);
      } else if constexpr (MODE == OUT_BF16) {
        store_rotated<Sh::PERM, P, true>(v, norm, out0, e0);
      } else if constexpr (MODE == OUT_INT4) {
        store_int4<Sh::PERM, P>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
      } else if constexpr (MODE == OUT_NVFP4) {
        store_nvfp4<Sh::PERM, P>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
      } else {
        store_mxfp4<Sh::PERM, P>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
      }
    }
  }
}

// Per-token int8, b >= 256: one CTA per row of n elements (n / b teams).
// blockDim = n / 128 rounded up to 32; dynamic shared memory = n / 128 rows.
template <int LOGB, bool IN_BF16, bool SG>
__global__ void __launch_bounds__(256)
team_row_int8_kernel(const void* __restrict__ x, int64_t rows, int64_t n, float norm, int8_t* __restrict__ codes,
                     float* __restrict__ scales, Signs sg) {
  using Sh = TeamShape<LOGB, 7>;   // 128 values per thread (blockDim = n / 128)
  grid_dependency_sync();
  extern __shared__ float4 smem_f4[];
  float* buf = reinterpret_cast<float*>(smem_f4);
  __shared__ float red[32];
  const int nthreads = static_cast<int>(n >> 7);
  const bool active = static_cast<int>(threadIdx.x) < nthreads;
  const int team = threadIdx.x >> Sh::t;
  const int tau = threadIdx.x & (Sh::T - 1);
  float* team_rows = buf + (active ? team * Sh::T * Sh::ROW : 0);
  const int64_t row_bytes = n * (IN_BF16 ? 2 : 4);
  uint32_t sm[Sh::W];
  if constexpr (SG) team_sign_mask<LOGB, 7>(sg, tau, sm);
  float v[128];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    if (threadIdx.x == 0 && r + gridDim.x < rows)
      prefetch_l2(static_cast<const char*>(x) + (r + gridDim.x) * row_bytes, static_cast<uint32_t>(row_bytes));
    const int64_t base = r * n + (static_cast<int64_t>(team) << LOGB);
    if (active) {
      team_rotate<LOGB, 7, IN_BF16, SG>(x, base, true, tau, team_rows, v, sg.side == SIGNS_BEFORE, sm);
      if constexpr (SG) {
        if (sg.side == SIGNS_AFTER) apply_signs<128>(v, sm);
      }
    } else {
      // Idle threads still take part in every barrier of team_rotate.
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = 0.f;
      team_sync<Sh::T>();
      team_sync<Sh::T>();
    }
    const float m = cta_max(absmax_regs(v, 0, 128), red) * norm;
    if (active) store_int8<Sh::PERM, 128>(v, norm, m, codes, base + tau * 128);
    if (threadIdx.x == 0) scales[r] = int8_scale(m);
  }
}

}  // namespace hadq
