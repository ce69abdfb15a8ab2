// Rotation of blocks of b = K * 2^m elements: the non-power-of-2 sizes.
//
// "Rotation Transform" (AutoRound docs), section 1.5: for a dimension that is
// not a power of 2, get_hadamard_K(n) factors n = K * 2^m and combines a base
// Hadamard matrix of order K with a Sylvester block.  The base matrix here is
// Paley's second construction (R. E. A. C. Paley, "On orthogonal matrices",
// J. Math. Phys. 12, 1933) over GF(q), q = K / 2 - 1 = 1 (mod 4):
//
//   C   = [[0, 1^T], [1, Q]],  Q[a][b] = chi(a - b)   (conference matrix,
//         chi the quadratic character of GF(q); index 0 is the point at
//         infinity, then the field elements, element a + b*i at index a + p b),
//   H_K = C (x) A + I (x) B,   A = [[1, 1], [1, -1]],  B = [[1, -1], [-1, -1]],
//   H_b = H_K (x) H_(2^m)      (element e = k 2^m + j).
//
// H_K is symmetric, so H_b / sqrt(b) is its own inverse like the Sylvester
// rotation.  The two factors commute as stages, (H_K (x) I)(I (x) H_(2^m)),
// so one CTA per block runs:
//
//   load      the block into shared memory (16-byte loads);
//   K stage   for each column j the K values z_k = x[k 2^m + j], k = 2i + u,
//             are mixed by H_K.  With the packed pairs w_i = (z_2i + z_2i+1,
//             z_2i - z_2i+1), F = sum_{i >= 1} w_i and P_i = the sum of the w_i'
//             with chi(a_i' - a_i) = +1 (a_i = field element of row i >= 1),
//               y_0 = F + (w_0.y, -w_0.x),
//               y_i = w_0 + 2 P_i - F + w_i + (w_i.y, -w_i.x),
//             since row i of C sums its field columns to 2 P_i - (F - w_i)
//             and adds w_0, and B adds (w_i.y, -w_i.x).  The sign pattern is a
//             compile-time table, so a column costs about q^2 / 2 + 5 q packed
//             f32x2 adds; results go to a shared fp32 buffer whose 64-value
//             runs are padded to 68 words (128-bit accesses without conflicts);
//   2^m stage each thread takes one 64-value run of one sub-block: 6 butterfly
//             stages in registers, m - 6 more with shuffles across the
//             2^(m-6) neighbouring lanes that hold the sub-block; then the
//             epilogue of the butterfly kernels (1/sqrt(b), quantize, store).
#pragma once

#include <utility>

#include "hadq_device.cuh"

namespace hadq {
namespace ksize {

// GF(q), q = p^e (e = 1 or 2); GF(p^2) = GF(p)[i] / (i^2 - nu), nu a
// quadratic non-residue mod p.
template <int K> struct PaleyField;
template <> struct PaleyField<12> { static constexpr int p = 5, e = 1, nu = 0; };
template <> struct PaleyField<20> { static constexpr int p = 3, e = 2, nu = 2; };
template <> struct PaleyField<28> { static constexpr int p = 13, e = 1, nu = 0; };
template <> struct PaleyField<36> { static constexpr int p = 17, e = 1, nu = 0; };
template <> struct PaleyField<52> { static constexpr int p = 5, e = 2, nu = 2; };
template <> struct PaleyField<60> { static constexpr int p = 29, e = 1, nu = 0; };
template <> struct PaleyField<108> { static constexpr int p = 53, e = 1, nu = 0; };

template <int K>
struct Paley {
  static constexpr int p = PaleyField<K>::p, nu = PaleyField<K>::nu;
  static constexpr int q = PaleyField<K>::e == 1 ? p : p * p;
  static_assert(K == 2 * (q + 1), "Paley II: K = 2 (q + 1)");
  static_assert(q % 4 == 1, "Paley II needs q = 1 (mod 4)");

  // Index of s - t, of t^2 (element a + b*i at index a + p b).
  static constexpr int sub(int s, int t) { return (s % p - t % p + p) % p + p * ((s / p - t / p + p) % p); }
  static constexpr int square(int t) {
    const int a = t % p, b = t / p;
    return (a * a + nu * b * b) % p + p * ((2 * a * b) % p);
  }
  struct Table {
    bool plus[q][q];   // plus[s][t]: chi(s - t) = +1
  };
  static constexpr Table make() {
    Table tab{};
    bool sq[q] = {};
    for (int t = 1; t < q; ++t) sq[square(t)] = true;
    for (int s = 0; s < q; ++s)
      for (int t = 0; t < q; ++t) {
        const int d = sub(s, t);
        tab.plus[s][t] = d != 0 && sq[d];
      }
    return tab;
  }
  static constexpr Table tab = make();
};

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pr;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "add.rn.f32x2 pr, pa, pb;\n\t"
      "mov.b64 {%0, %1}, pr;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pr;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "sub.rn.f32x2 pr, pa, pb;\n\t"
      "mov.b64 {%0, %1}, pr;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// acc += w[T + 1] where chi(a_T - a_(I-1)) = +1 (row I of C, field column T).
template <int K, int I, int T>
__device__ __forceinline__ void add_if_plus(float2& acc, const float2* w) {
  if constexpr (Paley<K>::tab.plus[T][I - 1]) acc = add2(acc, w[T + 1]);
}

template <int K, int I, int... Ts>
__device__ __forceinline__ float2 plus_sum(const float2* w, std::integer_sequence<int, Ts...>) {
  float2 acc = make_float2(0.f, 0.f);
  (add_if_plus<K, I, Ts>(acc, w), ...);
  return acc;
}

// Output pair I >= 1: y_I = w_0 + 2 P_I - F + w_I + (w_I.y, -w_I.x), written to
// column-major rows 2I, 2I + 1 of the shared buffer through `put`.
template <int K, int I, class Put>
__device__ __forceinline__ void output_pair(const float2* w, float2 f, Put& put) {
  const float2 pp = plus_sum<K, I>(w, std::make_integer_sequence<int, Paley<K>::q>{});
  float2 t = __ffma2_rn(pp, make_float2(2.f, 2.f), w[0]);
  t = sub2(t, f);
  t = add2(t, w[I]);
  t = add2(t, make_float2(w[I].y, -w[I].x));
  put(2 * I, t.x);
  put(2 * I + 1, t.y);
}

template <int K, class Put, int... Is>
__device__ __forceinline__ void output_pairs(const float2* w, float2 f, Put& put, std::integer_sequence<int, Is...>) {
  (output_pair<K, Is + 1>(w, f, put), ...);
}

// One column: z_k = get(k) for k < K; y = z . H_K written through put(k, y_k).
template <int K, class Get, class Put>
__device__ __forceinline__ void kstage_column(Get& get, Put& put) {
  constexpr int q = Paley<K>::q;
  float2 w[q + 1];
#pragma unroll
  for (int i = 0; i <= q; ++i) {
    const float a = get(2 * i), b = get(2 * i + 1);
    w[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  float2 f = w[1];
#pragma unroll
  for (int i = 2; i <= q; ++i) f = add2(f, w[i]);
  const float2 y0 = add2(f, make_float2(w[0].y, -w[0].x));
  put(0, y0.x);
  put(1, y0.y);
  output_pairs<K>(w, f, put, std::make_integer_sequence<int, q>{});
}

constexpr int kMaxThreads = 512;
constexpr int kRunPad = 68;   // words per 64-value run in the shared buffer

// Bytes of dynamic shared memory for a block of b elements.
__host__ __device__ constexpr int64_t smem_bytes(int64_t b, int esize, bool sg) {
  return b * esize + (b / 64) * kRunPad * 4 + (sg ? b : 0) + 32 * 4;
}

// Blocks of b = K * 2^logs elements (64 <= 2^logs, b / 64 <= kMaxThreads),
// `units` of them back to back; blockDim.x = b / 64 rounded up to 32.
// MODE: OutMode, or -1 for per-token int8 (then b = n and a unit is a row).
template <int K, bool IN_BF16, int MODE, bool SG>
__global__ void __launch_bounds__(kMaxThreads)
ksize_kernel(const void* __restrict__ x, int64_t units, int logs, float norm, int group, void* __restrict__ out0,
             void* __restrict__ out1, Signs sg) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int ES = IN_BF16 ? 2 : 4;
  const int S = 1 << logs;
  const int b = K * S;
  const int rps = S >> 6;                      // 64-value runs per sub-block
  const int runs = K * rps;
  uint8_t* xs = smem;                          // the staged block
  float* wbuf = reinterpret_cast<float*>(smem + static_cast<size_t>(b) * ES);
  int8_t* ssm = reinterpret_cast<int8_t*>(wbuf + static_cast<size_t>(runs) * kRunPad);
  float* red = reinterpret_cast<float*>(ssm + (SG ? b : 0));
  const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31;
  const int64_t block_bytes = static_cast<int64_t>(b) * ES;

  if (tid == 0 && blockIdx.x < units)
    prefetch_l2(static_cast<const uint8_t*>(x) + blockIdx.x * block_bytes, static_cast<uint32_t>(block_bytes));
  grid_dependency_sync();
  if constexpr (SG) {
    for (int c = tid; c < b / 16; c += T)
      reinterpret_cast<uint4*>(ssm)[c] = reinterpret_cast<const uint4*>(sg.s)[c];
  }
  const bool before = SG && sg.side == SIGNS_BEFORE;

  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const uint8_t* xu = static_cast<const uint8_t*>(x) + u * block_bytes;
    if (tid == 0 && u + gridDim.x < units)
      prefetch_l2(xu + gridDim.x * block_bytes, static_cast<uint32_t>(block_bytes));
    for (int c = tid; c < b * ES / 16; c += T)
      reinterpret_cast<uint4*>(xs)[c] = ldg_stream(reinterpret_cast<const uint4*>(xu) + c);
    __syncthreads();   // block staged (and the previous block's runs consumed)

    // ------------------------------------------------------------ K stage
    for (int j = tid; j < S; j += T) {
      auto get = [&](int k) {
        const int e = k * S + j;
        float v;
        if constexpr (IN_BF16) {
          v = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(xs)[e]) << 16);
        } else {
          v = reinterpret_cast<const float*>(xs)[e];
        }
        if constexpr (SG) {
          if (before && ssm[e] < 0) v = -v;
        }
        return v;
      };
      float* wcol = wbuf + (j >> 6) * kRunPad + (j & 63);
      auto put = [&](int k, float v) { wcol[k * rps * kRunPad] = v; };
      kstage_column<K>(get, put);
    }
    __syncthreads();   // every run of the block mixed

    // ---------------------------------------------------------- 2^m stage
    const int r = tid;
    const bool active = r < runs;
    float v[64];
    if (active) {
      const float4* src = reinterpret_cast<const float4*>(wbuf + r * kRunPad);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 t = src[i];
        v[4 * i] = t.x;
        v[4 * i + 1] = t.y;
        v[4 * i + 2] = t.z;
        v[4 * i + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = 0.f;
    }
    fwht_bits<64, 0, 6>(v);
    for (int d = 0; d < logs - 6; ++d) {   // j bits 6 and up: the sub-block's neighbouring lanes
      const float sgn = ((lane >> d) & 1) ? -1.f : 1.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], 1 << d);
        v[i] = fmaf(v[i], sgn, o);   // lower lane: own + other; upper lane: other - own
      }
    }
    const int64_t e0 = u * b + static_cast<int64_t>(r) * 64;   // run r holds block columns 64 r ..
    if constexpr (SG) {
      if (!before && active) {
        const uint32_t m[2] = {sign_bits32(ssm, r * 64), sign_bits32(ssm, r * 64 + 32)};
        apply_signs<64>(v, m);
      }
    }
    if constexpr (MODE == OUT_INT4) {
      if (group == 128) {
        store_int4_pair<false>(v, norm, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0, active);
      } else if (active) {
        store_int4<false, 64>(v, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
      }
    } else if constexpr (MODE == OUT_MXFP4) {
      if (active) store_mxfp4<false, 64>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
    } else if constexpr (MODE == OUT_NVFP4) {
      if (active) store_nvfp4<false, 64>(v, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
    } else if constexpr (MODE == OUT_BF16) {
      if (active) store_rotated<false, 64, true>(v, norm, out0, e0);
    } else if constexpr (MODE == OUT_F32) {
      if (active) store_rotated<false, 64, false>(v, norm, out0, e0);
    } else {
      static_assert(MODE == -1, "per-token int8");
      const float m = cta_max(absmax_regs(v, 0, 64), red) * norm;
      if (active) store_int8<false, 64>(v, norm, m, static_cast<int8_t*>(out0), e0);
      if (tid == 0) static_cast<float*>(out1)[u] = int8_scale(m);
    }
  }
}

}  // namespace ksize
}  // namespace hadq
