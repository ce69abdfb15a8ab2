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
//               y_i = w_0 + 2 P_i - F + w_i + (w_i.y, -w_i.x)
//                   = (w_0 - F) + 2 (P_i + (z_2i, -z_2i+1)),
//             since row i of C sums its field columns to 2 P_i - (F - w_i)
//             and adds w_0, and B adds (w_i.y, -w_i.x).  The sign pattern is a
//             compile-time table and the P_i share pair sums, so a column
//             costs about q^2 / 3 + 4 q packed f32x2 operations; results go to
//             a shared fp32 buffer whose 64-value runs are padded to 68 words
//             (128-bit accesses without conflicts);
//   2^m stage each thread takes one 64-value run of one sub-block: 6 butterfly
//             stages in registers, and those of the remaining S_lo points
//             with shuffles across the neighbouring lanes that hold the
//             piece (the column stage has already mixed the pieces); then the
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

// The residue sums P_I share work: for every output pair the set of field
// columns T with chi(T - a_(I-1)) = +1 is covered by neighbouring index pairs
// {t, t + 1 (mod q)} (their sums w_t + w_(t+1) computed once for all rows)
// and single columns.  For prime q the sets are translates of the residues,
// so every row finds the same pairs (q = 13: 2 pairs + 2 singles, 52 packed
// adds for all P_I instead of 65).
template <int K>
struct PaleyCover {
  static constexpr int q = Paley<K>::q;
  struct Table {
    int cnt[q];            // terms of row r (output pair r + 1)
    int term[q][q];        // field column index of each term
    bool pair[q][q];       // the term is the pair sum starting at that column
    bool pair_used[q];     // some row uses the pair sum starting at column t
  };
  static constexpr Table make() {
    Table tab{};
    for (int r = 0; r < q; ++r) {
      bool in[q] = {}, used[q] = {};
      for (int t = 0; t < q; ++t) in[t] = Paley<K>::tab.plus[t][r];
      int n = 0;
      for (int t = 0; t < q; ++t) {
        const int u = (t + 1) % q;
        if (in[t] && !used[t] && in[u] && !used[u]) {
          used[t] = used[u] = true;
          tab.term[r][n] = t;
          tab.pair[r][n] = true;
          tab.pair_used[t] = true;
          ++n;
        }
      }
      for (int t = 0; t < q; ++t)
        if (in[t] && !used[t]) {
          used[t] = true;
          tab.term[r][n] = t;
          tab.pair[r][n] = false;
          ++n;
        }
      tab.cnt[r] = n;
    }
    return tab;
  }
  static constexpr Table tab = make();
};

template <int K, int T>
__device__ __forceinline__ void pair_sum_if_used(const float2* w, float2* ps) {
  if constexpr (PaleyCover<K>::tab.pair_used[T]) ps[T] = add2(w[T + 1], w[(T + 1) % Paley<K>::q + 1]);
}

template <int K, int... Ts>
__device__ __forceinline__ void pair_sums(const float2* w, float2* ps, std::integer_sequence<int, Ts...>) {
  (pair_sum_if_used<K, Ts>(w, ps), ...);
}

template <int K, int R, int J>
__device__ __forceinline__ float2 cover_term(const float2* w, const float2* ps) {
  constexpr int t = PaleyCover<K>::tab.term[R][J];
  if constexpr (PaleyCover<K>::tab.pair[R][J]) return ps[t];
  else return w[t + 1];
}

template <int K, int R, int... Js>
__device__ __forceinline__ float2 cover_sum(const float2* w, const float2* ps, std::integer_sequence<int, Js...>) {
  float2 acc = cover_term<K, R, 0>(w, ps);
  ((acc = add2(acc, cover_term<K, R, Js + 1>(w, ps))), ...);
  return acc;
}

// w[L] + ... + w[L + N - 1] as a balanced tree (short dependency chains).
template <int L, int N>
__device__ __forceinline__ float2 tree_sum(const float2* w) {
  if constexpr (N == 1) return w[L];
  else return add2(tree_sum<L, N / 2>(w), tree_sum<L + N / 2, N - N / 2>(w));
}

// Output pair I >= 1.  With a_i + b_i = 2 z_2i and b_i - a_i = -2 z_2i+1,
//   y_I = w_0 + 2 P_I - F + w_I + (w_I.y, -w_I.x) = G + 2 (P_I + (z_2I, -z_2I+1)),
// G = w_0 - F: two packed fused multiply-adds per pair.
template <int K, int I, class Put>
__device__ __forceinline__ void output_pair(const float* z, const float2* w, const float2* ps, float2 g, Put& put) {
  const float2 p = cover_sum<K, I - 1>(w, ps, std::make_integer_sequence<int, PaleyCover<K>::tab.cnt[I - 1] - 1>{});
  const float2 t = __ffma2_rn(make_float2(z[2 * I], z[2 * I + 1]), make_float2(1.f, -1.f), p);
  const float2 y = __ffma2_rn(t, make_float2(2.f, 2.f), g);
  put(2 * I, y.x);
  put(2 * I + 1, y.y);
}

template <int K, class Put, int... Is>
__device__ __forceinline__ void output_pairs(const float* z, const float2* w, const float2* ps, float2 g, Put& put,
                                             std::integer_sequence<int, Is...>) {
  (output_pair<K, Is + 1>(z, w, ps, g, put), ...);
}

// Compact form for the large orders (K >= 52), where keeping the inputs and
// the pair sums live as well would spill registers: the residue sums taken
// column by column, y_I = w_0 + 2 P_I - F + w_I + (w_I.y, -w_I.x).
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

template <int K, int I, class Put>
__device__ __forceinline__ void output_pair_compact(const float2* w, float2 f, Put& put) {
  const float2 pp = plus_sum<K, I>(w, std::make_integer_sequence<int, Paley<K>::q>{});
  float2 t = __ffma2_rn(pp, make_float2(2.f, 2.f), w[0]);
  t = sub2(t, f);
  t = add2(t, w[I]);
  t = add2(t, make_float2(w[I].y, -w[I].x));
  put(2 * I, t.x);
  put(2 * I + 1, t.y);
}

template <int K, class Put, int... Is>
__device__ __forceinline__ void output_pairs_compact(const float2* w, float2 f, Put& put,
                                                     std::integer_sequence<int, Is...>) {
  (output_pair_compact<K, Is + 1>(w, f, put), ...);
}

// One column: z_k = get(k) for k < K; y = z . H_K written through put(k, y_k).
// Every get happens before the first put, so get and put may address the
// same storage.  Orders up to 36 share pair sums and use the two-FMA output
// form; the large orders take the compact form.
template <int K, class Get, class Put>
__device__ __forceinline__ void kstage_column(Get& get, Put& put) {
  constexpr int q = Paley<K>::q;
  if constexpr (K >= 52) {
    float2 w[q + 1];
#pragma unroll
    for (int i = 0; i <= q; ++i) {
      const float a = get(2 * i), b = get(2 * i + 1);
      w[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
    const float2 f = tree_sum<1, q>(w);
    const float2 y0 = add2(f, make_float2(w[0].y, -w[0].x));
    put(0, y0.x);
    put(1, y0.y);
    output_pairs_compact<K>(w, f, put, std::make_integer_sequence<int, q>{});
  } else {
    float z[K];
#pragma unroll
    for (int k = 0; k < K; ++k) z[k] = get(k);
    float2 w[q + 1];
#pragma unroll
    for (int i = 0; i <= q; ++i)
      w[i] = make_float2(__fadd_rn(z[2 * i], z[2 * i + 1]), __fsub_rn(z[2 * i], z[2 * i + 1]));
    const float2 f = tree_sum<1, q>(w);
    float2 ps[q];
    pair_sums<K>(w, ps, std::make_integer_sequence<int, q>{});
    put(0, __fadd_rn(f.x, w[0].y));
    put(1, __fsub_rn(f.y, w[0].x));
    const float2 g = sub2(w[0], f);
    output_pairs<K>(z, w, ps, g, put, std::make_integer_sequence<int, q>{});
  }
}

constexpr int kMaxThreads = 512;
constexpr int kRunPad = 68;   // words per 64-value run in the shared buffer
constexpr int kMaxSlo = 2048; // longest butterfly the 2^m stage runs inside one warp

// Sign variants: none; one sign per block column shared by every block (the
// random Hadamard of "Rotation Transform", section 1.5); or RPBH, a
// permutation of the row's columns and one sign per column ("orbitquant
// 0.2.0", Method Conformance).
enum StageSigns : int { SGK_NONE = 0, SGK_BLOCK = 1, SGK_RPBH = 2 };

// Everything a launch passes: the row (unit) layout, the rotation block
// b = K * SHI * S_lo and the quantizer.
struct StageArgs {
  const void* x;
  int64_t units;       // units of unit_len elements, back to back
  int unit_len;        // elements per unit: a block, or a whole row (per-row quantizers, RPBH)
  int b;               // rotation block (divides unit_len)
  int logs_lo;         // log2 S_lo: the butterfly the 2^m stage runs per column
  float norm;          // 1 / sqrt(b) (NVFP4: also divided by the per-tensor scale)
  int group;           // int4 group
  int bits;            // codebook bits (2 or 4)
  void* out0;
  void* out1;
  Signs sg;            // SGK_BLOCK: b signs; SGK_RPBH: unit_len signs
  const int32_t* perm; // SGK_RPBH: v_e = x_perm[e]
  const double* thr;   // codebook thresholds (2^bits - 1, ascending)
};

// Bytes of dynamic shared memory for a unit of u elements.
__host__ __device__ constexpr int64_t smem_bytes(int64_t u, int esize, int sgk, int64_t b) {
  return u * esize + (u / 64) * kRunPad * 4 + (sgk == SGK_BLOCK ? b : 0) + 32 * 8 + 16 * 8;
}

// Sum over the CTA in double (blockDim.x a multiple of 32, every thread calling).
__device__ __forceinline__ double cta_sum(double v, double* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  v = lane < nw ? red[lane] : 0.0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();
  return v;
}

// Codebook index of z: the number of thresholds tau_j = hi_j + lo_j below z
// (binary search over L - 1 thresholds in shared memory; z - hi_j is exact
// near the threshold, so the comparison is that of z with tau_j).
template <int L>
__device__ __forceinline__ uint32_t codebook_index(float z, const float2* tau) {
  uint32_t idx = 0;
#pragma unroll
  for (int step = L / 2; step >= 1; step >>= 1) {
    const float2 t = tau[idx + step - 1];
    if (__fsub_rn(z, t.x) > t.y) idx += step;
  }
  return idx;
}

// Units of unit_len elements; blockDim.x = unit_len / 64 rounded up to 32.
// MODE: OutMode, or -1 for per-token int8.  K: 1 (Sylvester) or a Paley
// order; SHI: how many S_lo-long pieces the 2^m factor is cut into: the
// column stage mixes those pieces (H_SHI) along with the K sub-blocks, the
// butterfly stage runs the S_lo points that remain.  The host takes SHI as
// large as K * SHI <= 64 registers and S_lo >= 64 allow, which keeps the
// lane-crossing butterfly stages (shuffles) few or none: a 4096-point block
// is 64 x 64, both halves in registers.
template <int K, int SHI, bool IN_BF16, int MODE, int SGK>
__global__ void __launch_bounds__(kMaxThreads)
staged_kernel(const __grid_constant__ StageArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int ES = IN_BF16 ? 2 : 4;
  constexpr int KH = K * SHI;                  // values mixed per column
  const int U = a.unit_len, b = a.b;
  const int slo = 1 << a.logs_lo;
  const int runs = U >> 6;
  uint8_t* xs = smem;                          // the staged unit
  float* wbuf = reinterpret_cast<float*>(smem + static_cast<size_t>(U) * ES);
  int8_t* ssm = reinterpret_cast<int8_t*>(wbuf + static_cast<size_t>(runs) * kRunPad);
  double* red = reinterpret_cast<double*>(ssm + (SGK == SGK_BLOCK ? b : 0));
  float2* tau = reinterpret_cast<float2*>(red + 32);
  const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31;
  const int64_t unit_bytes = static_cast<int64_t>(U) * ES;
  const float norm = a.norm;

  if (tid == 0 && blockIdx.x < a.units)
    prefetch_l2(static_cast<const uint8_t*>(a.x) + blockIdx.x * unit_bytes, static_cast<uint32_t>(unit_bytes));
  grid_dependency_sync();
  if constexpr (SGK == SGK_BLOCK) {
    for (int c = tid; c < b / 16; c += T) reinterpret_cast<uint4*>(ssm)[c] = reinterpret_cast<const uint4*>(a.sg.s)[c];
  }
  const bool before = SGK == SGK_BLOCK && a.sg.side == SIGNS_BEFORE;

  for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
    const uint8_t* xu = static_cast<const uint8_t*>(a.x) + u * unit_bytes;
    if (tid == 0 && u + gridDim.x < a.units)
      prefetch_l2(xu + gridDim.x * unit_bytes, static_cast<uint32_t>(unit_bytes));
    for (int c = tid; c < U * ES / 16; c += T)
      reinterpret_cast<uint4*>(xs)[c] = ldg_stream(reinterpret_cast<const uint4*>(xu) + c);
    __syncthreads();   // unit staged (and the previous unit's runs consumed)

    // ------------------------------------------------------- column stage
    // Column (blk, j), j < S_lo: the KH values at unit offsets
    // blk b + (k SHI + h) S_lo + j are permuted / signed as the variant
    // says, mixed by H_SHI over h and H_K over k, and written to the runs.
    const int ncols = U / KH;
    for (int col = tid; col < ncols; col += T) {
      const int blk = col >> a.logs_lo, j = col & (slo - 1);
      const int base = blk * b + j;
      auto get = [&](int kh) {
        const int e = base + kh * slo;
        float v;
        int src = e;
        if constexpr (SGK == SGK_RPBH) {   // an entry outside the row is clamped (memory-safe, result unspecified)
          src = static_cast<int>(min(static_cast<unsigned>(__ldg(a.perm + e)), static_cast<unsigned>(U - 1)));
        }
        if constexpr (IN_BF16) {
          v = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(xs)[src]) << 16);
        } else {
          v = reinterpret_cast<const float*>(xs)[src];
        }
        if constexpr (SGK == SGK_RPBH) {
          if (__ldg(a.sg.s + e) < 0) v = -v;
        } else if constexpr (SGK == SGK_BLOCK) {
          if (before && ssm[e - blk * b] < 0) v = -v;
        }
        return v;
      };
      auto put = [&](int kh, float v) {
        const int e = base + kh * slo;
        wbuf[(e >> 6) * kRunPad + (e & 63)] = v;
      };
      // z[k SHI + h] = the value at (k SHI + h) S_lo + j: H_SHI over h for
      // every k (Sylvester), then H_K over k for every h.
      float z[KH];
#pragma unroll
      for (int kh = 0; kh < KH; ++kh) z[kh] = get(kh);
#pragma unroll
      for (int d = 1; d < SHI; d <<= 1) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
#pragma unroll
          for (int h = 0; h < SHI; ++h) {
            if ((h & d) == 0) {
              const float u = z[k * SHI + h], w = z[k * SHI + h + d];
              z[k * SHI + h] = __fadd_rn(u, w);
              z[k * SHI + h + d] = __fsub_rn(u, w);
            }
          }
        }
      }
      if constexpr (K == 1) {
#pragma unroll
        for (int h = 0; h < SHI; ++h) put(h, z[h]);
      } else {
#pragma unroll
        for (int h = 0; h < SHI; ++h) {
          auto geth = [&](int k) { return z[k * SHI + h]; };
          auto puth = [&](int k, float v) { put(k * SHI + h, v); };
          kstage_column<K>(geth, puth);
        }
      }
    }
    __syncthreads();   // every run of the unit mixed

    // ---------------------------------------------------- butterfly stage
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
    if (a.logs_lo >= 6) {
      fwht_bits<64, 0, 6>(v);
      for (int d = 0; d < a.logs_lo - 6; ++d) {   // column bits 6 and up: neighbouring lanes
        const float sgn = ((lane >> d) & 1) ? -1.f : 1.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, v[i], 1 << d);
          v[i] = fmaf(v[i], sgn, o);   // lower lane: own + other; upper lane: other - own
        }
      }
    } else {
      fwht_low<64>(v, a.logs_lo);      // blocks shorter than a run
    }
    const int64_t e0 = u * U + static_cast<int64_t>(r) * 64;   // run r holds unit columns 64 r ..
    if constexpr (SGK == SGK_BLOCK) {
      if (!before && active) {
        const int c0 = (r * 64) % b;
        uint32_t m[2] = {0u, 0u};
        if (b >= 64) {
          m[0] = sign_bits32(ssm, c0);
          m[1] = sign_bits32(ssm, c0 + 32);
        } else {   // the run holds 64 / b blocks, each with the same b signs
          for (int i = 0; i < 64; ++i)
            if (ssm[i & (b - 1)] < 0) m[i >> 5] |= 1u << (i & 31);
        }
        apply_signs<64>(v, m);
      }
    }
    if constexpr (MODE == OUT_INT4) {
      if (a.group == 128) {
        store_int4_pair<false>(v, norm, static_cast<uint8_t*>(a.out0), static_cast<__half*>(a.out1), e0, active);
      } else if (active) {
        store_int4<false, 64>(v, norm, a.group, static_cast<uint8_t*>(a.out0), static_cast<__half*>(a.out1), e0);
      }
    } else if constexpr (MODE == OUT_MXFP4) {
      if (active) store_mxfp4<false, 64>(v, norm, static_cast<uint8_t*>(a.out0), static_cast<uint8_t*>(a.out1), e0);
    } else if constexpr (MODE == OUT_NVFP4) {
      if (active) store_nvfp4<false, 64>(v, norm, static_cast<uint8_t*>(a.out0), static_cast<uint8_t*>(a.out1), e0);
    } else if constexpr (MODE == OUT_BF16) {
      if (active) store_rotated<false, 64, true>(v, norm, a.out0, e0);
    } else if constexpr (MODE == OUT_F32) {
      if (active) store_rotated<false, 64, false>(v, norm, a.out0, e0);
    } else if constexpr (MODE == OUT_CODEBOOK) {
      // Per-token norm (double sum of squares of the unnormalised rotation),
      // then the thresholds in the same units, tau_j = ||z|| t_j, split as an
      // exact float pair.
      double ss = 0.0;
#pragma unroll
      for (int i = 0; i < 64; ++i) ss = fma(static_cast<double>(v[i]), static_cast<double>(v[i]), ss);
      const double zn = sqrt(cta_sum(ss, red));
      const double zs = zn > 0.0 ? zn : 1.0;   // a zero row codes u = 0
      const int levels = 1 << a.bits;
      if (tid < levels - 1) {
        const double t = zs * a.thr[tid];
        const float hi = static_cast<float>(t);
        tau[tid] = make_float2(hi, static_cast<float>(t - static_cast<double>(hi)));
      }
      if (tid == 0) static_cast<float*>(a.out1)[u] = static_cast<float>(zn * static_cast<double>(norm));
      __syncthreads();
      if (active) {
        uint8_t* codes = static_cast<uint8_t*>(a.out0);
        if (a.bits == 4) {
          uint32_t w[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= codebook_index<16>(v[8 * q + i], tau) << (4 * i);
            w[q] = word;
          }
          store32(codes + (e0 >> 1), make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
        } else {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) word |= codebook_index<4>(v[16 * q + i], tau) << (2 * i);
            w[q] = word;
          }
          reinterpret_cast<uint4*>(codes + (e0 >> 2))[0] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      __syncthreads();   // tau may be rewritten for the next unit
    } else {
      static_assert(MODE == -1, "per-token int8");
      const float m = cta_max(absmax_regs(v, 0, 64), reinterpret_cast<float*>(red)) * norm;
      if (active) store_int8<false, 64>(v, norm, m, static_cast<int8_t*>(a.out0), e0);
      if (tid == 0) static_cast<float*>(a.out1)[u] = int8_scale(m);
    }
  }
}

}  // namespace ksize
}  // namespace hadq
