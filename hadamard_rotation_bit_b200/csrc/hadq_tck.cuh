// Tensor-core variant for blocks of b = K * 2^m elements with 2^m = 128 * HI
// (K a Paley order, HI = 1, 2, 4, ...), bf16 input.
//
// "Rotation Transform" (AutoRound docs), section 1.5: a size that is not a
// power of 2 is rotated by a base Hadamard matrix of order K combined with a
// Sylvester block, H_b = H_K (x) H_(2^m).  With 2^m = HI * 128 the Sylvester
// block splits once more, H_(2^m) = H_HI (x) H_128, over the index split
//
//     e = c * 128 + i,   c = k * HI + h   (chunk c of the block),
//
// so a block is C = K * HI consecutive 128-element chunks.  One tcgen05 MMA
// per block rotates every chunk by H_128,
//
//     D[i', c] = sum_i H_128[i', i] * X[c * 128 + i]
//
// (M = 128, K = 128, N = C rounded up to a multiple of 16): A = H_128 in
// shared memory, B = the chunks exactly as they lie in global memory,
// K-major with the 128-byte swizzle, loaded by the block-128 kernel's pair of
// 2-D tensor maps (columns beyond C hold whatever follows the block and are
// never read).  Operands are exact in bf16; products accumulate in fp32 in
// tensor memory.  TMEM lane i' then holds output index i' of every chunk of
// the block, so the rest of the rotation -- H_HI over h (Sylvester stages),
// then the Paley K-point mix over k for each h (the compile-time residue table
// of hadq_ksize.cuh) -- needs no data exchange between threads.  Each thread
// works through its lane in passes, with tensor memory as scratch, so that
// only one step's values are in registers at a time (at most K plus the
// mix's temporaries, not K * HI): pass A, per window of 4 values of k, H_HI
// and a write-back that puts each h's values in 4-column pieces; pass B, per
// h, the K-point mix (rotation outputs leave from here); pass C, per-token
// int8 only, after the row absmax is known, the codes.  The small register
// footprint buys epilogue warps: up to four groups of 4, against two when a
// thread held a value of every chunk.  A thread's outputs y[c * 128 + i'] are
// one per chunk, so for each chunk a warp writes 32 consecutive outputs.
//
// Roles as in the block-128 kernel: warp 0 TMA producer, warp 1 TMEM
// allocator and single-thread MMA issuer, then EPI_GROUPS groups of 4
// epilogue warps (one TMEM lane quarter each) taking whole blocks round-robin,
// each holding its block's accumulator until pass C has read it.  Per-token
// int8 takes a whole row per block (b = n) and joins the row absmax of the
// group's 4 warps in shared memory.  Every wait is bounded (hadq_tc_fault),
// and thread 0 first asks L2 to prefetch the CTA's first PREFETCH blocks.
#pragma once

#include <utility>

#include "hadq_ksize.cuh"
#include "hadq_tc.cuh"

namespace hadq {
namespace tc {

template <int K_, int HI_, int STAGES_, int EPI_GROUPS_, int PREFETCH_, bool GROUPED_ = false>
struct TckCfg {
  // GROUPED: the grouped quantizers (int4, MXFP4, NVFP4), which read the
  // finished block back through a per-warp 32 x 32 transpose in shared
  // memory (pass C) and join int4 group maxima of 64 / 128 across warps.
  static constexpr bool GROUPED = GROUPED_;
  static constexpr int K = K_, HI = HI_, C = K * HI;   // chunks per block
  static constexpr int NP = (C + 15) / 16 * 16;         // MMA N
  static_assert(C % 4 == 0 && NP <= 128, "a thread holds one output of every chunk in registers");
  static constexpr int STAGES = STAGES_;
  static constexpr int EPI_GROUPS = EPI_GROUPS_;
  static constexpr int PREFETCH = PREFETCH_;            // blocks per CTA prefetched into L2 at entry
  static constexpr int PANEL_BYTES = NP * 128;          // NP chunks x 64 bf16 (one K-panel)
  static constexpr int TILE_BYTES = 2 * PANEL_BYTES;    // B operand per block
  static constexpr int ACC_BUFS = 4;                    // accumulators at TMEM columns 0, 128, 256, 384
  static constexpr int THREADS = 32 * (2 + 4 * EPI_GROUPS);
  // kind::f16, fp32 accumulate, bf16 A and B, both K-major, N = NP, M = 128.
  static constexpr uint32_t IDESC =
      (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(NP >> 3) << 17) | (8u << 24);
  static constexpr int SM_A = 0;                        // H_128
  static constexpr int SM_B = SM_A + kABytes;           // STAGES x TILE_BYTES
  static constexpr int SM_BARS = SM_B + STAGES * TILE_BYTES;
  static constexpr int SM_RED = SM_BARS + 8 * (2 * STAGES + 2 * ACC_BUFS);   // per-token row max
  static constexpr int TR_WORDS = 32 * 32;               // one warp's transpose tile (16-byte granules swizzled)
  static constexpr int SM_TR = SM_RED + 4 * 4 * EPI_GROUPS;
  static constexpr int SM_GMAX = SM_TR + (GROUPED ? 4 * TR_WORDS * 4 * EPI_GROUPS : 0);   // [group][quarter][32]
  static constexpr int SM_SLOT = SM_GMAX + (GROUPED ? 4 * 4 * 32 * EPI_GROUPS : 0);
  static constexpr int SMEM_BYTES = SM_SLOT + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
  static_assert(SM_TR % 16 == 0, "16-byte reads of the transpose tiles");
  static_assert(PANEL_BYTES % 1024 == 0, "swizzle atoms of 8 chunks");
};

// 16, 8 and 4 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float* v) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// Columns [0, C) of this thread's lane, C a multiple of 4.
template <int C>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&z)[C]) {
  constexpr int C32 = C / 32 * 32;
#pragma unroll
  for (int c = 0; c < C32; c += 32) tmem_ld32(taddr + c, &z[c]);
  constexpr int R = C - C32;
  if constexpr (R & 16) tmem_ld16(taddr + C32, &z[C32]);
  if constexpr (R & 8) tmem_ld8(taddr + C32 + (R & 16), &z[C32 + (R & 16)]);
  if constexpr (R & 4) tmem_ld4(taddr + C32 + (R & 24), &z[C32 + (R & 24)]);
}

// Tensor-memory stores of 4, 8 and 32 consecutive 32-bit columns of this
// thread's lane (16: tmem_st16), and N-column loads and stores by size.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  tmem_st16(taddr, r);
  tmem_st16(taddr + 16, r + 16);
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float* v) {
  static_assert(N == 4 || N == 8 || N == 16 || N == 32, "4, 8, 16 or 32 columns");
  if constexpr (N == 4) tmem_ld4(taddr, v);
  else if constexpr (N == 8) tmem_ld8(taddr, v);
  else if constexpr (N == 16) tmem_ld16(taddr, v);
  else tmem_ld32(taddr, v);
}

template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t* r) {
  static_assert(N == 4 || N == 8 || N == 16 || N == 32, "4, 8, 16 or 32 columns");
  if constexpr (N == 4) tmem_st4(taddr, r);
  else if constexpr (N == 8) tmem_st8(taddr, r);
  else if constexpr (N == 16) tmem_st16(taddr, r);
  else tmem_st32(taddr, r);
}

// Columns [0, C) of this thread's lane from registers, C a multiple of 4.
template <int C>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float (&z)[C]) {
  uint32_t r[C];
#pragma unroll
  for (int i = 0; i < C; ++i) r[i] = __float_as_uint(z[i]);
  constexpr int C32 = C / 32 * 32;
#pragma unroll
  for (int c = 0; c < C32; c += 32) tmem_st32(taddr + c, &r[c]);
  constexpr int R = C - C32;
  if constexpr (R & 16) tmem_st16(taddr + C32, &r[C32]);
  if constexpr (R & 8) tmem_st8(taddr + C32 + (R & 16), &r[C32 + (R & 16)]);
  if constexpr (R & 4) tmem_st4(taddr + C32 + (R & 24), &r[C32 + (R & 24)]);
}

// Scratch layout of the tensor-memory epilogue: with HI > 1 the columns are
// windows of 4 values of k, each window holding its 4 * HI values h-major
// (position j W + 4 h + kl for chunk (4 j + kl) HI + h, W = 4 HI); with HI = 1
// position and chunk coincide.
template <int HI>
__host__ __device__ constexpr int scratch_chunk(int p) {
  if (HI == 1) return p;
  return (4 * (p / (4 * HI)) + (p % (4 * HI)) % 4) * HI + (p % (4 * HI)) / 4;
}

// Outputs of the values v[0, N) read from scratch positions P0 .. P0 + N - 1:
// chunk c = scratch_chunk(P0 + i) goes to element e0 + 128 c.  Per-token int8
// uses the arithmetic of the other kernels (codes rne(v * rn) by the
// round-magic FMA; a tiny scale divides per element).
template <int HI, int P0, int N, int MODE>
__device__ __forceinline__ void tck_emit(const float* v, float norm, float s, float rn, bool tiny, void* out0,
                                         int64_t e0) {
  if constexpr (MODE < 0) {
    uint8_t* codes = static_cast<uint8_t*>(out0) + e0;
    if (!tiny) {
      const float2 r2 = make_float2(rn, rn), m2 = make_float2(kRoundMagic, kRoundMagic);
#pragma unroll
      for (int i = 0; i < N; i += 2) {
        const float2 q = __ffma2_rn(make_float2(v[i], v[i + 1]), r2, m2);
        codes[128 * scratch_chunk<HI>(P0 + i)] = static_cast<uint8_t>(__float_as_uint(q.x) & 0xFFu);
        codes[128 * scratch_chunk<HI>(P0 + i + 1)] = static_cast<uint8_t>(__float_as_uint(q.y) & 0xFFu);
      }
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const float q = fminf(fmaxf(__fdiv_rn(v[i] * norm, s), -127.f), 127.f);
        codes[128 * scratch_chunk<HI>(P0 + i)] =
            static_cast<uint8_t>((__float_as_uint(__fadd_rn(q, kRoundMagic)) - kRoundMagicBits) & 0xFFu);
      }
    }
  } else if constexpr (MODE == OUT_BF16) {
    uint16_t* o = static_cast<uint16_t*>(out0) + e0;
#pragma unroll
    for (int i = 0; i < N; ++i) o[128 * scratch_chunk<HI>(P0 + i)] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i] * norm));
  } else {
    float* o = static_cast<float*>(out0) + e0;
#pragma unroll
    for (int i = 0; i < N; ++i) o[128 * scratch_chunk<HI>(P0 + i)] = v[i] * norm;
  }
}

// Pass C of the scratch epilogue: positions [P0, C) in pieces of up to 32.
template <int HI, int C, int MODE, int P0>
__device__ __forceinline__ void tck_emit_from(uint32_t tb, float norm, float s, float rn, bool tiny, void* out0,
                                              int64_t e0) {
  if constexpr (P0 < C) {
    constexpr int L = C - P0;
    constexpr int N = L >= 32 ? 32 : (L >= 16 ? 16 : (L >= 8 ? 8 : 4));
    float v[N];
    tmem_ldn<N>(tb + P0, v);
    tmem_wait_ld();
    tck_emit<HI, P0, N, MODE>(v, norm, s, rn, tiny, out0, e0);
    tck_emit_from<HI, C, MODE, P0 + N>(tb, norm, s, rn, tiny, out0, e0);
  }
}

// One block through tensor memory (tb = this thread's lane, first column of
// the block's accumulator).  Pass A (HI > 1): per window of 4 values of k,
// H_HI over h, written back h-major.  Pass B: per h, the K-point mix of the K
// values of that h (one 4-column piece per window), written back; rotation
// outputs leave from here.  Per-token int8 then joins the row absmax of the
// group and, pass C, reads the block back and stores the codes.  Returns after
// the last tensor-memory read of the block.
// The grouped quantizers (int4, MXFP4, NVFP4) store the mixed values back as
// per-token int8 does and, pass C, read them in batches of 32 positions: each
// warp transposes its 32 lanes x 32 positions through its shared tile `tr`, so
// that lane l holds the 32 consecutive outputs 32 quarter .. of the chunk at
// position p0 + l -- one MXFP4 group, two NVFP4 groups, or 32 of an int4
// group, whose absmax is joined across the group's warps through `gmax`.
template <int MODE>
__host__ __device__ constexpr bool tck_grouped() {
  return MODE == OUT_INT4 || MODE == OUT_MXFP4 || MODE == OUT_NVFP4 || MODE == OUT_MXFP4_BLOCKED ||
         MODE == OUT_NVFP4_BLOCKED;
}

template <int K, int HI, int MODE>
__device__ __forceinline__ void tck_block_scratch(uint32_t tb, float norm, void* out0, void* out1, int64_t t,
                                                  int64_t e0, int lane, int quarter, float* gred, int bar,
                                                  float* tr, float* gmax, int group, int scale_cols) {
  constexpr int C = K * HI, W = 4 * HI;
  constexpr bool STORE_BACK = MODE < 0 || tck_grouped<MODE>();
  if constexpr (HI > 1) {
#pragma unroll 1
    for (int j = 0; j < K / 4; ++j) {
      float v[W];
      tmem_ldn<W>(tb + j * W, v);
      tmem_wait_ld();
#pragma unroll
      for (int d = 1; d < HI; d <<= 1) {
#pragma unroll
        for (int i = 0; i < W; ++i) {
          if (((i % HI) & d) == 0) {
            const float u = v[i], w = v[i + d];
            v[i] = __fadd_rn(u, w);
            v[i + d] = __fsub_rn(u, w);
          }
        }
      }
      uint32_t o[W];
#pragma unroll
      for (int kl = 0; kl < 4; ++kl)
#pragma unroll
        for (int h = 0; h < HI; ++h) o[4 * h + kl] = __float_as_uint(v[kl * HI + h]);
      tmem_stn<W>(tb + j * W, o);
    }
    tmem_wait_st();
  }
  float mz = 0.f;
#pragma unroll 1
  for (int h = 0; h < HI; ++h) {
    float z[K];
    if constexpr (HI == 1) {
      tmem_ld_cols<K>(tb, z);
    } else {
#pragma unroll
      for (int j = 0; j < K / 4; ++j) tmem_ld4(tb + j * W + 4 * h, &z[4 * j]);
    }
    tmem_wait_ld();
    auto get = [&](int k) { return z[k]; };
    auto put = [&](int k, float v) { z[k] = v; };
    ksize::kstage_column<K>(get, put);
    if constexpr (STORE_BACK) {
      if constexpr (MODE < 0) mz = fmaxf(mz, absmax_regs(z, 0, K));
      if constexpr (HI == 1) {
        tmem_st_cols<K>(tb, z);
      } else {
#pragma unroll
        for (int j = 0; j < K / 4; ++j) {
          const uint32_t r[4] = {__float_as_uint(z[4 * j]), __float_as_uint(z[4 * j + 1]), __float_as_uint(z[4 * j + 2]),
                                 __float_as_uint(z[4 * j + 3])};
          tmem_st4(tb + j * W + 4 * h, r);
        }
      }
    } else {
      // Value k of this h is chunk k HI + h.
      float* of = static_cast<float*>(out0) + e0;
      uint16_t* ob = static_cast<uint16_t*>(out0) + e0;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int64_t off = 128 * (static_cast<int64_t>(k) * HI + h);
        if constexpr (MODE == OUT_BF16) ob[off] = __bfloat16_as_ushort(__float2bfloat16_rn(z[k] * norm));
        else of[off] = z[k] * norm;
      }
    }
  }
  if constexpr (MODE < 0) {
    tmem_wait_st();
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, off));
    if (lane == 0) gred[quarter] = mz;
    asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
    const float m = fmaxf(fmaxf(gred[0], gred[1]), fmaxf(gred[2], gred[3])) * norm;
    asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");   // gred may be rewritten next block
    const float s = int8_scale(m);
    const bool tiny = s > 0.f && s < 1.0e-36f;
    const float rn = (s >= 1.0e-36f && s <= 3.0e38f) ? code_factor(norm, s) : 0.f;
    tck_emit_from<HI, C, MODE, 0>(tb, norm, s, rn, tiny, out0, e0);
    if (quarter == 0 && lane == 0) static_cast<float*>(out1)[t] = s;
  } else if constexpr (tck_grouped<MODE>()) {
    tmem_wait_st();
    const int64_t blk0 = t * (static_cast<int64_t>(C) * 128);
    uint8_t* codes = static_cast<uint8_t*>(out0);
#pragma unroll 1
    for (int p0 = 0; p0 < C; p0 += 32) {
      float v[32];
      tmem_ld32(tb + p0, v);   // positions past C read unused accumulator columns and are not stored
      tmem_wait_ld();
      // Row j of the tile holds position p0 + j; its 16-byte granules are
      // XOR-swizzled by j % 8, so both the column writes and the row reads
      // (8 x 16 bytes) are free of bank conflicts.
#pragma unroll
      for (int j = 0; j < 32; ++j) tr[j * 32 + ((((lane >> 2) ^ j) & 7) << 2) + (lane & 3)] = v[j];
      __syncwarp();
      float u[32];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float4 q = *reinterpret_cast<const float4*>(tr + lane * 32 + ((g ^ (lane & 7)) << 2));
        u[4 * g] = q.x;
        u[4 * g + 1] = q.y;
        u[4 * g + 2] = q.z;
        u[4 * g + 3] = q.w;
      }
      __syncwarp();            // the tile is rewritten by the next batch
      const int p = p0 + lane;
      const bool ok = p < C;
      const int64_t eo = blk0 + 128 * static_cast<int64_t>(scratch_chunk<HI>(ok ? p : 0)) + 32 * quarter;
      if constexpr (MODE == OUT_MXFP4 || MODE == OUT_MXFP4_BLOCKED) {
        if (ok)
          store_mxfp4<false, 32>(u, norm, codes, static_cast<uint8_t*>(out1), eo,
                                 MODE == OUT_MXFP4_BLOCKED ? scale_cols : 0);
      } else if constexpr (MODE == OUT_NVFP4 || MODE == OUT_NVFP4_BLOCKED) {
        if (ok)
          store_nvfp4<false, 32>(u, norm, codes, static_cast<uint8_t*>(out1), eo,
                                 MODE == OUT_NVFP4_BLOCKED ? scale_cols : 0);
      } else {
        float m32 = absmax_regs(u, 0, 32);
        if (group > 32) {        // 64: this quarter and its neighbour; 128: all four
          gmax[quarter * 32 + lane] = m32;
          asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
          m32 = group == 64 ? fmaxf(m32, gmax[(quarter ^ 1) * 32 + lane])
                            : fmaxf(fmaxf(gmax[lane], gmax[32 + lane]), fmaxf(gmax[64 + lane], gmax[96 + lane]));
          asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");   // gmax is rewritten by the next batch
        }
        if (ok) store_int4_piece32(u, norm, m32, group, codes, static_cast<__half*>(out1), eo);
      }
    }
  }
}

// MODE: OUT_F32 / OUT_BF16, -1 for per-token int8 (one block = one row), or
// a grouped quantizer (OUT_INT4 with `group`, OUT_MXFP4, OUT_NVFP4 and their
// tiled-scale forms with scale_cols scale columns per row; C::GROUPED).
template <class C, int MODE>
__global__ void __launch_bounds__(C::THREADS, 1)
tck_kernel(const __grid_constant__ CUtensorMap map_p0, const __grid_constant__ CUtensorMap map_p1,
           const uint16_t* __restrict__ x, int64_t blocks, float norm, int group, void* __restrict__ out0,
           void* __restrict__ out1, int scale_cols) {
  constexpr bool PER_TOKEN = MODE < 0;
  static_assert(PER_TOKEN || MODE == OUT_F32 || MODE == OUT_BF16 || (tck_grouped<MODE>() && C::GROUPED),
                "rotation, per-token int8 or a grouped quantizer with its shared tiles");
  constexpr int NC = C::C;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  float* red = reinterpret_cast<float*>(smem + C::SM_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int64_t kBlockElems = static_cast<int64_t>(NC) * 128;

  if (threadIdx.x == 0) {
    int64_t t = blockIdx.x;
    for (int i = 0; i < C::PREFETCH && t < blocks; ++i, t += gridDim.x)
      prefetch_l2(x + t * kBlockElems, static_cast<uint32_t>(kBlockElems * 2));
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);             // the 4 warps of the group that took the block
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      grid_dependency_sync();
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < blocks; t += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (it >= C::STAGES && !mbar_wait(&empty[s], ph ^ 1)) {
          atomicOr(&hadq_tc_fault, kFaultProducer);
          drain_loads(full, C::STAGES, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::TILE_BYTES);
        uint8_t* dst = smem + C::SM_B + s * C::TILE_BYTES;
        const int c0 = static_cast<int>(t * NC);   // first chunk of the block
        tma_load_2d(dst, &map_p0, 0, c0, &full[s]);
        tma_load_2d(dst + C::PANEL_BYTES, &map_p1, 0, c0, &full[s]);
      }
    }
  } else {
    // A = H_128, K-major with the 128-byte swizzle (row m holds H[m][k] over k).
    for (int i = threadIdx.x - 32; i < 128 * 16; i += C::THREADS - 32) {
      const int m = i >> 4, kc = i & 15;
      uint32_t w[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int k = kc * 8 + 2 * p;
        w[p] = 0x3F803F80u | ((__popc(m & k) & 1u) << 15) | ((__popc(m & (k + 1)) & 1u) << 31);
      }
      const int panel = kc >> 3, chunk = kc & 7;
      const uint32_t off = panel * 16384 + m * 128 + ((chunk ^ (m & 7)) << 4);
      *reinterpret_cast<uint4*>(smem + C::SM_A + off) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(512));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(C::THREADS - 32) : "memory");
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 1) {
      // ------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t h_base = smem_u32(smem + C::SM_A);
        uint32_t it = 0;
        for (int64_t t = blockIdx.x; t < blocks; t += gridDim.x, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          const int b = it % C::ACC_BUFS;
          const uint32_t aph = (it / C::ACC_BUFS) & 1;
          if (!mbar_wait(&full[s], ph) || (it >= C::ACC_BUFS && !mbar_wait(&acc_empty[b], aph ^ 1))) {
            atomicOr(&hadq_tc_fault, kFaultMma);
            drain_mmas(empty, C::STAGES, it);
            break;
          }
          tc_fence_after();
          const uint32_t x_base = smem_u32(smem + C::SM_B + s * C::TILE_BYTES);
          const uint32_t d = tmem_base + b * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff_h = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t koff_x = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
            mma_bf16(d, smem_desc(h_base + koff_h, 16, 1024, kSwizzle128),
                     smem_desc(x_base + koff_x, 16, 1024, kSwizzle128), C::IDESC, kk > 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          mma_commit(&acc_full[b]);
        }
      }
    } else {
      // --------------------------------------------------------- epilogue
      grid_dependency_sync();
      const int quarter = warp & 3;
      const int group_id = (warp - 2) >> 2;
      const int ip = quarter * 32 + lane;       // output index within each chunk = TMEM lane
      uint32_t it = 0;
      bool failed = false;   // a wait ran out: skip the work, keep joining the group's barriers
      float* gred = red + 4 * group_id;
      const int bar = 2 + group_id;
      float* tr = reinterpret_cast<float*>(smem + C::SM_TR) + (warp - 2) * C::TR_WORDS;   // grouped quantizers
      float* gmax = reinterpret_cast<float*>(smem + C::SM_GMAX) + group_id * 128;
      for (int64_t t = blockIdx.x; t < blocks; t += gridDim.x, ++it) {
        if (static_cast<int>(it % C::EPI_GROUPS) != group_id) continue;
        const int b = it % C::ACC_BUFS;
        const uint32_t aph = (it / C::ACC_BUFS) & 1;
        if (!failed && !mbar_wait(&acc_full[b], aph)) {
          atomicOr(&hadq_tc_fault, kFaultEpilogue);
          failed = true;
        }
        if (failed) {
          if constexpr (PER_TOKEN) {
            asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
            asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
          } else if constexpr (MODE == OUT_INT4) {
            if (group > 32) {
              for (int p0 = 0; p0 < NC; p0 += 32) {
                asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
                asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
              }
            }
          }
          continue;
        }
        tc_fence_after();
        tck_block_scratch<C::K, C::HI, MODE>(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * 128, norm,
                                             out0, out1, t, t * kBlockElems + ip, lane, quarter, gred, bar, tr, gmax,
                                             group, scale_cols);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512));
  }
}

}  // namespace tc
}  // namespace hadq
