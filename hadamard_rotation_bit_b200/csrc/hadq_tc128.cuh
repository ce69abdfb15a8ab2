// Tensor-core variant for block-diagonal rotations with b = 128 (R3 per-head
// Q/K, R4 block rotation_size 128; "Rotation Transform", AutoRound docs,
// sections 1.1 and 1.2), bf16 input.
//
// A row of n elements is n / 128 contiguous blocks; every block is a row of
// the matrix X_blk, and the rotation of all blocks at once is one product
//
//     D = X_blk . H_128      (M = 128 blocks, K = 128, N = 128 outputs),
//
// exact in bf16 operands, accumulated in fp32 in tensor memory.  TMEM lane m
// then holds the whole rotated block m: the epilogue only quantizes (every
// int4 / MXFP4 group lies inside one thread), with no butterflies and no
// data exchange between threads.  Per-token int8 takes one row per tile
// (n / 128 <= 128 blocks) and reduces the row absmax across the 4 warps of
// the epilogue group that owns the tile.
//
// A = X_blk is K-major with the 128-byte swizzle, loaded by TMA (each CTA
// its own tiles) as two 64-element K-panels per tile from two 2-D tensor maps
// whose bases differ by 128 bytes; B = H_128 (symmetric) is built in shared
// memory in the same layout.  Random Hadamard signs cost nothing per tile:
// they are folded into B when it is built, as diag(s) H_128 for signs before
// the rotation and H_128 diag(s) for signs after it (section 1.5), so the
// MMA applies the signed rotation and the epilogue is the unsigned one.  Roles as in hadq_tc.cuh: warp 0 TMA producer,
// warp 1 TMEM allocator + single-thread MMA issuer, warps 2.. EPI_GROUPS
// groups of 4 epilogue warps taking whole tiles round-robin.  Waits are
// bounded (hadq_tc_fault).  As there, thread 0 first asks L2 to prefetch the
// CTA's first PREFETCH tiles (a hint, so it may precede the wait for the
// previous kernel).  These kernels run for tens of microseconds or more, so a
// deep prefetch (8 tiles = 256 KB per CTA) pays: it keeps HBM busy through the
// previous kernel's drain and the dependency release, which a short prefetch
// leaves idle (8192 x 14336 int8: 54.5 us with 2 tiles, 51.5 us with 8).
#pragma once

#include "hadq_tc.cuh"

namespace hadq {
namespace tc {

template <int STAGES_, int EPI_GROUPS_, int PREFETCH_>
struct Tc128Cfg {
  static constexpr int STAGES = STAGES_;
  static constexpr int EPI_GROUPS = EPI_GROUPS_;
  static constexpr int PREFETCH = PREFETCH_;                    // tiles per CTA prefetched into L2 at entry
  static constexpr int PANEL_BYTES = 128 * 128;                 // 128 blocks x 64 bf16
  static constexpr int TILE_BYTES = 2 * PANEL_BYTES;            // A operand per tile (<= 128 blocks)
  static constexpr int ACC_BUFS = 4;                            // 4 x 128 TMEM columns
  static constexpr int THREADS = 32 * (2 + 4 * EPI_GROUPS);
  // kind::f16, fp32 accumulate, bf16 A and B, both K-major, N = 128, M = 128.
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (16u << 17) | (8u << 24);
  static constexpr int SM_B = 0;                                // H_128
  static constexpr int SM_A = SM_B + kABytes;                   // STAGES x TILE_BYTES
  static constexpr int SM_BARS = SM_A + STAGES * TILE_BYTES;
  static constexpr int SM_RED = SM_BARS + 8 * (2 * STAGES + 2 * ACC_BUFS);   // per-token row max
  static constexpr int SM_SLOT = SM_RED + 4 * 4 * EPI_GROUPS;
  static constexpr int SMEM_BYTES = SM_SLOT + 16 + 1024;
};

// MODE: OUT_F32 / OUT_BF16 / OUT_INT4 / OUT_MXFP4 / OUT_NVFP4, or -1 for
// per-token int8.  sg: none, or signs on either side (folded into B).
// E > 0: blocks of b = 2^E * 128, H_b = H_(2^E) (x) H_128 over the element
// index e = j * 128 + i.  The block's 2^E chunks j are 2^E neighbouring TMEM
// lanes of one warp, so after the MMA the remaining E stages pair lanes by
// shuffles (one shuffle and one fused multiply-add per value and stage); every
// quantizer group still lies inside one chunk.  No signs and no per-token
// int8 then (the host keeps those at b = 128).
template <class C, int MODE, int E = 0>
__global__ void __launch_bounds__(C::THREADS, 1)
tc128_kernel(const __grid_constant__ CUtensorMap map_p0, const __grid_constant__ CUtensorMap map_p1,
             const uint16_t* __restrict__ x, int64_t blocks, int blocks_per_tile, float norm, int group,
             void* __restrict__ out0, void* __restrict__ out1, Signs sg, int scale_cols) {
  constexpr bool PER_TOKEN = MODE < 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  float* red = reinterpret_cast<float*>(smem + C::SM_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles = (blocks + blocks_per_tile - 1) / blocks_per_tile;
  const uint32_t tile_bytes = static_cast<uint32_t>(blocks_per_tile) * 256u;   // both panels

  if (threadIdx.x == 0) {
    int64_t t = blockIdx.x;
    for (int i = 0; i < C::PREFETCH && t < tiles; ++i, t += gridDim.x) {
      const int64_t b0 = t * blocks_per_tile;   // a tile is blocks [b0, b1), contiguous
      const int64_t b1 = b0 + blocks_per_tile < blocks ? b0 + blocks_per_tile : blocks;
      prefetch_l2(x + b0 * 128, static_cast<uint32_t>((b1 - b0) * 256));
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);             // the 4 warps of the group that took the tile
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      grid_dependency_sync();
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (it >= C::STAGES && !mbar_wait(&empty[s], ph ^ 1)) {
          atomicOr(&hadq_tc_fault, kFaultProducer);
          drain_loads(full, C::STAGES, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], tile_bytes);
        uint8_t* dst = smem + C::SM_A + s * C::TILE_BYTES;
        const int b0 = static_cast<int>(t * blocks_per_tile);
        tma_load_2d(dst, &map_p0, 0, b0, &full[s]);
        tma_load_2d(dst + C::PANEL_BYTES, &map_p1, 0, b0, &full[s]);
      }
    }
  } else {
    // B = H_128, K-major with the 128-byte swizzle (row n holds B[n][k] over
    // k; D = A B^T).  With signs, B[n][k] = H[n][k] s[k] (before) or s[n]
    // H[n][k] (after): one XOR of the bf16 sign bit.  The signs are caller
    // memory, so they are read only after the previous kernel has completed.
    const bool signed_b = sg.side != SIGNS_NONE;
    if (signed_b) grid_dependency_sync();
    for (int i = threadIdx.x - 32; i < 128 * 16; i += C::THREADS - 32) {
      const int m = i >> 4, kc = i & 15;
      uint32_t w[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int k = kc * 8 + 2 * p;
        w[p] = 0x3F803F80u | ((__popc(m & k) & 1u) << 15) | ((__popc(m & (k + 1)) & 1u) << 31);
      }
      if (signed_b) {
        if (sg.side == SIGNS_BEFORE) {
          // s[kc*8 .. kc*8+7]: 8-byte aligned (s is 16-byte aligned); a negative
          // entry has bit 7 set, which lands on the bf16 sign bit.
          const uint2 q = *reinterpret_cast<const uint2*>(sg.s + kc * 8);
          const uint32_t q0 = q.x & 0x80808080u, q1 = q.y & 0x80808080u;
          w[0] ^= __byte_perm(q0, 0u, 0x1404);
          w[1] ^= __byte_perm(q0, 0u, 0x3424);
          w[2] ^= __byte_perm(q1, 0u, 0x1404);
          w[3] ^= __byte_perm(q1, 0u, 0x3424);
        } else if (neg_bit(sg.s, m)) {
#pragma unroll
          for (int p = 0; p < 4; ++p) w[p] ^= 0x80008000u;
        }
      }
      const int panel = kc >> 3, chunk = kc & 7;
      const uint32_t off = panel * 16384 + m * 128 + ((chunk ^ (m & 7)) << 4);
      *reinterpret_cast<uint4*>(smem + C::SM_B + off) = make_uint4(w[0], w[1], w[2], w[3]);
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
        const uint32_t h_base = smem_u32(smem + C::SM_B);
        uint32_t it = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
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
          const uint32_t a_base = smem_u32(smem + C::SM_A + s * C::TILE_BYTES);
          const uint32_t d = tmem_base + b * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16(d, smem_desc(a_base + koff, 16, 1024, kSwizzle128), smem_desc(h_base + koff, 16, 1024, kSwizzle128),
                     C::IDESC, kk > 0 ? 1u : 0u);
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
      const int m = quarter * 32 + lane;        // block within the tile = TMEM lane
      uint32_t it = 0;
      bool failed = false;   // a wait ran out: skip the work, keep joining the group's barriers
      float* gred = red + 4 * group_id;
      const int bar = 2 + group_id;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
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
          }
          continue;
        }
        tc_fence_after();
        float z[128];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * 128;
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld32(taddr + c, &z[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        if constexpr (E > 0) {
          static_assert(MODE >= 0 && E <= 5, "blocks of up to 32 chunks, one warp");
          // Chunk j = lane bits 0 .. E-1 of its block: the lower lane of each
          // pair takes z + z', the upper z' - z.
#pragma unroll
          for (int d = 0; d < E; ++d) {
            const float sgn = ((lane >> d) & 1) ? -1.f : 1.f;
#pragma unroll
            for (int i = 0; i < 128; ++i) z[i] = fmaf(z[i], sgn, __shfl_xor_sync(0xffffffffu, z[i], 1 << d));
          }
        }
        const int64_t blk = t * blocks_per_tile + m;
        const bool ok = m < blocks_per_tile && blk < blocks;
        const int64_t e0 = blk * 128;
        if constexpr (PER_TOKEN) {
          // One row per tile: the row absmax over the group's 128 threads.
          float mz = ok ? absmax_regs(z, 0, 128) : 0.f;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, off));
          if (lane == 0) gred[quarter] = mz;
          asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
          const float mrow = fmaxf(fmaxf(gred[0], gred[1]), fmaxf(gred[2], gred[3])) * norm;
          asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");   // gred may be rewritten next tile
          if (ok) store_int8<false, 128>(z, norm, mrow, static_cast<int8_t*>(out0), e0);
          if (m == 0) static_cast<float*>(out1)[t] = int8_scale(mrow);
        } else if constexpr (MODE == OUT_INT4) {
          if (ok) store_int4<false, 128>(z, norm, group, static_cast<uint8_t*>(out0), static_cast<__half*>(out1), e0);
        } else if constexpr (MODE == OUT_MXFP4 || MODE == OUT_MXFP4_BLOCKED) {
          // the tiled GEMM scale layout: scale_cols = n / 32 columns per row
          if (ok)
            store_mxfp4<false, 128>(z, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0,
                                    MODE == OUT_MXFP4_BLOCKED ? scale_cols : 0);
        } else if constexpr (MODE == OUT_NVFP4 || MODE == OUT_NVFP4_BLOCKED) {
          if (ok)
            store_nvfp4<false, 128>(z, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0,
                                    MODE == OUT_NVFP4_BLOCKED ? scale_cols : 0);
        } else if constexpr (MODE == OUT_BF16) {
          if (ok) store_rotated<false, 128, true>(z, norm, out0, e0);
        } else {
          if (ok) store_rotated<false, 128, false>(z, norm, out0, e0);
        }
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
