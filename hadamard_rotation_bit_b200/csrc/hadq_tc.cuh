// Tensor-core variant for large full-size rotations (b = n = 2^(7 + LO),
// LO = 5 or 6, i.e. n = 4096 or 8192), bf16 input.
//
// The Sylvester matrix factors as H_n = H_128 (x) H_(2^LO) over the index
// split e = hi * 2^LO + lo ("Rotation Transform", AutoRound docs, section
// 1.5 construction).  Per tile of R = 128 / 2^LO rows, one tcgen05 MMA applies
// H_128 to the high bits of every row at once,
//
//     D[hi', (r, lo)] = sum_hi H_128[hi', hi] * X[r][hi * 2^LO + lo],
//
// with M = 128 (hi'), K = 128 (hi), N = 128 (R rows x 2^LO lo values).  The
// operands are exact in bf16 (X is bf16, H is +/-1) and the products are
// accumulated in fp32 in tensor memory; this replaces 7 of the log2(n)
// butterfly stages.  The epilogue reads one TMEM lane (= one hi') per thread,
// runs the remaining LO butterfly stages over lo in registers and quantizes.
//
// Roles (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: X tiles (box 2^LO x 128 x R, 64B/128B swizzle,
//               no multicast) into a ring of kStages shared-memory stages;
//   warp 1      TMEM allocator and MMA issuer (one thread), double-buffered
//               accumulators (kAccBufs x 128 columns);
//   warps 2..5  epilogue, warp w reading TMEM lanes 32 * (w % 4) + [0, 32).
// Every mbarrier wait is bounded; on timeout the kernel records a fault in
// hadq_tc_fault and stops issuing work.
#pragma once

#include <cuda.h>
#include "hadq_device.cuh"

namespace hadq {
namespace tc {

constexpr int kStages = 5;
constexpr int kAccBufs = 4;
constexpr int kAccCols = 128;            // fp32 accumulator columns per tile
constexpr int kTmemCols = kAccBufs * kAccCols;
constexpr int kTileBytes = 128 * 128 * 2;  // B operand: K = 128 rows x N = 128 bf16
constexpr int kABytes = 128 * 128 * 2;     // A operand: H_128 in bf16
constexpr int kThreads = 192;
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded mbarrier waits (~seconds)

// Fault codes written to hadq_tc_fault.
constexpr unsigned kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Wait for the phase with parity `parity` to complete; false after kSpinLimit tries.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// UMMA shared-memory matrix descriptor (sm_100 format: start, leading and
// stride byte offsets in 16-byte units, version 1, swizzle mode in bits 61..63).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (static_cast<uint64_t>(swizzle) << 61);
}

constexpr uint32_t kSwizzle128 = 2, kSwizzle64 = 4;

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A K-major,
// B MN-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            (static_cast<uint32_t>(kAccCols >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ unsigned int hadq_tc_fault;   // sticky fault bits (bounded waits that ran out)

// Shared-memory layout (offsets from a 1024-byte aligned base).
struct Smem {
  static constexpr int kA = 0;                                   // H_128, 2 K-panels x 16 KB
  static constexpr int kB = kA + kABytes;                        // kStages x 32 KB
  static constexpr int kBars = kB + kStages * kTileBytes;        // mbarriers
  static constexpr int kTmemSlot = kBars + 8 * (2 * kStages + 2 * kAccBufs);
  static constexpr int kEnd = kTmemSlot + 16;
  static constexpr int kDynamicBytes = kEnd + 1024;              // + alignment slack
};

// Epilogue for one row of one tile: z holds the 2^LO values of TMEM lane hi'
// (after the tensor-core stage over hi); finish the butterfly over lo and emit.
template <int LO, int MODE>
__device__ __forceinline__ void tc_emit_row(float (&z)[1 << LO], int hi, int64_t row, bool row_ok, int n, float norm,
                                            int group, void* __restrict__ out0, void* __restrict__ out1) {
  constexpr int L = 1 << LO;
  fwht_bits<L, 0, LO>(z);
  const int64_t e0 = row * n + static_cast<int64_t>(hi) * L;   // first output element of this thread
  if constexpr (MODE == OUT_INT4) {
    // Groups of `group` outputs = L values x (group / L) consecutive lanes.
    float mz = absmax_regs(z, 0, L);
    if constexpr (L == 32) {
      if (group >= 64) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 1));
      if (group >= 128) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 2));
    } else {
      if (group == 128) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 1));
    }
    float mz_lo = mz, mz_hi = mz;
    if constexpr (L == 64) {
      if (group == 32) {
        mz_lo = absmax_regs(z, 0, 32);
        mz_hi = absmax_regs(z, 32, 32);
      }
    }
#pragma unroll
    for (int j = 0; j < L / 32; ++j) {
      const float m = (j == 0 ? mz_lo : mz_hi) * norm;
      const __half s16 = __float2half_rn(__fdiv_rn(m, 7.0f));
      const float s = __half2float(s16);
      const float r = (s > 0.f && s <= 65504.f) ? __frcp_rn(s) : 0.f;
      const float rn = r * norm;
      uint4 w;
      if ((j == 0 ? mz_lo : mz_hi) * rn < 7.25f) {
        w = make_uint4(pack_int4x8<false>(z, 32 * j, rn), pack_int4x8<false>(z, 32 * j + 8, rn),
                       pack_int4x8<false>(z, 32 * j + 16, rn), pack_int4x8<false>(z, 32 * j + 24, rn));
      } else {
        w = make_uint4(pack_int4x8_clamped<false>(z, 32 * j, rn), pack_int4x8_clamped<false>(z, 32 * j + 8, rn),
                       pack_int4x8_clamped<false>(z, 32 * j + 16, rn), pack_int4x8_clamped<false>(z, 32 * j + 24, rn));
      }
      if (row_ok) {
        reinterpret_cast<uint4*>(static_cast<uint8_t*>(out0) + ((e0 + 32 * j) >> 1))[0] = w;
        if (((e0 + 32 * j) % group) == 0) static_cast<__half*>(out1)[(e0 + 32 * j) / group] = s16;
      }
    }
  } else if constexpr (MODE == OUT_MXFP4) {
    if (row_ok) store_mxfp4<false, L>(z, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
  } else if constexpr (MODE == OUT_BF16) {
    if (row_ok) store_rotated<false, L, true>(z, norm, out0, e0);
  } else {
    if (row_ok) store_rotated<false, L, false>(z, norm, out0, e0);
  }
}

template <int LO, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_rotate_kernel(const __grid_constant__ CUtensorMap xmap, int64_t rows, int n, float norm, int group,
                 void* __restrict__ out0, void* __restrict__ out1) {
  constexpr int L = 1 << LO;          // lo values per row per TMEM lane
  constexpr int R = 128 / L;          // rows per tile
  static_assert(LO == 5 || LO == 6, "tensor-core path covers n = 4096 and 8192");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::kTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles = (rows + R - 1) / R;

  // A = H_128 (K-major, 128-byte swizzle, two K-panels of 64): element (m, k)
  // at panel (k / 64) + m * 128 + (k % 64) * 2 bytes, 16-byte chunk index
  // XOR-ed with (m % 8).
  for (int i = threadIdx.x; i < 128 * 128 / 8; i += kThreads) {
    const int m = i >> 4, kc = i & 15;                // 8 consecutive k per 16-byte chunk
    uint32_t w[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t h2 = 0;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int k = kc * 8 + p * 2 + q;
        const uint32_t neg = __popc(m & k) & 1;
        h2 |= (neg ? 0xBF80u : 0x3F80u) << (16 * q);  // bf16 -1 / +1
      }
      w[p] = h2;
    }
    const int panel = kc >> 3, chunk = kc & 7;
    const uint32_t off = panel * 16384 + m * 128 + ((chunk ^ (m & 7)) << 4);
    *reinterpret_cast<uint4*>(smem + Smem::kA + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);      // one arrival per epilogue warp
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // A visible to the tensor core
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  grid_dependency_sync();   // x may be written by the previous kernel in the stream

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (it >= kStages && !mbar_wait(&empty[s], ph ^ 1)) {
          atomicOr(&hadq_tc_fault, kFaultProducer);
          break;
        }
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_3d(smem + Smem::kB + s * kTileBytes, &xmap, 0, 0, static_cast<int>(t * R), &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t a_base = smem_u32(smem + Smem::kA);
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int b = it % kAccBufs;
        const uint32_t aph = (it / kAccBufs) & 1;
        if (!mbar_wait(&full[s], ph) || (it >= kAccBufs && !mbar_wait(&acc_empty[b], aph ^ 1))) {
          atomicOr(&hadq_tc_fault, kFaultMma);
          break;
        }
        tc_fence_after();
        const uint32_t b_base = smem_u32(smem + Smem::kB + s * kTileBytes);
        const uint32_t d = tmem_base + b * kAccCols;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // K = 128 in steps of 16
          const uint64_t a_desc = smem_desc(a_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSwizzle128);
          const uint64_t b_desc = (LO == 5) ? smem_desc(b_base + kk * 1024, 8192, 512, kSwizzle64)
                                            : smem_desc(b_base + kk * 2048, 16384, 1024, kSwizzle128);
          mma_bf16(d, a_desc, b_desc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);      // stage s may be refilled once these MMAs have read it
        mma_commit(&acc_full[b]);   // accumulator b is ready for the epilogue
      }
    }
  } else {
    const int quarter = warp & 3;            // TMEM lanes this warp may access
    const int hi = quarter * 32 + lane;      // the H_128 output index this thread owns
    uint32_t it = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
      const int b = it % kAccBufs;
      const uint32_t aph = (it / kAccBufs) & 1;
      if (!mbar_wait(&acc_full[b], aph)) {
        atomicOr(&hadq_tc_fault, kFaultEpilogue);
        ok = false;
        break;
      }
      tc_fence_after();
      float z[R][L];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * kAccCols;
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int c = 0; c < L; c += 32) tmem_ld32(taddr + r * L + c, &z[r][c]);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t row = t * R + r;
        tc_emit_row<LO, MODE>(z[r], hi, row, row < rows, n, norm, group, out0, out1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

}  // namespace tc
}  // namespace hadq
