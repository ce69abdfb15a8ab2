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
// Roles (one CTA per SM, persistent over tiles; tile = TILE_N columns =
// TILE_N / 2^LO rows, contiguous in global memory):
//   warp 0      TMA producer: X tiles (box 2^LO x 128 x R, 64B/128B swizzle,
//               each CTA loading its own) into a ring of STAGES stages;
//   warp 1      TMEM allocator and MMA issuer (one thread); accumulators in
//               512 / TILE_N tensor-memory buffers;
//   warps 2..   4 * SPLIT epilogue warps; warp w reads TMEM lanes
//               32 * (w % 4) + [0, 32) for the rows r = j (mod SPLIT) of every
//               tile, j = (w - 2) / 4, so each tile is finished by all of them.
// The producer starts streaming as soon as the barriers exist; the other
// warps build H_128 in shared memory and allocate tensor memory meanwhile.
// Before anything else, thread 0 asks L2 to prefetch the CTA's first
// PREFETCH tiles.  A prefetch is only a hint (no data reaches the CTA
// and nothing is observed), so it may precede the wait for the previous
// kernel in the stream; it lets the first TMA loads after that wait hit L2
// instead of starting cold from HBM.  Two tiles is the measured optimum for
// 4096 x 4096 (9.46 us per launch; 10.1 us with 4, 11.1 us with 8, where the
// prefetches of later tiles delay the first tile's loads).  With HALF, the MMAs of a tile are issued
// as two N/2 halves with their own commit, so the epilogue warps of the first
// half start while the tensor core still works on the second.
// Random Hadamard signs (section 1.5) after the rotation are applied in the
// epilogue to the finished outputs.  Signs before it must reach the operand
// ahead of the MMA, since every output mixes inputs with different signs:
// with SIDE == SIGNS_BEFORE extra warps (SIGN_THREADS) flip the bf16 sign bits of each
// landed tile in shared memory (one XOR per 32-bit word; each thread always
// owns the same 16 chunks of the swizzled tile, so its sign masks are loaded
// once) and release the stage to the MMA through a second mbarrier.
// Every mbarrier wait gives up after one second (globaltimer); on timeout the
// kernel records a fault in hadq_tc_fault, stops issuing work, waits (bounded
// the same way) for the loads and MMAs it already issued, and still releases
// its tensor memory.
#pragma once

#include <cuda.h>
#include "hadq_device.cuh"

namespace hadq {
namespace tc {

constexpr int kABytes = 128 * 128 * 2;     // A operand: H_128 in bf16
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // every mbarrier wait gives up after 1 s


template <int LO_, int TILE_N_, int STAGES_, int SPLIT_, bool HALF_, int PREFETCH_ = 2, bool AHEAD_ = false,
          bool A_TMEM_ = false>
struct TcCfg {
  // A_TMEM: H_128 lives in tensor memory (64 columns after the accumulators)
  // instead of shared memory, so the MMAs read only the B tile from shared
  // memory; one accumulator buffer fewer.
  static constexpr bool A_TMEM = A_TMEM_;
  static constexpr int PREFETCH = PREFETCH_;             // tiles per CTA prefetched into L2 at entry
  static constexpr bool AHEAD = AHEAD_;                  // keep the prefetch PREFETCH tiles ahead of the loads
  // Sign-flipping threads (signs before the rotation only): as many as the
  // register budget allows, since they sit between a tile's arrival and its
  // MMA (n = 4096: 60-register epilogue; n = 8192: up to 137 registers).
  static constexpr int SIGN_THREADS = LO_ == 5 ? 256 : 128;
  static constexpr int LO = LO_, L = 1 << LO;
  static constexpr int TILE_N = TILE_N_;                  // MMA N: columns per tile
  static constexpr int R = TILE_N / L;                    // rows per tile
  static constexpr int STAGES = STAGES_;
  static constexpr int TILE_BYTES = 128 * TILE_N * 2;     // B operand: K = 128 x N bf16
  static constexpr int TMEM_COLS = 512;                   // the whole tensor memory of the SM
  static constexpr int ACC_BUFS = (TMEM_COLS - (A_TMEM ? 64 : 0)) / TILE_N;
  static constexpr int A_COL = ACC_BUFS * TILE_N;         // A_TMEM: first column of H_128
  static constexpr int SPLIT = SPLIT_;                    // epilogue warps per TMEM lane quarter
  static constexpr int THREADS = 32 * (2 + 4 * SPLIT);
  static constexpr bool HALF = HALF_;                      // two N/2 MMA halves per tile, committed apart
  static_assert(!HALF || (R == SPLIT && R % 2 == 0),
                "HALF: one row per epilogue sub-group, so each half tile has its own sub-groups");
  static_assert(LO == 5 || LO == 6, "tensor-core path covers n = 4096 and 8192");
  static_assert(R >= 1 && (TILE_N == 64 || TILE_N == 128), "tile of 64 or 128 columns");
  // Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A K-major,
  // B MN-major, N = TILE_N, M = 128.
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                    (static_cast<uint32_t>(TILE_N >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
  static constexpr uint32_t IDESC_HALF = (IDESC & ~(63u << 17)) | (static_cast<uint32_t>(TILE_N >> 4) << 17);
  // Shared memory (offsets from a 1024-byte aligned base).
  static constexpr int SM_A = 0;                          // H_128, 2 K-panels x 16 KB (not A_TMEM)
  static constexpr int SM_B = SM_A + (A_TMEM ? 0 : kABytes);   // STAGES x TILE_BYTES
  static constexpr int SM_BARS = SM_B + STAGES * TILE_BYTES;
  static constexpr int SM_SLOT = SM_BARS + 8 * (3 * STAGES + 3 * ACC_BUFS);
  static constexpr int SMEM_BYTES = SM_SLOT + 16 + 1024;  // + alignment slack
};

// Fault codes written to hadq_tc_fault.
constexpr unsigned kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u, kFaultSign = 8u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The dynamic shared memory rounded up to a 1024-byte boundary (what the
// 128-byte swizzle atoms need), as an offset from the __shared__ array
// itself: the compiler then still knows every pointer derived from it to be
// shared memory and emits shared loads and stores (an integer round trip
// through uintptr_t would leave generic accesses, which take the longer
// global-memory path through the load/store unit).
__device__ __forceinline__ uint8_t* smem_align1024(uint8_t* base) {
  return base + ((1024u - (smem_u32(base) & 1023u)) & 1023u);
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

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with parity `parity` to complete; false after kWaitLimitNs.
// Each try_wait may suspend the warp in hardware for up to kSuspendHintNs (it
// resumes as soon as the phase completes), so waiting warps do not spin on
// issue slots the working warps need.
constexpr uint32_t kSuspendHintNs = 100000;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  if (ok) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    if (ok) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// UMMA shared-memory matrix descriptor (sm_100 format: start, leading and
// stride byte offsets in 16-byte units, version 1, swizzle mode in bits 61..63).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (static_cast<uint64_t>(swizzle) << 61);
}

constexpr uint32_t kSwizzle128 = 2, kSwizzle64 = 4;

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// The same with A in tensor memory (lane m = row m, column c = the bf16 pair
// k = 2c, 2c + 1).
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// 16 consecutive 32-bit columns of this thread's TMEM lane from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
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

// Sticky fault bits (bounded waits that ran out), one word per translation
// unit that instantiates these kernels; the host ORs them.
static __device__ unsigned int hadq_tc_fault;

// After a wait ran out, what this thread already issued must finish before
// the CTA exits: a TMA write into shared memory, or an MMA reading it, must
// not outlive the CTA.  Loads: the full phases of the last min(issued,
// stages) tiles.  MMAs complete in order, so the stage-release commit of the
// last issued tile covers all earlier ones.  Every wait is bounded like the
// others; one that runs out leaves the rest in flight (already a fault).
__device__ __forceinline__ void drain_loads(uint64_t* full, int stages, uint32_t issued) {
  for (uint32_t i = issued > static_cast<uint32_t>(stages) ? issued - stages : 0; i < issued; ++i)
    if (!mbar_wait(&full[i % stages], (i / stages) & 1)) return;
}

__device__ __forceinline__ void drain_mmas(uint64_t* empty, int stages, uint32_t issued) {
  if (issued > 0) (void)mbar_wait(&empty[(issued - 1) % stages], ((issued - 1) / stages) & 1);
}

// Epilogue for one row of one tile: z holds the 2^LO values of TMEM lane hi'
// (after the tensor-core stage over hi); finish the butterfly over lo and emit.
// Signs after the rotation (random Hadamard): SGK = 1, output column
// hi * 2^LO + c is negated where bit c of the mask words sm[c / 32] is set;
// SGK = 2, sm holds one XOR word (0 or the fp32 sign bit) per column c.
template <int LO, int MODE, int SGK>
__device__ __forceinline__ void tc_emit_row(float (&z)[1 << LO], int hi, int64_t row, bool row_ok, int n, float norm,
                                            int group, void* __restrict__ out0, void* __restrict__ out1,
                                            const uint32_t* sm) {
  constexpr int L = 1 << LO;
  fwht_bits<L, 0, LO>(z);
  if constexpr (SGK == 1) {
    apply_signs<L>(z, *reinterpret_cast<const uint32_t(*)[L / 32]>(sm));
  } else if constexpr (SGK == 2) {
#pragma unroll
    for (int c = 0; c < L; ++c) z[c] = __uint_as_float(__float_as_uint(z[c]) ^ sm[c]);
  }
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
      const __half s16 = __float2half_rn(int4_scale_f32(m));
      const float s = __half2float(s16);
      const float rn = (s > 0.f && s <= 65504.f) ? code_factor(norm, s) : 0.f;
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
        if (((e0 + 32 * j) & (group - 1)) == 0)   // group is a power of 2
          static_cast<__half*>(out1)[(e0 + 32 * j) >> (__ffs(group) - 1)] = s16;
      }
    }
  } else if constexpr (MODE == OUT_MXFP4 || MODE == OUT_MXFP4_BLOCKED) {
    // n = 2^(7 + LO): 2^(LO + 2) scales of 32 per row
    constexpr int LOG_C = MODE == OUT_MXFP4_BLOCKED ? LO + 2 : 0;
    if (row_ok) store_mxfp4<false, L, LOG_C>(z, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
  } else if constexpr (MODE == OUT_NVFP4 || MODE == OUT_NVFP4_BLOCKED) {
    constexpr int LOG_C = MODE == OUT_NVFP4_BLOCKED ? LO + 3 : 0;   // 2^(LO + 3) scales of 16 per row
    if (row_ok) store_nvfp4<false, L, LOG_C>(z, norm, static_cast<uint8_t*>(out0), static_cast<uint8_t*>(out1), e0);
  } else if constexpr (MODE == OUT_BF16) {
    if (row_ok) store_rotated<false, L, true>(z, norm, out0, e0);
  } else {
    if (row_ok) store_rotated<false, L, false>(z, norm, out0, e0);
  }
}

// Threads of tc_rotate_kernel<C, MODE, SIDE>.
template <class C, int SIDE>
__host__ __device__ constexpr int tc_threads() {
  return C::THREADS + (SIDE == SIGNS_BEFORE ? C::SIGN_THREADS : 0);
}

template <class C, int MODE, int SIDE>
__global__ void __launch_bounds__(tc_threads<C, SIDE>(), 1)
tc_rotate_kernel(const __grid_constant__ CUtensorMap xmap, const uint16_t* __restrict__ x, int64_t rows, int n,
                 float norm, int group, void* __restrict__ out0, void* __restrict__ out1, Signs sg) {
  constexpr int LO = C::LO, L = C::L, R = C::R;
  constexpr bool SG = SIDE == SIGNS_AFTER, SB = SIDE == SIGNS_BEFORE;
  constexpr int T = tc_threads<C, SIDE>();
  constexpr int kFirstSignWarp = 2 + 4 * C::SPLIT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint64_t* acc_full2 = acc_empty + C::ACC_BUFS;   // second half of a tile (HALF)
  uint64_t* flipped = acc_full2 + C::ACC_BUFS;     // stage signed (SB): the MMA may read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles = (rows + R - 1) / R;

  if (threadIdx.x == 0) {
    int64_t t = blockIdx.x;
    for (int i = 0; i < C::PREFETCH && t < tiles; ++i, t += gridDim.x) {
      const int64_t r1 = (t + 1) * R < rows ? (t + 1) * R : rows;   // a tile is rows [t R, r1), contiguous
      prefetch_l2(x + t * R * n, static_cast<uint32_t>((r1 - t * R) * n * 2));
    }
    if constexpr (SIDE != SIGNS_NONE) prefetch_l2(sg.s, 128 * L);   // the b signs (int8)
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&flipped[s], C::SIGN_THREADS / 32);   // one arrival per sign warp
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * C::SPLIT);  // every epilogue warp reads every tile
      mbar_init(&acc_full2[b], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      grid_dependency_sync();   // x may be written by the previous kernel in the stream
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (it >= C::STAGES && !mbar_wait(&empty[s], ph ^ 1)) {
          atomicOr(&hadq_tc_fault, kFaultProducer);
          drain_loads(full, C::STAGES, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::TILE_BYTES);
        tma_load_3d(smem + C::SM_B + s * C::TILE_BYTES, &xmap, 0, 0, static_cast<int>(t * R), &full[s]);
        if constexpr (C::AHEAD) {
          const int64_t tp = t + static_cast<int64_t>(C::PREFETCH) * gridDim.x;   // this CTA's tile it + PREFETCH
          if (tp < tiles) {
            const int64_t r1 = (tp + 1) * R < rows ? (tp + 1) * R : rows;
            prefetch_l2(x + tp * R * n, static_cast<uint32_t>((r1 - tp * R) * n * 2));
          }
        }
      }
    }
  } else {
    // A = H_128 (K-major, 128-byte swizzle, two K-panels of 64): element (m, k)
    // at panel (k / 64) + m * 128 + (k % 64) * 2 bytes, 16-byte chunk index
    // XOR-ed with (m % 8).  Entry (m, k) = (-1)^popcount(m & k) as bf16.
    if constexpr (!C::A_TMEM) {
      for (int i = threadIdx.x - 32; i < 128 * 16; i += T - 32) {
        const int m = i >> 4, kc = i & 15;              // 8 consecutive k per 16-byte chunk
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
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // A visible to the tensor core
    }
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(T - 32) : "memory");   // warps 1.. only
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if constexpr (C::A_TMEM) {
      // H_128 into tensor memory by the four warps of the first epilogue
      // group (warp w reaches lanes 32 (w % 4) ..): lane m holds row m,
      // column A_COL + c the bf16 pair (k = 2c, 2c + 1).
      if (warp >= 2 && warp < 6) {
        const int m = (warp & 3) * 32 + lane;
        for (int c0 = 0; c0 < 64; c0 += 16) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k = 2 * (c0 + i);
            w[i] = 0x3F803F80u | ((__popc(m & k) & 1u) << 15) | ((__popc(m & (k + 1)) & 1u) << 31);
          }
          tmem_st16(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + C::A_COL + c0, w);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"r"(T - 32) : "memory");   // A written before the first MMA
      tc_fence_after();
    }

    if (warp == 1) {
      // ------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t a_base = smem_u32(smem + C::SM_A);
        uint32_t it = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          const int b = it % C::ACC_BUFS;
          const uint32_t aph = (it / C::ACC_BUFS) & 1;
          if (!mbar_wait(SB ? &flipped[s] : &full[s], ph) ||
              (it >= C::ACC_BUFS && !mbar_wait(&acc_empty[b], aph ^ 1))) {
            atomicOr(&hadq_tc_fault, kFaultMma);
            drain_mmas(empty, C::STAGES, it);
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(smem + C::SM_B + s * C::TILE_BYTES);
          const uint32_t d = tmem_base + b * C::TILE_N;
          // A half tile is R/2 whole rows: half h starts TILE_BYTES/2 into the
          // stage (rows are the outermost box dimension) and TILE_N/2 columns
          // into the accumulator.
          constexpr int NH = C::HALF ? 2 : 1;
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            const uint32_t bh = b_base + h * (C::TILE_BYTES / 2);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {   // K = 128 in steps of 16
              const uint64_t b_desc = (LO == 5) ? smem_desc(bh + kk * 1024, 8192, 512, kSwizzle64)
                                                : smem_desc(bh + kk * 2048, 16384, 1024, kSwizzle128);
              if constexpr (C::A_TMEM) {
                mma_bf16_ta(d + h * (C::TILE_N / 2), tmem_base + C::A_COL + kk * 8, b_desc,
                            C::HALF ? C::IDESC_HALF : C::IDESC, kk > 0 ? 1u : 0u);
              } else {
                const uint64_t a_desc = smem_desc(a_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSwizzle128);
                mma_bf16(d + h * (C::TILE_N / 2), a_desc, b_desc, C::HALF ? C::IDESC_HALF : C::IDESC,
                         kk > 0 ? 1u : 0u);
              }
            }
            if (h == NH - 1) mma_commit(&empty[s]);   // stage s may be refilled once these MMAs have read it
            mma_commit(h == 0 ? &acc_full[b] : &acc_full2[b]);   // (this half of) accumulator b is ready
          }
        }
      }
    } else if (SB && warp >= kFirstSignWarp) {
      // ------------------------------------------- signs before the rotation
      // The stage holds the box (lo, hi, r) of the rows with lo innermost:
      // 2L-byte lines (hi, r), 16-byte chunks permuted by the 64-byte
      // (L = 32: chunk bits 4..5 ^= address bits 7..8) or 128-byte (L = 64:
      // bits 4..6 ^= bits 7..9) swizzle.  A chunk holds the 8 columns
      // hi * L + 8 * (logical chunk) + [0, 8) of one row; a negative int8
      // sign has bit 7 set, which byte_perm moves onto the bf16 sign bits.
      grid_dependency_sync();                  // the signs are caller memory
      constexpr int kChunks = C::TILE_BYTES / 16 / C::SIGN_THREADS;
      constexpr uint32_t kSwz = LO == 5 ? 3u : 7u;
      const int j = threadIdx.x - 32 * kFirstSignWarp;
      uint32_t q[kChunks][2];
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const uint32_t p = 16u * static_cast<uint32_t>(j + C::SIGN_THREADS * i);
        const uint32_t hi = (p / (2 * L)) & 127u;
        const uint32_t c = ((p % (2 * L)) >> 4) ^ ((p >> 7) & kSwz);
        const uint2 v = *reinterpret_cast<const uint2*>(sg.s + hi * L + 8 * c);
        q[i][0] = v.x & 0x80808080u;
        q[i][1] = v.y & 0x80808080u;
      }
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(&full[s], ph)) {
          atomicOr(&hadq_tc_fault, kFaultSign);
          break;
        }
        // Shared-window addresses (ld/st.shared, not generic accesses).
        const uint32_t stage = smem_u32(smem + C::SM_B + s * C::TILE_BYTES) + 16u * static_cast<uint32_t>(j);
        constexpr int kBatch = 8;              // loads in flight before the first store
#pragma unroll
        for (int i0 = 0; i0 < kChunks; i0 += kBatch) {
          uint4 v[kBatch];
#pragma unroll
          for (int i = 0; i < kBatch; ++i)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                         : "r"(stage + 16u * C::SIGN_THREADS * (i0 + i)));
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            v[i].x ^= __byte_perm(q[i0 + i][0], 0u, 0x1404);
            v[i].y ^= __byte_perm(q[i0 + i][0], 0u, 0x3424);
            v[i].z ^= __byte_perm(q[i0 + i][1], 0u, 0x1404);
            v[i].w ^= __byte_perm(q[i0 + i][1], 0u, 0x3424);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                         ::"r"(stage + 16u * C::SIGN_THREADS * (i0 + i)), "r"(v[i].x), "r"(v[i].y), "r"(v[i].z),
                           "r"(v[i].w)
                         : "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&flipped[s]);
      }
    } else {
      // --------------------------------------------------------- epilogue
      grid_dependency_sync();                  // outputs may still be read by the previous kernel
      const int quarter = warp & 3;            // TMEM lanes this warp may access
      const int sub = (warp - 2) >> 2;         // rows r = sub (mod SPLIT) of every tile
      const int hi = quarter * 32 + lane;      // the H_128 output index this thread owns
      // SG: signs after the rotation; this thread's outputs are block columns
      // hi * L + [0, L).
      // n = 4096 keeps one XOR word per column (32 registers; the epilogue
      // has room), n = 8192 the 2 bit-mask words.
      constexpr int SGK = !SG ? 0 : (LO == 5 ? 2 : 1);
      uint32_t sm[SGK == 2 ? L : L / 32];
      if constexpr (SGK == 1) {
#pragma unroll
        for (int w = 0; w < L / 32; ++w) sm[w] = sign_bits32(sg.s, hi * L + 32 * w);
      } else if constexpr (SGK == 2) {
        const uint32_t m = sign_bits32(sg.s, hi * L);
#pragma unroll
        for (int c = 0; c < L; ++c) sm[c] = (m << (31 - c)) & 0x80000000u;
      }
      // With HALF, sub-groups sub < SPLIT/2 own rows of the first half tile.
      const bool second_half = C::HALF && 2 * sub >= C::SPLIT;
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int b = it % C::ACC_BUFS;
        const uint32_t aph = (it / C::ACC_BUFS) & 1;
        if (!mbar_wait(second_half ? &acc_full2[b] : &acc_full[b], aph)) {
          atomicOr(&hadq_tc_fault, kFaultEpilogue);
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * C::TILE_N;
        constexpr int RW = (R + C::SPLIT - 1) / C::SPLIT;   // rows per warp per tile (at most)
        float z[RW][L];
#pragma unroll
        for (int j = 0; j < RW; ++j) {
          const int r = sub + C::SPLIT * j;
          if (r < R) {
#pragma unroll
            for (int c = 0; c < L; c += 32) tmem_ld32(taddr + r * L + c, &z[j][c]);
          }
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
#pragma unroll
        for (int j = 0; j < RW; ++j) {
          const int r = sub + C::SPLIT * j;
          if (r < R) {
            const int64_t row = t * R + r;
            tc_emit_row<LO, MODE, SGK>(z[j], hi, row, row < rows, n, norm, group, out0, out1, sm);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
  }
}

}  // namespace tc
}  // namespace hadq
