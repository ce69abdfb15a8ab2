// Tensor-core variant of orbitquant's RPBH rotation at full size 4096, bf16
// input ("orbitquant 0.2.0", Method Conformance: a random permutation of the
// row's columns and one Rademacher sign per column, then the block Hadamard
// rotation; here the block is the whole row).
//
// Row r of the output is y = H_4096 v / 64 with v_e = x[r][pi(e)] * s_e.  The
// rotation is the n = 4096 tensor-core kernel's (hadq_tc.cuh): tiles of 4
// rows, D = H_128 X_tile by one tcgen05 MMA per tile over the high 7 index
// bits, the low 5 in the epilogue's registers.  The permutation moves data
// across the whole row, so it cannot ride on the MMA operand or on the TMA
// box; gather warps build each operand tile in shared memory instead:
//
//   TMA       the raw 4-row tile into one of RAW_STAGES raw stages;
//   gather    for every output chunk of 8 columns e .. e + 7 of each row, 8
//             16-bit loads from the raw tile at the swizzled places of
//             pi(e) .. pi(e + 7), the signs applied by one XOR per pair, one
//             16-byte store into a permuted stage laid out exactly as a TMA
//             tile of v would be; then the raw stage goes back to the TMA
//             producer and the permuted stage to the MMA;
//   MMA       A = H_128 from tensor memory, B = the permuted stage;
//   epilogue  as the n = 4096 kernel (LO = 5 register stages, quantizer).
//
// Each gather thread always owns the same two output chunks of every row, so
// its 16 source offsets and signs (two of each per word) are computed once per
// launch from the caller's permutation and signs.  Roles: warp 0 TMA
// producer, warp 1 TMEM allocator and MMA issuer, warps 2..17 epilogue (one
// row of each tile per group of 4), warps 18..25 gather.  Every wait is
// bounded (hadq_tc_fault).
#pragma once

#include "hadq_tc.cuh"

namespace hadq {
namespace tc {

struct TcrCfg {
  static constexpr int LO = 5, L = 32, TILE_N = 128, R = 4, SPLIT = 4;
  static constexpr int RAW_STAGES = 3, P_STAGES = 2;
  static constexpr int PREFETCH = 2;                       // tiles per CTA prefetched into L2 at entry
  static constexpr int GATHER_THREADS = 256;               // 2 output chunks of each row per thread
  static constexpr int TILE_BYTES = 128 * TILE_N * 2;      // 4 rows of 4096 bf16
  static constexpr int ROW_BYTES = TILE_BYTES / R;
  static constexpr int ACC_BUFS = 3;                       // 3 x 128 TMEM columns, H_128 after them
  static constexpr int A_COL = ACC_BUFS * TILE_N;
  static constexpr int TMEM_COLS = 512;
  static constexpr int FIRST_GATHER_WARP = 2 + 4 * SPLIT;
  static constexpr int THREADS = 32 * FIRST_GATHER_WARP + GATHER_THREADS;
  // kind::f16, fp32 accumulate, bf16 A and B, A K-major, B MN-major, N = 128, M = 128.
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                    (static_cast<uint32_t>(TILE_N >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
  static constexpr int SM_RAW = 0;
  static constexpr int SM_P = SM_RAW + RAW_STAGES * TILE_BYTES;
  static constexpr int SM_BARS = SM_P + P_STAGES * TILE_BYTES;
  static constexpr int SM_RED = SM_BARS + 8 * (2 * RAW_STAGES + 2 * P_STAGES + 2 * ACC_BUFS);
  // Codebook quantizer: per epilogue sub-group (one row of each tile) 2 x 4
  // partial sums of squares (double; a buffer per tile parity), and per
  // epilogue warp up to 15 row thresholds (float).
  static constexpr int SM_CB = SM_RED + 8 * 2 * 4 * SPLIT;   // 16-byte aligned (quartile loads)
  static constexpr int SM_SLOT = SM_CB + 4 * 16 * 4 * SPLIT;
  static_assert(SM_CB % 16 == 0, "quartile loads of the row thresholds are 16-byte loads");
  static constexpr int SMEM_BYTES = SM_SLOT + 16 + 1024;
  static_assert(GATHER_THREADS * 2 * 8 == ROW_BYTES / 2, "two 8-column chunks of each row per gather thread");
};

// Byte offset within a row of the 64-byte-swizzled tile (the stage base is
// 1024-byte aligned and a row is 8192 bytes, so only the in-row offset
// decides the swizzle): 16-byte chunk bits 4..5 XOR address bits 7..8.
__device__ __forceinline__ uint32_t swz64(uint32_t off) { return off ^ (((off >> 7) & 3u) << 4); }

// Codebook quantizer ("orbitquant 0.2.0", Method Conformance: per-token norm,
// the normalised rotation, the nearest centroid of the unit-sphere Lloyd-Max
// codebook) for one row; z holds the thread's 32 values of the row after the
// tensor-core stage (output columns hi * 32 ..).  Every thread of the row's 4
// warps calls it for every tile (work = false after a failed wait: the
// barrier is still joined).  The code of u = y / ||y|| is the number of unit
// thresholds t_j below u, i.e. of row thresholds tau_j = ||z|| t_j below z;
// with h = fl(tau_j) and l = tau_j - h (double), z > tau_j exactly when
// z >= g_j = (l < 0 ? h : the next float above h), so one float per
// threshold decides exactly.  The norm is a double sum of squares (four
// accumulation chains), joined across the 4 warps by one named barrier; red
// holds the partial sums of this tile (a buffer per tile parity: a warp can be
// one tile ahead of the others when it writes, never two), and each warp
// computes the thresholds into its own table gtab, so no second barrier is
// needed.
__device__ __forceinline__ void tcr_codebook_row(float (&z)[32], bool work, int quarter, int lane, int64_t e0,
                                                 int64_t row, bool row_ok, float norm, int bits, const double* thr,
                                                 double* red, float* gtab, int bar, uint8_t* codes, float* norms) {
  double ss = 0.0;
  if (work) {
    fwht_bits<32, 0, 5>(z);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i & 3] = fma(static_cast<double>(z[i]), static_cast<double>(z[i]), acc[i & 3]);
    ss = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) red[quarter] = ss;
  asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
  const double zn = sqrt((red[0] + red[1]) + (red[2] + red[3]));
  const int levels = 1 << bits;
  if (lane < levels - 1) {
    const double t = (zn > 0.0 ? zn : 1.0) * thr[lane];   // a zero row codes u = 0
    const float h = __double2float_rn(t);
    gtab[lane] = (t - static_cast<double>(h) < 0.0) ? h : nextafterf(h, INFINITY);
  }
  if (quarter == 0 && lane == 0 && row_ok && work) norms[row] = static_cast<float>(zn * static_cast<double>(norm));
  __syncwarp();
  if (!work || !row_ok) return;
  if (bits == 4) {
    // The separators g_3, g_7, g_11 (registers) give the quartile Q of z; one
    // 16-byte load of g_4Q .. g_4Q+2 and two more compares finish the search.
    const float g3 = gtab[3], g7 = gtab[7], g11 = gtab[11];
    const float4* quart = reinterpret_cast<const float4*>(gtab);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = z[8 * q + i];
        const uint32_t b3 = v >= g7 ? 1u : 0u;
        const uint32_t b2 = v >= (b3 ? g11 : g3) ? 1u : 0u;
        const uint32_t Q = 2 * b3 + b2;
        const float4 f = quart[Q];
        const uint32_t b1 = v >= f.y ? 1u : 0u;
        const uint32_t b0 = v >= (b1 ? f.z : f.x) ? 1u : 0u;
        word |= (4 * Q + 2 * b1 + b0) << (4 * i);
      }
      w[q] = word;
    }
    *reinterpret_cast<uint4*>(codes + (e0 >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    const float g0 = gtab[0], g1 = gtab[1], g2 = gtab[2];
    uint32_t w[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v = z[16 * q + i];
        const uint32_t b1 = v >= g1 ? 1u : 0u;
        const uint32_t b0 = v >= (b1 ? g2 : g0) ? 1u : 0u;
        word |= (2 * b1 + b0) << (2 * i);
      }
      w[q] = word;
    }
    *reinterpret_cast<uint2*>(codes + (e0 >> 2)) = make_uint2(w[0], w[1]);
  }
}

// MODE: an OutMode of tc_emit_row (rotation, int4, MXFP4, NVFP4) or
// OUT_CODEBOOK (group = bits, 2 or 4; thr = the 2^bits - 1 ascending unit
// thresholds).  perm: n int32 source columns (entries outside [0, n) are
// clamped: memory-safe, result unspecified); signs: n int8, negative = -1.
template <int MODE>
__global__ void __launch_bounds__(TcrCfg::THREADS, 1)
tc_rpbh_kernel(const __grid_constant__ CUtensorMap xmap, const uint16_t* __restrict__ x, int64_t rows, int n,
               float norm, int group, void* __restrict__ out0, void* __restrict__ out1,
               const int32_t* __restrict__ perm, const int8_t* __restrict__ signs, const double* __restrict__ thr) {
  using C = TcrCfg;
  constexpr int LO = C::LO, L = C::L, R = C::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);   // raw tile landed
  uint64_t* empty = full + C::RAW_STAGES;                           // raw stage read by the gather
  uint64_t* gathered = empty + C::RAW_STAGES;                       // permuted stage written
  uint64_t* pfree = gathered + C::P_STAGES;                         // permuted stage read by the MMA
  uint64_t* acc_full = pfree + C::P_STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles = (rows + R - 1) / R;

  if (threadIdx.x == 0) {
    int64_t t = blockIdx.x;
    for (int i = 0; i < C::PREFETCH && t < tiles; ++i, t += gridDim.x) {
      const int64_t r1 = (t + 1) * R < rows ? (t + 1) * R : rows;
      prefetch_l2(x + t * R * n, static_cast<uint32_t>((r1 - t * R) * n * 2));
    }
    for (int s = 0; s < C::RAW_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::GATHER_THREADS / 32);
    }
    for (int p = 0; p < C::P_STAGES; ++p) {
      mbar_init(&gathered[p], C::GATHER_THREADS / 32);
      mbar_init(&pfree[p], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * C::SPLIT);
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
        const int s = it % C::RAW_STAGES;
        const uint32_t ph = (it / C::RAW_STAGES) & 1;
        if (it >= C::RAW_STAGES && !mbar_wait(&empty[s], ph ^ 1)) {
          atomicOr(&hadq_tc_fault, kFaultProducer);
          drain_loads(full, C::RAW_STAGES, it);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::TILE_BYTES);
        tma_load_3d(smem + C::SM_RAW + s * C::TILE_BYTES, &xmap, 0, 0, static_cast<int>(t * R), &full[s]);
      }
    }
  } else if (warp >= C::FIRST_GATHER_WARP) {
    // ----------------------------------------------------------------- gather
    grid_dependency_sync();                  // the permutation and signs are caller memory
    const int j = threadIdx.x - 32 * C::FIRST_GATHER_WARP;
    // src: per pair of output columns e, e + 1 the two 13-bit in-row source
    // offsets (bits 0..12, 16..28) and their signs (bit 15, 31 set for -1),
    // which are then exactly the XOR mask of the packed bf16 pair.
    uint32_t src[8], dst[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int c = j + C::GATHER_THREADS * q;   // output chunk: columns 8 c .. 8 c + 7
      dst[q] = swz64(16u * static_cast<uint32_t>(c));
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const uint32_t p0 = min(static_cast<uint32_t>(__ldg(perm + 8 * c + i)), static_cast<uint32_t>(n - 1));
        const uint32_t p1 = min(static_cast<uint32_t>(__ldg(perm + 8 * c + i + 1)), static_cast<uint32_t>(n - 1));
        const uint32_t s0 = __ldg(signs + 8 * c + i) < 0 ? 0x8000u : 0u;
        const uint32_t s1 = __ldg(signs + 8 * c + i + 1) < 0 ? 0x8000u : 0u;
        src[4 * q + i / 2] = (swz64(2u * p0) | s0) | ((swz64(2u * p1) | s1) << 16);
      }
    }
    uint32_t it = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
      const int s = it % C::RAW_STAGES, p = it % C::P_STAGES;
      const uint32_t sph = (it / C::RAW_STAGES) & 1, pph = (it / C::P_STAGES) & 1;
      if (!mbar_wait(&full[s], sph) || (it >= C::P_STAGES && !mbar_wait(&pfree[p], pph ^ 1))) {
        atomicOr(&hadq_tc_fault, kFaultSign);
        break;
      }
      const uint8_t* raw = smem + C::SM_RAW + s * C::TILE_BYTES;
      uint8_t* pb = smem + C::SM_P + p * C::TILE_BYTES;
#pragma unroll
      for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t off = ((i & 1) ? (src[4 * q + i / 2] >> 16) : src[4 * q + i / 2]) & 0x1FFFu;
            v[i] = *reinterpret_cast<const uint16_t*>(raw + r * C::ROW_BYTES + off);
          }
          uint4 w;
          w.x = __byte_perm(v[0], v[1], 0x5410) ^ (src[4 * q + 0] & 0x80008000u);
          w.y = __byte_perm(v[2], v[3], 0x5410) ^ (src[4 * q + 1] & 0x80008000u);
          w.z = __byte_perm(v[4], v[5], 0x5410) ^ (src[4 * q + 2] & 0x80008000u);
          w.w = __byte_perm(v[6], v[7], 0x5410) ^ (src[4 * q + 3] & 0x80008000u);
          *reinterpret_cast<uint4*>(pb + r * C::ROW_BYTES + dst[q]) = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the permuted stage, to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&gathered[p]);
        mbar_arrive(&empty[s]);
      }
    }
  } else {
    // Warps 1 .. FIRST_GATHER_WARP - 1: tensor memory, H_128, MMA, epilogue.
    constexpr int kSetupThreads = 32 * (C::FIRST_GATHER_WARP - 1);
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(kSetupThreads) : "memory");
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // H_128 into tensor memory (lane m = row m, column A_COL + c = the bf16
    // pair k = 2c, 2c + 1), by the warps of the first epilogue group.
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
    asm volatile("bar.sync 1, %0;" ::"r"(kSetupThreads) : "memory");
    tc_fence_after();

    if (warp == 1) {
      // ------------------------------------------------------- MMA issuer
      if (lane == 0) {
        uint32_t it = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
          const int p = it % C::P_STAGES;
          const uint32_t pph = (it / C::P_STAGES) & 1;
          const int b = it % C::ACC_BUFS;
          const uint32_t aph = (it / C::ACC_BUFS) & 1;
          if (!mbar_wait(&gathered[p], pph) || (it >= C::ACC_BUFS && !mbar_wait(&acc_empty[b], aph ^ 1))) {
            atomicOr(&hadq_tc_fault, kFaultMma);
            drain_mmas(pfree, C::P_STAGES, it);
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(smem + C::SM_P + p * C::TILE_BYTES);
          const uint32_t d = tmem_base + b * C::TILE_N;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ta(d, tmem_base + C::A_COL + kk * 8, smem_desc(b_base + kk * 1024, 8192, 512, kSwizzle64),
                        C::IDESC, kk > 0 ? 1u : 0u);
          mma_commit(&pfree[p]);
          mma_commit(&acc_full[b]);
        }
      }
    } else {
      // --------------------------------------------------------- epilogue
      grid_dependency_sync();
      const int quarter = warp & 3;
      const int sub = (warp - 2) >> 2;         // row `sub` of every tile
      const int hi = quarter * 32 + lane;
      double* red = reinterpret_cast<double*>(smem + C::SM_RED) + 8 * sub;      // [tile parity][quarter]
      float* gtab = reinterpret_cast<float*>(smem + C::SM_CB) + 16 * (warp - 2);  // this warp's thresholds
      uint32_t it = 0;
      bool failed = false;   // a wait ran out: skip the work (the codebook still joins its barriers)
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int b = it % C::ACC_BUFS;
        const uint32_t aph = (it / C::ACC_BUFS) & 1;
        if (!failed && !mbar_wait(&acc_full[b], aph)) {
          atomicOr(&hadq_tc_fault, kFaultEpilogue);
          failed = true;
        }
        if (failed && MODE != OUT_CODEBOOK) break;
        float z[L];
        if (!failed) {
          tc_fence_after();
          tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + b * C::TILE_N + sub * L, z);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        const int64_t row = t * R + sub;
        if constexpr (MODE == OUT_CODEBOOK) {
          tcr_codebook_row(z, !failed, quarter, lane, row * n + static_cast<int64_t>(hi) * L, row, row < rows, norm,
                           group, thr, red + 4 * (it & 1), gtab, 2 + sub, static_cast<uint8_t*>(out0),
                           static_cast<float*>(out1));
        } else {
          tc_emit_row<LO, MODE, 0>(z, hi, row, row < rows, n, norm, group, out0, out1, nullptr);
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
