// Kernel entry points as the host launcher sees them.
//
// The kernels are instantiated in their own translation units
// (kernels_segment.cu, kernels_team.cu, kernels_tc.cu, kernels_tck.cu, ...), which nvcc compiles in
// parallel; each exports a lookup that returns the instantiation for a call's
// shape, output mode and sign variant.  SG selects the random Hadamard
// (signed) instantiation; the deterministic ones are compiled without any
// sign code.  A nullptr / fn == nullptr result means "no such instantiation".
#pragma once

#include <cuda.h>
#include <cstdint>

#include "hadq_device.cuh"

namespace hadq {
namespace launch {

using SegFn = void (*)(const void*, int64_t, int, float, int, void*, void*, Signs);
using SegRowFn = void (*)(const void*, int64_t, int64_t, int, float, int8_t*, float*, Signs);
using TeamFn = void (*)(const void*, int64_t, float, int, void*, void*, Signs);
using TeamRowFn = void (*)(const void*, int64_t, int64_t, float, int8_t*, float*, Signs);
using TcFn = void (*)(const CUtensorMap, const uint16_t*, int64_t, int, float, int, void*, void*, Signs);
using Tc128Fn = void (*)(const CUtensorMap, const CUtensorMap, const uint16_t*, int64_t, int, float, int, void*, void*,
                         Signs, int);
}  // namespace launch
namespace ksize {
struct StageArgs;
}
namespace launch {
using KsFn = void (*)(const ksize::StageArgs);

struct TcVariant {
  TcFn fn;
  int threads, smem, tile_n;
};

struct Tc128Variant {
  Tc128Fn fn;
  int threads, smem;
};

using TckFn = void (*)(const CUtensorMap, const CUtensorMap, const uint16_t*, int64_t, float, int, void*, void*, int);
using TcrFn = void (*)(const CUtensorMap, const uint16_t*, int64_t, int, float, int, void*, void*, const int32_t*,
                       const int8_t*, const double*);

struct TcrVariant {
  TcrFn fn;
  int threads, smem;
};

struct TckVariant {
  TckFn fn;
  int threads, smem, np;   // np: MMA N = chunks per block rounded up to 16
};

// Segment kernels (b <= 128): log2 of the per-thread segment `logs`, FULL when
// b equals the segment.  mode: OutMode.
SegFn segment_kernel_for(bool bf16, bool full, int logs, int mode, bool sg);
SegRowFn segment_row_kernel_for(bool bf16, bool full, int logs, bool sg);

// Team kernels (256 <= b <= 8192); one unit per input dtype
// (kernels_team.cu: fp32 and the dispatch, kernels_team_bf16.cu: bf16).
TeamFn team_kernel_for(bool bf16, int logb, int mode, bool sg);
TeamRowFn team_row_kernel_for(bool bf16, int logb, bool sg);
TeamFn team_kernel_bf16(int logb, int mode, bool sg);
TeamRowFn team_row_kernel_bf16(int logb, bool sg);

// Tensor-core kernels: full size 2^(7 + lo), lo = 5 or 6; block 128 (mode -1 =
// per-token int8).
TcVariant tc_kernel_for(int lo, int mode, int side);   // side: hadq::SignSide
// Block-128 kernel; e > 0: blocks of 2^e * 128 (1 <= e <= 4), the last e
// stages across neighbouring lanes, no signs and no per-token int8.
Tc128Variant tc128_kernel_for(int mode, int e);   // e = 0: signs of either side folded into B
TcrVariant tcr_kernel_for(int mode);       // RPBH at full size 4096 (permutation gathered in shared memory)

// Shared-memory staged kernels: blocks of K * 2^m elements (K a covered Paley
// order 12 .. 108, or 1 with the RPBH permutation or the codebook quantizer);
// shi = pieces of the 2^m factor mixed in the column stage; mode -1 =
// per-token int8; sgk: ksize::StageSigns.  One unit per input dtype
// (kernels_ksize.cu: fp32 and the dispatch, kernels_ksize_bf16.cu: bf16).
KsFn staged_kernel_for(int k, int shi, bool bf16, int mode, int sgk);
KsFn staged_kernel_f32(int k, int shi, int mode, int sgk);
KsFn staged_kernel_bf16(int k, int shi, int mode, int sgk);

// Tensor-core kernels for blocks of K * 128 * hi elements (K a Paley order,
// K * hi <= 128 chunks of 128); mode OUT_F32 / OUT_BF16, -1 = per-token int8
// (block = row), or OUT_INT4 / OUT_MXFP4 / OUT_NVFP4.
TckVariant tck_kernel_for(int k, int hi, int mode);

// The tensor-core kernels' sticky fault words (bounded waits that ran out),
// one per translation unit; cleared when `clear` is non-zero.  -1 on a CUDA
// error.
int tc_fault_bits(int clear);
int tck_fault_bits(int clear);

}  // namespace launch
}  // namespace hadq
