// Instantiations of the K * 2^m rotation kernels (non-power-of-2 blocks) for
// one input dtype, and their lookup.  The unit is compiled twice: with
// HADQ_KSIZE_BF16 for bf16 input (kernels_ksize_bf16.cu) and without it for
// fp32 input.
#include "hadq_ksize.cuh"
#include "hadq_launch.h"

#ifndef HADQ_KSIZE_BF16
#define HADQ_KSIZE_BF16 0
#endif

namespace hadq {
namespace launch {
namespace {

constexpr bool kBf16 = HADQ_KSIZE_BF16 != 0;

template <int K, bool SG>
KsFn ks_mode(int mode) {
  switch (mode) {
    case OUT_F32: return &ksize::ksize_kernel<K, kBf16, OUT_F32, SG>;
    case OUT_BF16: return &ksize::ksize_kernel<K, kBf16, OUT_BF16, SG>;
    case OUT_INT4: return &ksize::ksize_kernel<K, kBf16, OUT_INT4, SG>;
    case OUT_MXFP4: return &ksize::ksize_kernel<K, kBf16, OUT_MXFP4, SG>;
    case OUT_NVFP4: return &ksize::ksize_kernel<K, kBf16, OUT_NVFP4, SG>;
    case -1: return &ksize::ksize_kernel<K, kBf16, -1, SG>;
    default: return nullptr;
  }
}

template <int K>
KsFn ks_sign(int mode, bool sg) {
  return sg ? ks_mode<K, true>(mode) : ks_mode<K, false>(mode);
}

}  // namespace

#if HADQ_KSIZE_BF16
KsFn ksize_kernel_bf16(int k, int mode, bool sg) {
#else
KsFn ksize_kernel_f32(int k, int mode, bool sg) {
#endif
  switch (k) {
    case 12: return ks_sign<12>(mode, sg);
    case 20: return ks_sign<20>(mode, sg);
    case 28: return ks_sign<28>(mode, sg);
    case 36: return ks_sign<36>(mode, sg);
    case 52: return ks_sign<52>(mode, sg);
    case 60: return ks_sign<60>(mode, sg);
    case 108: return ks_sign<108>(mode, sg);
    default: return nullptr;
  }
}

#if !HADQ_KSIZE_BF16
KsFn ksize_kernel_for(int k, bool bf16, int mode, bool sg) {
  return bf16 ? ksize_kernel_bf16(k, mode, sg) : ksize_kernel_f32(k, mode, sg);
}
#endif

}  // namespace launch
}  // namespace hadq
