// Instantiations of the shared-memory staged kernels (hadq_ksize.cuh) for one
// input dtype, and their lookup.  The unit is compiled twice: with
// HADQ_KSIZE_BF16 for bf16 input (kernels_ksize_bf16.cu) and without it for
// fp32 input.  Instantiated: every Paley base order K with the plain and
// block-signed rotations, all formats and the codebook quantizer; the pure
// Sylvester blocks (K = 1) with the RPBH permutation and the codebook
// quantizer, the variants no other kernel family covers.  SHI: the pieces of
// the 2^m factor mixed in the column stage (K * SHI <= 64).
#include "hadq_ksize.cuh"
#include "hadq_launch.h"

#ifndef HADQ_KSIZE_BF16
#define HADQ_KSIZE_BF16 0
#endif

namespace hadq {
namespace launch {
namespace {

using ksize::SGK_BLOCK;
using ksize::SGK_NONE;
using ksize::SGK_RPBH;
using ksize::staged_kernel;
constexpr bool kBf16 = HADQ_KSIZE_BF16 != 0;

template <int K, int SHI, int SGK>
KsFn with_mode(int mode) {
  switch (mode) {
    case OUT_F32: return &staged_kernel<K, SHI, kBf16, OUT_F32, SGK>;
    case OUT_BF16: return &staged_kernel<K, SHI, kBf16, OUT_BF16, SGK>;
    case OUT_INT4: return &staged_kernel<K, SHI, kBf16, OUT_INT4, SGK>;
    case OUT_MXFP4: return &staged_kernel<K, SHI, kBf16, OUT_MXFP4, SGK>;
    case OUT_NVFP4: return &staged_kernel<K, SHI, kBf16, OUT_NVFP4, SGK>;
    case -1: return &staged_kernel<K, SHI, kBf16, -1, SGK>;
    default: return nullptr;
  }
}

template <int K, int SHI>
KsFn pick(int mode, int sgk) {
  if (mode == OUT_CODEBOOK) {
    if (sgk == SGK_NONE) return &staged_kernel<K, SHI, kBf16, OUT_CODEBOOK, SGK_NONE>;
    if constexpr (K == 1) {
      if (sgk == SGK_RPBH) return &staged_kernel<K, SHI, kBf16, OUT_CODEBOOK, SGK_RPBH>;
    }
    return nullptr;
  }
  if constexpr (K == 1) {
    return sgk == SGK_RPBH ? with_mode<K, SHI, SGK_RPBH>(mode) : nullptr;
  } else {
    if (sgk == SGK_NONE) return with_mode<K, SHI, SGK_NONE>(mode);
    if (sgk == SGK_BLOCK) return with_mode<K, SHI, SGK_BLOCK>(mode);
    return nullptr;
  }
}

}  // namespace

#if HADQ_KSIZE_BF16
KsFn staged_kernel_bf16(int k, int shi, int mode, int sgk) {
#else
KsFn staged_kernel_f32(int k, int shi, int mode, int sgk) {
#endif
  if (k == 1) {
    switch (shi) {
      case 1: return pick<1, 1>(mode, sgk);
      case 2: return pick<1, 2>(mode, sgk);
      case 4: return pick<1, 4>(mode, sgk);
      case 8: return pick<1, 8>(mode, sgk);
      case 16: return pick<1, 16>(mode, sgk);
      case 32: return pick<1, 32>(mode, sgk);
      case 64: return pick<1, 64>(mode, sgk);
      default: return nullptr;
    }
  }
  switch (k) {
    case 12: return shi == 1 ? pick<12, 1>(mode, sgk) : shi == 2 ? pick<12, 2>(mode, sgk)
                  : shi == 4 ? pick<12, 4>(mode, sgk) : nullptr;
    case 20: return shi == 1 ? pick<20, 1>(mode, sgk) : shi == 2 ? pick<20, 2>(mode, sgk) : nullptr;
    case 28: return shi == 1 ? pick<28, 1>(mode, sgk) : shi == 2 ? pick<28, 2>(mode, sgk) : nullptr;
    case 36: return shi == 1 ? pick<36, 1>(mode, sgk) : nullptr;
    case 52: return shi == 1 ? pick<52, 1>(mode, sgk) : nullptr;
    case 60: return shi == 1 ? pick<60, 1>(mode, sgk) : nullptr;
    case 108: return shi == 1 ? pick<108, 1>(mode, sgk) : nullptr;
    default: return nullptr;
  }
}

#if !HADQ_KSIZE_BF16
KsFn staged_kernel_for(int k, int shi, bool bf16, int mode, int sgk) {
  return bf16 ? staged_kernel_bf16(k, shi, mode, sgk) : staged_kernel_f32(k, shi, mode, sgk);
}
#endif

}  // namespace launch
}  // namespace hadq
