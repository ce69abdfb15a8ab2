// Instantiations of the segment kernels (b <= 128) and their lookup.
#include "hadq_kernels.cuh"
#include "hadq_launch.h"

namespace hadq {
namespace launch {
namespace {

template <int LOGS, bool BF, bool FULL, bool SG>
SegFn seg_fn(int mode) {
  switch (mode) {
    case OUT_F32: return &segment_kernel<LOGS, BF, OUT_F32, FULL, SG>;
    case OUT_BF16: return &segment_kernel<LOGS, BF, OUT_BF16, FULL, SG>;
    case OUT_INT4:
      if constexpr (LOGS >= 5) return &segment_kernel<LOGS, BF, OUT_INT4, FULL, SG>;
      return nullptr;
    case OUT_NVFP4:
      if constexpr (LOGS >= 4) return &segment_kernel<LOGS, BF, OUT_NVFP4, FULL, SG>;
      return nullptr;
    case OUT_MXFP4:
      if constexpr (LOGS >= 5) return &segment_kernel<LOGS, BF, OUT_MXFP4, FULL, SG>;
      return nullptr;
    default:
      return nullptr;
  }
}

// The launcher makes a segment max(b, 16) or max(b, 32) elements (at most the
// largest power of 2 dividing n), so a segment longer than its block (!FULL)
// is at most 32 elements; 64- and 128-element segments are whole blocks.
template <bool BF, bool FULL, bool SG>
SegFn seg_fn_logs(int logs, int mode) {
  switch (logs) {
    case 3: return seg_fn<3, BF, FULL, SG>(mode);
    case 4: return seg_fn<4, BF, FULL, SG>(mode);
    case 5: return seg_fn<5, BF, FULL, SG>(mode);
    case 6:
      if constexpr (FULL) return seg_fn<6, BF, FULL, SG>(mode);
      return nullptr;
    case 7:
      if constexpr (FULL) return seg_fn<7, BF, FULL, SG>(mode);
      return nullptr;
    default: return nullptr;
  }
}

template <bool BF, bool FULL, bool SG>
SegRowFn seg_row_fn(int logs) {
  switch (logs) {
    case 3: return &segment_row_int8_kernel<3, BF, FULL, SG>;
    case 4: return &segment_row_int8_kernel<4, BF, FULL, SG>;
    case 5: return &segment_row_int8_kernel<5, BF, FULL, SG>;
    case 6: return &segment_row_int8_kernel<6, BF, FULL, SG>;
    case 7: return &segment_row_int8_kernel<7, BF, FULL, SG>;
    default: return nullptr;
  }
}

template <bool SG>
SegFn seg_any(bool bf16, bool full, int logs, int mode) {
  if (bf16) return full ? seg_fn_logs<true, true, SG>(logs, mode) : seg_fn_logs<true, false, SG>(logs, mode);
  return full ? seg_fn_logs<false, true, SG>(logs, mode) : seg_fn_logs<false, false, SG>(logs, mode);
}

template <bool SG>
SegRowFn seg_row_any(bool bf16, bool full, int logs) {
  if (bf16) return full ? seg_row_fn<true, true, SG>(logs) : seg_row_fn<true, false, SG>(logs);
  return full ? seg_row_fn<false, true, SG>(logs) : seg_row_fn<false, false, SG>(logs);
}

}  // namespace

SegFn segment_kernel_for(bool bf16, bool full, int logs, int mode, bool sg) {
  return sg ? seg_any<true>(bf16, full, logs, mode) : seg_any<false>(bf16, full, logs, mode);
}

SegRowFn segment_row_kernel_for(bool bf16, bool full, int logs, bool sg) {
  return sg ? seg_row_any<true>(bf16, full, logs) : seg_row_any<false>(bf16, full, logs);
}

}  // namespace launch
}  // namespace hadq
