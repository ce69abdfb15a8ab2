// Instantiations of the bf16-input team kernels (256 <= b <= 8192).
#include "hadq_kernels.cuh"
#include "hadq_launch.h"

namespace hadq {
namespace launch {
namespace {

template <int LOGB, bool BF, bool SG>
TeamFn team_fn(int mode) {
  switch (mode) {
    case OUT_F32: return &team_kernel<LOGB, BF, OUT_F32, SG>;
    case OUT_BF16: return &team_kernel<LOGB, BF, OUT_BF16, SG>;
    case OUT_INT4: return &team_kernel<LOGB, BF, OUT_INT4, SG>;
    case OUT_NVFP4: return &team_kernel<LOGB, BF, OUT_NVFP4, SG>;
    case OUT_MXFP4: return &team_kernel<LOGB, BF, OUT_MXFP4, SG>;
    default: return nullptr;
  }
}

template <bool BF, bool SG>
TeamFn team_fn_logb(int logb, int mode) {
  switch (logb) {
    case 8: return team_fn<8, BF, SG>(mode);
    case 9: return team_fn<9, BF, SG>(mode);
    case 10: return team_fn<10, BF, SG>(mode);
    case 11: return team_fn<11, BF, SG>(mode);
    case 12: return team_fn<12, BF, SG>(mode);
    case 13: return team_fn<13, BF, SG>(mode);
    default: return nullptr;
  }
}

template <bool BF, bool SG>
TeamRowFn team_row_fn(int logb) {
  switch (logb) {
    case 8: return &team_row_int8_kernel<8, BF, SG>;
    case 9: return &team_row_int8_kernel<9, BF, SG>;
    case 10: return &team_row_int8_kernel<10, BF, SG>;
    case 11: return &team_row_int8_kernel<11, BF, SG>;
    case 12: return &team_row_int8_kernel<12, BF, SG>;
    case 13: return &team_row_int8_kernel<13, BF, SG>;
    default: return nullptr;
  }
}

}  // namespace

TeamFn team_kernel_bf16(int logb, int mode, bool sg) {
  return sg ? team_fn_logb<true, true>(logb, mode) : team_fn_logb<true, false>(logb, mode);
}

TeamRowFn team_row_kernel_bf16(int logb, bool sg) {
  return sg ? team_row_fn<true, true>(logb) : team_row_fn<true, false>(logb);
}

}  // namespace launch
}  // namespace hadq
