// Instantiations of the tensor-core kernels and their lookup; this unit also
// owns the kernels' fault word (hadq_tc_fault).
#include "hadq_launch.h"
#include "hadq_tc.cuh"
#include "hadq_tc128.cuh"
#include "hadq_tcr.cuh"

#include <type_traits>

namespace hadq {
namespace launch {
namespace {

template <class C, int MODE, int SIDE>
TcVariant tc_variant() {
  return TcVariant{&tc::tc_rotate_kernel<C, MODE, SIDE>, tc::tc_threads<C, SIDE>(), C::SMEM_BYTES, C::TILE_N};
}

// n = 4096: 4 rows per tile, one row per epilogue warp, 3 stages, H_128 held
// in tensor memory (the MMAs read only the B tile from shared memory):
// 4096 x 4096 int4 9.57 us per launch against 9.62 with H_128 in shared
// memory; signs before the rotation 11.42 against 11.54 (the best shared-
// memory layout there, 4 stages).  n = 8192: 2 rows per tile, 4 stages; for
// int4 (whose epilogue is the heaviest) the MMAs are committed per row so the
// first row's epilogue starts early.
template <int SIDE>
TcVariant tc_pick(int lo, int mode) {
  using C5 = tc::TcCfg<5, 128, 3, 4, false, 2, false, true>;
  using C6 = tc::TcCfg<6, 128, 4, 2, false>;
  using C6H = tc::TcCfg<6, 128, 4, 2, true>;
  switch (mode) {
    case OUT_F32: return lo == 5 ? tc_variant<C5, OUT_F32, SIDE>() : tc_variant<C6, OUT_F32, SIDE>();
    case OUT_BF16: return lo == 5 ? tc_variant<C5, OUT_BF16, SIDE>() : tc_variant<C6, OUT_BF16, SIDE>();
    case OUT_INT4: return lo == 5 ? tc_variant<C5, OUT_INT4, SIDE>() : tc_variant<C6H, OUT_INT4, SIDE>();
    case OUT_NVFP4: return lo == 5 ? tc_variant<C5, OUT_NVFP4, SIDE>() : tc_variant<C6, OUT_NVFP4, SIDE>();
    case OUT_MXFP4: return lo == 5 ? tc_variant<C5, OUT_MXFP4, SIDE>() : tc_variant<C6, OUT_MXFP4, SIDE>();
    case OUT_MXFP4_BLOCKED:
      return lo == 5 ? tc_variant<C5, OUT_MXFP4_BLOCKED, SIDE>() : tc_variant<C6, OUT_MXFP4_BLOCKED, SIDE>();
    case OUT_NVFP4_BLOCKED:
      return lo == 5 ? tc_variant<C5, OUT_NVFP4_BLOCKED, SIDE>() : tc_variant<C6, OUT_NVFP4_BLOCKED, SIDE>();
    default: return TcVariant{nullptr, 0, 0, 0};
  }
}

using Tc128C = tc::Tc128Cfg<4, 2, 8>;

}  // namespace

namespace {
template <int E>
Tc128Fn tc128_fn(int mode) {
  switch (mode) {
    case OUT_F32: return &tc::tc128_kernel<Tc128C, OUT_F32, E>;
    case OUT_BF16: return &tc::tc128_kernel<Tc128C, OUT_BF16, E>;
    case OUT_INT4: return &tc::tc128_kernel<Tc128C, OUT_INT4, E>;
    case OUT_MXFP4: return &tc::tc128_kernel<Tc128C, OUT_MXFP4, E>;
    case OUT_NVFP4: return &tc::tc128_kernel<Tc128C, OUT_NVFP4, E>;
    case OUT_MXFP4_BLOCKED: return &tc::tc128_kernel<Tc128C, OUT_MXFP4_BLOCKED, E>;
    case OUT_NVFP4_BLOCKED: return &tc::tc128_kernel<Tc128C, OUT_NVFP4_BLOCKED, E>;
    default: return nullptr;
  }
}
}  // namespace

Tc128Variant tc128_kernel_for(int mode, int e) {
  Tc128Fn fn = nullptr;
  switch (e) {
    case 0: fn = mode == -1 ? &tc::tc128_kernel<Tc128C, -1> : tc128_fn<0>(mode); break;
    case 1: fn = tc128_fn<1>(mode); break;
    case 2: fn = tc128_fn<2>(mode); break;
    case 3: fn = tc128_fn<3>(mode); break;
    case 4: fn = tc128_fn<4>(mode); break;
    default: break;
  }
  return Tc128Variant{fn, Tc128C::THREADS, Tc128C::SMEM_BYTES};
}

TcrVariant tcr_kernel_for(int mode) {
  TcrFn fn = nullptr;
  switch (mode) {
    case OUT_F32: fn = &tc::tc_rpbh_kernel<OUT_F32>; break;
    case OUT_BF16: fn = &tc::tc_rpbh_kernel<OUT_BF16>; break;
    case OUT_INT4: fn = &tc::tc_rpbh_kernel<OUT_INT4>; break;
    case OUT_MXFP4: fn = &tc::tc_rpbh_kernel<OUT_MXFP4>; break;
    case OUT_NVFP4: fn = &tc::tc_rpbh_kernel<OUT_NVFP4>; break;
    case OUT_CODEBOOK: fn = &tc::tc_rpbh_kernel<OUT_CODEBOOK>; break;
    default: break;
  }
  return TcrVariant{fn, tc::TcrCfg::THREADS, tc::TcrCfg::SMEM_BYTES};
}

TcVariant tc_kernel_for(int lo, int mode, int side) {
  if (lo != 5 && lo != 6) return TcVariant{nullptr, 0, 0, 0};
  switch (side) {
    case SIGNS_NONE: return tc_pick<SIGNS_NONE>(lo, mode);
    case SIGNS_BEFORE: return tc_pick<SIGNS_BEFORE>(lo, mode);
    case SIGNS_AFTER: return tc_pick<SIGNS_AFTER>(lo, mode);
    default: return TcVariant{nullptr, 0, 0, 0};
  }
}

int tc_fault_bits(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tc::hadq_tc_fault, sizeof(v)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(tc::hadq_tc_fault, &z, sizeof(z)) != cudaSuccess) return -1;
  }
  return static_cast<int>(v);
}

}  // namespace launch
}  // namespace hadq
