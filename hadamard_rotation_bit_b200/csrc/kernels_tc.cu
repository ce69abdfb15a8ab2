// Instantiations of the tensor-core kernels and their lookup; this unit also
// owns the kernels' fault word (hadq_tc_fault).
#include "hadq_launch.h"
#include "hadq_tc.cuh"
#include "hadq_tc128.cuh"

namespace hadq {
namespace launch {
namespace {

template <class C, int MODE, bool SG>
TcVariant tc_variant() {
  return TcVariant{&tc::tc_rotate_kernel<C, MODE, SG>, C::THREADS, C::SMEM_BYTES, C::TILE_N};
}

// n = 4096: 4 rows per tile, one row per epilogue warp, 3 stages.  n = 8192:
// 2 rows per tile, 4 stages; for int4 (whose epilogue is the heaviest) the
// MMAs are committed per row so the first row's epilogue starts early.
template <bool SG>
TcVariant tc_pick(int lo, int mode) {
  using C5 = tc::TcCfg<5, 128, 3, 4, false>;
  using C6 = tc::TcCfg<6, 128, 4, 2, false>;
  using C6H = tc::TcCfg<6, 128, 4, 2, true>;
  switch (mode) {
    case OUT_F32: return lo == 5 ? tc_variant<C5, OUT_F32, SG>() : tc_variant<C6, OUT_F32, SG>();
    case OUT_BF16: return lo == 5 ? tc_variant<C5, OUT_BF16, SG>() : tc_variant<C6, OUT_BF16, SG>();
    case OUT_INT4: return lo == 5 ? tc_variant<C5, OUT_INT4, SG>() : tc_variant<C6H, OUT_INT4, SG>();
    case OUT_NVFP4: return lo == 5 ? tc_variant<C5, OUT_NVFP4, SG>() : tc_variant<C6, OUT_NVFP4, SG>();
    case OUT_MXFP4: return lo == 5 ? tc_variant<C5, OUT_MXFP4, SG>() : tc_variant<C6, OUT_MXFP4, SG>();
    default: return TcVariant{nullptr, 0, 0, 0};
  }
}

using Tc128C = tc::Tc128Cfg<4, 2>;

template <bool SG>
Tc128Variant tc128_pick(int mode) {
  Tc128Fn fn = nullptr;
  switch (mode) {
    case OUT_F32: fn = &tc::tc128_kernel<Tc128C, OUT_F32, SG>; break;
    case OUT_BF16: fn = &tc::tc128_kernel<Tc128C, OUT_BF16, SG>; break;
    case OUT_INT4: fn = &tc::tc128_kernel<Tc128C, OUT_INT4, SG>; break;
    case OUT_MXFP4: fn = &tc::tc128_kernel<Tc128C, OUT_MXFP4, SG>; break;
    case OUT_NVFP4: fn = &tc::tc128_kernel<Tc128C, OUT_NVFP4, SG>; break;
    case -1: fn = &tc::tc128_kernel<Tc128C, -1, SG>; break;
    default: break;
  }
  return Tc128Variant{fn, Tc128C::THREADS, Tc128C::SMEM_BYTES};
}

}  // namespace

TcVariant tc_kernel_for(int lo, int mode, bool sg) {
  if (lo != 5 && lo != 6) return TcVariant{nullptr, 0, 0, 0};
  return sg ? tc_pick<true>(lo, mode) : tc_pick<false>(lo, mode);
}

Tc128Variant tc128_kernel_for(int mode, bool sg) { return sg ? tc128_pick<true>(mode) : tc128_pick<false>(mode); }

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
