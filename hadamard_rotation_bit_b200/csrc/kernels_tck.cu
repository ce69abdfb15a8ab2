// Instantiations of the tensor-core kernels for blocks of K * 128 * HI
// elements (hadq_tck.cuh) and their lookup; this unit owns their fault word.
#include "hadq_launch.h"
#include "hadq_tck.cuh"

namespace hadq {
namespace launch {
namespace {

// 4 stages of one block each, 8 blocks per CTA prefetched into L2 at entry,
// the epilogue through tensor memory.  Its widest step is the K-point mix of
// one h (K values and the mix's temporaries in registers), so the number of
// epilogue groups follows K: four (18 warps, at most 96 registers) up to
// K = 28, three (14 warps, 128 registers) up to K = 60, one (6 warps) for
// K = 108; fewer would leave warps idle, more would spill.  The accumulators
// (4 x 128 TMEM columns) bound the groups at four.
template <int K>
constexpr int tck_groups() {
  return K <= 28 ? 4 : (K <= 60 ? 3 : 1);
}

template <int K, int HI, int MODE>
TckVariant tck_variant() {
  using C = tc::TckCfg<K, HI, 4, tck_groups<K>(), 8, tc::tck_grouped<MODE>()>;
  return TckVariant{&tc::tck_kernel<C, MODE>, C::THREADS, C::SMEM_BYTES, C::NP};
}

template <int K, int HI>
TckVariant tck_modes(int mode) {
  switch (mode) {
    case OUT_F32: return tck_variant<K, HI, OUT_F32>();
    case OUT_BF16: return tck_variant<K, HI, OUT_BF16>();
    case -1: return tck_variant<K, HI, -1>();
    case OUT_INT4: return tck_variant<K, HI, OUT_INT4>();
    case OUT_MXFP4: return tck_variant<K, HI, OUT_MXFP4>();
    case OUT_NVFP4: return tck_variant<K, HI, OUT_NVFP4>();
    case OUT_MXFP4_BLOCKED: return tck_variant<K, HI, OUT_MXFP4_BLOCKED>();
    case OUT_NVFP4_BLOCKED: return tck_variant<K, HI, OUT_NVFP4_BLOCKED>();
    default: return TckVariant{nullptr, 0, 0, 0};
  }
}

}  // namespace

// Every Paley order with K * HI <= 128 chunks.
TckVariant tck_kernel_for(int k, int hi, int mode) {
  switch (k * 1000 + hi) {
    case 12001: return tck_modes<12, 1>(mode);
    case 12002: return tck_modes<12, 2>(mode);
    case 12004: return tck_modes<12, 4>(mode);
    case 12008: return tck_modes<12, 8>(mode);
    case 20001: return tck_modes<20, 1>(mode);
    case 20002: return tck_modes<20, 2>(mode);
    case 20004: return tck_modes<20, 4>(mode);
    case 28001: return tck_modes<28, 1>(mode);
    case 28002: return tck_modes<28, 2>(mode);
    case 28004: return tck_modes<28, 4>(mode);
    case 36001: return tck_modes<36, 1>(mode);
    case 36002: return tck_modes<36, 2>(mode);
    case 52001: return tck_modes<52, 1>(mode);
    case 52002: return tck_modes<52, 2>(mode);
    case 60001: return tck_modes<60, 1>(mode);
    case 60002: return tck_modes<60, 2>(mode);
    case 108001: return tck_modes<108, 1>(mode);
    default: return TckVariant{nullptr, 0, 0, 0};
  }
}

int tck_fault_bits(int clear) {
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
