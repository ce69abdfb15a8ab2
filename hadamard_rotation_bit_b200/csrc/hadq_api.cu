// libhadq host side: argument validation, launch planning and the C ABI.
//
// Every check runs before the first CUDA call, so a failing call launches
// nothing and leaves all outputs untouched (validate first, then apply -- the
// rule the apply_spinquant docstring states for its rotation passes).  There
// is no CPU path: a missing device or kernel image surfaces as HADQ_ERR_CUDA.
#include "hadq.h"
#include "hadq_kernels.cuh"   // launch constants only; the kernels are instantiated elsewhere
#include "hadq_ksize.cuh"
#include "hadq_launch.h"

#include <cudaTypedefs.h>

#include <atomic>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <utility>
#include <mutex>
#include <string>
#include <tuple>

namespace {

thread_local std::string g_last_error;

hadq_status fail(hadq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

bool is_pow2(int64_t v) { return v >= 1 && (v & (v - 1)) == 0; }

int ilog2(int64_t v) {
  int k = 0;
  while ((int64_t(1) << k) < v) ++k;
  return k;
}

int64_t esize(hadq_dtype d) { return d == HADQ_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Span {
  uintptr_t lo = 0, hi = 0;
};

Span span(const void* p, int64_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return Span{a, a + static_cast<uintptr_t>(bytes)};
}

bool overlaps(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi; }

constexpr int kMaxBlock = 8192;
constexpr int64_t kMaxInt8N = 32768;

// What the kernels need to know about one call.
struct Shape {
  int64_t rows = 0, n = 0, b = 0;
  int kbase = 1;  // b = kbase * 2^logk: 1 for a power of 2, else a covered Paley order
  int logk = 0;
  int logb = 0;   // log2(b) when kbase == 1
  int logs = 0;   // segment kernels: log2 of the per-thread segment
  float norm = 1.f;
};

// Base orders K of the non-power-of-2 sizes b = K * 2^m (Paley II matrices;
// the kernels build the same ones at compile time).
constexpr int kPaleyOrders[] = {12, 20, 28, 36, 52, 60, 108};

// b = K * 2^m with a covered K: K (or 0 if none), and m.
int split_size(int64_t b, int* logk) {
  int64_t odd = b;
  int m = 0;
  while (odd % 2 == 0) {
    odd /= 2;
    ++m;
  }
  for (int k : kPaleyOrders)
    if (k == 4 * odd && m >= 2) {
      *logk = m - 2;
      return k;
    }
  return 0;
}

hadq_status check_shape(hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, Shape* sh) {
  if (x_dtype != HADQ_F32 && x_dtype != HADQ_BF16) return fail(HADQ_ERR_INVALID_ARG, "x_dtype must be HADQ_F32 or HADQ_BF16");
  if (rows < 0) return fail(HADQ_ERR_INVALID_ARG, "rows must be >= 0");
  if (n <= 0) return fail(HADQ_ERR_INVALID_ARG, "n must be > 0");
  if (block < -1) return fail(HADQ_ERR_INVALID_ARG, "block must be -1, 0 (full) or a block size dividing n");
  const bool full = block == -1 || block == 0 || block == n;
  const int64_t b = full ? n : block;
  if (n % b != 0) return fail(HADQ_ERR_INVALID_ARG, "block must divide n");
  if (n % 8 != 0) return fail(HADQ_ERR_UNSUPPORTED, "n must be a multiple of 8");
  if (rows > (INT64_MAX / 8) / n) return fail(HADQ_ERR_INVALID_ARG, "rows * n overflows");
  sh->rows = rows;
  sh->n = n;
  sh->b = b;
  sh->norm = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
  const int64_t low = n & (-n);                 // largest power of 2 dividing n
  sh->logs = ilog2(low < 128 ? low : 128);
  if (is_pow2(b)) {
    if (b > kMaxBlock) return fail(HADQ_ERR_UNSUPPORTED, "rotation blocks above 8192 are not supported");
    sh->kbase = 1;
    sh->logb = ilog2(b);
    return HADQ_OK;
  }
  int logk = 0;
  const int k = split_size(b, &logk);
  if (k == 0)
    return fail(HADQ_ERR_INVALID_ARG, full ? "a full rotation needs n = 2^m or K * 2^m with K in {12, 20, 28, 36, 52, 60, 108}"
                                           : "block must be 2^m or K * 2^m with K in {12, 20, 28, 36, 52, 60, 108}");
  if (logk < 6 || b / 64 > hadq::ksize::kMaxThreads)
    return fail(HADQ_ERR_UNSUPPORTED, "K * 2^m rotations need 2^m >= 64 and K * 2^m <= 32768");
  sh->kbase = k;
  sh->logk = logk;
  sh->logb = -1;
  return HADQ_OK;
}

hadq_status check_quant(hadq_fmt fmt, int64_t group, const Shape& sh, int* eff_group) {
  switch (fmt) {
    case HADQ_INT4_SYM:
      if (group != 32 && group != 64 && group != 128) return fail(HADQ_ERR_INVALID_ARG, "int4 group must be 32, 64 or 128");
      if (sh.n % group != 0) return fail(HADQ_ERR_INVALID_ARG, "int4 group must divide n");
      *eff_group = static_cast<int>(group);
      return HADQ_OK;
    case HADQ_INT8_SYM:
      if (group != 0 && group != sh.n) return fail(HADQ_ERR_INVALID_ARG, "int8 is per token: group must be 0 or n");
      if (sh.n > kMaxInt8N) return fail(HADQ_ERR_UNSUPPORTED, "per-token int8 supports n <= 32768");
      if (sh.kbase > 1 && sh.b != sh.n) return fail(HADQ_ERR_UNSUPPORTED, "per-token int8 with a K * 2^m block needs the full row");
      if (sh.kbase == 1 && sh.b <= 128 && (sh.n >> sh.logs) > 256)
        return fail(HADQ_ERR_UNSUPPORTED, "per-token int8: n / segment exceeds 256 threads");
      *eff_group = static_cast<int>(sh.n);
      return HADQ_OK;
    case HADQ_MXFP4:
      if (group != 0 && group != 32) return fail(HADQ_ERR_INVALID_ARG, "MXFP4 group must be 0 or 32");
      if (sh.n % 32 != 0) return fail(HADQ_ERR_INVALID_ARG, "MXFP4 needs n to be a multiple of 32");
      *eff_group = 32;
      return HADQ_OK;
    case HADQ_NVFP4:
      if (group != 0 && group != 16) return fail(HADQ_ERR_INVALID_ARG, "NVFP4 group must be 0 or 16");
      if (sh.n % 16 != 0) return fail(HADQ_ERR_INVALID_ARG, "NVFP4 needs n to be a multiple of 16");
      *eff_group = 16;
      return HADQ_OK;
    case HADQ_MXFP4_BLOCKED:
    case HADQ_NVFP4_BLOCKED: {
      const int blk = fmt == HADQ_MXFP4_BLOCKED ? 32 : 16;
      if (group != 0 && group != blk)
        return fail(HADQ_ERR_INVALID_ARG, fmt == HADQ_MXFP4_BLOCKED ? "MXFP4 group must be 0 or 32"
                                                                      : "NVFP4 group must be 0 or 16");
      if (sh.n % (4 * blk) != 0)
        return fail(HADQ_ERR_INVALID_ARG, "blocked scales need whole 4-column tiles: n a multiple of 4 x the block");
      *eff_group = blk;
      return HADQ_OK;
    }
    default:
      return fail(HADQ_ERR_INVALID_ARG,
                  "fmt must be HADQ_INT4_SYM, HADQ_INT8_SYM, HADQ_MXFP4, HADQ_NVFP4 or a blocked FP4 format");
  }
}

bool blocked_fmt(hadq_fmt fmt) { return fmt == HADQ_MXFP4_BLOCKED || fmt == HADQ_NVFP4_BLOCKED; }

int64_t codes_bytes(int64_t rows, int64_t n, hadq_fmt fmt) {
  return fmt == HADQ_INT8_SYM ? rows * n : rows * n / 2;
}

// The tiled GEMM scale layout pads the rows to a multiple of 128.
int64_t padded_scale_rows(int64_t rows) { return (rows + 127) / 128 * 128; }

int64_t scales_bytes(int64_t rows, int64_t n, hadq_fmt fmt, int group) {
  switch (fmt) {
    case HADQ_INT4_SYM: return rows * (n / group) * 2;
    case HADQ_INT8_SYM: return rows * 4;
    case HADQ_NVFP4: return rows * (n / 16);
    case HADQ_MXFP4_BLOCKED: return padded_scale_rows(rows) * (n / 32);
    case HADQ_NVFP4_BLOCKED: return padded_scale_rows(rows) * (n / 16);
    default: return rows * (n / 32);
  }
}

// ------------------------------------------------------------ kernel lookups

using hadq::Signs;
namespace hl = hadq::launch;

// ------------------------------------------------- per-device launch caches

std::mutex g_mu;
std::map<int, int> g_sms;                                    // device -> SM count
std::map<std::tuple<int, const void*, int, int>, int> g_occ; // (device, fn, block, smem) -> CTAs/SM

hadq_status device_sms(int* sms, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_sms.find(dev);
  if (it == g_sms.end()) {
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    it = g_sms.emplace(dev, v).first;
  }
  *sms = it->second;
  *dev_out = dev;
  return HADQ_OK;
}

// Resident CTAs per SM for `fn` at this block/smem size.  Also raises the
// dynamic shared memory limit of `fn` on this device when it needs more than
// 48 KB; the limit only ever grows (a kernel whose shared memory depends on
// the call must keep the largest size any earlier call of it needed).
std::map<std::pair<int, const void*>, int> g_smem_limit;   // (device, fn) -> dynamic smem limit set

hadq_status occupancy(const void* fn, int dev, int block, int smem, int* occ) {
  std::lock_guard<std::mutex> lk(g_mu);
  const auto key = std::make_tuple(dev, fn, block, smem);
  auto it = g_occ.find(key);
  if (it == g_occ.end()) {
    cudaError_t e = cudaSuccess;
    int& limit = g_smem_limit[std::make_pair(dev, fn)];
    if (smem > limit) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      limit = smem;
    }
    int v = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, block, smem);
    if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("occupancy query: ") + cudaGetErrorString(e));
    if (v < 1) return fail(HADQ_ERR_CUDA, "kernel does not fit on an SM");
    it = g_occ.emplace(key, v).first;
  }
  *occ = it->second;
  return HADQ_OK;
}

hadq_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return HADQ_OK;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream drains; it waits for that kernel's
// completion (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*fn)(KArgs...), int64_t grid, int block, int smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, args...);
}

hadq_status launch_result(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return check_launch(what);
}

// ------------------------------------------------------- tensor-core path

// Which implementation serves the calls both implementations cover (bf16
// input at full size 4096 / 8192 and at block 128): set process-wide through
// hadq_set_impl, HADQ_IMPL_AUTO (the tcgen05 + TMA kernels) by default.
std::atomic<int> g_impl{HADQ_IMPL_AUTO};

bool tc_eligible(hadq_dtype x_dtype, const Shape& sh, int mode) {
  return x_dtype == HADQ_BF16 && sh.kbase == 1 && (sh.logb == 12 || sh.logb == 13) && mode >= 0;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Blocks of b = 2^(7 + LO) bf16 elements, each rotated in full: the blocks are
// the rows of a (rows * n / b) x b matrix.
hadq_status launch_tc(const void* x, const Shape& sh, int mode, int group, void* out0, void* out1,
                      cudaStream_t stream, int sms, int dev, Signs sg) {
  const int lo = sh.logb - 7;
  const hl::TcVariant v = hl::tc_kernel_for(lo, mode, sg.side);
  if (v.fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no tensor-core kernel for this size and format");
  const int L = 1 << lo, R = v.tile_n / L;
  const int64_t rows = sh.rows * (sh.n >> sh.logb);
  if (rows > (int64_t(1) << 31) - R) return fail(HADQ_ERR_UNSUPPORTED, "tensor-core path: too many rows");
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (encode == nullptr) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  CUtensorMap map;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(L), 128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(L) * 2, static_cast<cuuint64_t>(sh.b) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(L), 128, static_cast<cuuint32_t>(R)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            lo == 5 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  int occ = 0;
  hadq_status st = occupancy(reinterpret_cast<const void*>(v.fn), dev, v.threads, v.smem, &occ);
  if (st != HADQ_OK) return st;
  const int64_t tiles = (rows + R - 1) / R;
  const int64_t grid = std::min<int64_t>(tiles, sms);
  return launch_result(launch_pdl(v.fn, grid, v.threads, v.smem, stream, map, static_cast<const uint16_t*>(x), rows,
                                  static_cast<int>(sh.b), sh.norm, group, out0, out1, sg),
                       "tensor-core kernel launch");
}

// Scale columns per row of the tiled-scale FP4 formats (0 otherwise).
int tiled_scale_cols(const Shape& sh, int mode) {
  if (mode == hadq::OUT_MXFP4_BLOCKED) return static_cast<int>(sh.n / 32);
  if (mode == hadq::OUT_NVFP4_BLOCKED) return static_cast<int>(sh.n / 16);
  return 0;
}

// Block-128 rotations of bf16 rows on the tensor cores: every 128-element
// chunk is a row of the MMA's A operand.  Per-token int8 takes one row per
// tile and so needs 32 <= n / 128 <= 128 with n / 128 a multiple of 8.
// Blocks of 256 .. 2048 (block or full size) take the same kernel with the
// remaining stages across neighbouring lanes: unsigned, rotation outputs and
// the grouped quantizers.
bool tc128_eligible(hadq_dtype x_dtype, const Shape& sh, int mode, Signs sg) {
  if (x_dtype != HADQ_BF16 || sh.kbase != 1 || sh.logb < 7 || sh.logb > 11) return false;
  if (sh.logb > 7) return mode >= 0 && mode != hadq::OUT_CODEBOOK && sg.side == hadq::SIGNS_NONE;
  if (mode >= 0) return true;
  const int64_t bpr = sh.n >> 7;            // whole 8-row swizzle atoms per tile
  return bpr >= 32 && bpr <= 128 && bpr % 8 == 0;
}

hadq_status launch_tc128(const void* x, const Shape& sh, int mode, int group, void* out0, void* out1,
                         cudaStream_t stream, int sms, int dev, Signs sg) {
  const int64_t blocks = sh.rows * (sh.n >> 7);
  if (blocks > (int64_t(1) << 31) - 256) return fail(HADQ_ERR_UNSUPPORTED, "tensor-core path: too many blocks");
  const int bpt = mode < 0 ? static_cast<int>(sh.n >> 7) : 128;   // blocks per tile
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (encode == nullptr) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  CUtensorMap maps[2];
  for (int p = 0; p < 2; ++p) {
    cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(blocks)};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(bpt)};
    cuuint32_t estr[2] = {1, 1};
    void* base = const_cast<char*>(static_cast<const char*>(x)) + 128 * p;
    const CUresult r = encode(&maps[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  }
  const hl::Tc128Variant v = hl::tc128_kernel_for(mode, sh.logb - 7);
  if (v.fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no block-128 tensor-core kernel for this format");
  int occ = 0;
  hadq_status st = occupancy(reinterpret_cast<const void*>(v.fn), dev, v.threads, v.smem, &occ);
  if (st != HADQ_OK) return st;
  const int64_t tiles = (blocks + bpt - 1) / bpt;
  const int64_t grid = std::min<int64_t>(tiles, sms);
  return launch_result(launch_pdl(v.fn, grid, v.threads, v.smem, stream, maps[0], maps[1],
                                  static_cast<const uint16_t*>(x), blocks, bpt, sh.norm, group, out0, out1, sg,
                                  tiled_scale_cols(sh, mode)),
                       "tensor-core block-128 kernel launch");
}

// RPBH at full size 4096, bf16 input, on the tensor cores (hadq_tcr.cuh): the
// permutation and signs applied by gather warps in shared memory, then the
// n = 4096 rotation and epilogue.  Rotation outputs, int4, MXFP4, NVFP4 and
// the codebook quantizer.
bool tcr_eligible(hadq_dtype x_dtype, const Shape& sh, int mode) {
  return x_dtype == HADQ_BF16 && sh.kbase == 1 && sh.n == 4096 && sh.b == 4096 && mode >= 0;
}

hadq_status launch_tcr(const void* x, const Shape& sh, int mode, int group, void* out0, void* out1,
                       cudaStream_t stream, int sms, int dev, const int32_t* perm, const int8_t* signs,
                       const double* thr) {
  const hl::TcrVariant v = hl::tcr_kernel_for(mode);
  if (v.fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no RPBH tensor-core kernel for this format");
  constexpr int L = 32, R = 4;
  if (sh.rows > (int64_t(1) << 31) - R) return fail(HADQ_ERR_UNSUPPORTED, "tensor-core path: too many rows");
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (encode == nullptr) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  CUtensorMap map;
  cuuint64_t dims[3] = {L, 128, static_cast<cuuint64_t>(sh.rows)};
  cuuint64_t strides[2] = {L * 2, static_cast<cuuint64_t>(sh.n) * 2};
  cuuint32_t box[3] = {L, 128, R};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  int occ = 0;
  hadq_status st = occupancy(reinterpret_cast<const void*>(v.fn), dev, v.threads, v.smem, &occ);
  if (st != HADQ_OK) return st;
  const int64_t tiles = (sh.rows + R - 1) / R;
  const int64_t grid = std::min<int64_t>(tiles, sms);
  return launch_result(launch_pdl(v.fn, grid, v.threads, v.smem, stream, map, static_cast<const uint16_t*>(x), sh.rows,
                                  static_cast<int>(sh.n), sh.norm, group, out0, out1, perm, signs, thr),
                       "RPBH tensor-core kernel launch");
}

// Blocks of b = K * 128 * hi bf16 elements on the tensor cores
// (hadq_tck.cuh): H_128 on every 128-element chunk by one MMA, the H_hi and
// Paley H_K factors by the thread that holds one output of every chunk
// (through tensor memory), so K * hi <= 128.  Rotation outputs, int4, MXFP4,
// NVFP4, and per-token int8 over whole rows (b = n); signs, the RPBH
// permutation and the codebook take the staged kernels.
bool tck_eligible(hadq_dtype x_dtype, const Shape& sh, int mode, Signs sg) {
  if (x_dtype != HADQ_BF16 || sh.kbase == 1 || sh.logk < 7 || sg.side != hadq::SIGNS_NONE) return false;
  if (static_cast<int64_t>(sh.kbase) << (sh.logk - 7) > 128) return false;
  if (mode < 0) return sh.b == sh.n;
  return mode == hadq::OUT_F32 || mode == hadq::OUT_BF16 || mode == hadq::OUT_INT4 || mode == hadq::OUT_MXFP4 ||
         mode == hadq::OUT_NVFP4 || mode == hadq::OUT_MXFP4_BLOCKED || mode == hadq::OUT_NVFP4_BLOCKED;
}


hadq_status launch_tck(const void* x, const Shape& sh, int mode, int group, void* out0, void* out1,
                       cudaStream_t stream, int sms, int dev) {
  const hl::TckVariant v = hl::tck_kernel_for(sh.kbase, 1 << (sh.logk - 7), mode);
  if (v.fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no K * 2^m tensor-core kernel for this size and format");
  const int64_t chunks = sh.rows * (sh.n >> 7);
  if (chunks > (int64_t(1) << 31) - 256) return fail(HADQ_ERR_UNSUPPORTED, "tensor-core path: too many blocks");
  const int64_t blocks = sh.rows * (sh.n / sh.b);
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (encode == nullptr) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  // The chunks are the rows of a chunks x 128 matrix, loaded as two 64-wide
  // K-panels of v.np chunks (the block's chunks, then padding that is never read).
  CUtensorMap maps[2];
  for (int p = 0; p < 2; ++p) {
    cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(chunks)};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(v.np)};
    cuuint32_t estr[2] = {1, 1};
    void* base = const_cast<char*>(static_cast<const char*>(x)) + 128 * p;
    const CUresult r = encode(&maps[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(HADQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  }
  int occ = 0;
  hadq_status st = occupancy(reinterpret_cast<const void*>(v.fn), dev, v.threads, v.smem, &occ);
  if (st != HADQ_OK) return st;
  const int64_t grid = std::min<int64_t>(blocks, sms);
  return launch_result(launch_pdl(v.fn, grid, v.threads, v.smem, stream, maps[0], maps[1],
                                  static_cast<const uint16_t*>(x), blocks, sh.norm, group, out0, out1,
                                  tiled_scale_cols(sh, mode)),
                       "K * 2^m tensor-core kernel launch");
}

// Blocks of b = K * 2^m elements (one CTA per block, persistent over blocks).
// What the shared-memory staged kernels need beyond the shape: the RPBH
// permutation (with n signs) and the codebook thresholds.
struct Extra {
  const int32_t* perm = nullptr;
  const int8_t* rpbh_signs = nullptr;
  const double* thr = nullptr;
  int bits = 0;
};

// Shared-memory staged kernels (hadq_ksize.cuh): blocks of K * 2^m elements,
// and any power-of-2 block with the RPBH permutation or the codebook
// quantizer.  A unit is a block, or the whole row when the quantizer needs
// row statistics (per-token int8, codebook) or the permutation spans the row.
hadq_status launch_staged(const void* x, hadq_dtype x_dtype, const Shape& sh, int mode, int group, void* out0,
                          void* out1, cudaStream_t stream, int sms, int dev, Signs sg, const Extra& ex) {
  namespace ks = hadq::ksize;
  const bool bf = x_dtype == HADQ_BF16;
  const int sgk = ex.perm != nullptr ? ks::SGK_RPBH : (sg.side != hadq::SIGNS_NONE ? ks::SGK_BLOCK : ks::SGK_NONE);
  const bool per_row = mode < 0 || mode == hadq::OUT_CODEBOOK || sgk == ks::SGK_RPBH;
  const int64_t unit = per_row ? sh.n : sh.b;
  if (unit % 64 != 0 || unit / 64 > ks::kMaxThreads)
    return fail(HADQ_ERR_UNSUPPORTED, per_row ? "this quantizer / permutation needs n a multiple of 64 and n <= 32768"
                                              : "K * 2^m blocks need 2^m >= 64 and K * 2^m <= 32768");
  // The column stage mixes K * SHI values per column in registers (at most
  // 64); the butterfly stage runs the S_lo = 2^m / SHI points left, 64 and
  // more in runs of 64 with shuffles across lanes for the rest.  SHI as large
  // as both allow, so as few shuffle stages as possible remain.
  const int logm = sh.kbase == 1 ? sh.logb : sh.logk;
  int logshi = 0;
  while ((sh.kbase << (logshi + 1)) <= 64 && logm - (logshi + 1) >= 6) ++logshi;
  const int shi = 1 << logshi, logs_lo = logm - logshi;
  const hl::KsFn fn = hl::staged_kernel_for(sh.kbase, shi, bf, mode, sgk);
  if (fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no staged kernel for this size, format and sign variant");
  const int64_t smem = ks::smem_bytes(unit, bf ? 2 : 4, sgk, sh.b);
  if (smem > 227 * 1024) return fail(HADQ_ERR_UNSUPPORTED, "row or block too large for the staged kernel's shared memory");
  // One thread per 64-value run in the butterfly stage and one per column in
  // the column stage, whichever needs more (threads beyond either sit out).
  const int64_t cols = unit / (int64_t(sh.kbase) * shi);
  const int threads = static_cast<int>(
      std::min<int64_t>(ceil_div(std::max<int64_t>(unit / 64, cols), 32) * 32, hadq::ksize::kMaxThreads));
  int occ = 0;
  hadq_status st = occupancy(reinterpret_cast<const void*>(fn), dev, threads, static_cast<int>(smem), &occ);
  if (st != HADQ_OK) return st;
  ks::StageArgs a;
  a.x = x;
  a.units = sh.rows * (sh.n / unit);
  a.unit_len = static_cast<int>(unit);
  a.b = static_cast<int>(sh.b);
  a.logs_lo = logs_lo;
  a.norm = sh.norm;
  a.group = group;
  a.bits = ex.bits;
  a.out0 = out0;
  a.out1 = out1;
  a.sg = sgk == ks::SGK_RPBH ? Signs{ex.rpbh_signs, hadq::SIGNS_BEFORE} : sg;
  a.perm = ex.perm;
  a.thr = ex.thr;
  const int64_t grid = std::min<int64_t>(a.units, int64_t(sms) * occ);
  return launch_result(launch_pdl(fn, grid, threads, static_cast<int>(smem), stream, a), "staged kernel launch");
}

// Launch the kernel for an already validated call.  mode: hadq::OutMode, or
// -1 for per-token int8.
hadq_status launch(const void* x, hadq_dtype x_dtype, const Shape& sh, int mode, int group, void* out0, void* out1,
                   cudaStream_t stream, Signs sg = Signs{nullptr, hadq::SIGNS_NONE}, const Extra& ex = Extra{}) {
  int sms = 0, dev = 0;
  hadq_status st = device_sms(&sms, &dev);
  if (st != HADQ_OK) return st;
  const bool bf = x_dtype == HADQ_BF16;
  const bool full_seg = sh.logb == sh.logs;
  const bool sgd = sg.side != hadq::SIGNS_NONE;
  // Segment kernels: a thread owns S = max(b, the quantizer's span, 16)
  // consecutive elements (at most 128 and at most the largest power of 2
  // dividing n), so a block of b >= 16 is a whole segment (fixed butterfly,
  // no run-time stage count) and smaller blocks keep short register arrays.
  // The span is 32 for int4 (larger groups span 2 or 4 neighbouring
  // segments, joined by shuffles) and MXFP4, 16 for NVFP4 and rotations.
  int seg_logs = sh.logs;
  if (mode >= 0 && sh.b <= 128) {
    const int need = mode == hadq::OUT_INT4 || mode == hadq::OUT_MXFP4 ? 32 : 16;
    seg_logs = std::min(sh.logs, std::max(std::max(sh.logb, ilog2(need)), 4));
  }
  (void)cudaGetLastError();   // launch errors below must be ours
  if (ex.perm != nullptr && g_impl.load(std::memory_order_relaxed) != HADQ_IMPL_BUTTERFLY &&
      tcr_eligible(x_dtype, sh, mode))
    return launch_tcr(x, sh, mode, mode == hadq::OUT_CODEBOOK ? ex.bits : group, out0, out1, stream, sms, dev, ex.perm,
                      ex.rpbh_signs, ex.thr);
  if (ex.perm == nullptr && g_impl.load(std::memory_order_relaxed) != HADQ_IMPL_BUTTERFLY &&
      tck_eligible(x_dtype, sh, mode, sg))
    return launch_tck(x, sh, mode, group, out0, out1, stream, sms, dev);
  if (sh.kbase > 1 || ex.perm != nullptr || mode == hadq::OUT_CODEBOOK)
    return launch_staged(x, x_dtype, sh, mode, group, out0, out1, stream, sms, dev, sg, ex);
  if (g_impl.load(std::memory_order_relaxed) != HADQ_IMPL_BUTTERFLY) {
    if (tc_eligible(x_dtype, sh, mode)) return launch_tc(x, sh, mode, group, out0, out1, stream, sms, dev, sg);
    if (tc128_eligible(x_dtype, sh, mode, sg))
      return launch_tc128(x, sh, mode, group, out0, out1, stream, sms, dev, sg);
  }
  if (mode >= 0) {
    if (sh.b <= 128) {
      const hl::SegFn fn = hl::segment_kernel_for(bf, sh.logb == seg_logs, seg_logs, mode, sgd);
      if (fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no kernel for this segment size and format");
      const int64_t segs = sh.rows * (sh.n >> seg_logs);
      int occ = 0;
      st = occupancy(reinterpret_cast<const void*>(fn), dev, hadq::kThreads, 0, &occ);
      if (st != HADQ_OK) return st;
      const int64_t grid = std::min<int64_t>(ceil_div(segs, hadq::kThreads), int64_t(sms) * occ);
      return launch_result(launch_pdl(fn, grid, hadq::kThreads, 0, stream, x, segs, sh.logb, sh.norm, group, out0, out1,
                                      sg),
                           "segment kernel launch");
    }
    const hl::TeamFn fn = hl::team_kernel_for(bf, sh.logb, mode, sgd);
    if (fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no kernel for this block size and format");
    const int smem = hadq::team_smem_bytes(sh.logb);
    int occ = 0;
    st = occupancy(reinterpret_cast<const void*>(fn), dev, hadq::kThreads, smem, &occ);
    if (st != HADQ_OK) return st;
    const int teams = hadq::kThreads >> (sh.logb - hadq::team_logp(sh.logb));
    const int64_t units = sh.rows * (sh.n >> sh.logb);
    const int64_t grid = std::min<int64_t>(ceil_div(units, teams), int64_t(sms) * occ);
    return launch_result(launch_pdl(fn, grid, hadq::kThreads, smem, stream, x, units, sh.norm, group, out0, out1, sg),
                         "team kernel launch");
  }
  // per-token int8
  int8_t* codes = static_cast<int8_t*>(out0);
  float* scales = static_cast<float*>(out1);
  if (sh.b <= 128) {
    const hl::SegRowFn fn = hl::segment_row_kernel_for(bf, full_seg, sh.logs, sgd);
    if (fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no per-token kernel for this segment size");
    const int block = static_cast<int>(ceil_div(sh.n >> sh.logs, 32) * 32);
    int occ = 0;
    st = occupancy(reinterpret_cast<const void*>(fn), dev, block, 0, &occ);
    if (st != HADQ_OK) return st;
    const int64_t grid = std::min<int64_t>(sh.rows, int64_t(sms) * occ);
    return launch_result(launch_pdl(fn, grid, block, 0, stream, x, sh.rows, sh.n, sh.logb, sh.norm, codes, scales, sg),
                         "per-token int8 kernel launch");
  }
  const hl::TeamRowFn fn = hl::team_row_kernel_for(bf, sh.logb, sgd);
  if (fn == nullptr) return fail(HADQ_ERR_UNSUPPORTED, "no per-token kernel for this block size");
  const int block = static_cast<int>(ceil_div(sh.n >> 7, 32) * 32);
  const int smem = static_cast<int>((sh.n >> 7) * hadq::kRowFloats * 4);
  int occ = 0;
  st = occupancy(reinterpret_cast<const void*>(fn), dev, block, smem, &occ);
  if (st != HADQ_OK) return st;
  const int64_t grid = std::min<int64_t>(sh.rows, int64_t(sms) * occ);
  return launch_result(launch_pdl(fn, grid, block, smem, stream, x, sh.rows, sh.n, sh.norm, codes, scales, sg),
                       "per-token int8 kernel launch");
}

// Random Hadamard signs: a signed entry point passes its caller's side
// (which must be HADQ_SIGNS_AFTER or HADQ_SIGNS_BEFORE); the unsigned entry
// points pass kUnsigned, which no caller value can reach.
constexpr int kUnsigned = -1;

struct SideArg {
  bool is_signed;
  int side;
};

hadq_status check_side(SideArg a) {
  if (a.is_signed && a.side != HADQ_SIGNS_AFTER && a.side != HADQ_SIGNS_BEFORE)
    return fail(HADQ_ERR_INVALID_ARG, "side must be HADQ_SIGNS_AFTER or HADQ_SIGNS_BEFORE");
  return HADQ_OK;
}

// For rows > 0: the signs array (b bytes) must exist and must not overlap an
// output, since every CTA reads it while others may already be writing.
hadq_status make_signs(const int8_t* signs, SideArg a, const Shape& sh, const Span* outs, int nouts, Signs* sg) {
  *sg = Signs{nullptr, hadq::SIGNS_NONE};
  if (!a.is_signed) return HADQ_OK;
  if (signs == nullptr) return fail(HADQ_ERR_INVALID_ARG, "null signs");
  if (!aligned16(signs)) return fail(HADQ_ERR_MISALIGNED, "signs must be 16-byte aligned");
  const Span ss = span(signs, sh.b);
  for (int i = 0; i < nouts; ++i)
    if (overlaps(ss, outs[i])) return fail(HADQ_ERR_INVALID_ARG, "signs must not overlap an output");
  *sg = Signs{signs, a.side == HADQ_SIGNS_AFTER ? hadq::SIGNS_AFTER : hadq::SIGNS_BEFORE};
  return HADQ_OK;
}

// RPBH: n int32 permutation entries and n int8 signs on the device; they
// are read while outputs are written, so they must not overlap an output.
hadq_status make_rpbh(const int32_t* perm, const int8_t* signs, const Shape& sh, const Span* outs, int nouts,
                      Extra* ex) {
  if (perm == nullptr || signs == nullptr) return fail(HADQ_ERR_INVALID_ARG, "RPBH needs both perm and signs");
  if (!aligned16(perm) || !aligned16(signs)) return fail(HADQ_ERR_MISALIGNED, "perm and signs must be 16-byte aligned");
  const Span sp = span(perm, sh.n * 4), ss = span(signs, sh.n);
  for (int i = 0; i < nouts; ++i)
    if (overlaps(sp, outs[i]) || overlaps(ss, outs[i]))
      return fail(HADQ_ERR_INVALID_ARG, "perm and signs must not overlap an output");
  ex->perm = perm;
  ex->rpbh_signs = signs;
  return HADQ_OK;
}

hadq_status rotate_impl(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, void* out,
                        hadq_dtype out_dtype, void* stream, const int8_t* signs = nullptr,
                        SideArg side = SideArg{false, kUnsigned}, const int32_t* perm = nullptr) {
  g_last_error.clear();
  Shape sh;
  hadq_status st = check_shape(x_dtype, rows, n, block, &sh);
  if (st != HADQ_OK) return st;
  if (out_dtype != HADQ_F32 && out_dtype != HADQ_BF16) return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_F32 or HADQ_BF16");
  st = check_side(side);
  if (st != HADQ_OK) return st;
  if (rows == 0) return HADQ_OK;
  if (x == nullptr || out == nullptr) return fail(HADQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(out)) return fail(HADQ_ERR_MISALIGNED, "x and out must be 16-byte aligned");
  const Span sx = span(x, rows * n * esize(x_dtype));
  const Span so = span(out, rows * n * esize(out_dtype));
  if (overlaps(sx, so) && !(x == out && x_dtype == out_dtype))
    return fail(HADQ_ERR_INVALID_ARG, "out overlaps x (only exact in-place with equal dtypes is allowed)");
  Signs sg{nullptr, hadq::SIGNS_NONE};
  Extra ex;
  st = perm != nullptr ? make_rpbh(perm, signs, sh, &so, 1, &ex) : make_signs(signs, side, sh, &so, 1, &sg);
  if (st != HADQ_OK) return st;
  return launch(x, x_dtype, sh, out_dtype == HADQ_F32 ? hadq::OUT_F32 : hadq::OUT_BF16, 0, out, nullptr,
                static_cast<cudaStream_t>(stream), sg, ex);
}


hadq_status quant_checks(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, hadq_fmt fmt,
                         int64_t group, const void* codes, const void* scales, Shape* sh, int* g) {
  hadq_status st = check_shape(x_dtype, rows, n, block, sh);
  if (st != HADQ_OK) return st;
  st = check_quant(fmt, group, *sh, g);
  if (st != HADQ_OK) return st;
  if (rows == 0) return HADQ_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return fail(HADQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales))
    return fail(HADQ_ERR_MISALIGNED, "x, codes and scales must be 16-byte aligned");
  const Span sx = span(x, rows * n * esize(x_dtype));
  const Span sc = span(codes, codes_bytes(rows, n, fmt));
  const Span ss = span(scales, scales_bytes(rows, n, fmt, *g));
  if (overlaps(sx, sc) || overlaps(sx, ss) || overlaps(sc, ss))
    return fail(HADQ_ERR_INVALID_ARG, "x, codes and scales must not overlap");
  return HADQ_OK;
}

int quant_mode(hadq_fmt fmt) {
  switch (fmt) {
    case HADQ_INT4_SYM: return hadq::OUT_INT4;
    case HADQ_MXFP4: return hadq::OUT_MXFP4;
    case HADQ_NVFP4: return hadq::OUT_NVFP4;
    case HADQ_MXFP4_BLOCKED: return hadq::OUT_MXFP4_BLOCKED;
    case HADQ_NVFP4_BLOCKED: return hadq::OUT_NVFP4_BLOCKED;
    default: return -1;
  }
}

hadq_status rotate_quant_impl(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                              hadq_fmt fmt, int64_t group, void* codes, void* scales, void* stream,
                              const int8_t* signs = nullptr, SideArg side = SideArg{false, kUnsigned},
                              double tensor_scale = 1.0, const int32_t* perm = nullptr) {
  g_last_error.clear();
  Shape sh;
  int g = 0;
  hadq_status st = check_side(side);
  if (st != HADQ_OK) return st;
  if (!(std::isfinite(tensor_scale) && tensor_scale > 0))
    return fail(HADQ_ERR_INVALID_ARG, "tensor_scale must be finite and > 0");
  st = quant_checks(x, x_dtype, rows, n, block, fmt, group, codes, scales, &sh, &g);
  if (st != HADQ_OK || rows == 0) return st;
  // NVFP4 quantizes y / tensor_scale: fold the division into the rotation's
  // normalisation (one rounding, on the host, in double).
  if (fmt == HADQ_NVFP4 || fmt == HADQ_NVFP4_BLOCKED)
    sh.norm = static_cast<float>(1.0 / std::sqrt(static_cast<double>(sh.b)) / tensor_scale);
  const Span outs[2] = {span(codes, codes_bytes(rows, n, fmt)), span(scales, scales_bytes(rows, n, fmt, g))};
  Signs sg{nullptr, hadq::SIGNS_NONE};
  Extra ex;
  st = perm != nullptr ? make_rpbh(perm, signs, sh, outs, 2, &ex) : make_signs(signs, side, sh, outs, 2, &sg);
  if (st != HADQ_OK) return st;
  if (blocked_fmt(fmt)) {
    // Only the tensor-core kernels write the tiled layout; the padding rows of
    // the last 128-row tile are zeroed first (the kernel writes every other entry).
    const int qm = quant_mode(fmt);
    if (perm != nullptr || g_impl.load(std::memory_order_relaxed) == HADQ_IMPL_BUTTERFLY ||
        !(tc_eligible(x_dtype, sh, qm) || tc128_eligible(x_dtype, sh, qm, sg) || tck_eligible(x_dtype, sh, qm, sg)))
      return fail(HADQ_ERR_UNSUPPORTED, "blocked FP4 scales: bf16 input on a tensor-core shape (no RPBH)");
    if (rows % 128 != 0) {
      const int64_t cols = n / g;   // scale columns per row
      const int64_t tile_row_bytes = cols / 4 * 512;
      const cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(scales) + rows / 128 * tile_row_bytes, 0,
                                            static_cast<size_t>(tile_row_bytes), static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("zero the scale padding: ") + cudaGetErrorString(e));
    }
  }
  return launch(x, x_dtype, sh, quant_mode(fmt), g, codes, scales, static_cast<cudaStream_t>(stream), sg, ex);
}

// The codebook quantizer: per-token norm, nearest centroid of the normalized
// rotated row; codes bits / 8 bytes per element, one fp32 norm per row.
hadq_status codebook_impl(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                          const int32_t* perm, const int8_t* signs, int bits, const double* thresholds, void* codes,
                          float* norms, void* stream) {
  g_last_error.clear();
  Shape sh;
  hadq_status st = check_shape(x_dtype, rows, n, block, &sh);
  if (st != HADQ_OK) return st;
  if (bits != 2 && bits != 4) return fail(HADQ_ERR_UNSUPPORTED, "codebook bits must be 2 or 4");
  if ((perm == nullptr) != (signs == nullptr)) return fail(HADQ_ERR_INVALID_ARG, "give both perm and signs, or neither");
  if (rows == 0) return HADQ_OK;
  if (x == nullptr || codes == nullptr || norms == nullptr || thresholds == nullptr)
    return fail(HADQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(norms) || !aligned16(thresholds))
    return fail(HADQ_ERR_MISALIGNED, "x, codes, norms and thresholds must be 16-byte aligned");
  const int64_t cb = rows * n * bits / 8;
  const Span sx = span(x, rows * n * esize(x_dtype)), sc = span(codes, cb), sn = span(norms, rows * 4);
  const Span st_thr = span(thresholds, ((int64_t(1) << bits) - 1) * 8);
  if (overlaps(sx, sc) || overlaps(sx, sn) || overlaps(sc, sn) || overlaps(st_thr, sc) || overlaps(st_thr, sn))
    return fail(HADQ_ERR_INVALID_ARG, "x, codes, norms and thresholds must not overlap");
  const Span outs[2] = {sc, sn};
  Extra ex;
  if (perm != nullptr) {
    st = make_rpbh(perm, signs, sh, outs, 2, &ex);
    if (st != HADQ_OK) return st;
  }
  ex.thr = thresholds;
  ex.bits = bits;
  return launch(x, x_dtype, sh, hadq::OUT_CODEBOOK, 0, codes, norms, static_cast<cudaStream_t>(stream),
                Signs{nullptr, hadq::SIGNS_NONE}, ex);
}

// ----------------------------------------------- allocation-free host path
// Device staging for hadq_rotate_quant_host_static: one file-scope array that
// every GPU loading this library holds until the process exits.  In host code
// `g_static_scratch` only names the symbol; its device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 32 MiB per GPU
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::map<int, void*> g_static_scratch_ptr;   // device -> device address of g_static_scratch (under g_mu)

hadq_status static_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_static_scratch_ptr.find(dev);
  if (it == g_static_scratch_ptr.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(HADQ_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") + cudaGetErrorString(e));
    it = g_static_scratch_ptr.emplace(dev, p).first;
  }
  *ptr = it->second;
  return HADQ_OK;
}

size_t align256(int64_t v) { return (static_cast<size_t>(v) + 255) & ~size_t(255); }

}  // namespace

extern "C" {

hadq_status hadq_rotate(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, void* out,
                        hadq_dtype out_dtype, void* stream) {
  return rotate_impl(x, x_dtype, rows, n, block, out, out_dtype, stream);
}

hadq_status hadq_rotate_inverse(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, void* out,
                                hadq_dtype out_dtype, void* stream) {
  return rotate_impl(x, x_dtype, rows, n, block, out, out_dtype, stream);
}

hadq_status hadq_rotate_quant(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block, hadq_fmt fmt,
                              int64_t group, void* codes, void* scales, void* stream) {
  return rotate_quant_impl(x, x_dtype, rows, n, block, fmt, group, codes, scales, stream);
}

hadq_status hadq_rotate_quant_nvfp4(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                    float tensor_scale, void* codes, void* scales, void* stream) {
  return rotate_quant_impl(x, x_dtype, rows, n, block, HADQ_NVFP4, 16, codes, scales, stream, nullptr,
                           SideArg{false, kUnsigned}, static_cast<double>(tensor_scale));
}

hadq_status hadq_rotate_signed(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                               const int8_t* signs, hadq_sign_side side, void* out, hadq_dtype out_dtype,
                               void* stream) {
  return rotate_impl(x, x_dtype, rows, n, block, out, out_dtype, stream, signs, SideArg{true, static_cast<int>(side)});
}

hadq_status hadq_rotate_quant_signed(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                     const int8_t* signs, hadq_sign_side side, hadq_fmt fmt, int64_t group,
                                     void* codes, void* scales, void* stream) {
  return rotate_quant_impl(x, x_dtype, rows, n, block, fmt, group, codes, scales, stream, signs,
                           SideArg{true, static_cast<int>(side)});
}

hadq_status hadq_rotate_rpbh(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                             const int32_t* perm, const int8_t* signs, void* out, hadq_dtype out_dtype, void* stream) {
  if (perm == nullptr && rows > 0) {
    g_last_error.clear();
    return fail(HADQ_ERR_INVALID_ARG, "null perm");
  }
  return rotate_impl(x, x_dtype, rows, n, block, out, out_dtype, stream, signs, SideArg{false, kUnsigned}, perm);
}

hadq_status hadq_rotate_quant_rpbh(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                   const int32_t* perm, const int8_t* signs, hadq_fmt fmt, int64_t group, void* codes,
                                   void* scales, void* stream) {
  if (perm == nullptr && rows > 0) {
    g_last_error.clear();
    return fail(HADQ_ERR_INVALID_ARG, "null perm");
  }
  return rotate_quant_impl(x, x_dtype, rows, n, block, fmt, group, codes, scales, stream, signs,
                           SideArg{false, kUnsigned}, 1.0, perm);
}

hadq_status hadq_rotate_quant_codebook(const void* x, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                       const int32_t* perm, const int8_t* signs, int bits, const double* thresholds,
                                       void* codes, float* norms, void* stream) {
  return codebook_impl(x, x_dtype, rows, n, block, perm, signs, bits, thresholds, codes, norms, stream);
}

hadq_status hadq_rotate_quant_host(const void* x_host, hadq_dtype x_dtype, int64_t rows, int64_t n, int64_t block,
                                   hadq_fmt fmt, int64_t group, void* codes_host, void* scales_host, void* x_dev,
                                   void* codes_dev, void* scales_dev, void* stream) {
  g_last_error.clear();
  Shape sh;
  int g = 0;
  hadq_status st = quant_checks(x_dev, x_dtype, rows, n, block, fmt, group, codes_dev, scales_dev, &sh, &g);
  if (st != HADQ_OK || rows == 0) return st;
  if (x_host == nullptr || codes_host == nullptr || scales_host == nullptr)
    return fail(HADQ_ERR_INVALID_ARG, "null host pointer");
  if (!aligned16(x_host) || !aligned16(codes_host) || !aligned16(scales_host))
    return fail(HADQ_ERR_MISALIGNED, "host buffers must be 16-byte aligned");
  const int64_t xb = rows * n * esize(x_dtype), cb = codes_bytes(rows, n, fmt), sb = scales_bytes(rows, n, fmt, g);
  const Span hx = span(x_host, xb), hc = span(codes_host, cb), hs = span(scales_host, sb);
  if (overlaps(hx, hc) || overlaps(hx, hs) || overlaps(hc, hs))
    return fail(HADQ_ERR_INVALID_ARG, "host x, codes and scales must not overlap");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, static_cast<size_t>(xb), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy x to device: ") + cudaGetErrorString(e));
  st = launch(x_dev, x_dtype, sh, quant_mode(fmt), g, codes_dev, scales_dev, s);
  if (st != HADQ_OK) return st;
  e = cudaMemcpyAsync(codes_host, codes_dev, static_cast<size_t>(cb), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy codes to host: ") + cudaGetErrorString(e));
  e = cudaMemcpyAsync(scales_host, scales_dev, static_cast<size_t>(sb), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy scales to host: ") + cudaGetErrorString(e));
  return HADQ_OK;
}

hadq_status hadq_rotate_quant_host_static(const void* x_host, hadq_dtype x_dtype, int64_t rows, int64_t n,
                                          int64_t block, hadq_fmt fmt, int64_t group, void* codes_host,
                                          void* scales_host, void* stream) {
  g_last_error.clear();
  Shape sh;
  int g = 0;
  hadq_status st = check_shape(x_dtype, rows, n, block, &sh);
  if (st != HADQ_OK) return st;
  st = check_quant(fmt, group, sh, &g);
  if (st != HADQ_OK || rows == 0) return st;
  if (x_host == nullptr || codes_host == nullptr || scales_host == nullptr)
    return fail(HADQ_ERR_INVALID_ARG, "null host pointer");
  if (!aligned16(x_host) || !aligned16(codes_host) || !aligned16(scales_host))
    return fail(HADQ_ERR_MISALIGNED, "host buffers must be 16-byte aligned");
  const int64_t xb = rows * n * esize(x_dtype), cb = codes_bytes(rows, n, fmt), sb = scales_bytes(rows, n, fmt, g);
  const Span hx = span(x_host, xb), hc = span(codes_host, cb), hs = span(scales_host, sb);
  if (overlaps(hx, hc) || overlaps(hx, hs) || overlaps(hc, hs))
    return fail(HADQ_ERR_INVALID_ARG, "host x, codes and scales must not overlap");
  if (align256(xb) + align256(cb) + align256(sb) > kStaticScratchBytes)
    return fail(HADQ_ERR_UNSUPPORTED,
                "input + codes + scales exceed the 32 MiB static device scratch of hadq_rotate_quant_host_static; "
                "use hadq_rotate_quant_host with caller-owned device buffers");
  void* scratch = nullptr;
  st = static_scratch(&scratch);   // first call on a device: resolve the symbol's device address
  if (st != HADQ_OK) return st;
  unsigned char* base = static_cast<unsigned char*>(scratch);
  void* x_dev = base;
  void* codes_dev = base + align256(xb);
  void* scales_dev = base + align256(xb) + align256(cb);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, static_cast<size_t>(xb), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy x to static scratch: ") + cudaGetErrorString(e));
  st = launch(x_dev, x_dtype, sh, quant_mode(fmt), g, codes_dev, scales_dev, s);
  if (st != HADQ_OK) return st;
  e = cudaMemcpyAsync(codes_host, codes_dev, static_cast<size_t>(cb), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy codes to host: ") + cudaGetErrorString(e));
  e = cudaMemcpyAsync(scales_host, scales_dev, static_cast<size_t>(sb), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, std::string("copy scales to host: ") + cudaGetErrorString(e));
  return HADQ_OK;
}

int64_t hadq_codes_bytes(int64_t rows, int64_t n, hadq_fmt fmt) {
  if (rows < 0 || n <= 0 || n % 2 != 0) return 0;
  if (fmt != HADQ_INT4_SYM && fmt != HADQ_INT8_SYM && fmt != HADQ_MXFP4 && fmt != HADQ_NVFP4 && !blocked_fmt(fmt))
    return 0;
  return codes_bytes(rows, n, fmt);
}

int64_t hadq_scales_bytes(int64_t rows, int64_t n, hadq_fmt fmt, int64_t group) {
  if (rows < 0 || n <= 0) return 0;
  switch (fmt) {
    case HADQ_INT4_SYM:
      if ((group != 32 && group != 64 && group != 128) || n % group != 0) return 0;
      return scales_bytes(rows, n, fmt, static_cast<int>(group));
    case HADQ_INT8_SYM:
      return (group == 0 || group == n) ? rows * 4 : 0;
    case HADQ_MXFP4:
      return ((group == 0 || group == 32) && n % 32 == 0) ? rows * (n / 32) : 0;
    case HADQ_NVFP4:
      return ((group == 0 || group == 16) && n % 16 == 0) ? rows * (n / 16) : 0;
    case HADQ_MXFP4_BLOCKED:
      return ((group == 0 || group == 32) && n % 128 == 0) ? scales_bytes(rows, n, fmt, 32) : 0;
    case HADQ_NVFP4_BLOCKED:
      return ((group == 0 || group == 16) && n % 64 == 0) ? scales_bytes(rows, n, fmt, 16) : 0;
    default:
      return 0;
  }
}

const char* hadq_status_string(hadq_status status) {
  switch (status) {
    case HADQ_OK: return "ok";
    case HADQ_ERR_INVALID_ARG: return "invalid argument";
    case HADQ_ERR_UNSUPPORTED: return "unsupported size or format";
    case HADQ_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case HADQ_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

const char* hadq_last_error(void) { return g_last_error.c_str(); }

int hadq_version(void) { return 200; }

hadq_status hadq_set_impl(hadq_impl impl) {
  g_last_error.clear();
  if (impl != HADQ_IMPL_AUTO && impl != HADQ_IMPL_BUTTERFLY && impl != HADQ_IMPL_TENSOR)
    return fail(HADQ_ERR_INVALID_ARG, "impl must be HADQ_IMPL_AUTO, HADQ_IMPL_BUTTERFLY or HADQ_IMPL_TENSOR");
  g_impl.store(static_cast<int>(impl), std::memory_order_relaxed);
  return HADQ_OK;
}

hadq_impl hadq_get_impl(void) { return static_cast<hadq_impl>(g_impl.load(std::memory_order_relaxed)); }

int hadq_device_faults(int clear) {
  const int a = hadq::launch::tc_fault_bits(clear), b = hadq::launch::tck_fault_bits(clear);
  return a < 0 || b < 0 ? -1 : (a | b);
}

}  // extern "C"
