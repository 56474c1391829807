// libfp8q.so: the C ABI declared in include/fp8q.h.
//
// Host side: argument validation (before any launch), TMA tensor-map encoding
// (cuTensorMapEncodeTiled through the runtime's driver entry point, so the library
// needs no -lcuda), kernel attribute setup and launches on the caller's stream.
// All device code lives in quant.cuh and gemm.cuh (one translation unit).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/fp8q.h"
#include "gemm.cuh"
#include "gemm_ue8m0.cuh"
#include "quant.cuh"

namespace {

using fp8q::GemmArgs;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The tensor-map encoder is a driver call and needs the device's context current on the
// calling thread.  A thread that has made no runtime call yet (a framework's worker
// thread, say) may have none bound: make the current device's primary context current.
bool bind_current_context() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess;
}

// 2D K-major E4M3 operand: [rows, K] with a row stride of `ld` bytes; box = 128 bytes of K
// by `box_rows` rows, 128-byte swizzle (the canonical layout the MMA descriptors expect).
int encode_operand(CUtensorMap* tm, const void* base, uint64_t K, uint64_t rows, uint64_t ld,
                   uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc || !bind_current_context()) return FP8Q_ERR_CUDA;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// bf16 output C [rows, N] with a row stride of `ldc` elements, stored by TMA: boxes of 64
// columns (128 bytes) by 32 rows, 128-byte swizzle (the promoted GEMM's staging layout).
int encode_output_bf16(CUtensorMap* tm, void* base, uint64_t N, uint64_t rows, uint64_t ldc) {
  auto enc = tensor_map_encoder();
  if (!enc || !bind_current_context()) return FP8Q_ERR_CUDA;
  cuuint64_t dims[2] = {N, rows};
  cuuint64_t strides[1] = {ldc * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Tile shape of the promoted GEMMs: one CTA per 128 x 256 tile (the same shape for both
// B scale modes and output paths).
using Cfg1 = fp8q::GemmCfg<false>;

template <bool PROMOTE, bool ROW_B, bool GROUPED, bool OUT_BF16, bool QOUT = false>
struct GemmLauncher {
  using Cfg = fp8q::GemmCfgOf<PROMOTE, ROW_B, OUT_BF16, QOUT>;
  static constexpr auto kern = fp8q::gemm_fp8_blockscaled_kernel<PROMOTE, ROW_B, GROUPED, OUT_BF16, QOUT>;
  static_assert(Cfg::kTileM == Cfg1::kTileM && Cfg::kN == Cfg1::kN, "one tile shape");

  // Co-resident CTAs on the current device; sets the kernel's attributes on first use.
  // 0 on failure.
  static int max_units() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int units = cached[dev].load(std::memory_order_acquire);
    if (units) return units;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Cfg::smem_bytes)) != cudaSuccess)
      return 0;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, fp8q::kGemmThreads,
                                                      Cfg::smem_bytes) != cudaSuccess ||
        per_sm <= 0) {
      (void)cudaGetLastError();   // the query's failure is handled here, not by the next launch check
      return 0;
    }
    units = sms * per_sm;
    cached[dev].store(units, std::memory_order_release);
    return units;
  }

  static int launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                    const GemmArgs& args, int64_t grid, cudaStream_t stream) {
    if (grid <= 0) return FP8Q_OK;
    kern<<<static_cast<unsigned>(grid), fp8q::kGemmThreads, Cfg::smem_bytes, stream>>>(tmA, tmB, tmC, args);
    return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
  }
};

// Work split of a dense GEMM over `units` co-resident CTAs: whole tiles in full waves,
// and, when the last wave would leave most CTAs idle, its R tiles split into S K-chunks
// (S = min(units / R, G / 2) >= 2) whose partials need a workspace of R*S tiles.
struct SplitPlan {
  int64_t tiles_full, tail_tiles, tail_split, grid_units;
  size_t ws_bytes;
};

SplitPlan plan_split(int64_t tiles, int64_t G, int64_t units) {
  SplitPlan sp{tiles, 0, 1, tiles < units ? tiles : units, 0};
  if (units <= 0) return sp;
  const int64_t full_waves = tiles / units, tail = tiles % units;
  if (tail == 0) return sp;
  int64_t split = units / tail;
  if (split > G / 2) split = G / 2;
  if (split < 2) return sp;
  sp.tiles_full = full_waves * units;
  sp.tail_tiles = tail;
  sp.tail_split = split;
  sp.grid_units = full_waves > 0 ? units : tail * split;
  sp.ws_bytes = static_cast<size_t>(tail * split) * Cfg1::kTileM * Cfg1::kN * sizeof(float);
  return sp;
}

int check_gemm_common(const uint8_t* A, const uint8_t* B, const void* C, int out_dtype,
                             int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                             int64_t ldc) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (out_dtype != FP8Q_OUT_BF16 && out_dtype != FP8Q_OUT_FP32) return FP8Q_ERR_UNSUPPORTED;
  if (!A || !B || !C) return FP8Q_ERR_NULL;
  if (K == 0 || K % 128 != 0 || N == 0 || N % 128 != 0) return FP8Q_ERR_SHAPE;
  if (lda < K || ldb < K || ldc < N) return FP8Q_ERR_SHAPE;
  const int64_t esz = out_dtype == FP8Q_OUT_BF16 ? 2 : 4;
  if (lda % 16 != 0 || ldb % 16 != 0 || (ldc * esz) % 16 != 0) return FP8Q_ERR_ALIGN;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16)) return FP8Q_ERR_ALIGN;
  if (K / 128 > 0x7FFFFF || M > 0x7FFFFFFF || N > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  return FP8Q_OK;
}

// Host checks of the dense block-scaled GEMMs' arguments (everything but a workspace).
int check_dense_blockscaled(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                            const float* sB, int64_t ld_sb, int b_scale_mode, const void* C,
                            int out_dtype, int64_t M, int64_t N, int64_t K, int64_t lda,
                            int64_t ldb, int64_t ldc) {
  int st = check_gemm_common(A, B, C, out_dtype, M, N, K, lda, ldb, ldc);
  if (st != FP8Q_OK) return st;
  if (!sA || !sB) return FP8Q_ERR_NULL;
  if (b_scale_mode != FP8Q_BSCALE_BLOCK128x128 && b_scale_mode != FP8Q_BSCALE_ROW1x128)
    return FP8Q_ERR_UNSUPPORTED;
  if (ld_sa < M) return FP8Q_ERR_SHAPE;
  if (b_scale_mode == FP8Q_BSCALE_ROW1x128 && ld_sb < N) return FP8Q_ERR_SHAPE;
  if (!aligned(sA, 4) || !aligned(sB, 4)) return FP8Q_ERR_ALIGN;
  return FP8Q_OK;
}

// Launch one GEMM instantiation.  work: tiles (a bound for grouped).  Dense GEMMs given a
// large enough workspace split their last partial wave along K and finish with a
// reduction launch on the same stream.  tmC: the bf16 output's tensor map for the
// instantiations that store through TMA (GemmCfgOf's TSTORE), otherwise unused.
template <bool PROMOTE, bool ROW_B, bool GROUPED, bool OUT_BF16, bool QOUT = false>
int run_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC, GemmArgs a,
             int64_t work, void* ws, size_t ws_bytes, cudaStream_t st) {
  using L = GemmLauncher<PROMOTE, ROW_B, GROUPED, OUT_BF16, QOUT>;
  const int units = L::max_units();
  if (units <= 0) return FP8Q_ERR_CUDA;
  a.ws = nullptr;
  a.tiles_full = static_cast<int>(work);
  a.tail_tiles = 0;
  a.tail_split = 1;
  int64_t grid = work < units ? work : units;
  if (!GROUPED && PROMOTE && ws != nullptr) {
    const SplitPlan sp = plan_split(work, a.G, units);
    if (sp.tail_tiles > 0 && sp.ws_bytes <= ws_bytes) {
      a.ws = static_cast<float*>(ws);
      a.tiles_full = static_cast<int>(sp.tiles_full);
      a.tail_tiles = static_cast<int>(sp.tail_tiles);
      a.tail_split = static_cast<int>(sp.tail_split);
      grid = sp.grid_units;
    }
  }
  int st_code = L::launch(tmA, tmB, tmC, a, grid, st);
  if (st_code != FP8Q_OK || a.tail_tiles == 0) return st_code;
  const int mt_total = static_cast<int>((a.M + Cfg1::kTileM - 1) / Cfg1::kTileM);
  fp8q::splitk_reduce_kernel<OUT_BF16, Cfg1::kTileM, Cfg1::kN>
      <<<a.tail_tiles * Cfg1::kTileM, Cfg1::kN, 0, st>>>(a, mt_total);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Promoted dense GEMM: B scale mode and output type chosen at run time; a quantized
// output (bf16, no workspace) takes its own instantiation.
int dispatch_dense(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                   const GemmArgs& a, bool row_b, bool bf16, int64_t work, void* ws, size_t ws_bytes,
                   cudaStream_t st) {
  if (a.qc != nullptr) {
    return row_b ? run_gemm<true, true, false, true, true>(tmA, tmB, tmC, a, work, nullptr, 0, st)
                 : run_gemm<true, false, false, true, true>(tmA, tmB, tmC, a, work, nullptr, 0, st);
  }
  if (row_b) {
    return bf16 ? run_gemm<true, true, false, true>(tmA, tmB, tmC, a, work, ws, ws_bytes, st)
                : run_gemm<true, true, false, false>(tmA, tmB, tmC, a, work, ws, ws_bytes, st);
  }
  return bf16 ? run_gemm<true, false, false, true>(tmA, tmB, tmC, a, work, ws, ws_bytes, st)
              : run_gemm<true, false, false, false>(tmA, tmB, tmC, a, work, ws, ws_bytes, st);
}

int64_t dense_tiles(int64_t M, int64_t N) {
  return ((M + Cfg1::kTileM - 1) / Cfg1::kTileM) * ((N + Cfg1::kN - 1) / Cfg1::kN);
}

static_assert(fp8q::kErrScale == FP8Q_ERR_SCALE, "device status code of a bad scale");

// Launch of the power-of-two-scale GEMM: one persistent CTA per SM (kernel attributes set
// and the co-resident count cached per device on first use).  work: tiles (a bound for
// grouped).
template <bool ROW_B, bool OUT_BF16, bool GROUPED>
int run_gemm_ue8m0(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                   int64_t work, cudaStream_t st) {
  using Cfg = fp8q::Ue8m0Cfg<GROUPED>;
  static constexpr auto kern = fp8q::gemm_fp8_ue8m0_kernel<ROW_B, OUT_BF16, GROUPED>;
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  int units = cached[dev].load(std::memory_order_acquire);
  if (units == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Cfg::smem_bytes)) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::kThreads, Cfg::smem_bytes) !=
            cudaSuccess || per_sm <= 0)
      return FP8Q_ERR_CUDA;
    units = sms * per_sm;
    cached[dev].store(units, std::memory_order_release);
  }
  const int64_t grid = work < units ? work : units;
  if (grid <= 0) return FP8Q_OK;
  kern<<<static_cast<unsigned>(grid), Cfg::kThreads, Cfg::smem_bytes, st>>>(tmA, tmB, a);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace

namespace fp8q {
// Self-test of the bounded wait: one thread waits on a barrier that nothing arrives on;
// the wait gives up after timeout_ns and records (site 7 << 8) | FP8Q_ERR_TIMEOUT.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    mbar_wait_ns(smem_u32(&bar), 0, 7, nullptr, timeout_ns);
  }
}
}  // namespace fp8q

// ---------------------------------------------------------------------------------------
// Fixed scratch for fp8_gemm_blockscaled_noalloc.
//
// Some callers cannot allocate device memory at the moment they run a GEMM: code that
// runs under a memory budget fixed in advance (a pre-sized arena), allocator hooks or
// callbacks that must not re-enter the allocator, or runtimes that forbid cudaMalloc
// on their hot path.  For them the split-K workspace lives in this file-scope device
// array instead of a caller buffer.  It is sized for the largest split plan on a 148-SM
// B200 (at most one 128 x 256 FP32 partial tile per SM: 18.5 MiB), and every GPU that
// loads this library keeps it for the life of the process.
constexpr size_t kStaticScratchBytes = size_t(20) << 20;   // 20 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

// Device address of g_static_scratch on the current device.  On the host the array's
// name only stands for the symbol, so it is looked up once per device (with that device
// current) and cached.  nullptr on failure.
void* static_scratch_address() {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int fp8q_abi_version(void) { return 1; }

const char* fp8q_status_string(int status) {
  switch (status & 0xFF) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_NULL: return "null pointer argument";
    case FP8Q_ERR_SHAPE: return "invalid shape or leading dimension";
    case FP8Q_ERR_ALIGN: return "pointer or leading dimension misaligned";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported mode, dtype or device";
    case FP8Q_ERR_SCALE: return "a scale is not a power of two representable as UE8M0";
    case FP8Q_ERR_CUDA: return "CUDA call failed";
    case FP8Q_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int fp8q_get_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int h = 0;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, fp8q::g_device_error) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (cudaMemcpyAsync(&h, addr, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (cudaMemsetAsync(addr, 0, sizeof(h), s) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP8Q_ERR_CUDA;
  return static_cast<int>(h);
}

int fp8q_quant_act_1x128(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                         float* scales, int64_t ld_scale, int pow2_scale, void* stream) {
  if (M < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!x || !q || !scales) return FP8Q_ERR_NULL;
  if (K % 128 != 0 || ldx < K || ldq < K || ld_scale < M) return FP8Q_ERR_SHAPE;
  if (ldx % 8 != 0 || ldq % 8 != 0 || !aligned(x, 16) || !aligned(q, 8) || !aligned(scales, 4))
    return FP8Q_ERR_ALIGN;
  const int64_t G = K / 128;
  const int64_t row_blocks = M / fp8q::kActRowsPerBlock + (M % fp8q::kActRowsPerBlock != 0);
  if (row_blocks > 0x7FFFFFFF / G) return FP8Q_ERR_SHAPE;   // one-dimensional grid
  const unsigned grid = static_cast<unsigned>(row_blocks * G);
  auto st = static_cast<cudaStream_t>(stream);
  const auto* xs = static_cast<const uint16_t*>(x);
  const auto g32 = static_cast<uint32_t>(G);
  if (pow2_scale)
    fp8q::quant_act_1x128_kernel<true><<<grid, 256, 0, st>>>(xs, M, ldx, q, ldq, scales, ld_scale, g32);
  else
    fp8q::quant_act_1x128_kernel<false><<<grid, 256, 0, st>>>(xs, M, ldx, q, ldq, scales, ld_scale, g32);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int fp8q_quant_act_dual(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                        int64_t ldq, float* s, int64_t ld_s, uint8_t* qt, int64_t ldqt,
                        float* st, int64_t ld_st, int pow2_scale, void* stream) {
  if (M < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!x || !q || !s || !qt || !st) return FP8Q_ERR_NULL;
  if (M % 128 != 0 || K % 128 != 0 || ldx < K || ldq < K || ld_s < M || ldqt < M || ld_st < K)
    return FP8Q_ERR_SHAPE;
  if (ldx % 8 != 0 || ldq % 8 != 0 || ldqt % 16 != 0 || !aligned(x, 16) || !aligned(q, 8) ||
      !aligned(qt, 16) || !aligned(s, 4) || !aligned(st, 4))
    return FP8Q_ERR_ALIGN;
  if (M / 128 > 0x7FFFFFFF / (K / 128)) return FP8Q_ERR_SHAPE;   // one-dimensional grid
  static std::atomic<unsigned long long> ready{0};   // per-device bit: attributes set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  if (!(ready.load(std::memory_order_acquire) & (1ull << dev))) {
    if (cudaFuncSetAttribute(fp8q::quant_act_dual_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kDualSmem) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::quant_act_dual_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kDualSmem) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    ready.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  // the bf16 tile arrives by TMA: boxes of 128 rows x 64 columns, 128-byte swizzle
  CUtensorMap tmx;
  {
    auto enc = tensor_map_encoder();
    if (!enc || !bind_current_context()) return FP8Q_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldx) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tmx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return FP8Q_ERR_CUDA;
  }
  const unsigned grid = static_cast<unsigned>((M / 128) * (K / 128));
  const auto g32 = static_cast<uint32_t>(K / 128);
  auto stm = static_cast<cudaStream_t>(stream);
  if (pow2_scale)
    fp8q::quant_act_dual_kernel<true><<<grid, 256, fp8q::kDualSmem, stm>>>(tmx, q, ldq, s, ld_s, qt, ldqt,
                                                                           st, ld_st, g32);
  else
    fp8q::quant_act_dual_kernel<false><<<grid, 256, fp8q::kDualSmem, stm>>>(tmx, q, ldq, s, ld_s, qt, ldqt,
                                                                            st, ld_st, g32);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int fp8q_transpose_blocks(const uint8_t* q, const float* s, int64_t N, int64_t K, int64_t ldq,
                          uint8_t* qt, float* st, int64_t ldqt, void* stream) {
  if (N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (!q || !s || !qt || !st) return FP8Q_ERR_NULL;
  if (N % 128 != 0 || K % 128 != 0 || ldq < K || ldqt < N) return FP8Q_ERR_SHAPE;
  if (ldq % 16 != 0 || ldqt % 16 != 0 || !aligned(q, 16) || !aligned(qt, 16) || !aligned(s, 4) ||
      !aligned(st, 4))
    return FP8Q_ERR_ALIGN;
  if (N / 128 > 65535 || K / 128 > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  dim3 grid(static_cast<unsigned>(K / 128), static_cast<unsigned>(N / 128));
  fp8q::transpose_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      q, s, ldq, static_cast<int>(K / 128), qt, st, ldqt, static_cast<int>(N / 128));
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int fp8q_quant_weight_128x128(const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q,
                              int64_t ldq, float* scales, int pow2_scale, void* stream) {
  if (N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (!w || !q || !scales) return FP8Q_ERR_NULL;
  if (N % 128 != 0 || K % 128 != 0 || ldw < K || ldq < K) return FP8Q_ERR_SHAPE;
  if (ldw % 8 != 0 || ldq % 8 != 0 || !aligned(w, 16) || !aligned(q, 8) || !aligned(scales, 4))
    return FP8Q_ERR_ALIGN;
  const int64_t G = K / 128, NB = N / 128;
  if (NB > 65535 || G > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  dim3 grid(static_cast<unsigned>(G), static_cast<unsigned>(NB));
  auto st = static_cast<cudaStream_t>(stream);
  const auto* ws = static_cast<const uint16_t*>(w);
  if (pow2_scale)
    fp8q::quant_weight_128x128_kernel<true><<<grid, 256, 0, st>>>(ws, ldw, q, ldq, scales, G);
  else
    fp8q::quant_weight_128x128_kernel<false><<<grid, 256, 0, st>>>(ws, ldw, q, ldq, scales, G);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int fp8q_quant_rowwise(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                       float* scales, int pow2_scale, void* stream) {
  if (M < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (!x || !q || !scales) return FP8Q_ERR_NULL;
  if (K % 128 != 0 || ldx < K || ldq < K) return FP8Q_ERR_SHAPE;
  if (ldx % 8 != 0 || ldq % 8 != 0 || !aligned(x, 16) || !aligned(q, 8) || !aligned(scales, 4))
    return FP8Q_ERR_ALIGN;
  if (M > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  auto st = static_cast<cudaStream_t>(stream);
  const auto* xs = static_cast<const uint16_t*>(x);
  if (pow2_scale)
    fp8q::quant_rowwise_kernel<true><<<static_cast<unsigned>(M), 256, 0, st>>>(xs, K, ldx, q, ldq, scales);
  else
    fp8q::quant_rowwise_kernel<false><<<static_cast<unsigned>(M), 256, 0, st>>>(xs, K, ldx, q, ldq, scales);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int fp8_gemm_blockscaled_ws(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                            const float* sB, int64_t ld_sb, int b_scale_mode, void* C, int out_dtype,
                            int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (M == 0 && N >= 0 && K >= 0) return FP8Q_OK;
  int st = check_dense_blockscaled(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode, C, out_dtype, M, N, K,
                                   lda, ldb, ldc);
  if (st != FP8Q_OK) return st;
  if (workspace != nullptr && !aligned(workspace, 16)) return FP8Q_ERR_ALIGN;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, M, lda, 128)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, B, K, N, ldb, Cfg1::kBBox)) != FP8Q_OK) return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = ld_sa; a.sB = sB; a.ld_sb = ld_sb; a.C = C; a.ldc = ldc;
  a.M = M; a.N = N; a.G = static_cast<int>(K / 128); a.m_offsets = nullptr; a.num_experts = 0;
  a.n_fastest = M > N;
  const int64_t tiles = dense_tiles(M, N);
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const bool row_b = b_scale_mode == FP8Q_BSCALE_ROW1x128, bf16 = out_dtype == FP8Q_OUT_BF16;
  CUtensorMap tmC = tmA;   // a placeholder unless the output leaves through TMA
  if (bf16 && !row_b && (st = encode_output_bf16(&tmC, C, N, M, ldc)) != FP8Q_OK) return st;
  return dispatch_dense(tmA, tmB, tmC, a, row_b, bf16, tiles, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream));
}

int fp8_gemm_blockscaled(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                         const float* sB, int64_t ld_sb, int b_scale_mode, void* C, int out_dtype,
                         int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                         void* stream) {
  return fp8_gemm_blockscaled_ws(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode, C, out_dtype, M, N, K,
                                 lda, ldb, ldc, nullptr, 0, stream);
}

int fp8_gemm_blockscaled_quant(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                               const float* sB, int64_t ld_sb, int b_scale_mode, void* C, int64_t ldc,
                               uint8_t* qC, int64_t ldq, float* sC, int64_t ld_sc, int pow2_scale,
                               int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                               void* stream) {
  if (M == 0 && N >= 0 && K >= 0) return FP8Q_OK;
  // C is optional: without it the C checks run on stand-ins that always pass them.
  int st = check_dense_blockscaled(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode,
                                   C != nullptr ? C : static_cast<void*>(qC), FP8Q_OUT_BF16, M, N,
                                   K, lda, ldb, C != nullptr ? ldc : N);
  if (st != FP8Q_OK) return st;
  if (!qC || !sC) return FP8Q_ERR_NULL;
  if (ldq < N || ld_sc < M) return FP8Q_ERR_SHAPE;
  if (ldq % 16 != 0 || !aligned(qC, 16) || !aligned(sC, 4)) return FP8Q_ERR_ALIGN;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, M, lda, 128)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, B, K, N, ldb, Cfg1::kBBox)) != FP8Q_OK) return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = ld_sa; a.sB = sB; a.ld_sb = ld_sb; a.C = C; a.ldc = ldc;
  a.M = M; a.N = N; a.G = static_cast<int>(K / 128); a.m_offsets = nullptr; a.num_experts = 0;
  a.n_fastest = M > N;
  a.qc = qC; a.ldq = ldq; a.sc = sC; a.ld_sc = ld_sc; a.qpow2 = pow2_scale != 0;
  const int64_t tiles = dense_tiles(M, N);
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  // no workspace: every tile is finished by one CTA, which quantizes its rows
  return dispatch_dense(tmA, tmB, tmA, a, b_scale_mode == FP8Q_BSCALE_ROW1x128, true, tiles, nullptr, 0,
                        static_cast<cudaStream_t>(stream));
}

int fp8_gemm_blockscaled_ue8m0(const uint8_t* A, const float* sA, int64_t ld_sa,
                               const uint8_t* B, const float* sB, int64_t ld_sb, int b_scale_mode,
                               void* C, int out_dtype, int64_t M, int64_t N, int64_t K,
                               int64_t lda, int64_t ldb, int64_t ldc, void* stream) {
  using Cfg = fp8q::Ue8m0Cfg<false>;
  if (M == 0 && N >= 0 && K >= 0) return FP8Q_OK;
  int st = check_dense_blockscaled(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode, C, out_dtype, M, N, K,
                                   lda, ldb, ldc);
  if (st != FP8Q_OK) return st;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, M, lda, Cfg::kTileM)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, B, K, N, ldb, Cfg::kN)) != FP8Q_OK) return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = ld_sa; a.sB = sB; a.ld_sb = ld_sb; a.C = C; a.ldc = ldc;
  a.M = M; a.N = N; a.G = static_cast<int>(K / 128); a.m_offsets = nullptr; a.num_experts = 0;
  a.n_fastest = M > N;
  const int64_t tiles = ((M + Cfg::kTileM - 1) / Cfg::kTileM) * ((N + Cfg::kN - 1) / Cfg::kN);
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const auto s = static_cast<cudaStream_t>(stream);
  const bool row_b = b_scale_mode == FP8Q_BSCALE_ROW1x128;
  if (out_dtype == FP8Q_OUT_BF16)
    return row_b ? run_gemm_ue8m0<true, true, false>(tmA, tmB, a, tiles, s)
                 : run_gemm_ue8m0<false, true, false>(tmA, tmB, a, tiles, s);
  return row_b ? run_gemm_ue8m0<true, false, false>(tmA, tmB, a, tiles, s)
               : run_gemm_ue8m0<false, false, false>(tmA, tmB, a, tiles, s);
}

int fp8_gemm_grouped_ue8m0(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* W,
                           const float* sW, void* C, int out_dtype, const int32_t* m_offsets,
                           int num_groups, int64_t max_sum_M, int64_t N, int64_t K, void* stream) {
  using Cfg = fp8q::Ue8m0Cfg<true>;
  if (max_sum_M < 0 || N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (num_groups < 1 || num_groups > fp8q::kMaxGroups) return FP8Q_ERR_UNSUPPORTED;
  if (max_sum_M == 0) return FP8Q_OK;
  int st = check_gemm_common(A, W, C, out_dtype, max_sum_M, N, K, K, K, N);
  if (st != FP8Q_OK) return st;
  if (!sA || !sW || !m_offsets) return FP8Q_ERR_NULL;
  if (ld_sa < max_sum_M) return FP8Q_ERR_SHAPE;
  if (!aligned(sA, 4) || !aligned(sW, 4) || !aligned(m_offsets, 4)) return FP8Q_ERR_ALIGN;
  if (static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, max_sum_M, K, Cfg::kTileM)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, W, K, static_cast<uint64_t>(num_groups) * N, K, Cfg::kN)) != FP8Q_OK)
    return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = ld_sa; a.sB = sW; a.ld_sb = 0; a.C = C; a.ldc = N;
  a.M = max_sum_M; a.N = N; a.G = static_cast<int>(K / 128);
  a.m_offsets = m_offsets; a.num_experts = num_groups;
  // Upper bound on tiles (every group may add one partial m-tile) sizes the persistent grid.
  const int64_t bound = ((max_sum_M + Cfg::kTileM - 1) / Cfg::kTileM + num_groups) *
                        ((N + Cfg::kN - 1) / Cfg::kN);
  if (bound > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const auto s = static_cast<cudaStream_t>(stream);
  return out_dtype == FP8Q_OUT_BF16 ? run_gemm_ue8m0<false, true, true>(tmA, tmB, a, bound, s)
                                    : run_gemm_ue8m0<false, false, true>(tmA, tmB, a, bound, s);
}

int fp8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, size_t* bytes) {
  if (!bytes) return FP8Q_ERR_NULL;
  *bytes = 0;
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (M == 0 || N == 0 || K == 0) return FP8Q_OK;
  if (K % 128 != 0 || N % 128 != 0) return FP8Q_ERR_SHAPE;
  // both B scale modes and output types share the plan
  const int units = GemmLauncher<true, false, false, true>::max_units();
  if (units <= 0) return FP8Q_ERR_CUDA;
  *bytes = plan_split(dense_tiles(M, N), K / 128, units).ws_bytes;
  return FP8Q_OK;
}

int fp8_gemm_grouped(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* W,
                     const float* sW, void* C, int out_dtype, const int32_t* m_offsets,
                     int num_groups, int64_t max_sum_M, int64_t N, int64_t K, void* stream) {
  if (max_sum_M < 0 || N < 0 || K < 0) return FP8Q_ERR_SHAPE;
  if (num_groups < 1 || num_groups > fp8q::kMaxGroups) return FP8Q_ERR_UNSUPPORTED;
  if (max_sum_M == 0) return FP8Q_OK;
  int st = check_gemm_common(A, W, C, out_dtype, max_sum_M, N, K, K, K, N);
  if (st != FP8Q_OK) return st;
  if (!sA || !sW || !m_offsets) return FP8Q_ERR_NULL;
  if (ld_sa < max_sum_M) return FP8Q_ERR_SHAPE;
  if (!aligned(sA, 4) || !aligned(sW, 4) || !aligned(m_offsets, 4)) return FP8Q_ERR_ALIGN;
  if (static_cast<int64_t>(num_groups) * N > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, max_sum_M, K, 128)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, W, K, static_cast<uint64_t>(num_groups) * N, K, Cfg1::kBBox)) !=
      FP8Q_OK)
    return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = ld_sa; a.sB = sW; a.ld_sb = 0; a.C = C; a.ldc = N;
  a.M = max_sum_M; a.N = N; a.G = static_cast<int>(K / 128);
  a.m_offsets = m_offsets; a.num_experts = num_groups;
  // Upper bound on tiles (every group may add one partial m-tile) sizes the persistent grid.
  const int64_t bound = ((max_sum_M + Cfg1::kTileM - 1) / Cfg1::kTileM + num_groups) *
                        ((N + Cfg1::kN - 1) / Cfg1::kN);
  if (bound > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const auto s = static_cast<cudaStream_t>(stream);
  if (out_dtype == FP8Q_OUT_BF16) {
    CUtensorMap tmC;
    if ((st = encode_output_bf16(&tmC, C, N, max_sum_M, N)) != FP8Q_OK) return st;
    return run_gemm<true, false, true, true>(tmA, tmB, tmC, a, bound, nullptr, 0, s);
  }
  return run_gemm<true, false, true, false>(tmA, tmB, tmA, a, bound, nullptr, 0, s);
}

int fp8_gemm_nopromo(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB, float* C,
                     int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                     void* stream) {
  if (M == 0 && N >= 0 && K >= 0) return FP8Q_OK;
  int st = check_gemm_common(A, B, C, FP8Q_OUT_FP32, M, N, K, lda, ldb, ldc);
  if (st != FP8Q_OK) return st;
  if (!sA || !sB) return FP8Q_ERR_NULL;
  if (!aligned(sA, 4) || !aligned(sB, 4)) return FP8Q_ERR_ALIGN;
  CUtensorMap tmA, tmB;
  if ((st = encode_operand(&tmA, A, K, M, lda, 128)) != FP8Q_OK) return st;
  if ((st = encode_operand(&tmB, B, K, N, ldb, Cfg1::kBBox)) != FP8Q_OK) return st;
  GemmArgs a{};
  a.sA = sA; a.ld_sa = 0; a.sB = sB; a.ld_sb = 0; a.C = C; a.ldc = ldc;
  a.M = M; a.N = N; a.G = static_cast<int>(K / 128); a.m_offsets = nullptr; a.num_experts = 0;
  a.n_fastest = M > N;
  const int64_t tiles = dense_tiles(M, N);
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  return run_gemm<false, false, false, false>(tmA, tmB, tmA, a, tiles, nullptr, 0,
                                                     static_cast<cudaStream_t>(stream));
}

// The split-K GEMM with its workspace in the library's fixed device scratch (see
// g_static_scratch above); allocates nothing.
int fp8_gemm_blockscaled_noalloc(const uint8_t* A, const float* sA, int64_t ld_sa,
                                 const uint8_t* B, const float* sB, int64_t ld_sb,
                                 int b_scale_mode, void* C, int out_dtype, int64_t M, int64_t N,
                                 int64_t K, int64_t lda, int64_t ldb, int64_t ldc, void* stream) {
  if (M == 0 && N >= 0 && K >= 0) return FP8Q_OK;
  // The argument errors are those of fp8_gemm_blockscaled, checked before the plan is sized.
  int st = check_dense_blockscaled(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode, C, out_dtype, M, N, K,
                                   lda, ldb, ldc);
  if (st != FP8Q_OK) return st;
  size_t need = 0;
  if ((st = fp8_gemm_workspace_size(M, N, K, &need)) != FP8Q_OK) return st;
  if (need > kStaticScratchBytes) return FP8Q_ERR_SHAPE;   // the plan would overflow the array
  void* scratch = static_scratch_address();
  if (scratch == nullptr) return FP8Q_ERR_CUDA;
  // Nothing in the scratch has to start at zero: in a call that completes, every partial
  // tile the reduction reads is written earlier in the same call.  After a device-side
  // timeout (reported by fp8q_get_device_error) a partial may not have been written, and
  // the reduction then adds a previous call's leftovers: C is undefined in that case.
  return fp8_gemm_blockscaled_ws(A, sA, ld_sa, B, sB, ld_sb, b_scale_mode, C, out_dtype, M, N, K,
                                 lda, ldb, ldc, scratch, kStaticScratchBytes, stream);
}

// Launches a one-thread kernel whose bounded wait cannot be satisfied; it returns after
// timeout_ns with the timeout recorded in the device error word (read it with
// fp8q_get_device_error).  Exercises the failure path without faulting the GPU.
int fp8q_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 1000000000ull) return FP8Q_ERR_SHAPE;
  fp8q::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // extern "C"
