// Block-scaled FP8 GEMM with per-128-K promotion for sm_100a (tcgen05 + TMEM + TMA).
//
// C[m, n] = sum_g  P_g[m, n] * sA[m, g] * sB(n, g),   P_g = sum_{k in group g} qA[m,k] qB[n,k]
//
// the-good.kr wr_id=2169793 para 1: per-group scaling factors along the inner
// dimension K, multiplied in on the CUDA cores as dequantization.
// pkd.ac.th webboard 78017 para 3 and why-be.co.kr wr_id=57820 para 3: once an
// interval of 128 K elements is accumulated on the tensor cores, the partial
// result is copied out, multiplied by the scaling factors and added into FP32
// registers.  On Hopper two warpgroups ping-pong so that one promotes while the
// other issues MMAs (pkd.ac.th webboard 78017 para 4); here the analogue is a
// double-buffered TMEM accumulator: the tensor core fills buffer g+1 while the
// epilogue warps drain buffer g.
//
// Roles (one 384-thread CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A tile [128 x 128 B] and B tile [256 x 128 B] per
//               K-group into a 4-stage shared-memory ring (128-byte swizzle).
//   warp 1      TMEM owner + MMA issuer: 4 x tcgen05.mma kind::f8f6f4 (K = 32 each)
//               per group into TMEM buffer (group parity), then tcgen05.commit to
//               free the smem stage and to publish the partial.
//   warps 2-3   idle (they complete the first warpgroup).
//   warps 4-11  promotion/epilogue: warp w reads TMEM lanes 32*(w%4).., columns
//               128*((w-4)/4)..; per group: tcgen05.ld -> acc += P * scale in FP32
//               registers; at tile end: convert and store C.
//
// Registers: the launch gives 168 per thread (3 warps per SM sub-partition).  The
// first warpgroup gives registers back (setmaxnreg 56) and the two epilogue
// warpgroups take them (setmaxnreg 224) for the 128-float running sum per thread:
// 128 * 56 + 256 * 224 = 384 * 168, and per sub-partition 56 + 2 * 224 <= 512.
//
// PROMOTE = false is the bench-only no-promotion variant: the whole K is
// accumulated in one TMEM buffer and per-row / per-column (1xK) scales are applied
// once at the end.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace fp8q {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 4;                      // first epilogue warp (second warpgroup)
constexpr int kGemmThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kRegsCtl = 56, kRegsEpi = 224;      // setmaxnreg split (see above)
constexpr uint32_t kABytes = kBM * kBK;
constexpr uint32_t kBBytes = kBN * kBK;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 1024;

// Error sites recorded with a timeout.
enum : unsigned int {
  kSiteProducer = 1,
  kSiteMmaFull = 2,
  kSiteMmaEmpty = 3,
  kSiteEpilogue = 4,
  kSiteDrain = 5
};

struct GemmArgs {
  const float* sA;      // PROMOTE: group-major [G][ld_sa]; no-promote: [M]
  int64_t ld_sa;
  const float* sB;      // BLOCK: [E][N/128][G]; ROW: group-major [G][ld_sb]; no-promote: [N]
  int64_t ld_sb;
  void* C;
  int64_t ldc;
  int64_t M;            // dense: rows; grouped: bound on sum of rows (A's allocation)
  int64_t N;
  int G;                // K / 128
  const int32_t* m_offsets;  // grouped: [E + 1] on the device
  int num_experts;
};

constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

struct SmemLayout {
  // byte offsets from the 1024-aligned base
  static constexpr uint32_t a = 0;                                   // kStages x 16 KB
  static constexpr uint32_t b = a + kStages * kABytes;               // kStages x 32 KB
  static constexpr uint32_t bars = b + kStages * kBBytes;
  // barriers: full[S], empty[S], tfull[2], tempty[2], drain
  static constexpr uint32_t n_bars = 2 * kStages + 5;
  static constexpr uint32_t misc = align_up(bars + 8 * n_bars, 16);  // tmem slot, abort flag
  static constexpr uint32_t sched = align_up(misc + 16, 16);         // int[kMaxGroups + 1]
  static constexpr uint32_t sbrow = align_up(sched + 4 * (kMaxGroups + 1), 128);  // float[2][2][128]
  static constexpr uint32_t end = sbrow + 4 * 2 * 2 * 128;
  static constexpr uint32_t bytes = end + 1024;                      // + base alignment slack
};
static_assert(SmemLayout::a % 1024 == 0 && SmemLayout::b % 1024 == 0, "swizzle atoms");
static_assert(SmemLayout::sbrow % 16 == 0, "float4 reads of the scale slots");
static_assert(SmemLayout::bytes <= 232448, "fits the 227 KB opt-in shared memory");

// Output tile of index t: first row of A, row bound for stores, first row of B (in the
// stacked [E*N, K] weights), first output column, expert.
struct Tile {
  int64_t row0, row_end, brow0, col0;
  int expert;
};

// Rows of expert e, clamped to [0, M] so that inconsistent offsets can never make a
// tile read or write outside A / C.
__device__ __forceinline__ void expert_rows(const GemmArgs& p, int e, int64_t& r_begin,
                                            int64_t& r_end) {
  int64_t b = p.m_offsets[e], en = p.m_offsets[e + 1];
  b = b < 0 ? 0 : (b > p.M ? p.M : b);
  en = en < b ? b : (en > p.M ? p.M : en);
  r_begin = b;
  r_end = en;
}

template <bool GROUPED>
__device__ __forceinline__ Tile decode_tile(int t, const GemmArgs& p, int mt_total, int nt_total,
                                            const int* sched) {
  Tile tl;
  if (!GROUPED) {
    const int mt = t % mt_total, nt = t / mt_total;
    tl.row0 = static_cast<int64_t>(mt) * kBM;
    tl.row_end = p.M;
    tl.col0 = static_cast<int64_t>(nt) * kBN;
    tl.brow0 = tl.col0;
    tl.expert = 0;
  } else {
    // sched[e] = first tile of expert e (prefix over experts), sched[E] = total.
    int lo = 0, hi = p.num_experts;  // find e with sched[e] <= t < sched[e + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sched[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    int64_t r_begin, r_end;
    expert_rows(p, e, r_begin, r_end);
    const int mte = static_cast<int>((r_end - r_begin + kBM - 1) / kBM);
    const int local = t - sched[e];
    const int mt = local % mte, nt = local / mte;
    tl.row0 = r_begin + static_cast<int64_t>(mt) * kBM;
    tl.row_end = r_end;
    tl.col0 = static_cast<int64_t>(nt) * kBN;
    tl.brow0 = static_cast<int64_t>(e) * p.N + tl.col0;
    tl.expert = e;
  }
  return tl;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <bool PROMOTE, bool ROW_B, bool GROUPED, bool OUT_BF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_fp8_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA,
                                const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SmemLayout::bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 4);
  int* sched = reinterpret_cast<int*>(smem + SmemLayout::sched);
  float* sbrow = reinterpret_cast<float*>(smem + SmemLayout::sbrow);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 32 * kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }

  const int nt_total = static_cast<int>((p.N + kBN - 1) / kBN);
  int mt_total = 0, num_tiles = 0;
  if (!GROUPED) {
    mt_total = static_cast<int>((p.M + kBM - 1) / kBM);
    num_tiles = mt_total * nt_total;
  } else {
    // per-expert tile counts, then an exclusive prefix (E is small)
    for (int e = threadIdx.x; e < p.num_experts; e += blockDim.x) {
      int64_t rb, re;
      expert_rows(p, e, rb, re);
      const int64_t rows = re - rb;
      sched[e + 1] = rows > 0 ? static_cast<int>((rows + kBM - 1) / kBM) * nt_total : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      sched[0] = 0;
      for (int e = 1; e <= p.num_experts; ++e) sched[e] += sched[e - 1];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (GROUPED) num_tiles = sched[p.num_experts];
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kEpiWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        const Tile tl = decode_tile<GROUPED>(t, p, mt_total, nt_total, sched);
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u, kSiteProducer, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(s), kABytes + kBBytes);
          tma_load_2d(sbase + SmemLayout::a + s * kABytes, &tmA, full_bar(s), g * kBK,
                      static_cast<int32_t>(tl.row0));
          tma_load_2d(sbase + SmemLayout::b + s * kBBytes, &tmB, full_bar(s), g * kBK,
                      static_cast<int32_t>(tl.brow0));
        }
      }
      // Every issued load lands before the CTA can exit (bounded; loads finish on their own).
      const uint32_t first = it > kStages ? it - kStages : 0;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait(full_bar(j % kStages), (j / kStages) & 1u, kSiteDrain, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kBM, kBN);
      uint32_t it = 0, acc_it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        uint32_t buf = 0;
        for (int g = 0; g < G; ++g, ++it) {
          if (PROMOTE || g == 0) {
            buf = acc_it & 1u;
            if (!mbar_wait(tempty_bar(buf), ((acc_it >> 1) & 1u) ^ 1u, kSiteMmaEmpty, abort_flag)) {
              ok = false;
              break;
            }
          }
          const int s = it % kStages;
          if (!mbar_wait(full_bar(s), (it / kStages) & 1u, kSiteMmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + buf * kBN;
          const uint32_t a_addr = sbase + SmemLayout::a + s * kABytes;
          const uint32_t b_addr = sbase + SmemLayout::b + s * kBBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {
            const uint32_t accumulate = PROMOTE ? (kk > 0) : (g > 0 || kk > 0);
            mma_f8(d, smem_desc_k_sw128(a_addr + 32 * kk), smem_desc_k_sw128(b_addr + 32 * kk),
                   idesc, accumulate);
          }
          mma_commit(empty_bar(s));
          if (PROMOTE || g == G - 1) {
            mma_commit(tfull_bar(buf));
            ++acc_it;
          }
        }
      }
      // All MMAs this thread issued complete before TMEM is released.
      mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, kSiteDrain, nullptr);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // ------------------------------------------------------------ promotion + epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;              // TMEM lanes this warp may access
    const int set = ew >> 2;                // column half of the tile
    const int row_in_tile = quad * 32 + lane;
    const int tid_in_set = (ew & 3) * 32 + lane;
    float* sb_slots = sbrow + set * 2 * 128;
    // The epilogue never leaves its loops early: after an abort it keeps walking the
    // (uniform) tile/group structure without touching TMEM, so that every thread of a
    // column set reaches the same named barriers.
    uint32_t acc_it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const Tile tl = decode_tile<GROUPED>(t, p, mt_total, nt_total, sched);
      const int64_t m = tl.row0 + row_in_tile;
      const bool row_ok = m < tl.row_end;
      const int64_t n0 = tl.col0 + set * 128;
      const bool cols_ok = n0 < p.N;
      float acc[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.0f;

      if (PROMOTE) {
        const float* sB_tile = nullptr;
        if (!ROW_B)
          sB_tile = p.sB + (static_cast<int64_t>(tl.expert) * (p.N / 128) + n0 / 128) * G;
        auto load_sa = [&](int g) -> float {
          return row_ok ? __ldg(p.sA + static_cast<int64_t>(g) * p.ld_sa + m) : 0.0f;
        };
        auto load_sb = [&](int g) -> float {
          if (ROW_B) {
            const int64_t n = n0 + tid_in_set;
            return cols_ok ? __ldg(p.sB + static_cast<int64_t>(g) * p.ld_sb + n) : 0.0f;
          }
          return cols_ok ? __ldg(sB_tile + g) : 0.0f;
        };
        float sa_cur = load_sa(0), sb_cur = load_sb(0);
        for (int g = 0; g < G; ++g) {
          const bool more = g + 1 < G;
          const float sa_nxt = more ? load_sa(g + 1) : 0.0f;
          const float sb_nxt = more ? load_sb(g + 1) : 0.0f;
          // ROW mode: the set's 128 column scales of this group go through a 2-slot
          // ring that alternates with every group of every tile.
          float* slot = sb_slots + (acc_it & 1u) * 128;
          if (ROW_B) {
            slot[tid_in_set] = sb_cur;
            named_bar_sync(1 + set, 128);
          }
          const uint32_t buf = acc_it & 1u;
          if (ok) ok = mbar_wait(tfull_bar(buf), (acc_it >> 1) & 1u, kSiteEpilogue, abort_flag);
          if (ok) {
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * kBN + set * 128;
            const float sc = sa_cur * sb_cur;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld_32cols(taddr + c * 32, r);
              tmem_ld_wait();
              if (c == 3) {
                tc_fence_before();
                mbar_arrive(tempty_bar(buf));
              }
              if (ROW_B) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                  const float4 b4 = *reinterpret_cast<const float4*>(slot + c * 32 + j);
                  acc[c * 32 + j + 0] = __fmaf_rn(__uint_as_float(r[j + 0]) * b4.x, sa_cur, acc[c * 32 + j + 0]);
                  acc[c * 32 + j + 1] = __fmaf_rn(__uint_as_float(r[j + 1]) * b4.y, sa_cur, acc[c * 32 + j + 1]);
                  acc[c * 32 + j + 2] = __fmaf_rn(__uint_as_float(r[j + 2]) * b4.z, sa_cur, acc[c * 32 + j + 2]);
                  acc[c * 32 + j + 3] = __fmaf_rn(__uint_as_float(r[j + 3]) * b4.w, sa_cur, acc[c * 32 + j + 3]);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  acc[c * 32 + j] = __fmaf_rn(__uint_as_float(r[j]), sc, acc[c * 32 + j]);
              }
            }
          }
          ++acc_it;
          sa_cur = sa_nxt;
          sb_cur = sb_nxt;
        }
      } else {
        // no promotion: one accumulator over all of K, scaled once by sA[m] * sB[n]
        const float sa = row_ok ? __ldg(p.sA + m) : 0.0f;
        float* slot = sb_slots;
        named_bar_sync(1 + set, 128);   // previous tile's readers are done with the slot
        slot[tid_in_set] = cols_ok ? __ldg(p.sB + n0 + tid_in_set) : 0.0f;
        named_bar_sync(1 + set, 128);
        const uint32_t buf = acc_it & 1u;
        if (ok) ok = mbar_wait(tfull_bar(buf), (acc_it >> 1) & 1u, kSiteEpilogue, abort_flag);
        if (ok) {
          tc_fence_after();
          const uint32_t taddr =
              tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * kBN + set * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld_32cols(taddr + c * 32, r);
            tmem_ld_wait();
            if (c == 3) {
              tc_fence_before();
              mbar_arrive(tempty_bar(buf));
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
              acc[c * 32 + j] = (__uint_as_float(r[j]) * sa) * slot[c * 32 + j];
          }
        }
        ++acc_it;
      }

      // ---- store the tile's rows: this thread owns row m, columns n0 .. n0+127
      if (ok && row_ok && cols_ok) {
        if (OUT_BF16) {
          __nv_bfloat16* crow = reinterpret_cast<__nv_bfloat16*>(p.C) + m * p.ldc + n0;
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
            uint4 o;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j + 0], acc[j + 1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
            o.x = *reinterpret_cast<uint32_t*>(&h0);
            o.y = *reinterpret_cast<uint32_t*>(&h1);
            o.z = *reinterpret_cast<uint32_t*>(&h2);
            o.w = *reinterpret_cast<uint32_t*>(&h3);
            *reinterpret_cast<uint4*>(crow + j) = o;
          }
        } else {
          float* crow = reinterpret_cast<float*>(p.C) + m * p.ldc + n0;
#pragma unroll
          for (int j = 0; j < 128; j += 4)
            *reinterpret_cast<float4*>(crow + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace fp8q
