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
// other issues MMAs (pkd.ac.th webboard 78017 para 4); here the analogue is a ring of
// TMEM accumulator slices: the tensor core fills the next slices while the epilogue
// warps drain the finished ones.
//
// Roles (384-thread CTAs, one per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per K-group, the A tile [128 rows x 128 B] and the B tile
//               [256 rows x 128 B] into a shared-memory ring (128-byte swizzle; 4 stages,
//               3 where the bf16 output is staged for TMA stores).
//   warp 1      TMEM owner and MMA issuer: per group 4 x tcgen05.mma kind::f8f6f4 (M128
//               N256 K32) into a fresh 256-column TMEM accumulator (two, alternating),
//               then one tcgen05.commit on the stage's barrier, which both frees the smem
//               stage and publishes the partial to the epilogue.  It waits for the
//               stage's operands before the accumulator: the operands are normally in
//               place long before, while the accumulator comes free just in time, and
//               the MMAs should follow its release with nothing in between.
//   warp 2      scale producer: for every group, ahead of the epilogue, copies the
//               tile's 128 row scales of A and its B scales (2 block scales, or 256
//               column scales) into a shared-memory ring of four-group slots with
//               cp.async (20-24 groups ahead for block scales, 16 for column scales).
//   warp 3      idle (it completes the first warpgroup).
//   warps 4-11  promotion/epilogue: warp w reads TMEM lanes 32*(w%4).. and the tile's
//               columns 128*((w-4)/4)..; per group two 64-column tcgen05.ld and
//               acc += P * scale in FP32 registers (f32x2 FMAs); the accumulator is freed
//               after the second load; at the end of the tile: convert and store C (bf16
//               with block scales: through a per-warp shared-memory slice and TMA stores).
//
// Measured on B200 and not kept (same operands, same parity): a CTA pair with 256 x 256
// tiles (a third less L2 traffic per FLOP, but the cross-CTA accumulator release slowed
// every group); MMAs issued as two N = 128 halves into four TMEM slices, and 128 x 128
// tiles with four accumulators (more slack per accumulator, but more operand traffic and
// twice the per-group synchronisation); 32-column TMEM loads pipelined with the FMAs
// (the extra registers spill); releases as one arrival per warp; block scales loaded by
// the epilogue itself instead of the scale ring.
//
// Registers: the launch gives 168 per thread (3 warps per SM sub-partition).  The
// first warpgroup gives registers back (setmaxnreg 40) and the two epilogue
// warpgroups take them (setmaxnreg 232) for the 128-float running sum per thread:
// 128 * 40 + 256 * 232 <= 384 * 168, and per sub-partition 40 + 2 * 232 <= 512.
//
// PROMOTE = false is the bench-only no-promotion variant: the whole K is
// accumulated in one TMEM buffer and per-row / per-column (1xK) scales are applied
// once at the end.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "quant.cuh"

namespace fp8q {

constexpr int kBK = 128;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 4;                      // first epilogue warp (second warpgroup)
constexpr int kGemmThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kRegsCtl = 40, kRegsEpi = 232;      // setmaxnreg split (see above)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 1024;

// Error sites recorded with a timeout.
enum : unsigned int {
  kSiteProducer = 1,
  kSiteMmaFull = 2,
  kSiteMmaEmpty = 3,
  kSiteEpilogue = 4,
  kSiteDrain = 5,
  kSiteScales = 6
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
  // Split-K of the last partial wave (dense only).  Tiles [0, tiles_full) are computed
  // whole; the remaining tail_tiles are split into tail_split K-chunks, one per CTA (or
  // CTA pair) of the last wave, whose FP32 partial tiles go to ws and are summed by
  // splitk_reduce_kernel.  tail_tiles == 0: no split, ws unused.
  float* ws;
  int tiles_full;
  int tail_tiles;
  int tail_split;
  // Quantized output (dense, bf16, no split): when qc is set, every 1x128 row segment of
  // the bf16 C is also quantized as fp8q_quant_act_1x128 would (codes qc[m * ldq + n],
  // scales sc[(n / 128) * ld_sc + m], power-of-two scales when qpow2); C itself is
  // stored only when C is set.
  uint8_t* qc;
  int64_t ldq;
  float* sc;
  int64_t ld_sc;
  int qpow2;
  // Dense tile order: m fastest (0), so that the CTAs of a wave share B tiles and re-read
  // A once per wave, or n fastest (1), the reverse; the host takes n fastest when A is
  // the larger operand (M > N).
  int n_fastest;
};

// A unit of work of one CTA (or CTA pair): a tile and a range of its K-groups, written
// to C (ws_index < 0) or as a partial tile to the workspace.
struct Unit {
  int tile, g0, g1, ws_index;
};

__device__ __forceinline__ int units_of(const GemmArgs& p, int num_tiles, int unit0, int units) {
  if (p.tail_tiles == 0) return unit0 < num_tiles ? (num_tiles - unit0 + units - 1) / units : 0;
  int n = unit0 < p.tiles_full ? (p.tiles_full - unit0 + units - 1) / units : 0;
  if (unit0 < p.tail_tiles * p.tail_split) ++n;
  return n;
}

__device__ __forceinline__ Unit unit_at(int i, const GemmArgs& p, int unit0, int units, int G) {
  Unit u;
  const int n_whole = p.tail_tiles == 0
                          ? 0x7FFFFFFF
                          : (unit0 < p.tiles_full ? (p.tiles_full - unit0 + units - 1) / units : 0);
  if (i < n_whole) {
    u.tile = unit0 + i * units;
    u.g0 = 0;
    u.g1 = G;
    u.ws_index = -1;
  } else {
    const int r = unit0 / p.tail_split, ch = unit0 % p.tail_split;
    u.tile = p.tiles_full + r;
    u.g0 = static_cast<int>(static_cast<int64_t>(G) * ch / p.tail_split);
    u.g1 = static_cast<int>(static_cast<int64_t>(G) * (ch + 1) / p.tail_split);
    u.ws_index = unit0;
  }
  return u;
}

constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// TSTORE: the tile's bf16 output leaves through shared memory and TMA stores (a 64 KB
// staging area, one 8 KB slice per epilogue warp), so the epilogue warps go on to the next
// tile while the stores drain; the operand ring then has 3 stages instead of 4.
template <bool ROW_B = false, bool TSTORE = false>
struct GemmCfg {
  static constexpr int kN = 256;                        // output columns per tile (MMA N)
  static constexpr int kTileM = 128;                    // output rows per tile (MMA M)
  static constexpr int kAccBufs = kTmemCols / kN;       // TMEM accumulators (groups in flight)
  static constexpr int kSetCols = kN / 2;               // columns per epilogue warpgroup
  static constexpr int kStages = TSTORE ? 3 : 4;
  static constexpr int kBBox = kN;                      // B rows per TMA box
  static constexpr uint32_t kABytes = 128 * kBK;        // per stage
  static constexpr uint32_t kBBytes = kN * kBK;
  static constexpr uint32_t kStageTx = kABytes + kBBytes;  // bytes per full barrier phase
  // shared memory, byte offsets from the 1024-aligned base
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + kStages * kABytes;
  static constexpr uint32_t bars = b + kStages * kBBytes;
  // Scale ring: a slot holds the scales of kSlotGroups consecutive groups of the CTA's
  // stream; per group its 128 A row scales and its B scales (the tile's kN column scales
  // in ROW mode; its kN / 128 block scales, padded to 4, otherwise).  One barrier wait
  // and one release per slot, not per group.
  static constexpr int kSlotGroups = 4;
  static constexpr int kScaleSlots = ROW_B ? 4 : (TSTORE ? 5 : 6);
  static constexpr uint32_t kGroupFloats = 128 + (ROW_B ? kN : 4);
  static constexpr uint32_t kSlotFloats = kSlotGroups * kGroupFloats;
  // full[S], empty[S], tfull[NB], tempty[NB], drain, sfull[R], sempty[R]
  static constexpr uint32_t n_bars = 2 * kStages + 2 * kAccBufs + 1 + 2 * kScaleSlots;
  static constexpr uint32_t misc = align_up(bars + 8 * n_bars, 16);   // tmem slot, abort flag
  static constexpr uint32_t sched = align_up(misc + 16, 16);          // int[kMaxGroups + 1]
  static constexpr uint32_t sbrow = align_up(sched + 4 * (kMaxGroups + 1), 128);  // float[2][2][128]
  static constexpr uint32_t sring = align_up(sbrow + 4 * 2 * 2 * 128, 128);  // float[R][kSlotFloats]
  static constexpr uint32_t kStageWarpBytes = 32 * kSetCols * 2;     // 32 rows of bf16
  static constexpr uint32_t stage = align_up(sring + 4 * kScaleSlots * kSlotFloats, 1024);
  static constexpr uint32_t end = TSTORE ? stage + kEpiWarps * kStageWarpBytes
                                         : sring + 4 * kScaleSlots * kSlotFloats;
  static constexpr uint32_t smem_bytes = end + 1024;                  // + base alignment slack
  static_assert(a % 1024 == 0 && b % 1024 == 0 && kABytes % 1024 == 0 && kBBytes % 1024 == 0,
                "swizzle atoms");
  static_assert(sbrow % 16 == 0 && sring % 16 == 0 && kGroupFloats % 4 == 0 && kN / 128 <= 4,
                "float4 reads of the scale slots");
  static_assert(kSetCols % 64 == 0 && kAccBufs >= 2, "64-column loads; two accumulators");
  static_assert(kN % 16 == 0 && kN <= 256 && kBBox <= 256, "MMA N and TMA box");
  static_assert(smem_bytes <= 232448, "fits the 227 KB opt-in shared memory");
  static_assert(!TSTORE || (kSetCols == 128 && stage % 1024 == 0), "two 64-column swizzled boxes per warp");
};

// The configuration a promoted-GEMM instantiation runs with (host and device agree on it).
template <bool PROMOTE, bool ROW_B, bool OUT_BF16, bool QOUT>
using GemmCfgOf = GemmCfg<ROW_B, PROMOTE && !ROW_B && OUT_BF16 && !QOUT>;

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

template <bool GROUPED, int TILE_M, int TILE_N>
__device__ __forceinline__ Tile decode_tile(int t, const GemmArgs& p, int mt_total, int nt_total,
                                            const int* sched) {
  Tile tl;
  if (!GROUPED) {
    const int fast = p.n_fastest ? nt_total : mt_total;   // tiles along the fast axis
    const int q = t / fast, r = t - q * fast;
    const int mt = p.n_fastest ? q : r, nt = p.n_fastest ? r : q;
    tl.row0 = static_cast<int64_t>(mt) * TILE_M;
    tl.row_end = p.M;
    tl.col0 = static_cast<int64_t>(nt) * TILE_N;
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
    // n-fastest inside an expert: concurrent tiles share a few row tiles of A and sweep
    // the expert's weight columns, so A stays in L2 for large experts and the 1-2 row
    // tiles of a small expert meet the same weight tile within one wave.
    const int local = t - sched[e];
    const int nt = local % nt_total, mt = local / nt_total;
    tl.row0 = r_begin + static_cast<int64_t>(mt) * TILE_M;
    tl.row_end = r_end;
    tl.col0 = static_cast<int64_t>(nt) * TILE_N;
    tl.brow0 = static_cast<int64_t>(e) * p.N + tl.col0;
    tl.expert = e;
  }
  return tl;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Promotion of one 32-column chunk of a slice into this thread's running sums:
// acc[j] += P * s (BLOCK: one scale for the whole chunk) or acc[j] += (P * sB[n]) * sA
// (ROW: a scale per column, read from shared memory as float4).
template <bool ROW_B>
__device__ __forceinline__ void promote_chunk(float2* acc, const uint32_t* r, float2 sc2,
                                              float2 sa2, const float* sbv) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float2 p0 = make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
    const float2 p1 = make_float2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
    float2& a0 = acc[j / 2];
    float2& a1 = acc[j / 2 + 1];
    if (ROW_B) {
      const float4 b4 = *reinterpret_cast<const float4*>(sbv + j);
      a0 = __ffma2_rn(__fmul2_rn(p0, make_float2(b4.x, b4.y)), sa2, a0);
      a1 = __ffma2_rn(__fmul2_rn(p1, make_float2(b4.z, b4.w)), sa2, a1);
    } else {
      a0 = __ffma2_rn(p0, sc2, a0);
      a1 = __ffma2_rn(p1, sc2, a1);
    }
  }
}

// Stores a row segment held one row per lane: lane i of each quad (4 lanes, rows r0 .. r0 + 3)
// holds chunks v[0 .. NC) (16 bytes each) of its row, destined for row_ptr(row) + 16 c.
// Groups of four chunks are transposed inside the quad (shuffles), so that each store
// instruction writes 64 contiguous bytes of one row per quad: 8 row pieces per warp
// instruction instead of 32 scattered 16-byte pieces.  `valid` is whether this lane's row
// is inside C; the quad's rows are exchanged with it.
template <int NC>
__device__ __forceinline__ void store_rows_by_quads(uint4 (&v)[NC], uint8_t* my_row, bool valid) {
  static_assert(NC % 4 == 0, "groups of four chunks");
  const int lane = threadIdx.x & 31, i = lane & 3;
  uint8_t* rows[4];
  bool ok[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {          // the quad's rows, row k from lane 4 (lane / 4) + k
    rows[k] = reinterpret_cast<uint8_t*>(
        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<uintptr_t>(my_row), (lane & ~3) + k));
    ok[k] = __shfl_sync(0xFFFFFFFFu, valid, (lane & ~3) + k);
  }
#pragma unroll
  for (int c0 = 0; c0 < NC; c0 += 4) {
    uint32_t w[4][4];                      // w[word][j]: word of chunk c0 + j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[0][j] = v[c0 + j].x;
      w[1][j] = v[c0 + j].y;
      w[2][j] = v[c0 + j].z;
      w[3][j] = v[c0 + j].w;
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) quad_transpose4(w[x], i);   // now w[x][k]: chunk c0 + i of row k
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (ok[k])
        *reinterpret_cast<uint4*>(rows[k] + 16 * (c0 + i)) = make_uint4(w[0][k], w[1][k], w[2][k], w[3][k]);
  }
}

// QOUT: the bf16 output is also quantized in 1x128 tiles (codes and scales through
// p.qc / p.sc; C only when p.C is set); a separate instantiation, so that the plain
// GEMM's registers are not shaped by it.
template <bool PROMOTE, bool ROW_B, bool GROUPED, bool OUT_BF16, bool QOUT = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_fp8_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA,
                                const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
  using Cfg = GemmCfgOf<PROMOTE, ROW_B, OUT_BF16, QOUT>;
  constexpr bool TSTORE = PROMOTE && !ROW_B && OUT_BF16 && !QOUT;
  constexpr int S = Cfg::kStages;
  constexpr int NB = Cfg::kAccBufs;
  constexpr int kN = Cfg::kN;
  constexpr int kSetCols = Cfg::kSetCols;
  static_assert(S >= NB, "a stage barrier's phase outlives the epilogue's wait for it");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + NB + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 2 * NB);
  constexpr int R = Cfg::kScaleSlots;
  auto sfull_bar = [&](int r) { return bar0 + 8u * (2 * S + 2 * NB + 1 + r); };
  auto sempty_bar = [&](int r) { return bar0 + 8u * (2 * S + 2 * NB + 1 + R + r); };
  float* sring = reinterpret_cast<float*>(smem + Cfg::sring);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::misc + 4);
  int* sched = reinterpret_cast<int*>(smem + Cfg::sched);
  float* sbrow = reinterpret_cast<float*>(smem + Cfg::sbrow);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;
  const int unit0 = blockIdx.x, units = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 32 * kEpiWarps);   // every epilogue thread frees it
    }
    mbar_init(drain_bar, 1);
    for (int r = 0; r < R; ++r) {
      mbar_init(sfull_bar(r), 32);                 // one cp.async arrival per producer lane
      mbar_init(sempty_bar(r), 32 * kEpiWarps);    // every epilogue thread frees the slot
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish<1>();
  }

  const int nt_total = static_cast<int>((p.N + kN - 1) / kN);
  int mt_total = 0, num_tiles = 0;
  if (!GROUPED) {
    mt_total = static_cast<int>((p.M + Cfg::kTileM - 1) / Cfg::kTileM);
    num_tiles = mt_total * nt_total;
  } else {
    // per-expert tile counts, then an exclusive prefix (E is small)
    for (int e = threadIdx.x; e < p.num_experts; e += blockDim.x) {
      int64_t rb, re;
      expert_rows(p, e, rb, re);
      const int64_t rows = re - rb;
      sched[e + 1] = rows > 0 ? static_cast<int>((rows + Cfg::kTileM - 1) / Cfg::kTileM) * nt_total : 0;
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
  const int n_units = units_of(p, num_tiles, unit0, units);
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kEpiWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        for (int ui = 0; ok && ui < n_units; ++ui) {
          const Unit u = unit_at(ui, p, unit0, units, G);
          const Tile tl = decode_tile<GROUPED, Cfg::kTileM, kN>(u.tile, p, mt_total, nt_total, sched);
          for (int g = u.g0; g < u.g1; ++g, ++it) {
            const int s = it % S;
            if (!mbar_wait(empty_bar(s), ((it / S) & 1u) ^ 1u, kSiteProducer, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(full_bar(s), Cfg::kStageTx);
            tma_load_2d(sbase + Cfg::a + s * Cfg::kABytes, &tmA, full_bar(s), g * kBK,
                        static_cast<int32_t>(tl.row0));
            tma_load_2d(sbase + Cfg::b + s * Cfg::kBBytes, &tmB, full_bar(s), g * kBK,
                        static_cast<int32_t>(tl.brow0));
          }
        }
        // every issued load lands before the CTA can exit (bounded; loads end on their own)
        const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0;
        for (uint32_t j = first; j < it; ++j)
          mbar_wait(full_bar(j % S), (j / S) & 1u, kSiteDrain, nullptr);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_e4m3_f32(Cfg::kTileM, kN);
        uint32_t it = 0, acc_it = 0;
        bool ok = true;
        for (int ui = 0; ok && ui < n_units; ++ui) {
          const Unit u = unit_at(ui, p, unit0, units, G);
          uint32_t buf = 0;
          for (int g = u.g0; g < u.g1; ++g, ++it) {
            const bool fresh = PROMOTE || g == u.g0;   // a new accumulator for this group
            const bool publish = PROMOTE || g == u.g1 - 1;
            const int s = it % S;
            // The stage's operands first (normally long in place), then the accumulator,
            // which comes free just in time: nothing should separate its release from
            // the MMAs.
            if (!mbar_wait(full_bar(s), (it / S) & 1u, kSiteMmaFull, abort_flag)) {
              ok = false;
              break;
            }
            if (fresh) {
              buf = acc_it % NB;
              if (!mbar_wait(tempty_bar(buf), ((acc_it / NB) & 1u) ^ 1u, kSiteMmaEmpty, abort_flag)) {
                ok = false;
                break;
              }
            }
            tc_fence_after();
            const uint32_t d = tmem_base + buf * kN;
            const uint32_t a_addr = sbase + Cfg::a + s * Cfg::kABytes;
            const uint32_t b_addr = sbase + Cfg::b + s * Cfg::kBBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 32; ++kk) {
              const uint32_t accumulate = PROMOTE ? (kk > 0) : (g > u.g0 || kk > 0);
              mma_f8<1>(d, smem_desc_k_sw128(a_addr + 32 * kk), smem_desc_k_sw128(b_addr + 32 * kk),
                        idesc, accumulate);
            }
            if (PROMOTE) {
              // One commit per group: its arrival on the stage's barrier both frees the
              // stage for the producer and publishes the group's partial to the epilogue
              // (group it uses stage it % S and accumulator it % NB).
              mma_commit<1>(empty_bar(s));
              ++acc_it;
            } else {
              mma_commit<1>(empty_bar(s));
              if (publish) {
                mma_commit<1>(tfull_bar(buf));
                ++acc_it;
              }
            }
          }
        }
        // All MMAs this thread issued complete before TMEM is released.
        mma_commit<1>(drain_bar);
        mbar_wait(drain_bar, 0, kSiteDrain, nullptr);
      }
    } else if (warp == 2 && PROMOTE) {
      // ---------------------------------------------------------- scale producer
      // Slot layout: [0, 128) A scales of the tile's 128 rows; then the B scales: the
      // tile's kN column scales (ROW mode) or, for 128x128 weight blocks, the kN / 128
      // blocks' scales.
      // `it` counts the CTA's groups; group it goes to slot (it / kSlotGroups) % R, part
      // it % kSlotGroups.  A slot is published after its last group, or after the CTA's
      // last group when that slot is only partly filled.
      constexpr uint32_t SG = Cfg::kSlotGroups;
      uint32_t it = 0;
      bool ok = true;
      for (int ui = 0; ok && ui < n_units; ++ui) {
        const Unit u = unit_at(ui, p, unit0, units, G);
        const Tile tl = decode_tile<GROUPED, Cfg::kTileM, kN>(u.tile, p, mt_total, nt_total, sched);
        const float* sB_tile =
            ROW_B ? nullptr : p.sB + (static_cast<int64_t>(tl.expert) * (p.N / 128) + tl.col0 / 128) * G;
        for (int g = u.g0; g < u.g1; ++g, ++it) {
          const uint32_t sl = it / SG;
          const int r = sl % R;
          if (it % SG == 0 &&
              !mbar_wait(sempty_bar(r), ((sl / R) & 1u) ^ 1u, kSiteScales, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t slot = sbase + Cfg::sring + 4u * (Cfg::kSlotFloats * r + Cfg::kGroupFloats * (it % SG));
          const float* sa_g = p.sA + static_cast<int64_t>(g) * p.ld_sa;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int64_t m = tl.row0 + 32 * j + lane;
            cp_async_4(slot + 4u * (32 * j + lane), sa_g + (m < tl.row_end ? m : 0), m < tl.row_end);
          }
          if (ROW_B) {
            const float* sb_g = p.sB + static_cast<int64_t>(g) * p.ld_sb;
#pragma unroll
            for (int j = 0; j < kN / 32; ++j) {
              const int64_t n = tl.col0 + 32 * j + lane;
              cp_async_4(slot + 4u * (128 + 32 * j + lane), sb_g + (n < p.N ? n : 0), n < p.N);
            }
          } else if (lane < kN / 128) {
            const bool v = tl.col0 + 128 * lane < p.N;
            cp_async_4(slot + 4u * (128 + lane), sB_tile + (v ? lane * G + g : 0), v);
          }
          if (it % SG == SG - 1) cp_async_arrive(sfull_bar(r));
        }
      }
      if (ok && it % SG != 0) cp_async_arrive(sfull_bar((it / SG) % R));   // the last, partial slot
      cp_async_wait_all();     // no copy into shared memory outlives the CTA
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
    auto release = [&](uint32_t buf) {      // every epilogue thread arrives
      tc_fence_before();
      mbar_arrive(tempty_bar(buf));
    };
    // The epilogue never leaves its loops early: after an abort it keeps walking the
    // (uniform) tile/group structure without touching TMEM, so that every thread of a
    // column set reaches the same named barriers.
    uint32_t acc_it = 0;
    bool ok = true;
    uint32_t rbuf[64];                      // one 64-column TMEM load
    float sa4[4] = {0.f, 0.f, 0.f, 0.f}, sb4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ui = 0; ui < n_units; ++ui) {
      const Unit u = unit_at(ui, p, unit0, units, G);
      bool warp_idle;
      {
        // warp-uniform: none of this warp's 32 rows is inside the tile's rows (an expert's
        // short last row tile), so its partials are never read.  (The tile is decoded
        // again for the stores, so that nothing of it stays live through the group loop.)
        const Tile tl = decode_tile<GROUPED, Cfg::kTileM, kN>(u.tile, p, mt_total, nt_total, sched);
        warp_idle = tl.row0 + row_in_tile - lane >= tl.row_end;
      }
      // acc[i] holds columns 2i, 2i+1 of this thread's row (packed FP32 pairs: the
      // promotion runs on the f32x2 FMA path, two accumulations per instruction).
      float2 acc[kSetCols / 2];
#pragma unroll
      for (int j = 0; j < kSetCols / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);

      if (PROMOTE) {
        for (int g = u.g0; g < u.g1; ++g) {
          // This group's scales, staged by the scale producer (the ring advances with
          // every group of every tile, in the same order as acc_it).
          constexpr uint32_t SG = Cfg::kSlotGroups;
          const uint32_t sl = acc_it / SG;
          const int r = sl % R;
          const int slot = Cfg::kSlotFloats * r + Cfg::kGroupFloats * (acc_it % SG);
          float sa_cur, sb_cur;
          if (ROW_B) {
            if (ok && acc_it % SG == 0) ok = mbar_wait(sfull_bar(r), (sl / R) & 1u, kSiteScales, abort_flag);
            sa_cur = sring[slot + quad * 32 + lane];
            sb_cur = 0.0f;
          } else {
            // Block-scaled B: at a slot's first group the slot's four groups of scales go to
            // registers and the slot is freed at once; its other groups read no shared
            // memory and pass no wait (on B200, 3% off the dense launch).  Entries of a last,
            // partly filled slot past the CTA's last group are read but never used.
            if (acc_it % SG == 0) {
              if (ok) ok = mbar_wait(sfull_bar(r), (sl / R) & 1u, kSiteScales, abort_flag);
              const int base = Cfg::kSlotFloats * r;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                sa4[j] = sring[base + Cfg::kGroupFloats * j + quad * 32 + lane];
                sb4[j] = sring[base + Cfg::kGroupFloats * j + 128 + set * kSetCols / 128];
              }
              mbar_arrive(sempty_bar(r));      // the slot is in registers: free it now
            }
            sa_cur = sa4[0];
            sb_cur = sb4[0];
            sa4[0] = sa4[1]; sa4[1] = sa4[2]; sa4[2] = sa4[3];
            sb4[0] = sb4[1]; sb4[1] = sb4[2]; sb4[2] = sb4[3];
          }
          const int sb = slot + 128 + set * kSetCols;        // ROW mode column scales
          const uint32_t buf = acc_it % NB;
          // group acc_it's MMAs have completed: the commit on its operand stage's barrier
          // (the epilogue cannot lag by a phase: group acc_it + S needs the accumulator
          // that this thread frees after group acc_it + S - NB)
          if (ok)
            ok = mbar_wait(empty_bar(acc_it % S), (acc_it / S) & 1u, kSiteEpilogue, abort_flag);
          ok = __all_sync(0xFFFFFFFFu, ok);  // warp-uniform: TMEM loads are per warp
          if (ok && !warp_idle) {
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * kN + set * kSetCols;
            const float2 sc2 = make_float2(sa_cur * sb_cur, sa_cur * sb_cur);
            const float2 sa2 = make_float2(sa_cur, sa_cur);
#pragma unroll
            for (int h = 0; h < kSetCols / 64; ++h) {
              tmem_ld_64cols(taddr + h * 64, rbuf);
              tmem_ld_wait_regs(rbuf);
              if (h == kSetCols / 64 - 1) release(buf);   // TMEM buffer free for group g + NB
              promote_chunk<ROW_B>(acc + 32 * h, rbuf, sc2, sa2, sring + sb + 64 * h);
              promote_chunk<ROW_B>(acc + 32 * h + 16, rbuf + 32, sc2, sa2, sring + sb + 64 * h + 32);
            }
          } else if (ok) {
            release(buf);
          }
          if (ROW_B && acc_it % SG == SG - 1) mbar_arrive(sempty_bar(r));   // the slot's groups consumed
          ++acc_it;
        }
      } else {
        // no promotion: one accumulator over all of K, scaled once by sA[m] * sB[n]
        const Tile tl = decode_tile<GROUPED, Cfg::kTileM, kN>(u.tile, p, mt_total, nt_total, sched);
        const int64_t m = tl.row0 + row_in_tile;
        const bool row_ok = m < tl.row_end;
        const int64_t n0 = tl.col0 + set * kSetCols;
        const bool cols_ok = n0 < p.N;
        const float sa = row_ok ? __ldg(p.sA + m) : 0.0f;
        float* slot = sb_slots;
        named_bar_sync(1 + set, 128);   // previous tile's readers are done with the slot
        if (tid_in_set < kSetCols)
          slot[tid_in_set] = cols_ok ? __ldg(p.sB + n0 + tid_in_set) : 0.0f;
        named_bar_sync(1 + set, 128);
        const uint32_t buf = acc_it % NB;
        if (ok) ok = mbar_wait(tfull_bar(buf), (acc_it / NB) & 1u, kSiteEpilogue, abort_flag);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) {
          tc_fence_after();
          const uint32_t taddr =
              tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + buf * kN + set * kSetCols;
          const float2 sa2 = make_float2(sa, sa);
#pragma unroll
          for (int h = 0; h < kSetCols / 64; ++h) {
            tmem_ld_64cols(taddr + h * 64, rbuf);
            tmem_ld_wait_regs(rbuf);
            if (h == kSetCols / 64 - 1) release(buf);
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const float2 pr = make_float2(__uint_as_float(rbuf[j]), __uint_as_float(rbuf[j + 1]));
              const float2 sb2 = *reinterpret_cast<const float2*>(slot + h * 64 + j);
              acc[(h * 64 + j) / 2] = __fmul2_rn(__fmul2_rn(pr, sa2), sb2);
            }
          }
        }
        ++acc_it;
      }

      // ---- store the tile's rows: this thread owns row m, columns n0 .. n0 + kSetCols
      const Tile tl = decode_tile<GROUPED, Cfg::kTileM, kN>(u.tile, p, mt_total, nt_total, sched);
      const int64_t m = tl.row0 + row_in_tile;
      const bool row_ok = m < tl.row_end;
      const int64_t n0 = tl.col0 + set * kSetCols;
      const bool cols_ok = n0 < p.N;
      if (ok && u.ws_index >= 0) {
        // split-K partial: the whole tile row (zeros outside C), summed later in fixed order
        float* wrow = p.ws + (static_cast<int64_t>(u.ws_index) * Cfg::kTileM + row_in_tile) * kN +
                      set * kSetCols;
#pragma unroll
        for (int j = 0; j < kSetCols / 2; j += 2)
          *reinterpret_cast<float4*>(wrow + 2 * j) =
              make_float4(acc[j].x, acc[j].y, acc[j + 1].x, acc[j + 1].y);
      } else if (ok && cols_ok) {          // warp-uniform: the row stores shuffle inside quads
        if (OUT_BF16) {
          // hv[j]: columns 8j .. 8j + 7 of the row segment, rounded to bf16
          uint4 hv[kSetCols / 8];
#pragma unroll
          for (int j = 0; j < kSetCols / 8; ++j) {
            __nv_bfloat162 h0 = __float22bfloat162_rn(acc[4 * j + 0]);
            __nv_bfloat162 h1 = __float22bfloat162_rn(acc[4 * j + 1]);
            __nv_bfloat162 h2 = __float22bfloat162_rn(acc[4 * j + 2]);
            __nv_bfloat162 h3 = __float22bfloat162_rn(acc[4 * j + 3]);
            hv[j].x = *reinterpret_cast<uint32_t*>(&h0);
            hv[j].y = *reinterpret_cast<uint32_t*>(&h1);
            hv[j].z = *reinterpret_cast<uint32_t*>(&h2);
            hv[j].w = *reinterpret_cast<uint32_t*>(&h3);
          }
          if constexpr (TSTORE) {
            // Rows of this warp all inside C's tile rows (always, dense: TMA drops rows past
            // M): through this warp's staging slice and two TMA stores.  A warp whose rows
            // cross an expert's end stores directly, masked by row.
            if (tl.row0 + row_in_tile - lane + 32 <= tl.row_end || !GROUPED) {
              const uint32_t stg = sbase + Cfg::stage + ew * Cfg::kStageWarpBytes;
              if (lane == 0) bulk_wait_read_all();   // the previous tile's stores have read it
              __syncwarp();
              // two boxes of 64 columns x 32 rows, 128-byte rows, 128-byte swizzle: chunk c
              // of row r at position c ^ (r % 8), so each quarter-warp covers all banks
#pragma unroll
              for (int j = 0; j < kSetCols / 8; ++j)
                st_shared_v4(stg + (j >> 3) * 4096 + lane * 128 + (((j & 7) ^ (lane & 7)) << 4), hv[j]);
              fence_proxy_async_shared();
              __syncwarp();
              if (lane == 0) {
                const int32_t y = static_cast<int32_t>(tl.row0 + row_in_tile - lane);
                tma_store_2d(&tmC, stg, static_cast<int32_t>(n0), y);
                tma_store_2d(&tmC, stg + 4096, static_cast<int32_t>(n0 + 64), y);
                bulk_commit_group();
              }
            } else {
              store_rows_by_quads(hv, reinterpret_cast<uint8_t*>(reinterpret_cast<__nv_bfloat16*>(p.C) + m * p.ldc + n0),
                                  row_ok);
            }
          } else if (p.C != nullptr) {
            store_rows_by_quads(hv, reinterpret_cast<uint8_t*>(reinterpret_cast<__nv_bfloat16*>(p.C) + m * p.ldc + n0),
                                row_ok);
          }
          if constexpr (QOUT) {
            // this thread's segment is exactly one 1x128 tile of the output row
            static_assert(kSetCols == 128 && !GROUPED, "one 1x128 output tile per epilogue thread");
            const float s_out = tile_scale(amax_vectors<kSetCols / 8>(hv), p.qpow2 != 0);
            uint2 o[kSetCols / 8];
            // f32x2 quotients, the rule voted once per warp (every lane's row has its own
            // tile scale)
            with_pair_quotient<true>(Quotient(s_out), [&](const auto& qd) {
#pragma unroll
              for (int j = 0; j < kSetCols / 8; ++j) {
                const float2 p0 = qd(hv[j].x), p1 = qd(hv[j].y), p2 = qd(hv[j].z), p3 = qd(hv[j].w);
                o[j].x = __byte_perm(cvt_e4m3x2(p0.x, p0.y), cvt_e4m3x2(p1.x, p1.y), 0x5410);
                o[j].y = __byte_perm(cvt_e4m3x2(p2.x, p2.y), cvt_e4m3x2(p3.x, p3.y), 0x5410);
              }
            });
            uint4 qv[kSetCols / 16];
#pragma unroll
            for (int j = 0; j < kSetCols / 16; ++j)
              qv[j] = make_uint4(o[2 * j].x, o[2 * j].y, o[2 * j + 1].x, o[2 * j + 1].y);
            store_rows_by_quads(qv, p.qc + m * p.ldq + n0, row_ok);
            if (row_ok) p.sc[(n0 / 128) * p.ld_sc + m] = s_out;
          }
        } else {
          uint4 fv[kSetCols / 4];
#pragma unroll
          for (int j = 0; j < kSetCols / 4; ++j)
            fv[j] = make_uint4(__float_as_uint(acc[2 * j].x), __float_as_uint(acc[2 * j].y),
                               __float_as_uint(acc[2 * j + 1].x), __float_as_uint(acc[2 * j + 1].y));
          store_rows_by_quads(fv, reinterpret_cast<uint8_t*>(reinterpret_cast<float*>(p.C) + m * p.ldc + n0),
                              row_ok);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  if (TSTORE && warp >= kEpiWarp0 && (threadIdx.x & 31) == 0) bulk_wait_all();   // stores done
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, kTmemCols);
  }
}

// Sum of the split-K partial tiles of the last wave, in chunk order, written to C.
// Grid: tail_tiles * TILE_M blocks (one tile row each) of TILE_N threads (one column each).
template <bool OUT_BF16, int TILE_M, int TILE_N>
__global__ void __launch_bounds__(TILE_N) splitk_reduce_kernel(const GemmArgs p, int mt_total) {
  const int r = blockIdx.x / TILE_M, row = blockIdx.x % TILE_M, col = threadIdx.x;
  const int t = p.tiles_full + r;
  const int nt_total = static_cast<int>((p.N + TILE_N - 1) / TILE_N);
  const int64_t m = static_cast<int64_t>(p.n_fastest ? t / nt_total : t % mt_total) * TILE_M + row;
  const int64_t n = static_cast<int64_t>(p.n_fastest ? t % nt_total : t / mt_total) * TILE_N + col;
  const float* w = p.ws + (static_cast<int64_t>(r) * p.tail_split * TILE_M + row) * TILE_N + col;
  float acc = 0.0f;
  for (int c = 0; c < p.tail_split; ++c) acc += w[static_cast<int64_t>(c) * TILE_M * TILE_N];
  if (m < p.M && n < p.N) {
    if (OUT_BF16)
      reinterpret_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(acc);
    else
      reinterpret_cast<float*>(p.C)[m * p.ldc + n] = acc;
  }
}

}  // namespace fp8q
