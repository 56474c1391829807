// Block-scaled FP8 GEMM for power-of-two scales, with the scaling done by the tensor core
// (sm_100a tcgen05.mma kind::mxf8f6f4.block_scale, UE8M0 scale factors in TMEM).
//
// C[m, n] = sum_g  P_g[m, n] * sA[m, g] * sB(n, g),   P_g = sum_{k in group g} qA[m,k] qB[n,k]
//
// why-be.co.kr wr_id=57820 para 4 and why-be.co.kr wr_id=72410 para 3 ask for tensor
// cores that take the per-group scaling factors themselves, so that the MMA applies the
// group scaling and the CUDA-core promotion step disappears.  B200's block-scaled MMA is
// that instruction for power-of-two scales: every 32-element K block of A and of B is
// multiplied by 2^(e - 127) of its UE8M0 scale byte inside the MMA, which is exact, and
// the products accumulate in FP32 in TMEM over the whole of K.  With the 1x128 and
// 128x128 scales of the quantizers the four 32-blocks of a 128-group share one scale.
//
// The result equals the promoted GEMM's up to the order of FP32 rounding (both are
// inside the same acceptance band against the oracle).  Scales that are not powers of
// two in [2^-127, 2^127] cannot be expressed in UE8M0: the kernel records
// (kSiteScaleFormat << 8) | FP8Q_ERR_SCALE in the device error word for them and goes on
// with scale 1.
//
// Tiles of 128 x 224 (224 divides 7168; two 224-column FP32 accumulators and the scale
// region fill the 512 TMEM columns), persistent CTAs, 12 warps.  GROUPED: the MoE form of
// fp8_gemm_grouped -- tiles come from a per-expert table built from m_offsets on the
// device (n fastest inside an expert), A rows past an expert's end are masked, B rows
// come from the stacked expert weights with that expert's block scales, and the ring has
// 4 stages to leave room for the table.
//   warp 0       TMA producer: A [128 x 128 B] and B [224 x 128 B] per K-group into a
//                5-stage ring (4 when grouped; 128-byte swizzle).
//   warp 1       TMEM owner and MMA issuer.  Per slot of four groups it copies the slot's
//                scale words from shared memory into TMEM (tcgen05.cp 32x128b.warpx4: a
//                32-row x 16-byte block into 4 columns of every 32-lane sub-partition),
//                then issues the groups' block-scaled MMAs (K = 32 each).  tcgen05.cp and
//                tcgen05.mma of one thread run in issue order, so a scale slot in TMEM is
//                rewritten only after the MMAs that read it.  Commits free smem stages,
//                scale slots and finished accumulators.
//   warp 2       scale producer.  For a slot (groups 4k .. 4k+3 of one tile) lane l packs
//                the UE8M0 bytes of A rows l, 32+l, 64+l, 96+l (byte j = group 4k+j) into
//                one 16-byte row of the A block, and those of B rows l + 32j (j < 7) into
//                two 16-byte rows of the B blocks, in a 3-slot shared-memory ring.  After
//                the copies the MMA reads, for A row m, lane m and column m/32, and for B
//                row n, column 4 + n/32 and lane n % 32 of its own sub-partition: the
//                layout of kind::mxf8f6f4 scale factors (checked on B200 with probes).
//   warp 3       idle.
//   warps 4-11   epilogue: warp w drains TMEM lanes 32*(w%4).. and 112 of the 224
//                columns of a finished accumulator, converts and stores C, and frees the
//                buffer for the tile after next.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "gemm.cuh"

namespace fp8q {

constexpr unsigned int kSiteScaleFormat = 8;
constexpr unsigned int kErrScale = 7;            // FP8Q_ERR_SCALE

template <bool GROUPED>
struct Ue8m0Cfg {
  static constexpr int kTileM = 128;
  static constexpr int kN = 224;                  // tile columns = MMA N
  static constexpr int kStages = GROUPED ? 4 : 5; // grouped: room for the tile table
  static constexpr int kAccCols = 2 * kN;         // two accumulator buffers
  static constexpr int kSfSmemSlots = 3;          // scale slots in shared memory, 4 groups each
  static constexpr int kSfTmemSlots = 4;          // scale slots in TMEM
  static constexpr int kSfSlotCols = 12;          // A: 4 columns, B: 8
  static constexpr int kSfCol0 = kAccCols;        // first scale column
  static constexpr int kSfWarp = 2, kEpiWarp0 = 4, kEpiWarps = 8;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kSetCols = kN / 2;         // columns per epilogue warp
  static constexpr uint32_t kABytes = 128 * kBK;
  static constexpr uint32_t kBBytes = kN * kBK;
  static constexpr uint32_t kStageTx = kABytes + kBBytes;
  static constexpr uint32_t kSfA = 32 * 16;       // one 32 x 16 B copy block
  static constexpr uint32_t kSfBytes = 3 * kSfA;  // A block, two B blocks
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + kStages * kABytes;
  static constexpr uint32_t sf = b + kStages * kBBytes;
  static constexpr uint32_t bars = sf + kSfSmemSlots * kSfBytes;
  // full[S], empty[S], tfull[2], tempty[2], sfull[SF], sempty[SF], drain
  static constexpr uint32_t n_bars = 2 * kStages + 4 + 2 * kSfSmemSlots + 1;
  static constexpr uint32_t misc = align_up(bars + 8 * n_bars, 16);   // tmem slot, abort flag
  static constexpr uint32_t sched = misc + 16;                        // grouped: int[E + 1]
  static constexpr uint32_t end = sched + (GROUPED ? 4 * (kMaxGroups + 1) : 0);
  static constexpr uint32_t smem_bytes = end + 1024;
  static_assert(kAccCols + kSfTmemSlots * kSfSlotCols <= static_cast<int>(kTmemCols), "TMEM budget");
  static_assert((kN + 31) / 32 <= 8, "B scales fit two copy blocks");
  static_assert(kN % 16 == 0 && kN <= 256, "MMA N for M = 128");
  static_assert(kSetCols % 16 == 0, "16-column epilogue loads");
  static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0 && sf % 1024 == 0, "alignment");
  static_assert(smem_bytes <= 232448, "fits the 227 KB opt-in shared memory");
};

// Shared-memory descriptor of a 32-row x 16-byte block (no swizzle: 8-row core matrices of
// 128 bytes, stacked) for tcgen05.cp; fields as in smem_desc_k_sw128, layout 0.
__device__ __forceinline__ uint64_t smem_desc_copy32x16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(128 >> 4) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

__device__ __forceinline__ void tmem_copy_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// UE8M0 byte of a power-of-two FP32 scale; sets `bad` for anything else.
__device__ __forceinline__ uint32_t ue8m0_of(float s, bool& bad) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t e = b >> 23;                     // sign and exponent
  if ((b & 0x7FFFFFu) == 0 && e >= 1 && e <= 254) return e;
  if (b == 0x00400000u) return 0;                 // 2^-127, the smallest UE8M0 value
  bad = true;
  return 127;
}

template <bool ROW_B, bool OUT_BF16, bool GROUPED>
__global__ void __launch_bounds__(Ue8m0Cfg<GROUPED>::kThreads, 1)
    gemm_fp8_ue8m0_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  using Cfg = Ue8m0Cfg<GROUPED>;
  static_assert(!(GROUPED && ROW_B), "grouped GEMMs take 128x128 weight-block scales");
  constexpr int S = Cfg::kStages;
  constexpr int SF = Cfg::kSfSmemSlots;
  constexpr int TS = Cfg::kSfTmemSlots;
  constexpr int kN = Cfg::kN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
  auto sfull_bar = [&](int r) { return bar0 + 8u * (2 * S + 4 + r); };
  auto sempty_bar = [&](int r) { return bar0 + 8u * (2 * S + 4 + SF + r); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 4 + 2 * SF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 32 * Cfg::kEpiWarps);   // every epilogue thread
    }
    for (int r = 0; r < SF; ++r) {
      mbar_init(sfull_bar(r), 1);                       // the scale producer
      mbar_init(sempty_bar(r), 1);                      // the MMA thread's commit
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
    tmem_alloc<1>(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish<1>();
  }
  const int nt_total = static_cast<int>((p.N + kN - 1) / kN);
  int* sched = reinterpret_cast<int*>(smem + Cfg::sched);
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
  const uint32_t tmem_base = *tmem_slot;
  if (GROUPED) num_tiles = sched[p.num_experts];
  // Tiles of this CTA: blockIdx.x, + gridDim.x, ...; dense: m-fastest so that the CTAs
  // of a wave share B tiles; grouped: expert by expert, n-fastest inside an expert.
  const int n_tiles = blockIdx.x < num_tiles ? (num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto tile_of = [&](int i) -> Tile {
    return decode_tile<GROUPED, Cfg::kTileM, kN>(blockIdx.x + i * gridDim.x, p, mt_total, nt_total, sched);
  };

  if (warp == 0) {
    // -------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int i = 0; ok && i < n_tiles; ++i) {
        const Tile tl = tile_of(i);
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % S;
          if (!mbar_wait(empty_bar(s), ((it / S) & 1u) ^ 1u, kSiteProducer, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), Cfg::kStageTx);
          tma_load_2d(sbase + Cfg::a + s * Cfg::kABytes, &tmA, full_bar(s), g * kBK,
                      static_cast<int32_t>(tl.row0));
          tma_load_2d(sbase + Cfg::b + s * Cfg::kBBytes, &tmB, full_bar(s), g * kBK,
                      static_cast<int32_t>(tl.brow0));
        }
      }
      // every issued load lands before the CTA can exit (bounded; loads end on their own)
      const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0;
      for (uint32_t j = first; j < it; ++j) mbar_wait(full_bar(j % S), (j / S) & 1u, kSiteDrain, nullptr);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, sc = 0;     // groups and scale slots issued so far
      bool ok = true;
      for (int i = 0; ok && i < n_tiles; ++i) {
        const uint32_t buf = i & 1;
        if (!mbar_wait(tempty_bar(buf), ((i >> 1) & 1u) ^ 1u, kSiteMmaEmpty, abort_flag)) break;
        const uint32_t d = tmem_base + buf * kN;
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % S;
          const int r = sc % SF;
          const uint32_t sfa = tmem_base + Cfg::kSfCol0 + (sc % TS) * Cfg::kSfSlotCols;
          if ((g & 3) == 0) {
            if (!mbar_wait(sfull_bar(r), (sc / SF) & 1u, kSiteScales, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t src = sbase + Cfg::sf + r * Cfg::kSfBytes;
            tmem_copy_32x128b_x4(sfa, smem_desc_copy32x16(src));
            tmem_copy_32x128b_x4(sfa + 4, smem_desc_copy32x16(src + Cfg::kSfA));
            tmem_copy_32x128b_x4(sfa + 8, smem_desc_copy32x16(src + 2 * Cfg::kSfA));
          }
          if (!mbar_wait(full_bar(s), (it / S) & 1u, kSiteMmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t byte = static_cast<uint32_t>(g & 3);
          const uint32_t idesc = idesc_e4m3_ue8m0(Cfg::kTileM, kN, byte);
          const uint32_t sfa_b = sfa | (byte << 30), sfb_b = (sfa + 4) | (byte << 30);
          const uint32_t a_addr = sbase + Cfg::a + s * Cfg::kABytes;
          const uint32_t b_addr = sbase + Cfg::b + s * Cfg::kBBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk)
            mma_f8_ue8m0(d, smem_desc_k_sw128(a_addr + 32 * kk), smem_desc_k_sw128(b_addr + 32 * kk),
                         idesc, (g > 0 || kk > 0) ? 1u : 0u, sfa_b, sfb_b);
          mma_commit<1>(empty_bar(s));
          if ((g & 3) == 3 || g == G - 1) {       // the slot's last group: free it when read
            mma_commit<1>(sempty_bar(r));
            ++sc;
          }
        }
        if (!ok) break;
        mma_commit<1>(tfull_bar(buf));
      }
      mma_commit<1>(drain_bar);
      mbar_wait(drain_bar, 0, kSiteDrain, nullptr);
    }
  } else if (warp == Cfg::kSfWarp) {
    // -------------------------------------------------------------- scale producer
    // Slots hold four groups of one tile (4k .. 4k + 3; a tile's last slot may be
    // partial); the CTA's slots run in order (tile i, slot k), and the raw scales of the
    // next slot are loaded before the current one is stored.
    //   A: lane l loads the 4 groups' scales of rows l + 32j, j < 4.
    //   B, 128x128 blocks: the tile's 224 rows touch at most 3 blocks; lane l < 12 loads
    //     block nb0 + l / 4, group 4k + l % 4, and shuffles build the packed words (every
    //     32-row chunk of the tile lies inside one block).
    //   B, 1x128 rows: lane l loads the 4 groups' scales of rows l + 32j, j < 7.
    constexpr int kRawB = ROW_B ? 28 : 1;
    struct Raw {
      float a[16];
      float b[kRawB];
    };
    bool bad = false;
    auto fetch = [&](int i, int k, Raw& raw) {
#pragma unroll
      for (int j = 0; j < 16; ++j) raw.a[j] = 1.0f;
#pragma unroll
      for (int j = 0; j < kRawB; ++j) raw.b[j] = 1.0f;
      if (i >= n_tiles) return;
      const Tile tl = tile_of(i);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t m = tl.row0 + 32 * j + lane;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int g = 4 * k + b;
          if (g < G && m < tl.row_end) raw.a[4 * j + b] = __ldg(p.sA + static_cast<int64_t>(g) * p.ld_sa + m);
        }
      }
      if (ROW_B) {
#pragma unroll
        for (int j = 0; j < 7; ++j) {
          const int64_t n = tl.col0 + 32 * j + lane;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int g = 4 * k + b;
            if (g < G && n < p.N) raw.b[4 * j + b] = __ldg(p.sB + static_cast<int64_t>(g) * p.ld_sb + n);
          }
        }
      } else {
        const int64_t nb = tl.col0 / 128 + (lane >> 2);
        const int g = 4 * k + (lane & 3);
        if (lane < 12 && g < G && nb * 128 < p.N)
          raw.b[0] = __ldg(p.sB + (static_cast<int64_t>(tl.expert) * (p.N / 128) + nb) * G + g);
      }
    };
    // Packs the slot into its shared-memory blocks once the MMA thread has copied the
    // ring slot's previous contents.  Returns false (warp-uniform) on abort or timeout.
    auto emit = [&](int i, int64_t sc, const Raw& raw) -> bool {
      const Tile tl = tile_of(i);
      uint32_t wa[4], wb[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wa[j] = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) wa[j] |= ue8m0_of(raw.a[4 * j + b], bad) << (8 * b);
      }
      if (ROW_B) {
#pragma unroll
        for (int j = 0; j < 7; ++j) {
          wb[j] = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) wb[j] |= ue8m0_of(raw.b[4 * j + b], bad) << (8 * b);
        }
      } else {
        const uint32_t byte = ue8m0_of(raw.b[0], bad);
        uint32_t w[3];
#pragma unroll
        for (int jb = 0; jb < 3; ++jb) {
          w[jb] = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) w[jb] |= __shfl_sync(0xFFFFFFFFu, byte, 4 * jb + b) << (8 * b);
        }
        const int nb0 = static_cast<int>(tl.col0 / 128);
#pragma unroll
        for (int j = 0; j < 7; ++j) {
          const int jb = static_cast<int>((tl.col0 + 32 * j) / 128) - nb0;
          wb[j] = jb == 0 ? w[0] : (jb == 1 ? w[1] : w[2]);
        }
      }
      wb[7] = 0;
      const int r = static_cast<int>(sc % SF);
      // warp-uniform outcome (the warp writes the slot together)
      const bool got = mbar_wait(sempty_bar(r), static_cast<uint32_t>(((sc / SF) & 1) ^ 1), kSiteScales,
                                 abort_flag);
      if (!__all_sync(0xFFFFFFFFu, got)) return false;
      uint8_t* blk = smem + Cfg::sf + r * Cfg::kSfBytes;
      *reinterpret_cast<uint4*>(blk + 16 * lane) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
      *reinterpret_cast<uint4*>(blk + Cfg::kSfA + 16 * lane) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
      *reinterpret_cast<uint4*>(blk + 2 * Cfg::kSfA + 16 * lane) = make_uint4(wb[4], wb[5], wb[6], wb[7]);
      fence_proxy_async_smem();                          // visible to tcgen05.cp
      __syncwarp();
      if (lane == 0) mbar_arrive(sfull_bar(r));
      return true;
    };
    const int G4 = (G + 3) / 4;
    Raw cur, nxt;
    fetch(0, 0, cur);
    int64_t sc = 0;
    for (int i = 0, k = 0; i < n_tiles; ++sc) {
      const int i2 = k + 1 < G4 ? i : i + 1, k2 = k + 1 < G4 ? k + 1 : 0;
      fetch(i2, k2, nxt);
      if (!emit(i, sc, cur)) break;
      cur = nxt;
      i = i2;
      k = k2;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_error((kSiteScaleFormat << 8) | kErrScale);
  } else if (warp >= Cfg::kEpiWarp0) {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - Cfg::kEpiWarp0;
    const int q = warp & 3;
    const int set = ew >> 2;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const Tile tl = tile_of(i);
      const uint32_t buf = i & 1;
      // warp-uniform outcome: the TMEM loads below are whole-warp instructions
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(tfull_bar(buf), (i >> 1) & 1u, kSiteEpilogue, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int64_t m = tl.row0 + 32 * q + lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + buf * kN +
                             set * Cfg::kSetCols;
      const int64_t n_set = tl.col0 + set * Cfg::kSetCols;
      const bool row_ok = m < tl.row_end;
      uint8_t* crow = reinterpret_cast<uint8_t*>(p.C) + (m * p.ldc + n_set) * (OUT_BF16 ? 2 : 4);
      // Stores go through store_rows_by_quads (64 contiguous bytes of 8 rows per warp
      // instruction): bf16 in 32-column steps, fp32 in 16-column steps; a bf16 step that
      // would cross N, and the set's last 16 bf16 columns, store 32 bytes per row directly.
      // Every condition on columns is warp-uniform (n_set is the warp's).
#pragma unroll 1
      for (int c = 0; c < Cfg::kSetCols; c += (OUT_BF16 && c + 32 <= Cfg::kSetCols) ? 32 : 16) {
        const int64_t n0 = n_set + c;
        if (OUT_BF16 && c + 32 <= Cfg::kSetCols && n0 + 32 <= p.N) {
          uint32_t r[32];
          tmem_ld_32cols(taddr + c, r);
          tmem_ld_wait();
          uint4 hv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t h[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 2 * t]),
                                                       __uint_as_float(r[8 * j + 2 * t + 1]));
              h[t] = *reinterpret_cast<uint32_t*>(&v);
            }
            hv[j] = make_uint4(h[0], h[1], h[2], h[3]);
          }
          store_rows_by_quads(hv, crow + 2 * c, row_ok);
          continue;
        }
        uint32_t r[16];
        tmem_ld_16cols(taddr + c, r);
        tmem_ld_wait();
        if (n0 >= p.N) continue;                         // N % 16 == 0: whole 16-column chunks
        if (OUT_BF16) {
          if (row_ok) {
            uint32_t h[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
              h[j] = *reinterpret_cast<uint32_t*>(&v);
            }
            uint4* dst = reinterpret_cast<uint4*>(crow + 2 * c);
            dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
            dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
          }
        } else {
          uint4 fv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) fv[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          store_rows_by_quads(fv, crow + 4 * c, row_ok);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(buf));                      // accumulator free for tile i + 2
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, kTmemCols);
  }
}

}  // namespace fp8q
