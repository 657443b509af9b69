// Persistent, warp-specialised tcgen05 GEMM for sm_100a with fused epilogues.
//
//   D[M, N] = A[M, K] * B[N, K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// Roles (one CTA per SM, 64 + 32*EPI_WARPS threads):
//   warp 0 lane 0 : TMA producer, STAGES-deep shared-memory ring of (A, B) k-blocks;
//   warp 1        : TMEM allocator; lane 0 issues tcgen05.mma (M=128, N=BN, K=16);
//   warps 2..     : epilogue; two TMEM accumulators so the epilogue of one tile
//                   overlaps the main loop of the next.
// Operands may be K-major (rows of K contiguous) or MN-major (rows of M/N
// contiguous); both are staged by TMA with the 128-byte swizzle and described to
// the tensor core directly, so no transpose is ever materialised.
//
// Every wait is bounded: a wait that runs out raises DEV_TIMEOUT in the status
// word, every role leaves its loop, in-flight copies and MMAs are drained (with
// bounded waits too) and TMEM is freed before the kernel returns.
#pragma once
#include "sm100.cuh"



namespace flce {

enum class Major : int { K = 0, MN = 1 };

template <int BN_, int STAGES_, Major AMAJ_, Major BMAJ_, int EPI_WARPS_>
struct GemmCfg {
  static constexpr bool PAIR = false;
  static constexpr int BM = 128;
  static constexpr int BM_CTA = 128;
  static constexpr int BN = BN_;
  static constexpr int BN_CTA = BN_;
  static constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row
  static constexpr int STAGES = STAGES_;
  static constexpr Major AMAJ = AMAJ_;
  static constexpr Major BMAJ = BMAJ_;
  static constexpr int EPI_WARPS = EPI_WARPS_;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr int COL_SPLIT = EPI_WARPS / 4;       // warps sharing one TMEM lane quarter
  static constexpr int COLS_PER_WARP = BN / COL_SPLIT;  // columns each epilogue thread owns
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(EPI_WARPS % 4 == 0, "epilogue warps must cover the four TMEM lane quarters");
  static_assert(COLS_PER_WARP % 32 == 0, "epilogue works in 32-column TMEM loads");
  static_assert(BN % 64 == 0 || BMAJ_ == Major::K, "MN-major tiles are whole 64-wide blocks");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0, N <= 256");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert((2 * STAGES + 5) * 8 + 4 <= BAR_BYTES, "barrier area too small");
  static_assert(SMEM_BYTES <= 232448, "more than 227 KB of shared memory");
};

struct GemmArgs {
  int M, N, K;          // problem extents (M rows of A, N rows of B, K shared)
  int m_fastest;        // tile order: 1 = consecutive tiles walk M first
  uint32_t* status;     // device status word (DEV_TIMEOUT is or-ed in)
  uint64_t limit_ns;    // bound on every wait
};

// ----------------------------------------------------------------------------------------------
// Tile loaders: K-major -> one TMA box {64 (K), rows}; MN-major -> rows/64 boxes {64 (MN), 64 (K)}
template <Major MAJ, int ROWS>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             int row0, int k0) {
  if constexpr (MAJ == Major::K) {
    tma_load_2d(dst, map, bar, k0, row0);
  } else {
#pragma unroll
    for (int q = 0; q < ROWS / 64; ++q) tma_load_2d(dst + q * 8192, map, bar, row0 + 64 * q, k0);
  }
}

// Descriptor of the k-th 16-deep slice of a staged operand tile.
template <Major MAJ>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  if constexpr (MAJ == Major::K) {
    return smem_desc_sw128(base + 32u * k, 16u, 1024u);
  } else {
    return smem_desc_sw128(base + 2048u * k, 8192u, 1024u);
  }
}

template <class C, class Epi>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs args, const __grid_constant__ typename Epi::Params ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m_tiles = (args.M + C::BM - 1) / C::BM;
  const int n_tiles = (args.N + C::BN - 1) / C::BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (args.K + C::BK - 1) / C::BK;
  auto tile_coords = [&](int t, int& mb, int& nb) {
    if (args.m_fastest) {
      mb = t % m_tiles;
      nb = t / m_tiles;
    } else {
      nb = t % n_tiles;
      mb = t / n_tiles;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long long arms = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, mb, nb);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, args.limit_ns)) {
            *abort_flag = 1;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          load_operand<C::AMAJ, C::BM>(sA, &tmA, &full[stage], mb * C::BM, kb * C::BK);
          load_operand<C::BMAJ, C::BN>(sB, &tmB, &full[stage], nb * C::BN, kb * C::BK);
          ++arms;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      const long long first = arms > C::STAGES ? arms - C::STAGES : 0;
      for (long long a = first; a < arms; ++a) {
        mbar_wait_bounded(&full[a % C::STAGES], static_cast<uint32_t>((a / C::STAGES) & 1),
                          args.status, args.limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc =
          instr_desc_bf16_f32(C::BM, C::BN, C::AMAJ == Major::MN, C::BMAJ == Major::MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, args.status, args.limit_ns)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, args.limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            mma_bf16_ss(d_tmem, operand_desc<C::AMAJ>(a_base, k), operand_desc<C::BMAJ>(b_base, k),
                        idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (issued) {  // drain: all MMAs complete before TMEM is released
        mma_commit(drain);
        mbar_wait_bounded(drain, 0, args.status, args.limit_ns);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int slab = ew >> 2;                  // which column slab of the tile
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, mb, nb);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, args.status, args.limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * C::BN + slab * C::COLS_PER_WARP);
      Epi::template apply<C::COLS_PER_WARP>(ep, mb * C::BM + row_in_tile,
                                            nb * C::BN + slab * C::COLS_PER_WARP, taddr,
                                            nb * C::COL_SPLIT + slab);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ==============================================================================================
// The same GEMM on SM pairs (cta_group::2): a 256 x BN tile per pair of CTAs in a 2-CTA cluster.
// Each CTA stages its own 128 rows of A and its own BN/2 rows of B (no multicast); both CTAs'
// copies complete on the leader's (rank 0) stage barrier; the leader issues
// tcgen05.mma.cta_group::2 (M = 256), which reads each half from its own CTA's shared memory and
// leaves rows 0-127 of the accumulator in the leader's TMEM and rows 128-255 in the peer's.
// Commits arrive on both CTAs' barriers; each CTA's epilogue drains its own TMEM half and
// releases the accumulator on the leader.  Per SM and k-block this stages 16 KB of A and
// BN/2 x 128 B of B, against 16 KB + BN x 128 B on a single SM.
template <int BN_, int STAGES_, Major AMAJ_, Major BMAJ_, int EPI_WARPS_>
struct GemmPairCfg {
  static constexpr bool PAIR = true;
  static constexpr int BM = 256;         // rows per pair tile
  static constexpr int BM_CTA = 128;     // rows per CTA (one TMEM lane each)
  static constexpr int BN = BN_;         // columns per pair tile
  static constexpr int BN_CTA = BN_ / 2; // B rows staged by each CTA
  static constexpr int BK = 64;
  static constexpr int STAGES = STAGES_;
  static constexpr Major AMAJ = AMAJ_;
  static constexpr Major BMAJ = BMAJ_;
  static constexpr int EPI_WARPS = EPI_WARPS_;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int A_BYTES = BM_CTA * BK * 2;
  static constexpr int B_BYTES = BN_CTA * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  static constexpr int COL_SPLIT = EPI_WARPS / 4;
  static constexpr int COLS_PER_WARP = BN / COL_SPLIT;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(EPI_WARPS % 4 == 0, "epilogue warps must cover the four TMEM lane quarters");
  static_assert(COLS_PER_WARP % 32 == 0, "epilogue works in 32-column TMEM loads");
  static_assert(BN_CTA % 64 == 0 || BMAJ_ == Major::K, "MN-major tiles are whole 64-wide blocks");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "cta_group::2 M=256 needs N % 16 == 0");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area too small");
  static_assert(SMEM_BYTES <= 232448, "more than 227 KB of shared memory");
};

template <class C, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmArgs args, const __grid_constant__ typename Epi::Params ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                 // used on the leader only
  uint64_t* empty = bars + C::STAGES;    // both CTAs
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;          // used on the leader only
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * C::EPI_WARPS);   // one arrival per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t leader_full = mapa_shared(smem_u32(full), 0);
  const uint32_t leader_tempty = mapa_shared(smem_u32(tempty), 0);

  const int m_tiles = (args.M + C::BM - 1) / C::BM;
  const int n_tiles = (args.N + C::BN - 1) / C::BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (args.K + C::BK - 1) / C::BK;
  auto tile_coords = [&](int t, int& mb, int& nb) {
    if (args.m_fastest) {
      mb = t % m_tiles;
      nb = t / m_tiles;
    } else {
      nb = t % n_tiles;
      mb = t / n_tiles;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      long long arms = 0;
      for (int t = pair; t < num_tiles && !*abort_flag; t += npairs) {
        int mb, nb;
        tile_coords(t, mb, nb);
        const int a_row = mb * C::BM + static_cast<int>(rank) * C::BM_CTA;
        const int b_row = nb * C::BN + static_cast<int>(rank) * C::BN_CTA;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, args.limit_ns)) {
            *abort_flag = 1;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          const uint32_t bar = leader_full + 8u * stage;
          if constexpr (C::AMAJ == Major::K) {
            tma_load_2d_pair(sA, &tmA, bar, kb * C::BK, a_row);
          } else {
#pragma unroll
            for (int q = 0; q < C::BM_CTA / 64; ++q)
              tma_load_2d_pair(sA + q * 8192, &tmA, bar, a_row + 64 * q, kb * C::BK);
          }
          if constexpr (C::BMAJ == Major::K) {
            tma_load_2d_pair(sB, &tmB, bar, kb * C::BK, b_row);
          } else {
#pragma unroll
            for (int q = 0; q < C::BN_CTA / 64; ++q)
              tma_load_2d_pair(sB + q * 8192, &tmB, bar, b_row + 64 * q, kb * C::BK);
          }
          ++arms;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {
        // Drain: the last phases of every stage include both CTAs' copies.
        const long long first = arms > C::STAGES ? arms - C::STAGES : 0;
        for (long long a = first; a < arms; ++a)
          mbar_wait_bounded(&full[a % C::STAGES], static_cast<uint32_t>((a / C::STAGES) & 1),
                            args.status, args.limit_ns);
      } else if (*abort_flag) {
        // After an abort the leader may not wait for this CTA's last copies: give them time
        // to land before the CTA can exit (copies take microseconds).
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader only)
      constexpr uint32_t idesc =
          instr_desc_bf16_f32(C::BM, C::BN, C::AMAJ == Major::MN, C::BMAJ == Major::MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int t = pair; t < num_tiles && !*abort_flag; t += npairs) {
        if (!mbar_wait_bounded_cluster(&tempty[acc], acc_phase ^ 1u, args.status, args.limit_ns)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, args.status, args.limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            mma_bf16_ss_pair(d_tmem, operand_desc<C::AMAJ>(a_base, k),
                             operand_desc<C::BMAJ>(b_base, k), idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit_pair_both(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_both(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (issued) {
        mma_commit_pair_both(drain);
        mbar_wait_bounded(drain, 0, args.status, args.limit_ns);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int slab = ew >> 2;
    const int row_in_cta = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < num_tiles && !*abort_flag; t += npairs) {
      int mb, nb;
      tile_coords(t, mb, nb);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, args.status, args.limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * C::BN + slab * C::COLS_PER_WARP);
      Epi::template apply<C::COLS_PER_WARP>(
          ep, mb * C::BM + static_cast<int>(rank) * C::BM_CTA + row_in_cta,
          nb * C::BN + slab * C::COLS_PER_WARP, taddr, nb * C::COL_SPLIT + slab);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty + 8u * acc);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // both CTAs done with TMEM, shared memory and barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ==============================================================================================
// Epilogue 1: softcapped logits -> softmax statistics, target capture, and (optionally) the
// unnormalised gradient operand A.
//
// With a softcap, s = cap*tanh(z/cap) < cap, so exp(s - cap) lies in (e^{-2 cap}, 1]: for
// moderate caps (fixed_ref) the row's softmax can be accumulated against the fixed reference
// `cap` with no running maximum and no overflow.  Then
//     softmax(s)_ij = exp(s_ij - cap) / S_i,            S_i = sum_{j < Vreal} exp(s_ij - cap),
//     lse_i = cap + log S_i,
//     dz_ij = g/Nv * (softmax_ij - [j = t_i]) * (1 - tanh^2(z_ij/cap))
//           = r_i * A'_ij,  r_i = g/(Nv S_i),
//     A'_ij = exp(s_ij - cap) (1 - tanh^2(z_ij/cap))  except  A'_{i,t_i} = (1 - tanh^2)(e_{i,t_i} - S_i).
// So the epilogue can write A (the unpatched A') before S_i is known; a per-row kernel later
// patches the one target element and folds r_i into the dX epilogue and into the X operand of
// the dW contraction.  Without a fixed reference (no softcap, or a very large one) the
// statistics pass keeps a per-slab (max, sum-exp) pair instead, and the operand pass uses the
// row's lse as the reference (then S_i = 1).
//
// tanh is evaluated from u = exp(-2|z|/cap) in (0, 1]:
//     tanh(|z|/cap) = (1-u)/(1+u),   1 - tanh^2 = 4u/(1+u)^2,
//     s - cap = -2 cap u/(1+u) (z >= 0)  or  -2 cap/(1+u) (z < 0),
// which keeps 1 - tanh^2 and s - cap free of cancellation at saturation.
struct Softcapped {
  float s, der, e;
};

// s = cap tanh(z/cap), der = 1 - tanh^2(z/cap) and e = exp(s - cap), from u = exp(-2|z|/cap):
// three special-function operations (exp2, reciprocal, exp2) and a handful of FMAs per logit.
// (Moving the reciprocal or the second exp2 to FMA-pipe Newton / polynomial forms measured
// slower on B200: the extra instructions cost more than the special-function unit saves.)
__device__ __forceinline__ Softcapped softcap_fixed_ref(float z, float k_u, float m2c_log2e,
                                                        float cap) {
  const float u = ex2_approx(-fabsf(z) * k_u);        // exp(-2|z|/cap) in (0, 1]
  const float q = rcp_approx(1.0f + u);               // 1/(1+u)
  const float uq = u * q;
  Softcapped r;
  r.der = 4.0f * uq * q;                               // 4u/(1+u)^2
  // s - cap = -2 cap u/(1+u) for z >= 0, -2 cap/(1+u) for z < 0
  r.e = ex2_approx((z >= 0.f ? uq : q) * m2c_log2e);
  r.s = copysignf(cap * (q - uq), z);                  // cap (1-u)/(1+u)
  return r;
}

enum LogitsMode : int { LOGITS_STATS = 0, LOGITS_FUSED = 1, LOGITS_RECOMPUTE = 2 };

struct LogitsParams {
  int rows;                  // rows of this pass; rows >= rows are padding of the last tile
  int Vreal, Vpad;
  int mode;                  // LogitsMode
  int fixed_ref;             // 1: exp reference is cap (requires cap > 0); 0: online / lse
  float cap;                 // > 0: softcap value; <= 0: no softcap
  float k_u;                 // 2/cap * log2(e)
  float m2c_log2e;           // -2 cap log2(e)
  const int* tgt;            // [rows] target id, -1 when the row is not in the loss
  const float* ref;          // [rows] exp reference (lse) when !fixed_ref and mode == RECOMPUTE
  float* partial;            // [rows][n_slabs] sum-exp (pairs (max, sum-exp) when !fixed_ref)
  int n_slabs;
  float* s_t;                // [rows] softcapped target logit
  float* der_t;              // [rows] 1 - tanh^2 at the target
  float* e_t;                // [rows] exp(s_t - reference)
  __nv_bfloat16* A;          // [rows][Vpad] gradient operand (modes FUSED / RECOMPUTE)
};

struct LogitsEpi {
  using Params = LogitsParams;
  static constexpr float LOG2E = 1.4426950408889634f;

  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int slab_index) {
    const bool row_ok = row < p.rows;
    const int t = row_ok ? __ldg(p.tgt + row) : -1;
    const bool capped = p.cap > 0.f;
    const bool write_a = p.mode != LOGITS_STATS;
    const bool online = !p.fixed_ref && p.mode == LOGITS_STATS;
    const float ref = p.fixed_ref ? p.cap
                                  : ((p.mode == LOGITS_RECOMPUTE && row_ok) ? __ldg(p.ref + row) : 0.f);
    float sum = 0.f;
    float run_max = -INFINITY;
    float tv_s = 0.f, tv_der = 0.f, tv_e = 0.f;
    bool has_t = false;
    __nv_bfloat16* arow = write_a && row_ok ? p.A + static_cast<size_t>(row) * p.Vpad : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      const int cbase = col0 + c * 32;
      if (p.fixed_ref) {
        // softcap with the fixed reference: e = exp(s - cap), A = e (1 - tanh^2)
        if (static_cast<unsigned>(t - cbase) < 32u) {   // this row's target is in this chunk
          float zt = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k == t - cbase) zt = v[k];
          const Softcapped sc = softcap_fixed_ref(zt, p.k_u, p.m2c_log2e, p.cap);
          tv_s = sc.s;
          tv_der = sc.der;
          tv_e = sc.e;
          has_t = true;
        }
        if (cbase + 32 <= p.Vreal) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const Softcapped sc = softcap_fixed_ref(v[k], p.k_u, p.m2c_log2e, p.cap);
            sum += sc.e;
            v[k] = sc.e * sc.der;
          }
        } else {                                            // last vocabulary tile: padded columns
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const Softcapped sc = softcap_fixed_ref(v[k], p.k_u, p.m2c_log2e, p.cap);
            const float e = cbase + k < p.Vreal ? sc.e : 0.f;
            sum += e;
            v[k] = e * sc.der;
          }
        }
      } else {
        float der[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          if (capped) {
            const float z = v[k];
            const float u = ex2_approx(-fabsf(z) * p.k_u);
            const float q = rcp_approx(1.0f + u);
            der[k] = 4.0f * u * q * q;
            v[k] = copysignf(p.cap * (1.0f - u) * q, z);
          } else {
            der[k] = 1.0f;
          }
        }
        if (online) {
          float cmax = -INFINITY;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (cbase + k < p.Vreal) cmax = fmaxf(cmax, v[k]);
          if (cmax > run_max) {
            sum = (run_max == -INFINITY) ? 0.f : sum * ex2_approx((run_max - cmax) * LOG2E);
            run_max = cmax;
          }
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int col = cbase + k;
            if (col < p.Vreal) sum += ex2_approx((v[k] - run_max) * LOG2E);
            if (col == t) {
              tv_s = v[k];
              tv_der = der[k];
              has_t = true;
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int col = cbase + k;
            float e = ex2_approx((v[k] - ref) * LOG2E);
            if (col >= p.Vreal) e = 0.f;
            sum += e;
            if (col == t) {
              tv_s = v[k];
              tv_der = der[k];
              tv_e = e;
              has_t = true;
            }
            v[k] = e * der[k];
          }
        }
      }
      if (arow != nullptr) {
        uint32_t packed[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) packed[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = cbase + 8 * g;
          if (col < p.Vpad) {
            *reinterpret_cast<uint4*>(arow + col) =
                make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
          }
        }
      }
    }
    if (!row_ok) return;
    if (p.mode != LOGITS_RECOMPUTE) {
      if (!online) {
        p.partial[static_cast<size_t>(row) * p.n_slabs + slab_index] = sum;
      } else {
        float* pp = p.partial + (static_cast<size_t>(row) * p.n_slabs + slab_index) * 2;
        pp[0] = run_max;
        pp[1] = sum;
      }
    }
    if (has_t) {
      p.s_t[row] = tv_s;
      p.der_t[row] = tv_der;
      p.e_t[row] = tv_e;
    }
  }
};

// ==============================================================================================
// Epilogue 2: dX rows = r_i * (A' W)_i, stored as bf16.
struct DxParams {
  int rows, d;
  const float* r;            // [rows] row scale g/(Nv S_i); 0 for rows not in the loss
  __nv_bfloat16* dX;         // [rows][d]
};

struct DxEpi {
  using Params = DxParams;
  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int) {
    const bool row_ok = row < p.rows;
    const float sc = row_ok ? __ldg(p.r + row) : 0.f;
    __nv_bfloat16* out = row_ok ? p.dX + static_cast<size_t>(row) * p.d : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (out == nullptr) continue;
      const int cbase = col0 + c * 32;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = cbase + 8 * g;
        if (col < p.d) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * g + 0] * sc, v[8 * g + 1] * sc);
          w.y = pack_bf16x2(v[8 * g + 2] * sc, v[8 * g + 3] * sc);
          w.z = pack_bf16x2(v[8 * g + 4] * sc, v[8 * g + 5] * sc);
          w.w = pack_bf16x2(v[8 * g + 6] * sc, v[8 * g + 7] * sc);
          *reinterpret_cast<uint4*>(out + col) = w;
        }
      }
    }
  }
};

// ==============================================================================================
// Epilogue 3: dW rows (vocabulary rows) = (A'^T (r . X))_j, written or accumulated in fp32.
struct DwParams {
  int Vpad, d;
  int accumulate;            // 1: dW += tile, 0: dW = tile
  float* dW;                 // [Vpad][d]
};

struct DwEpi {
  using Params = DwParams;
  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int) {
    const bool row_ok = row < p.Vpad;
    float* out = row_ok ? p.dW + static_cast<size_t>(row) * p.d : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (out == nullptr) continue;
      const int cbase = col0 + c * 32;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int col = cbase + 4 * g;
        if (col < p.d) {
          float4* dst = reinterpret_cast<float4*>(out + col);
          float4 w = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
          if (p.accumulate) {
            const float4 o = *dst;
            w.x += o.x;
            w.y += o.y;
            w.z += o.z;
            w.w += o.w;
          }
          *dst = w;
        }
      }
    }
  }
};

}  // namespace flce
