// Persistent, warp-specialised tcgen05 GEMM for sm_100a with fused epilogues.
//
//   D[M, N] = A[M, K] * B[N, K]^T, bf16 (or e4m3) operands, fp32 accumulation in TMEM.
//
// Runs on pairs of SMs (2-CTA clusters, tcgen05 cta_group::2).  Roles in each CTA
// (64 + 32*EPI_WARPS threads, one CTA per SM):
//   warp 0 lane 0 : TMA producer, STAGES-deep shared-memory ring of (A, B) k-blocks;
//   warp 1        : TMEM allocator; lane 0 of the leader CTA issues tcgen05.mma
//                   (M=256 across the pair, N=BN, K = 32 bytes of each operand row);
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

// 32 accumulator columns of this thread's TMEM lane, or zeros (warp-uniform `zero`).
__device__ __forceinline__ void tmem_ld32_or_zero(uint32_t taddr, float (&v)[32], bool zero) {
  if (zero) {
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = 0.f;
  } else {
    tmem_ld32(taddr, v);
  }
}

// ----------------------------------------------------------------------------------------------
// Staged operand tiles, all in 128-byte swizzled rows (EB = bytes per element: 2 bf16, 1 fp8).
//   K-major : one TMA box {128 bytes of K, rows}.
//   MN-major: rows / (128/EB) boxes {128/EB (MN), 128/EB (K)}: each box is one 128-byte-wide
//             block of M/N elements over the k-block's K rows, boxes laid out one after the
//             other (the descriptor's leading byte offset is the box size).
// The copy completes on the pair leader's barrier (shared::cluster address).
template <Major MAJ, int ROWS, int EB = 2>
__device__ __forceinline__ void load_operand_pair(uint8_t* dst, const CUtensorMap* map,
                                                  uint32_t leader_bar, int row0, int k0,
                                                  uint64_t policy) {
  if constexpr (MAJ == Major::K) {
    tma_load_2d_pair_hint(dst, map, leader_bar, k0, row0, policy);
  } else {
    constexpr int MNB = 128 / EB;               // elements of one 128-byte block
    constexpr int BOX = 128 * (128 / EB);       // bytes of one box (k-block rows x 128 bytes)
    static_assert(ROWS % MNB == 0, "MN-major tiles are whole 128-byte blocks");
#pragma unroll
    for (int q = 0; q < ROWS / MNB; ++q)
      tma_load_2d_pair_hint(dst + q * BOX, map, leader_bar, row0 + MNB * q, k0, policy);
  }
}

// Descriptor increment between consecutive MMA slices (start address field, 16-byte units);
// one slice is 32 bytes of K: 32 bytes along a K-major row, or 32/EB K rows of 128 bytes of an
// MN-major tile.  Staged tiles sit below 256 KB, so adding to the 14-bit field never carries
// out of it.
template <Major MAJ, int EB = 2>
__device__ __forceinline__ constexpr uint64_t desc_step() {
  return MAJ == Major::K ? 2u : static_cast<uint64_t>(256 / EB);
}

// Descriptor of the k-th MMA slice of a staged operand tile.
template <Major MAJ, int EB = 2>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  if constexpr (MAJ == Major::K) {
    return smem_desc_sw128(base + 32u * k, 16u, 1024u);
  } else {
    return smem_desc_sw128(base + (4096u / EB) * k, 128u * (128u / EB), 1024u);
  }
}

// One tcgen05.mma on an SM pair: kind::f16 (bf16) or kind::f8f6f4 (8-bit formats).
template <int EB>
__device__ __forceinline__ void mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
  if constexpr (EB == 2)
    mma_bf16_ss_pair(d, a, b, idesc, acc);
  else
    mma_e4m3_ss_pair(d, a, b, idesc, acc);
}

// ==============================================================================================
// The GEMM on SM pairs (cta_group::2): a 256 x BN tile per pair of CTAs in a 2-CTA cluster.
// Each CTA stages its own 128 rows of A and its own BN/2 rows of B (no multicast); both CTAs'
// copies complete on the leader's (rank 0) stage barrier; the leader issues
// tcgen05.mma.cta_group::2 (M = 256), which reads each half from its own CTA's shared memory and
// leaves rows 0-127 of the accumulator in the leader's TMEM and rows 128-255 in the peer's.
// Commits arrive on both CTAs' barriers; each CTA's epilogue drains its own TMEM half and
// releases the accumulator on the leader.  Per SM and k-block this stages 16 KB of A and
// BN/2 x 128 B of B, against 16 KB + BN x 128 B on a single SM.
//
// One launch may carry two problems (e.g. dX = A'W and dW = A'^T Xs, whose tiles differ in
// length by 12x): each pair first takes its round-robin share of problem 0's tiles, then its
// share of problem 1's tiles, handed out so that every pair ends with about the same number of
// k-blocks while concurrently running tiles stay neighbours (pair_schedule).  A launch with one
// problem is the plain round-robin persistent schedule.
// KSUB: k-blocks (128-byte swizzle rows of K) per ring slot.  Two per slot halve the barrier
// waits, fences and commits of the single MMA-issuing thread per MMA.
template <int BN_, int STAGES_, int EPI_WARPS_, int ELEM_BYTES_ = 2, int KSUB_ = 1>
struct PairCfg {
  static constexpr bool PAIR = true;
  static constexpr int ELEM_BYTES = ELEM_BYTES_;  // 2: bf16 (kind::f16), 1: e4m3 (kind::f8f6f4)
  static constexpr int BM = 256;         // rows per pair tile
  static constexpr int BM_CTA = 128;     // rows per CTA (one TMEM lane each)
  static constexpr int BN = BN_;         // columns per pair tile
  static constexpr int BN_CTA = BN_ / 2; // B rows staged by each CTA
  static constexpr int BK = 128 / ELEM_BYTES;  // one 128-byte swizzle row of K per k-block
  static constexpr int KSUB = KSUB_;           // k-blocks per ring slot
  static constexpr int KSLOT = BK * KSUB;      // K per ring slot
  static constexpr int MMA_K = 32 / ELEM_BYTES; // K per tcgen05.mma: 32 bytes of each row
  static constexpr int STAGES = STAGES_;
  static constexpr int EPI_WARPS = EPI_WARPS_;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int A_SUB = BM_CTA * 128;   // one k-block of A (this CTA's rows)
  static constexpr int B_SUB = BN_CTA * 128;
  static constexpr int A_BYTES = A_SUB * KSUB;
  static constexpr int B_BYTES = B_SUB * KSUB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  static constexpr int COL_SPLIT = EPI_WARPS / 4;
  static constexpr int COLS_PER_WARP = BN / COL_SPLIT;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static_assert(EPI_WARPS % 4 == 0, "epilogue warps must cover the four TMEM lane quarters");
  static_assert(COLS_PER_WARP % 32 == 0, "epilogue works in 32-column TMEM loads");
  static_assert(BN_CTA % 32 == 0, "B halves are whole 32-row groups (64-wide when MN-major)");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "cta_group::2 M=256 needs N % 16 == 0");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert((2 * STAGES + 5) * 8 + 32 <= BAR_BYTES, "barrier area too small");
  static_assert(SMEM_BYTES <= 232448, "more than 227 KB of shared memory");
  static_assert(KSUB >= 1 && KSUB <= 4, "1 to 4 k-blocks per slot");
};

template <int V>
struct IntC {
  static constexpr int value = V;
};

struct PairProblem {
  int M, N, K;          // extents; M == 0 marks an absent second problem
  int m_fastest;        // tile order: 1 = consecutive tiles walk M first
  int wide;             // problem 0 only: 1 = wide tiles (see below)
  int l2_a, l2_b;       // L2 priority of the A / B operand reads (l2_policy: 0, 1 first, 2 last)
  int dyn;              // DYN_M / DYN_K: that extent is min(extent, *PairArgs::dyn)
  int serpentine;       // 1: tiles of every other wave walk K backwards, so the operand rows
                        //    the previous wave read last (still in L2) are read first.  The
                        //    wave is (m_off + m block) * N tiles + n block over the pair count:
                        //    a property of the tile, so a tile's arithmetic does not depend on
                        //    the launch it runs in (vocabulary buckets give identical results)
  int m_off;            // M tiles before this problem's first (a launch over part of M)
  int n_groups;         // > 1 (tiles walking N fastest): the N blocks are taken in n_groups
                        //    consecutive groups, all M blocks of one group before the next, so
                        //    the tiles running at one time touch 1/n_groups of the B operand
};

enum : int { DYN_M = 1, DYN_K = 2 };

struct PairArgs {
  PairProblem prob[2];
  uint32_t* status;     // device status word (DEV_TIMEOUT is or-ed in)
  uint64_t limit_ns;    // bound on every wait
  const int* dyn;       // device count bounding the extents flagged in PairProblem::dyn
};

// Extents of a problem after the device-side bound (a count formed by an earlier kernel of the
// same stream, e.g. a chunk's number of rows in the loss).
struct Extents {
  int M, N, K;
};
__device__ __forceinline__ Extents extents_of(const PairProblem& p, int dynv) {
  Extents e{p.M, p.N, p.K};
  if (p.dyn & DYN_M) e.M = dynv < e.M ? dynv : e.M;
  if (p.dyn & DYN_K) e.K = dynv < e.K ? dynv : e.K;
  return e;
}

// Pair `pair` of `P` takes n0 tiles of problem 0 (pair, pair + P, ...).  Problem 0 has
// a = T0 / P tiles per pair plus one more on the first T0 % P pairs ("heavy" pairs).  Problem 1
// then runs in two interleaved phases so that concurrently running tiles stay neighbours (and
// share their operand slabs in L2):
//   phase A: the light pairs alone take k = round(c0 / c1) tiles each, round-robin among
//            themselves (tiles [0, TA)), making up for the problem-0 tile they lack;
//   phase B: the remaining tiles [TA, T1) round-robin over all pairs.
struct PairSchedule {
  int n0;        // problem-0 tiles
  int qa;        // phase-A tiles (light pairs only)
  int qb;        // phase-B tiles
  int la;        // index of this pair among the light pairs
  int p_light;   // number of light pairs
  int ta;        // problem-1 tiles handed out in phase A
};

__host__ __device__ inline PairSchedule pair_schedule(int pair, int P, int T0, int c0, int T1,
                                                     int c1) {
  PairSchedule s{0, 0, 0, 0, 1, 0};
  const int a = T0 / P, n_hi = T0 % P;
  s.n0 = a + (pair < n_hi ? 1 : 0);
  if (T1 <= 0) return s;
  s.p_light = P - n_hi;
  int k = n_hi > 0 ? (c0 + c1 / 2) / c1 : 0;
  if (static_cast<long long>(s.p_light) * k > T1) k = T1 / s.p_light;
  s.ta = s.p_light * k;
  s.qa = pair >= n_hi ? k : 0;
  s.la = pair - n_hi;
  const int rest = T1 - s.ta;
  s.qb = pair < rest ? (rest - pair + P - 1) / P : 0;
  return s;
}

// The i-th tile (0 <= i < n0 + qa + qb) of pair `pair`: its problem and its index t within that
// problem's tiles.  Compiled for the host too, where the library checks that every tile of both
// problems goes to exactly one (pair, i).
struct PairTile {
  int prob, t;
};
__host__ __device__ inline PairTile pair_tile(const PairSchedule& s, int pair, int P, int i) {
  if (i < s.n0) return PairTile{0, pair + i * P};
  const int j = i - s.n0;
  return PairTile{1, j < s.qa ? s.la + j * s.p_light : s.ta + pair + (j - s.qa) * P};
}

// WIDE0: problem 0 may run in wide tiles (below).  ROUND: ring slots per MMA-issue round of
// the other tiles (1 or 2).  FMT: with 8-bit operands, which of them are e5m2 (F8_A0, F8_B0,
// F8_A1, F8_B1 bits; the others are e4m3).
enum : int { F8_A0 = 1, F8_B0 = 2, F8_A1 = 4, F8_B1 = 8 };
template <class C, class E0, class E1, Major A0, Major B0, Major A1, Major B1, bool WIDE0 = false,
          int ROUND = 1, int FMT = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const PairArgs args, const __grid_constant__ typename E0::Params ep0,
                     const __grid_constant__ typename E1::Params ep1) {
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
  int* sched = reinterpret_cast<int*>(tmem_slot + 2);   // PairSchedule fields

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());

  // extents (the device-side bound was written by an earlier kernel of this stream)
  const int dynv = args.dyn != nullptr ? *args.dyn : 0x7fffffff;
  const Extents ex0 = extents_of(args.prob[0], dynv);
  const Extents ex1 = extents_of(args.prob[1], dynv);
  const int m_tiles0 = (ex0.M + C::BM - 1) / C::BM;
  const int n_tiles0 = (ex0.N + C::BN - 1) / C::BN;
  const int nkb0 = (ex0.K + C::KSLOT - 1) / C::KSLOT;   // ring slots per tile
  const int m_tiles1 = (ex1.M + C::BM - 1) / C::BM;
  const int n_tiles1 = (ex1.N + C::BN - 1) / C::BN;
  const int nkb1 = (ex1.K + C::KSLOT - 1) / C::KSLOT;
  // Wide tiles (problem 0, bf16): two adjacent BN-column blocks share every staged k-block of
  // A, one TMEM accumulator each, so a pair stages 256 + 512 operand rows per k-block instead
  // of 2 x (256 + 256).  The second B block goes into the next ring slot (its A area unused),
  // so a wide k-block takes two slots and the ring stays in step as long as the slot count and
  // the number of N blocks are even.  Meant for long-K problems: while a wide tile runs, no
  // accumulator is free for the epilogue of the previous tile to overlap with.
  const bool wide0 = WIDE0 && args.prob[0].wide != 0 && C::KSUB == 1 &&
                     (C::STAGES % 2) == 0 && (n_tiles0 % 2) == 0;
  const int w_tiles0 = wide0 ? n_tiles0 / 2 : n_tiles0;

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
    const PairSchedule mine = pair_schedule(pair, npairs, m_tiles0 * w_tiles0,
                                            wide0 ? 2 * nkb0 : nkb0,
                                            ex1.M > 0 ? m_tiles1 * n_tiles1 : 0,
                                            nkb1 > 0 ? nkb1 : 1);
    sched[0] = mine.n0;
    sched[1] = mine.qa;
    sched[2] = mine.qb;
    sched[3] = mine.la;
    sched[4] = mine.p_light;
    sched[5] = mine.ta;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (ex1.M > 0) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised, schedule written, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  PairSchedule ps;
  ps.n0 = sched[0];
  ps.qa = sched[1];
  ps.qb = sched[2];
  ps.la = sched[3];
  ps.p_light = sched[4];
  ps.ta = sched[5];
  const int n0 = ps.n0, total = ps.n0 + ps.qa + ps.qb;
  const uint32_t leader_full = mapa_shared(smem_u32(full), 0);
  const uint32_t leader_tempty = mapa_shared(smem_u32(tempty), 0);

  // i-th tile of this pair -> (problem, m block, n block, k-blocks); in a wide problem 0,
  // nb indexes pairs of N blocks (2 nb and 2 nb + 1).
  auto tile_of = [&](int i, int& prob, int& mb, int& nb, int& kbs) {
    const PairTile pt = pair_tile(ps, pair, npairs, i);
    const int t = pt.t;
    int mt, nt, mf;
    prob = pt.prob;
    if (prob == 0) {
      mt = m_tiles0;
      nt = w_tiles0;
      mf = args.prob[0].m_fastest;
      kbs = nkb0;
    } else {
      mt = m_tiles1;
      nt = n_tiles1;
      mf = args.prob[1].m_fastest;
      kbs = nkb1;
    }
    if (mf) {
      mb = t % mt;
      nb = t / mt;
    } else {
      const int ng = args.prob[prob].n_groups;
      if (ng > 1 && nt % ng == 0) {
        const int ntg = nt / ng, per = mt * ntg;
        const int grp = t / per, u = t - grp * per;
        nb = grp * ntg + u % ntg;
        mb = u / ntg;
      } else {
        nb = t % nt;
        mb = t / nt;
      }
    }
  };
  // Every role walks this pair's tiles in order; the wide tiles (all of problem 0, when wide0)
  // come first and run with NSUB = 2 known at compile time, everything else with NSUB = 1.
  auto for_each_run = [&](auto&& run) {
    if constexpr (WIDE0) {
      if (wide0) {
        run(IntC<2>{}, 0, n0);
        run(IntC<1>{}, n0, total);
        return;
      }
    }
    run(IntC<1>{}, 0, total);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      long long arms = 0;
      const uint64_t pol_a0 = l2_policy(args.prob[0].l2_a), pol_b0 = l2_policy(args.prob[0].l2_b);
      const uint64_t pol_a1 = l2_policy(args.prob[1].l2_a), pol_b1 = l2_policy(args.prob[1].l2_b);
      for_each_run([&](auto nsub_c, int i0, int i1) {
        constexpr int NSUB = decltype(nsub_c)::value;
        for (int i = i0; i < i1 && !*abort_flag; ++i) {
          int prob, mb, nb, kbs;
          tile_of(i, prob, mb, nb, kbs);
          const int a_row = mb * C::BM + static_cast<int>(rank) * C::BM_CTA;
          const int b_row = nb * NSUB * C::BN + static_cast<int>(rank) * C::BN_CTA;
          const int nt_all = prob == 0 ? n_tiles0 : n_tiles1;
          const bool rev = args.prob[prob].serpentine &&
                           ((((args.prob[prob].m_off + mb) * nt_all + nb * NSUB) / npairs) & 1);
          for (int kb = 0; kb < kbs; ++kb) {
            // a wide k-block starts on an even slot, so stage + 1 is in the same ring phase
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.status, args.limit_ns)) {
              *abort_flag = 1;
              break;
            }
            if constexpr (NSUB == 2) {
              if (!mbar_wait_bounded(&empty[stage + 1], phase ^ 1u, args.status, args.limit_ns)) {
                *abort_flag = 1;
                break;
              }
            }
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
              if constexpr (NSUB == 2) mbar_arrive_expect_tx(&full[stage + 1], 2 * C::B_BYTES);
            }
            uint8_t* sA = smem + stage * C::STAGE_BYTES;
            uint8_t* sB = sA + C::A_BYTES;
            const uint32_t bar = leader_full + 8u * stage;
#pragma unroll
            for (int j = 0; j < C::KSUB; ++j) {
              const int k0 = (rev ? kbs - 1 - kb : kb) * C::KSLOT + j * C::BK;
              if (prob == 0) {
                load_operand_pair<A0, C::BM_CTA, C::ELEM_BYTES>(sA + j * C::A_SUB, &tmA0, bar,
                                                                a_row, k0, pol_a0);
                load_operand_pair<B0, C::BN_CTA, C::ELEM_BYTES>(sB + j * C::B_SUB, &tmB0, bar,
                                                                b_row, k0, pol_b0);
                if constexpr (NSUB == 2)
                  load_operand_pair<B0, C::BN_CTA, C::ELEM_BYTES>(sB + C::STAGE_BYTES, &tmB0,
                                                                  bar + 8u, b_row + C::BN, k0,
                                                                  pol_b0);
              } else {
                load_operand_pair<A1, C::BM_CTA, C::ELEM_BYTES>(sA + j * C::A_SUB, &tmA1, bar,
                                                                a_row, k0, pol_a1);
                load_operand_pair<B1, C::BN_CTA, C::ELEM_BYTES>(sB + j * C::B_SUB, &tmB1, bar,
                                                                b_row, k0, pol_b1);
              }
            }
            arms += NSUB;
            stage += NSUB;
            if (stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      });
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
      constexpr int EB = C::ELEM_BYTES;
      static_assert((B0 == Major::K || C::BN_CTA % (128 / EB) == 0) &&
                        (B1 == Major::K || C::BN_CTA % (128 / EB) == 0),
                    "MN-major B halves are whole 128-byte blocks");
      static_assert(EB == 1 || FMT == 0, "operand formats are for 8-bit operands");
      constexpr uint32_t idesc0 =
          EB == 1 ? instr_desc_f8_f32(C::BM, C::BN, (FMT & F8_A0) ? F8_E5M2 : F8_E4M3,
                                      (FMT & F8_B0) ? F8_E5M2 : F8_E4M3, A0 == Major::MN,
                                      B0 == Major::MN)
                  : instr_desc_bf16_f32(C::BM, C::BN, A0 == Major::MN, B0 == Major::MN);
      constexpr uint32_t idesc1 =
          EB == 1 ? instr_desc_f8_f32(C::BM, C::BN, (FMT & F8_A1) ? F8_E5M2 : F8_E4M3,
                                      (FMT & F8_B1) ? F8_E5M2 : F8_E4M3, A1 == Major::MN,
                                      B1 == Major::MN)
                  : instr_desc_bf16_f32(C::BM, C::BN, A1 == Major::MN, B1 == Major::MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for_each_run([&](auto nsub_c, int i0, int i1) {
        constexpr int NSUB = decltype(nsub_c)::value;
        for (int i = i0; i < i1 && !*abort_flag; ++i) {
          int prob, mb, nb, kbs;
          tile_of(i, prob, mb, nb, kbs);
          // a wide tile takes both accumulators: acc, then the other one
          const int acc2 = acc ^ 1;
          const uint32_t acc2_phase = acc == 1 ? acc_phase ^ 1u : acc_phase;
          if (!mbar_wait_bounded_cluster(&tempty[acc], acc_phase ^ 1u, args.status,
                                         args.limit_ns)) {
            *abort_flag = 1;
            return;
          }
          if constexpr (NSUB == 2) {
            if (!mbar_wait_bounded_cluster(&tempty[acc2], acc2_phase ^ 1u, args.status,
                                           args.limit_ns)) {
              *abort_flag = 1;
              return;
            }
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
          if constexpr (NSUB == 2) {
            for (int kb = 0; kb < kbs; ++kb) {
              if (!mbar_wait_bounded(&full[stage], phase, args.status, args.limit_ns) ||
                  !mbar_wait_bounded(&full[stage + 1], phase, args.status, args.limit_ns)) {
                *abort_flag = 1;
                return;
              }
              tc_fence_after();
              const uint32_t a_base = smem_u32(smem + stage * C::STAGE_BYTES);
              const uint32_t b_base = a_base + C::A_BYTES;
              // both N blocks from one staged A k-block; the second B block is in the next slot
              const uint32_t d_tmem2 = tmem_base + static_cast<uint32_t>(acc2 * C::BN);
              const uint32_t b_base2 = b_base + C::STAGE_BYTES;
              const uint64_t da = operand_desc<A0, EB>(a_base, 0);
              const uint64_t db = operand_desc<B0, EB>(b_base, 0);
              const uint64_t db2 = operand_desc<B0, EB>(b_base2, 0);
#pragma unroll
              for (int k = 0; k < C::BK / C::MMA_K; ++k) {
                mma_pair<EB>(d_tmem, da + desc_step<A0, EB>() * k, db + desc_step<B0, EB>() * k,
                             idesc0, (kb | k) != 0 ? 1u : 0u);
                mma_pair<EB>(d_tmem2, da + desc_step<A0, EB>() * k,
                             db2 + desc_step<B0, EB>() * k, idesc0, (kb | k) != 0 ? 1u : 0u);
              }
              issued = true;
              mma_commit_pair_both(&empty[stage]);
              mma_commit_pair_both(&empty[stage + 1]);
              stage += 2;
              if (stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
              }
            }
          } else {
            // the MMAs of one staged k-block into d_tmem
            // the MMAs of one ring slot (KSUB k-blocks) into d_tmem
            auto issue = [&](int st, int kb) {
#pragma unroll
              for (int j = 0; j < C::KSUB; ++j) {
                const uint32_t a_base = smem_u32(smem + st * C::STAGE_BYTES + j * C::A_SUB);
                const uint32_t b_base = smem_u32(smem + st * C::STAGE_BYTES + C::A_BYTES +
                                                 j * C::B_SUB);
                const int first = kb | j;   // 0 only for the first k-block of the tile
                if (prob == 0) {
                  const uint64_t da = operand_desc<A0, EB>(a_base, 0);
                  const uint64_t db = operand_desc<B0, EB>(b_base, 0);
#pragma unroll
                  for (int k = 0; k < C::BK / C::MMA_K; ++k)
                    mma_pair<EB>(d_tmem, da + desc_step<A0, EB>() * k,
                                 db + desc_step<B0, EB>() * k, idesc0, (first | k) != 0 ? 1u : 0u);
                } else {
                  const uint64_t da1 = operand_desc<A1, EB>(a_base, 0);
                  const uint64_t db1 = operand_desc<B1, EB>(b_base, 0);
#pragma unroll
                  for (int k = 0; k < C::BK / C::MMA_K; ++k)
                    mma_pair<EB>(d_tmem, da1 + desc_step<A1, EB>() * k,
                                 db1 + desc_step<B1, EB>() * k, idesc1,
                                 (first | k) != 0 ? 1u : 0u);
                }
              }
            };
            // ROUND = 2: two ring slots per round, one fence and one loop step for both.  The
            // single MMA-issuing thread is what limits slots of one k-block (4 MMAs): its waits,
            // fence and commit take about as long as the MMAs run.  The logits use slots of two
            // k-blocks instead (KSUB = 2: one wait and one commit per 8 MMAs); the dW tiles keep
            // one (two per round measured slower there: their MN-major loads arrive later).
            static_assert(ROUND == 1 || ROUND == 2, "one or two ring slots per round");
            for (int kb = 0; kb < kbs; kb += ROUND) {
              const bool two = ROUND == 2 && kb + 1 < kbs;
              const int st2 = stage + 1 == C::STAGES ? 0 : stage + 1;
              const uint32_t ph2 = stage + 1 == C::STAGES ? phase ^ 1u : phase;
              if (!mbar_wait_bounded(&full[stage], phase, args.status, args.limit_ns) ||
                  (two && !mbar_wait_bounded(&full[st2], ph2, args.status, args.limit_ns))) {
                *abort_flag = 1;
                return;
              }
              tc_fence_after();
              issue(stage, kb);
              if (two) issue(st2, kb + 1);
              issued = true;
              mma_commit_pair_both(&empty[stage]);
              if (two) mma_commit_pair_both(&empty[st2]);
              stage = two ? st2 : stage;
              phase = two ? ph2 : phase;
              if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
          mma_commit_pair_both(&tfull[acc]);
          if constexpr (NSUB == 2) mma_commit_pair_both(&tfull[acc2]);
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub) {
            if (++acc == 2) {
              acc = 0;
              acc_phase ^= 1u;
            }
          }
        }
      });
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
    for_each_run([&](auto nsub_c, int i0, int i1) {
      constexpr int NSUB = decltype(nsub_c)::value;
      for (int i = i0; i < i1 && !*abort_flag; ++i) {
        int prob, mb, nb, kbs;
        tile_of(i, prob, mb, nb, kbs);
#pragma unroll
        for (int sub = 0; sub < NSUB; ++sub) {   // a wide tile: its two N blocks in turn
          if (!mbar_wait_bounded(&tfull[acc], acc_phase, args.status, args.limit_ns)) {
            *abort_flag = 1;
            return;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 static_cast<uint32_t>(acc * C::BN + slab * C::COLS_PER_WARP);
          const int nbs = nb * NSUB + sub;
          const int row = mb * C::BM + static_cast<int>(rank) * C::BM_CTA + row_in_cta;
          const int col0 = nbs * C::BN + slab * C::COLS_PER_WARP;
          // a tile with no k-blocks (a device-bounded K of 0) contributes a zero tile
          const bool zero = kbs == 0;
          if (prob == 0)
            E0::template apply<C::COLS_PER_WARP>(ep0, row, col0, taddr, nbs * C::COL_SPLIT + slab,
                                                 zero);
          else
            E1::template apply<C::COLS_PER_WARP>(ep1, row, col0, taddr, nbs * C::COL_SPLIT + slab,
                                                 zero);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(leader_tempty + 8u * acc);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
    });
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
  int a_ld;                  // row stride of A (elements, >= Vpad)
  int mode;                  // LogitsMode
  int fixed_ref;             // 1: exp reference is cap (requires cap > 0); 0: online / lse
  float cap;                 // > 0: softcap value; <= 0: no softcap
  float k_u;                 // 2/cap * log2(e)
  float m2c_log2e;           // -2 cap log2(e)
  const float* scale_a;      // e4m3 operands: z = acc * (*scale_a) * (*scale_b); null for bf16
  const float* scale_b;
  const int* tgt;            // [rows] target id, -1 when the row is not in the loss
  const float* ref;          // [rows] exp reference (lse) when !fixed_ref and mode == RECOMPUTE
  float* partial;            // [rows][n_slabs] sum-exp (pairs (max, sum-exp) when !fixed_ref)
  int n_slabs;
  float* s_t;                // [rows] softcapped target logit
  float* der_t;              // [rows] 1 - tanh^2 at the target
  float* e_t;                // [rows] exp(s_t - reference)
  __nv_bfloat16* A;          // [rows][Vpad] gradient operand (modes FUSED / RECOMPUTE)
  const int* pos;            // [rows] row of A for each row (-1: not written), or null: same row
  // The final RMSNorm's backward folded into dX (fixed reference only): per slab the sum of
  // A_ij z_ij over its columns (z the logit before the softcap), and the target's z.  With the
  // row sum S_i they give sum_j dz_ij z_ij, which is d times the RMSNorm's row term.
  float* q_partial;          // [rows][n_slabs], or null
  float* z_t;                // [rows] (with q_partial)
};

// FOLD: also the per-slab sums of A_ij z_ij and the target's z (q_partial, z_t), for the final
// RMSNorm's backward; a separate instantiation, so that the plain epilogue carries none of it.
template <bool FOLD>
struct LogitsEpiT {
  using Params = LogitsParams;
  static constexpr float LOG2E = 1.4426950408889634f;

  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int slab_index, bool zero) {
    const bool row_ok = row < p.rows;
    const int t = row_ok ? __ldg(p.tgt + row) : -1;
    const bool capped = p.cap > 0.f;
    const bool write_a = p.mode != LOGITS_STATS;
    // Tensorwise scales of e4m3 operands: folded into the exp2 argument on the fixed-reference
    // path (only |z| and the sign of z are used there), applied to z elsewhere.
    const float zs = p.scale_a != nullptr ? __ldg(p.scale_a) * __ldg(p.scale_b) : 1.0f;
    const float k_u = p.k_u * zs;
    const bool online = !p.fixed_ref && p.mode == LOGITS_STATS;
    const float ref = p.fixed_ref ? p.cap
                                  : ((p.mode == LOGITS_RECOMPUTE && row_ok) ? __ldg(p.ref + row) : 0.f);
    float sum = 0.f;
    float run_max = -INFINITY;
    float tv_s = 0.f, tv_der = 0.f, tv_e = 0.f, tv_z = 0.f;
    bool has_t = false;
    float qsum = 0.f;                                  // FOLD: sum of A_ij z_ij / zs
    __nv_bfloat16* arow = nullptr;
    if (write_a && row_ok) {
      const int at = p.pos != nullptr ? __ldg(p.pos + row) : row;
      if (at >= 0) arow = p.A + static_cast<size_t>(at) * p.a_ld;
    }
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32_or_zero(taddr + c * 32, v, zero);
      const int cbase = col0 + c * 32;
      if (p.fixed_ref) {
        // softcap with the fixed reference: e = exp(s - cap), A = e (1 - tanh^2)
        if (static_cast<unsigned>(t - cbase) < 32u) {   // this row's target is in this chunk
          float zt = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k == t - cbase) zt = v[k];
          const Softcapped sc = softcap_fixed_ref(zt, k_u, p.m2c_log2e, p.cap);
          tv_s = sc.s;
          tv_der = sc.der;
          tv_e = sc.e;
          if constexpr (FOLD) tv_z = zt * zs;
          has_t = true;
        }
        if (cbase + 32 <= p.Vreal) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float z = v[k];
            const Softcapped sc = softcap_fixed_ref(z, k_u, p.m2c_log2e, p.cap);
            sum += sc.e;
            v[k] = sc.e * sc.der;
            if constexpr (FOLD) qsum = fmaf(v[k], z, qsum);
          }
        } else {                                            // last vocabulary tile: padded columns
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float z = v[k];
            const Softcapped sc = softcap_fixed_ref(z, k_u, p.m2c_log2e, p.cap);
            const float e = cbase + k < p.Vreal ? sc.e : 0.f;
            sum += e;
            v[k] = e * sc.der;
            if constexpr (FOLD) qsum = fmaf(v[k], z, qsum);
          }
        }
      } else {
        float der[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          v[k] *= zs;
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
        if ((p.a_ld & 15) == 0) {
          // rows start on 32-byte boundaries: two full-sector stores per 32 columns
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int col = cbase + 16 * g;
            if (col < p.Vpad) {
              const uint32_t w[8] = {packed[8 * g],     packed[8 * g + 1], packed[8 * g + 2],
                                     packed[8 * g + 3], packed[8 * g + 4], packed[8 * g + 5],
                                     packed[8 * g + 6], packed[8 * g + 7]};
              st_global_v8(arow + col, w);
            }
          }
        } else {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = cbase + 8 * g;
            if (col < p.Vpad) {
              *reinterpret_cast<uint4*>(arow + col) = make_uint4(
                  packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
            }
          }
        }
      }
    }
    if (!row_ok) return;
    if (p.mode != LOGITS_RECOMPUTE) {
      if (!online) {
        p.partial[static_cast<size_t>(row) * p.n_slabs + slab_index] = sum;
        if constexpr (FOLD)
          p.q_partial[static_cast<size_t>(row) * p.n_slabs + slab_index] = qsum * zs;
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
      if constexpr (FOLD) p.z_t[row] = tv_z;
    }
  }
};
using LogitsEpi = LogitsEpiT<false>;
using LogitsFoldEpi = LogitsEpiT<true>;

// ==============================================================================================
// Epilogue 2: dX rows = r_i * (A' W)_i, stored as bf16.
struct DxParams {
  int rows, d;
  int sector32;              // 1: dX rows and base are 32-byte aligned (full-sector stores)
  const float* r;            // [rows] row scale g/(Nv S_i); 0 for rows not in the loss
  __nv_bfloat16* dX;         // [rows][d]
  const int* orig;           // compacted rows: dX row of each (null: same row)
  const int* dyn_rows;       // compacted rows: their device-side count (null: rows)
  const float* uscale;       // one scale for every row instead of r (8-bit operands), or null
  // The final RMSNorm x = h rstd gamma folded in (H != null): the rows are written as
  //   dH = rstd (gamma . dX - xh c),  xh = h rstd,  c = mean_k x_k dX_k
  // in place of dX, and for every block of 32 rows the column sums of dX . xh (the terms of
  // dgamma) go to dg_part.
  const __nv_bfloat16* H;    // [rows][d] the rows before the norm (indexed like dX)
  const __nv_bfloat16* gamma;// [d]
  const float* rstd;         // [rows] (indexed like dX)
  const float* cdot;         // [rows] c of each row (indexed like r)
  float* dg_part;            // [row blocks of 32][d] (blocks of the rows indexed like r)
};

struct DxEpi {
  using Params = DxParams;

  // On return lane L holds in a[0] the sum over the warp's 32 lanes of a[L]: five exchange
  // rounds, each halving the columns a lane keeps (the lanes with the round's bit set keep the
  // upper half).
  __device__ static __forceinline__ void warp_column_sums(float (&a)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int k = 0; k < s; ++k) {
        const float send = upper ? a[k] : a[k + s];
        const float keep = upper ? a[k + s] : a[k];
        a[k] = keep + __shfl_xor_sync(0xffffffffu, send, s);
      }
    }
  }

  template <int NCOLS>
  __device__ static __forceinline__ void apply_rmsnorm(const Params& p, int row, int col0,
                                                       uint32_t taddr, bool zero) {
    const int lane = threadIdx.x & 31;
    const int rows = p.dyn_rows != nullptr ? __ldg(p.dyn_rows) : p.rows;
    const bool row_ok = row < rows;
    const float sc = row_ok ? __ldg(p.r + row) : 0.f;
    const float c = row_ok ? __ldg(p.cdot + row) : 0.f;
    const int out_row = row_ok && p.orig != nullptr ? __ldg(p.orig + row) : row;
    const float rs = row_ok ? __ldg(p.rstd + out_row) : 0.f;
    const __nv_bfloat16* hrow = p.H + static_cast<size_t>(row_ok ? out_row : 0) * p.d;
    __nv_bfloat16* out = row_ok ? p.dX + static_cast<size_t>(out_row) * p.d : nullptr;
    float* dgp = p.dg_part + static_cast<size_t>(row >> 5) * p.d;   // the warp's 32-row block
    // h is read one 32-column chunk ahead of its use, so that the load's latency overlaps the
    // previous chunk's arithmetic (this epilogue is not overlapped with MMAs in wide tiles)
    uint4 hn[4];
    auto load_h = [&](int cbase) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = cbase + 8 * g;
        hn[g] = (row_ok && col < p.d) ? __ldg(reinterpret_cast<const uint4*>(hrow + col))
                                      : make_uint4(0, 0, 0, 0);
      }
    };
    load_h(col0);
#pragma unroll 1
    for (int cc = 0; cc < NCOLS / 32; ++cc) {
      float v[32];
      tmem_ld32_or_zero(taddr + cc * 32, v, zero);
      const int cbase = col0 + cc * 32;
      if (cbase >= p.d) continue;                      // the same for the whole warp
      uint4 hc[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) hc[g] = hn[g];
      if (cc + 1 < NCOLS / 32) load_h(cbase + 32);
      float dg[32];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = cbase + 8 * g;
        const uint4 gr = col < p.d ? __ldg(reinterpret_cast<const uint4*>(p.gamma + col))
                                   : make_uint4(0, 0, 0, 0);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hc[g]);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gr);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 hf = __bfloat1622float2(h2[q]);
          const float2 gf = __bfloat1622float2(g2[q]);
          const int k = 8 * g + 2 * q;
          const float xh0 = hf.x * rs, xh1 = hf.y * rs;
          const float dx0 = v[k] * sc, dx1 = v[k + 1] * sc;
          v[k] = rs * (gf.x * dx0 - xh0 * c);
          v[k + 1] = rs * (gf.y * dx1 - xh1 * c);
          dg[k] = dx0 * xh0;
          dg[k + 1] = dx1 * xh1;
        }
      }
      if (out != nullptr) store_row32(p, out, cbase, v);
      warp_column_sums(dg, lane);
      if (cbase + lane < p.d) dgp[cbase + lane] = dg[0];
    }
  }

  // 32 values of one row as bf16 at columns [cbase, cbase + 32) (those below d).
  __device__ static __forceinline__ void store_row32(const Params& p, __nv_bfloat16* out,
                                                     int cbase, const float (&v)[32]) {
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) w[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
    if (p.sector32) {
      // two full 32-byte sectors per 32 columns
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int col = cbase + 16 * g;
        if (col < p.d) {
          const uint32_t q[8] = {w[8 * g],     w[8 * g + 1], w[8 * g + 2], w[8 * g + 3],
                                 w[8 * g + 4], w[8 * g + 5], w[8 * g + 6], w[8 * g + 7]};
          st_global_v8(out + col, q);
        }
      }
    } else {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = cbase + 8 * g;
        if (col < p.d)
          *reinterpret_cast<uint4*>(out + col) =
              make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
      }
    }
  }

  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int, bool zero) {
    if (p.H != nullptr) {
      apply_rmsnorm<NCOLS>(p, row, col0, taddr, zero);
      return;
    }
    const int rows = p.dyn_rows != nullptr ? __ldg(p.dyn_rows) : p.rows;
    const bool row_ok = row < rows;
    const float sc = !row_ok ? 0.f : (p.uscale != nullptr ? __ldg(p.uscale) : __ldg(p.r + row));
    const int out_row = row_ok && p.orig != nullptr ? __ldg(p.orig + row) : row;
    __nv_bfloat16* out = row_ok ? p.dX + static_cast<size_t>(out_row) * p.d : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32_or_zero(taddr + c * 32, v, zero);
      if (out == nullptr) continue;
#pragma unroll
      for (int k = 0; k < 32; ++k) v[k] *= sc;
      store_row32(p, out, col0 + c * 32, v);
    }
  }
};

// ==============================================================================================
// Epilogue 3: dW rows (vocabulary rows) = (A'^T (r . X))_j, written or accumulated, in fp32 or in
// bf16 (bf16: the tile is added to the stored values in fp32 and rounded once).
struct DwParams {
  int Vpad, d;
  int accumulate;            // 1: dW += tile, 0: dW = tile
  int sector32;              // 1: dW rows and base are 32-byte aligned (full-sector accesses)
  int bf16;                  // 1: dW is bf16, 0: fp32
  void* dW;                  // [Vpad][d]
  const float* scale;        // factor applied to the tile (8-bit operands), or null
};

struct DwEpi {
  using Params = DwParams;

  // 16 bf16 values <-> 8 packed words
  __device__ static __forceinline__ void add_bf16x16(float* v, const uint32_t (&o)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o[k]));
      v[2 * k] += f.x;
      v[2 * k + 1] += f.y;
    }
  }

  template <int NCOLS>
  __device__ static __forceinline__ void apply(const Params& p, int row, int col0, uint32_t taddr,
                                               int, bool zero) {
    const bool row_ok = row < p.Vpad;
    float* out = row_ok ? static_cast<float*>(p.dW) + static_cast<size_t>(row) * p.d : nullptr;
    __nv_bfloat16* out16 =
        row_ok ? static_cast<__nv_bfloat16*>(p.dW) + static_cast<size_t>(row) * p.d : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
      float v[32];
      tmem_ld32_or_zero(taddr + c * 32, v, zero);
      if (!row_ok) continue;
      if (p.scale != nullptr) {
        const float f = __ldg(p.scale);
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] *= f;
      }
      const int cbase = col0 + c * 32;
      if (p.bf16) {
        if (p.sector32) {
          // two full 32-byte sectors (16 bf16 each) per 32 columns; d % 16 == 0
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int col = cbase + 16 * g;
            if (col < p.d) {
              __nv_bfloat16* dst = out16 + col;
              if (p.accumulate) {
                float f[8];
                ld_global_v8f(reinterpret_cast<const float*>(dst), f);
                uint32_t o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) o[k] = __float_as_uint(f[k]);
                add_bf16x16(v + 16 * g, o);
              }
              uint32_t q[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) q[k] = pack_bf16x2(v[16 * g + 2 * k], v[16 * g + 2 * k + 1]);
              st_global_v8(dst, q);
            }
          }
        } else {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = cbase + 8 * g;
            if (col < p.d) {
              uint4* dst = reinterpret_cast<uint4*>(out16 + col);
              if (p.accumulate) {
                const uint4 raw = *dst;
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 f = __bfloat1622float2(h[k]);
                  v[8 * g + 2 * k] += f.x;
                  v[8 * g + 2 * k + 1] += f.y;
                }
              }
              *dst = make_uint4(pack_bf16x2(v[8 * g], v[8 * g + 1]),
                                pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                pack_bf16x2(v[8 * g + 4], v[8 * g + 5]),
                                pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
            }
          }
        }
      } else if (p.sector32) {
        // whole 32-byte sectors: a partly written sector never reaches the L2 on its own
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = cbase + 8 * g;
          if (col < p.d) {
            float* dst = out + col;
            if (p.accumulate) {
              float o[8];
              ld_global_v8f(dst, o);
#pragma unroll
              for (int k = 0; k < 8; ++k) v[8 * g + k] += o[k];
            }
            const uint32_t q[8] = {
                __float_as_uint(v[8 * g]),     __float_as_uint(v[8 * g + 1]),
                __float_as_uint(v[8 * g + 2]), __float_as_uint(v[8 * g + 3]),
                __float_as_uint(v[8 * g + 4]), __float_as_uint(v[8 * g + 5]),
                __float_as_uint(v[8 * g + 6]), __float_as_uint(v[8 * g + 7])};
            st_global_v8(dst, q);
          }
        }
      } else {
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
  }
};

}  // namespace flce
