// fp4_gemm_pair.cuh -- the block-scaled NVFP4 GEMM of fp4_gemm.cuh on CTA
// pairs: each cluster of 2 CTAs (one TPC) computes 256 x 256 output tiles
// with tcgen05 cta_group::2 MMAs (M = 256, N = 256, K = 64).
//
//   Y = bf16( D . L2  +  deq(Xq) . deq(Rq)^T  +  bias )
//
// "Most operations happen in 4-bit tensor cores, while the low-rank correction
// runs in higher precision" (imaginepro.ai "Nunchaku 4-Bit Diffusion Inference
// in Diffusers: A Practical Guide", section "Under the Hood").
//
// CTA r of the pair stages the 128 rows [128 r, 128 r + 128) of the tile's A
// (activation codes) and of its B (weight codes) with A's scale rows; the
// pair's MMAs read A from each CTA for its half of M and B from both CTAs, so
// every byte of B's codes is loaded once per pair instead of once per CTA (38 KB
// of operands per CTA per 256-wide K stage instead of 54 KB).  B's scales are
// needed whole in each CTA's tensor memory (each CTA computes all 256 columns
// of its rows), so both CTAs load the scale rows of the full 256-row B tile.
// The leader (rank 0) issues the MMAs; the code tiles of both CTAs complete on
// the leader's stage barrier, each CTA's scale tiles on its own, and each CTA's
// scale warps write its tensor-memory scale buffers with tcgen05.st (as in the
// single-CTA kernel) and report to the leader; MMA completion is signalled to
// the barriers of both CTAs.  Each CTA's tensor memory holds its 128 rows of the
// fp32 accumulator (two alternating 256-column buffers sharing 64 columns, as
// in the single-CTA kernel) and its scale columns.  Each CTA's epilogue stores
// its own 128 rows and releases the shared columns to the leader.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"
#include "fp4_gemm.cuh"

namespace svdq {

constexpr int GP_THREADS = 384;
constexpr int GP_BM = 256;                 // tile rows per pair (128 per CTA)
constexpr int GP_BN = 256;                 // tile columns per pair (128 B rows per CTA)
constexpr uint32_t GP_A_TILE = 128 * 128;  // 16 KB per CTA and stage
constexpr uint32_t GP_B_TILE = 128 * 128;  // 16 KB
constexpr uint32_t GP_SF_TILE = 4 * 512;   // 2 KB: 128 rows x 4 k-groups of scales
constexpr uint32_t GP_SFB_TILE = 2 * GP_SF_TILE;   // B scales of all 256 tile columns

struct GemmPairCfg {
  static constexpr uint32_t kStage = GP_A_TILE + GP_B_TILE + GP_SF_TILE + GP_SFB_TILE;   // 38 KB
  static constexpr int kStages = 5;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSfaCol0 = 416;   // + 16 j: 4 k-blocks x 4 columns
  static constexpr uint32_t kSfbCol0 = 448;   // + 32 j: 4 k-blocks x 8 columns (all 256 B rows)
  static constexpr uint32_t kAcc1Col = 160;
  static constexpr int kOverlapChunks = 3;
  static constexpr uint32_t kOutBytes = 4 * GEMM_STAGE_OUT;
  static constexpr uint32_t kBarBytes = (3 * kStages + 8) * 8 + 16;
  static constexpr uint32_t kSmemBytes = kStages * kStage + kOutBytes + kBarBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kStage % 1024 == 0, "stage alignment");
};

struct GemmPairParams {
  const uint16_t* bias;
  int M, N, K, r;
  int m_tiles, n_tiles, num_tiles, kblocks;
};

template <int R_PAD>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GP_THREADS, 1)
    fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                         const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_l2,
                         const __grid_constant__ CUtensorMap tm_y, const GemmPairParams p) {
  using Cfg = GemmPairCfg;
  constexpr int S = Cfg::kStages;
  constexpr uint32_t kLRLayout = (R_PAD == 64 ? LAYOUT_SW128 : R_PAD == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
  constexpr uint32_t kLRSbo = 8 * R_PAD * 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* out_stage = smem + S * Cfg::kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + Cfg::kOutBytes);
  // bars[0..S) full (code tiles; the leader's counts both CTAs), [S..2S) empty,
  // 2S/2S+1 tmem_full[2], 2S+2 tmem_free (the leader's counts both epilogues), 2S+3 drain,
  // 2S+4/2S+5 sf_ready[2] (the leader's counts both CTAs' scale warps),
  // 2S+6/2S+7 sf_free[2], [2S+8..3S+8) sf_full (this CTA's scale tiles)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const uint32_t smem_base = smem_u32(smem);
  auto stage_a = [&](int s) { return smem_base + s * Cfg::kStage; };
  auto stage_b = [&](int s) { return smem_base + s * Cfg::kStage + GP_A_TILE; };
  auto stage_sfa = [&](int s) { return smem_base + s * Cfg::kStage + GP_A_TILE + GP_B_TILE; };
  auto stage_sfb = [&](int s) {
    return smem_base + s * Cfg::kStage + GP_A_TILE + GP_B_TILE + GP_SF_TILE;
  };
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto tmem_full = [&](int b) { return smem_u32(bars + 2 * S + b); };
  const uint32_t tmem_free = smem_u32(bars + 2 * S + 2);
  const uint32_t drain_bar = smem_u32(bars + 2 * S + 3);
  auto sf_ready = [&](uint32_t b) { return smem_u32(bars + 2 * S + 4 + b); };
  auto sf_free = [&](uint32_t b) { return smem_u32(bars + 2 * S + 6 + b); };
  auto sf_full = [&](int st) { return smem_u32(bars + 2 * S + 8 + st); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 2);      // the leader's arm + the peer's arrive
      mbar_init(empty_bar(s), 1);     // one multicast MMA commit
    }
    mbar_init(tmem_full(0), 1);
    mbar_init(tmem_full(1), 1);
    mbar_init(tmem_free, 2 * 4);      // both CTAs' epilogue warps
    mbar_init(drain_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sf_ready(b), 2 * 4);  // both CTAs' scale warps
      mbar_init(sf_free(b), 1);         // one multicast MMA commit
    }
    for (int st = 0; st < S; ++st) mbar_init(sf_full(st), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();   // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int kb_per_tile = p.kblocks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_sfa);
      tma_prefetch_desc(&tm_sfb);
      if (R_PAD > 0) {
        tma_prefetch_desc(&tm_d);
        tma_prefetch_desc(&tm_l2);
      }
      const uint32_t peer_full0 = mapa_shared(full_bar(0), 0);   // leader's full[0]
      int stage = 0;
      uint32_t phase = 0;
      int8_t fill_parity[S];
      for (int s = 0; s < S; ++s) fill_parity[s] = -1;
      const uint32_t tx_main = 2 * (GP_A_TILE + GP_B_TILE);      // both CTAs' code tiles
      const uint32_t tx_lr = 2 * (128 + 128) * R_PAD * 2;
      // arm (leader) or announce (peer) this CTA's loads for a stage
      auto post = [&](int s, uint32_t tx) {
        if (leader) mbar_arrive_expect_tx(full_bar(s), tx);
        else mbar_arrive_cluster(peer_full0 + s * 8);
      };
      bool ok = true;
      for (int t = pair; t < p.num_tiles && ok; t += num_pairs) {
        const int mb = t % p.m_tiles, nb = t / p.m_tiles;
        const int m0 = mb * GP_BM + 128 * rank, n0 = nb * GP_BN + 128 * rank;
        if (R_PAD > 0) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, KID_GEMM, 11)) { ok = false; break; }
          const uint32_t lb = leader_bar(full_bar(stage));
          tma_load_2d_pair(stage_a(stage), &tm_d, lb, 0, m0);
          tma_load_2d_pair(stage_b(stage), &tm_l2, lb, 0, n0);
          post(stage, tx_lr);
          mbar_arrive(sf_full(stage));   // keeps sf_full's phases in step with the ring
          fill_parity[stage] = static_cast<int8_t>(phase);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < kb_per_tile; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, KID_GEMM, 12)) { ok = false; break; }
          const uint32_t lb = leader_bar(full_bar(stage));
          tma_load_2d_pair(stage_a(stage), &tm_a, lb, kb * 128, m0);
          tma_load_2d_pair(stage_b(stage), &tm_b, lb, kb * 128, n0);
          post(stage, tx_main);
          mbar_arrive_expect_tx(sf_full(stage), GP_SF_TILE + GP_SFB_TILE);
          tma_load_2d(stage_sfa(stage), &tm_sfa, sf_full(stage), kb * 256, m0 / 128);
          tma_load_2d(stage_sfb(stage), &tm_sfb, sf_full(stage), kb * 256, (n0 - 128 * rank) / 128);
          fill_parity[stage] = static_cast<int8_t>(phase);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < S; ++s)
          if (fill_parity[s] >= 0) {
            if (leader) mbar_wait_drain(full_bar(s), static_cast<uint32_t>(fill_parity[s]));
            mbar_wait_drain(sf_full(s), static_cast<uint32_t>(fill_parity[s]));
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      const uint32_t idf = idesc_nvfp4(GP_BM, GP_BN);
      const uint32_t idb = idesc_bf16(GP_BM, GP_BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any_issued = false;
      int local = 0;
      uint32_t n = 0;
      for (int t = pair; t < p.num_tiles && ok; t += num_pairs, ++local) {
        const int buf = local & 1;
        const uint32_t acc = tmem_base + (buf ? Cfg::kAcc1Col : 0u);
        if (local > 0) {
          if (!mbar_wait(tmem_free, static_cast<uint32_t>(local - 1) & 1u, abort_flag, KID_GEMM, 14)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        uint32_t accumulate = 0;
        if (R_PAD > 0) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, KID_GEMM, 15)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = make_smem_desc(stage_a(stage), kLRLayout, kLRSbo, 0);
          const uint64_t bd = make_smem_desc(stage_b(stage), kLRLayout, kLRSbo, 0);
#pragma unroll
          for (int kk = 0; kk < R_PAD / 16; ++kk) {
            tc_mma_bf16_pair(acc, ad + 2 * kk, bd + 2 * kk, idb, accumulate);
            accumulate = 1;
          }
          tc_commit_pair(empty_bar(stage));
          any_issued = true;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < kb_per_tile; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, KID_GEMM, 16)) { ok = false; break; }
          const uint32_t sb = n & 1u;
          if (!mbar_wait(sf_ready(sb), (n >> 1) & 1u, abort_flag, KID_GEMM, 17)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa = tmem_base + Cfg::kSfaCol0 + 16 * sb;
          const uint32_t sfb = tmem_base + Cfg::kSfbCol0 + 32 * sb;
          const uint64_t ad = make_smem_desc(stage_a(stage), LAYOUT_SW128, 1024, 0);
          const uint64_t bd = make_smem_desc(stage_b(stage), LAYOUT_SW128, 1024, 0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tc_mma_nvfp4_pair(acc, ad + 2 * i, bd + 2 * i, idf, sfa + 4 * i, sfb + 8 * i, accumulate);
            accumulate = 1;
          }
          tc_commit_pair(empty_bar(stage));
          tc_commit_pair(sf_free(sb));
          ++n;
          any_issued = true;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(tmem_full(buf));
      }
      if (*abort_flag && any_issued) {
        tc_commit_pair(drain_bar);
        mbar_wait_drain(drain_bar, 0);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    uint8_t* stg = out_stage + q * GEMM_STAGE_OUT;
    const uint32_t stg_u = smem_u32(stg);
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t leader_free = mapa_shared(tmem_free, 0);
    int local = 0;
    for (int t = pair; t < p.num_tiles; t += num_pairs, ++local) {
      const int mb = t % p.m_tiles, nb = t / p.m_tiles;
      const int m0 = mb * GP_BM + 128 * rank, n0 = nb * GP_BN;
      const int buf = local & 1;
      const uint32_t acc = tmem_base + (buf ? Cfg::kAcc1Col : 0u);
      const uint4 tile_bias = load_tile_bias<GP_BN>(p.bias, n0, lane);
      if (!mbar_wait(tmem_full(buf), static_cast<uint32_t>(local >> 1) & 1u, abort_flag, KID_GEMM, 18))
        break;
      tc_fence_after();
      constexpr int kPieces = GP_BN / 16, kOv = 2 * Cfg::kOverlapChunks;
      epilogue_tile<GP_BN, kOv>(
          acc, lane_addr, lane, p.bias != nullptr, tile_bias, n0, m0 + q * 32, &tm_y, stg, stg_u,
          [&](int i) { return buf ? i : (i + kPieces - kOv) % kPieces; },
          [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_free);
          });
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ scale warps (both CTAs)
    // this CTA's tensor memory: A scales of its 128 rows, B scales of all 256
    // tile columns, each lane quarter its replica (see fp4_gemm.cuh)
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t leader_ready0 = mapa_shared(sf_ready(0), 0);
    int stage = 0;
    uint32_t phase = 0, n = 0;
    bool ok = true;
    for (int t = pair; t < p.num_tiles && ok; t += num_pairs) {
      if (R_PAD > 0) {
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      for (int kb = 0; kb < kb_per_tile; ++kb) {
        if (!mbar_wait(sf_full(stage), phase, abort_flag, KID_GEMM, 20)) { ok = false; break; }
        const uint32_t sb = n & 1u;
        if (n >= 2 && !mbar_wait(sf_free(sb), ((n >> 1) - 1) & 1u, abort_flag, KID_GEMM, 21)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* sa = smem + (stage_sfa(stage) - smem_base) + lane * 16;
        const uint8_t* sbp = smem + (stage_sfb(stage) - smem_base) + lane * 16;
        uint32_t va[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 x = *reinterpret_cast<const uint4*>(sa + i * 512);
          va[4 * i] = x.x; va[4 * i + 1] = x.y; va[4 * i + 2] = x.z; va[4 * i + 3] = x.w;
        }
        tmem_st_32x32b_x16(tmem_base + lane_addr + Cfg::kSfaCol0 + 16 * sb, va);
        uint32_t vb[32];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const uint4 x = *reinterpret_cast<const uint4*>(sbp + g * GP_SF_TILE + i * 512);
            vb[8 * i + 4 * g] = x.x; vb[8 * i + 4 * g + 1] = x.y;
            vb[8 * i + 4 * g + 2] = x.z; vb[8 * i + 4 * g + 3] = x.w;
          }
        tmem_st_32x32b_x32(tmem_base + lane_addr + Cfg::kSfbCol0 + 32 * sb, vb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_ready0 + 8 * sb);
        ++n;
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
  }

  // every role of both CTAs is done (remote arrivals delivered, MMAs drained
  // by the epilogues' last waits) before tensor memory is released
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace svdq
