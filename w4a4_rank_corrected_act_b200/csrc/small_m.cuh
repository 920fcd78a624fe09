// small_m.cuh -- the SVDQuant W4A4 linear layer for few tokens (M <= 32).
//
// With a handful of token rows (adaLN modulation, low-resolution previews) the
// layer is a weight stream: the NVFP4 residual of an N x K weight (N K / 2
// bytes of codes, N K / 16 of scales) is read once and each element meets at
// most 32 tokens, far below the tensor cores' ridge.  Its bound is HBM, so the
// design goal is that every SM streams its share of the weight from the first
// microsecond to the last.  Two kernels, chained by programmatic dependent
// launch:
//
//   act_quant_small_kernel  K/256 CTAs; CTA c quantises columns [256 c, 256 c +
//     256) of every token row (smoothing, one E4M3 scale per 16, E2M1 codes:
//     the "A4" of W4A4, aiphreaks.com "Bringing Nunchaku 4-bit Diffusion
//     Inference to Diffusers", section "Technical Breakdown and Performance
//     Metrics") and the matching slice of the low-rank down-projection,
//     D_c = bf16(Xhat[:, slice]) . L1[slice, :], as a float32 partial.
//
//   fp4_gemm_small_m_kernel  one CTA per 128 weight rows.  Operands swapped:
//     the weight tile is the MMA's A (M = 128 rows of R) and the tokens its
//     B (N = 16 or 32), so the 5th-generation tensor cores run the block-scaled
//     product Y^T = deq(Rq) deq(Xq)^T with no padding of the weight side
//     ("most operations ... in 4-bit tensor cores", imaginepro.ai practical
//     guide, section "Under the Hood").  The CTA's weight codes stream through
//     a TMA ring from the kernel's first instructions -- before the activation
//     kernel has finished, which the launch overlaps -- and the tile's weight
//     scales for the whole K sit in tensor memory (K/16 columns), so no scale
//     pipeline runs beside the MMAs.  After the activation kernel completes,
//     the activation codes (TMA), its scales (tensor memory) and the sum of
//     the D partials (shared memory) are brought in, the 4-bit MMAs drain the
//     ring, and the low-rank term D . L2 is added by bf16 MMAs into the same
//     accumulator (the 16-bit branch, same page).  The epilogue adds the bias
//     and stores bf16.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr int SMALL_MAX_TOKENS = 32;
constexpr int SMALL_ACT_COLS = 256;          // columns per activation CTA
constexpr int SMALL_THREADS = 256;
constexpr int SMALL_MAX_STAGES = 8;
constexpr int SMALL_IN_FLIGHT = 4;           // weight stages requested and not yet landed, per CTA
// Tensor memory: the accumulator in columns [0, 32), then for each 64-column
// block j of K a group of 4 columns of activation scales at 32 + 4 j (only the
// group's first column is read: it holds the 4 scales of token = lane) and a
// group of 4 columns of weight scales at 32 + 4 K/64 + 4 j.  Every scale
// address handed to the MMA is a multiple of 4 columns, the form the
// block-scaled MMA is given everywhere in this library.  32 + 8 K/64 <= 512
// bounds K.
constexpr int SMALL_MAX_K = 3840;
constexpr uint32_t SMALL_STAGE_BYTES = 128 * 128;   // 128 weight rows x 256 codes
constexpr uint32_t SMALL_ACC_COL = 0;
constexpr uint32_t SMALL_SFB_COL = 32;
constexpr uint32_t SMALL_TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t small_sfa_col(int K) { return SMALL_SFB_COL + 4u * static_cast<uint32_t>(K / 64); }
enum : uint32_t { KID_SMALL_ACT = 6, KID_SMALL_GEMM = 7 };

struct SmallActParams {
  const uint16_t* X;          // M x K bf16
  const float* inv_lambda;    // K
  const uint32_t* L1f;        // L1 in mma.m16n8k16 B-fragment order (l1_fragment_word)
  uint8_t* x_codes;           // M x K/2
  uint32_t* sfb;              // [K/64][32]: token t's 4 scale codes of 64-column block j (0 for t >= M)
  float* dpart;               // [K/256][M][r] float32 partial down-projections
  int M, K, r;
};

// ---------------------------------------------------------------------------
// Activation kernel for M <= 32.  A warp quantises one token row of the
// CTA's 256 columns (lane l: columns 8 l .. 8 l + 7, lane pairs forming the
// 16-element blocks), writes the codes and the scale words, and keeps
// bf16(Xhat) in shared memory; then each warp computes one 16 x 8 block of the
// partial D with bf16 mma.sync over the 256 columns.
// ---------------------------------------------------------------------------
template <int R_PAD>
__global__ void __launch_bounds__(SMALL_THREADS, 2) act_quant_small_kernel(const SmallActParams p) {
  constexpr int kRowStride = SMALL_ACT_COLS + 8;   // bf16 elements; 528-byte rows, conflict-free ldmatrix
  constexpr int kRowsPerWarp = SMALL_MAX_TOKENS / (SMALL_THREADS / 32);
  constexpr int kTilesPerWarp = R_PAD > 32 ? 2 : 1;   // 8-column blocks of D per warp
  __shared__ __align__(16) uint16_t xs[SMALL_MAX_TOKENS * kRowStride];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col0 = blockIdx.x * SMALL_ACT_COLS;
  // Nothing in global memory is touched before the previous kernel of the
  // stream has completed; only then may the GEMM launch (it reads X, which
  // that kernel may have written, and it waits for this grid before it reads
  // the D partials).
  pdl_wait();
  pdl_launch_dependents();

  // Every load of the kernel is issued here, before any of it is used, so
  // that the CTA pays one memory round trip: 1/lambda of the lane's 8 columns,
  // the warp's token rows, and the L1 fragments of its block of D.
  const float4 i0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + col0 + 8 * lane));
  const float4 i1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + col0 + 8 * lane + 4));
  uint4 raw[kRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = warp + 8 * i;
    raw[i] = row < p.M ? __ldg(reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(row) * p.K + col0) + lane)
                       : make_uint4(0u, 0u, 0u, 0u);
  }
  const int mt = warp >> 2, nt_count = p.r >> 3;
  const bool d_rows = R_PAD > 0 && mt * 16 < p.M;
  uint2 bfr[kTilesPerWarp][SMALL_ACT_COLS / 16];
  const uint2* f = reinterpret_cast<const uint2*>(p.L1f);
#pragma unroll
  for (int u = 0; u < kTilesPerWarp; ++u) {
    const int t = (warp & 3) + 4 * u;
#pragma unroll
    for (int ks = 0; ks < SMALL_ACT_COLS / 16; ++ks)
      bfr[u][ks] = (d_rows && t < nt_count)
                       ? __ldg(f + ((static_cast<size_t>(col0 / 16 + ks) * nt_count + t) * 32 + lane))
                       : make_uint2(0u, 0u);
  }

  const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = warp + 8 * i;
    uint32_t sc = 0;
    uint4 hx = make_uint4(0u, 0u, 0u, 0u);
    if (row < p.M) {   // uniform over the warp
      const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
      float v[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[2 * u] = __fmul_rn(__uint_as_float(w4[u] << 16), inv[2 * u]);
        v[2 * u + 1] = __fmul_rn(__uint_as_float(w4[u] & 0xFFFF0000u), inv[2 * u + 1]);
      }
      const uint32_t codes = nvfp4_quant_half_block(v, sc);
      *reinterpret_cast<uint32_t*>(p.x_codes + static_cast<size_t>(row) * (p.K / 2) + col0 / 2 + 4 * lane) = codes;
      hx = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
    }
    // the four block scales of a 64-column group sit on lanes 8 g, 8 g + 2, 8 g + 4, 8 g + 6
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 2);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 4);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 6);
    if ((lane & 7) == 0)
      p.sfb[(col0 / 64 + lane / 8) * SMALL_MAX_TOKENS + row] = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
    *reinterpret_cast<uint4*>(xs + row * kRowStride + 8 * lane) = hx;
  }
  __syncthreads();
  // partial D of this CTA's columns: warp w takes the 16-row block w / 4 and
  // the 8-column blocks w % 4 (+ 4) of D
  const uint32_t xs_u = smem_u32(xs);
#pragma unroll
  for (int u = 0; u < kTilesPerWarp; ++u) {
    const int t = (warp & 3) + 4 * u;
    if (!d_rows || t >= nt_count) break;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int ks = 0; ks < SMALL_ACT_COLS / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(xs_u + static_cast<uint32_t>(((16 * mt + (lane & 15)) * kRowStride + 16 * ks + 8 * (lane >> 4)) * 2),
                  a0, a1, a2, a3);
      mma_bf16_16816(acc, a0, a1, a2, a3, bfr[u][ks].x, bfr[u][ks].y);
    }
    const int rlo = 16 * mt + (lane >> 2), col = 8 * t + 2 * (lane & 3);
    float* out = p.dpart + static_cast<size_t>(blockIdx.x) * p.M * p.r;
    if (rlo < p.M) {
      out[static_cast<size_t>(rlo) * p.r + col] = acc[0];
      out[static_cast<size_t>(rlo) * p.r + col + 1] = acc[1];
    }
    if (rlo + 8 < p.M) {
      out[static_cast<size_t>(rlo + 8) * p.r + col] = acc[2];
      out[static_cast<size_t>(rlo + 8) * p.r + col + 1] = acc[3];
    }
  }
}

struct SmallGemmParams {
  const uint8_t* w_scales;    // weight scales, tile layout (128-row tiles, contiguous over K)
  const uint8_t* x_codes;     // activation codes M x K/2 (act_quant_small_kernel)
  const uint32_t* sfb;        // activation scales [K/64][32] (act_quant_small_kernel)
  const float* dpart;         // [K/256][M][r] (act_quant_small_kernel)
  const uint16_t* bias;       // N, or null
  uint16_t* Y;                // M x N row-major, or head-major [N / head_dim][M][head_dim]
  int M, N, K, r, head_dim;
  int stages;                 // depth of the weight ring
  uint32_t off_act, off_sfb, off_sfa, off_l2, off_d, off_bar;   // shared-memory layout (small_gemm_layout)
};

// Shared memory of fp4_gemm_small_m_kernel<TN, R_PAD> for a given K and ring
// depth: the weight ring, the activation codes of all of K (TN rows x 128 B
// per 256 columns, the MMA's K-major 128-byte-swizzled layout), the
// activation scale words (128 B per 64 columns), the tile's weight scales
// (512 B per 64 columns), the L2^T tile (128 x R_PAD bf16) and
// the D tile (TN x R_PAD bf16), each 1024-aligned, then the barriers.
// Returns the total including the alignment slack.
__host__ __device__ inline uint32_t small_gemm_layout(int TN, int R_PAD, int K, int stages, SmallGemmParams* p) {
  auto up = [](uint32_t x) { return (x + 1023u) & ~1023u; };
  const uint32_t nkb = static_cast<uint32_t>(K) / 256u;
  uint32_t off = static_cast<uint32_t>(stages) * SMALL_STAGE_BYTES;
  const uint32_t act = off;
  off = up(off + nkb * static_cast<uint32_t>(TN) * 128u);
  const uint32_t sfb = off;
  off = up(off + static_cast<uint32_t>(K) / 64u * SMALL_MAX_TOKENS * 4u);
  const uint32_t sfa = off;
  off = up(off + static_cast<uint32_t>(K) / 64u * 512u);
  const uint32_t l2 = off;
  off = up(off + 128u * static_cast<uint32_t>(R_PAD) * 2u);
  const uint32_t d = off;
  off = up(off + static_cast<uint32_t>(TN) * static_cast<uint32_t>(R_PAD) * 2u);
  const uint32_t bar = off;
  off += (2 * SMALL_MAX_STAGES + 9) * 8 + 16;
  if (p != nullptr) {
    p->off_act = act;
    p->off_sfb = sfb;
    p->off_sfa = sfa;
    p->off_l2 = l2;
    p->off_d = d;
    p->off_bar = bar;
    p->stages = stages;
  }
  return off + 1024u;
}

// Warp roles (256 threads): warp 0 streams the weight (TMA) from its first
// instruction; warp 1 issues the MMAs; warp 2 owns tensor memory; warps 2-7
// fetch the activation codes into shared memory once the activation kernel
// has completed (16-byte cp.async copies through the load/store unit, which
// do not queue behind the weight stream in the TMA engine); warps 4-7 also
// move the scales into
// tensor memory (each its lane quarter), sum the D partials and run the
// epilogue.  Two CTAs' worth of registers (<= 128 per thread), so that a CTA
// of the activation kernel can share an SM with this kernel's CTA.
template <int TN, int R_PAD>
__global__ void __launch_bounds__(SMALL_THREADS, 2)
    fp4_gemm_small_m_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_l2,
                            const SmallGemmParams p) {
  static_assert(TN == 16 || TN == 32, "token tile");
  constexpr uint32_t kLRLayout = (R_PAD == 64 ? LAYOUT_SW128 : R_PAD == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
  constexpr uint32_t kLRSwz = (R_PAD == 64 ? 3u : R_PAD == 32 ? 2u : 1u);
  constexpr uint32_t kLRSbo = 8 * R_PAD * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t base = smem_u32(smem);
  const int S = p.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  // bars: [0, 8) full, [8, 16) empty, 16 sfa_full, 17 l2_full, 18 act_ready,
  // 19 sf_ready, 20 d_ready, 21 acc_full, 22 drain, 23 tmem_done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SMALL_MAX_STAGES + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + SMALL_MAX_STAGES + s); };
  const uint32_t sfa_full = smem_u32(bars + 16), l2_full = smem_u32(bars + 17), act_ready = smem_u32(bars + 18);
  const uint32_t sf_ready = smem_u32(bars + 19), d_ready = smem_u32(bars + 20), acc_full = smem_u32(bars + 21);
  const uint32_t drain_bar = smem_u32(bars + 22), tmem_done = smem_u32(bars + 23);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128;
  const int nkb = p.K / 256, nk64 = p.K / 64;
  const uint32_t sfa_col = small_sfa_col(p.K);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SMALL_MAX_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(sfa_full, 1);
    mbar_init(l2_full, 1);
    mbar_init(act_ready, 6);   // warps 2-7
    mbar_init(sf_ready, 4);
    mbar_init(d_ready, 4);
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    mbar_init(tmem_done, 5);   // the MMA thread and the four epilogue warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), SMALL_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Only the weight (never written by the kernel before this one) is read
    // here, so none of it waits for the activation kernel.
    if (lane == 0) {
      tma_prefetch_desc(&tm_w);
      if (R_PAD > 0) tma_prefetch_desc(&tm_l2);
      // the tile's weight scales for all of K: one contiguous run of 128-row tiles
      const uint32_t sfa_bytes = static_cast<uint32_t>(nk64) * 512u;
      mbar_arrive_expect_tx(sfa_full, sfa_bytes);
      bulk_load(base + p.off_sfa, p.w_scales + static_cast<size_t>(n0 / 128) * sfa_bytes, sfa_bytes, sfa_full);
      if (R_PAD > 0) {
        mbar_arrive_expect_tx(l2_full, 128u * R_PAD * 2u);
        tma_load_2d(base + p.off_l2, &tm_l2, l2_full, 0, n0);
      }
      // At most SMALL_IN_FLIGHT stages are requested and not yet landed: all
      // SMs together then keep enough reads in flight to saturate HBM, but not
      // so many that every other request of the chip (the activation kernel's
      // among them) waits behind the weight stream's queue.
      int kb = 0;
      bool ok = true;
      for (; kb < nkb; ++kb) {
        const int s = kb % S;
        if (kb >= S && !mbar_wait(empty_bar(s), ((kb / S) & 1) ^ 1, abort_flag, KID_SMALL_GEMM, 1)) {
          ok = false;
          break;
        }
        const int k_landed = kb - SMALL_IN_FLIGHT;
        if (k_landed >= 0 &&
            !mbar_wait(full_bar(k_landed % S), (k_landed / S) & 1, abort_flag, KID_SMALL_GEMM, 7)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full_bar(s), SMALL_STAGE_BYTES);
        tma_load_2d(base + s * SMALL_STAGE_BYTES, &tm_w, full_bar(s), kb * 128, n0);
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        for (int k = (kb > S ? kb - S : 0); k < kb; ++k) mbar_wait_drain(full_bar(k % S), (k / S) & 1);
        mbar_wait_drain(sfa_full, 0);
        if (R_PAD > 0) mbar_wait_drain(l2_full, 0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(sf_ready, 0, abort_flag, KID_SMALL_GEMM, 2) &&
                mbar_wait(act_ready, 0, abort_flag, KID_SMALL_GEMM, 3);
      bool any = false;
      if (ok) {
        tc_fence_after();
        const uint32_t idf = idesc_nvfp4(128, TN);
        const uint32_t acc = tmem_base + SMALL_ACC_COL;
        uint32_t accumulate = 0;
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = kb % S;
          if (!mbar_wait(full_bar(s), (kb / S) & 1, abort_flag, KID_SMALL_GEMM, 4)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = make_smem_desc(base + s * SMALL_STAGE_BYTES, LAYOUT_SW128, 1024, 0);
          const uint64_t bd = make_smem_desc(base + p.off_act + kb * (TN * 128), LAYOUT_SW128, 1024, 0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t j = 4u * kb + i;   // 64-column block
            tc_mma_nvfp4(acc, ad + 2 * i, bd + 2 * i, idf, tmem_base + sfa_col + 4u * j,
                         tmem_base + SMALL_SFB_COL + 4u * j, accumulate);
            accumulate = 1;
          }
          any = true;
          tc_commit(empty_bar(s));
        }
        if (ok && R_PAD > 0) {
          // the low-rank term: acc[n][t] += sum_j L2^T[n][j] D[t][j]
          ok = mbar_wait(l2_full, 0, abort_flag, KID_SMALL_GEMM, 5) &&
               mbar_wait(d_ready, 0, abort_flag, KID_SMALL_GEMM, 6);
          if (ok) {
            tc_fence_after();
            const uint32_t idb = idesc_bf16(128, TN);
            const uint64_t ad = make_smem_desc(base + p.off_l2, kLRLayout, kLRSbo, 0);
            const uint64_t bd = make_smem_desc(base + p.off_d, kLRLayout, kLRSbo, 0);
#pragma unroll
            for (int kk = 0; kk < R_PAD / 16; ++kk) tc_mma_bf16(acc, ad + 2 * kk, bd + 2 * kk, idb, 1);
          }
        }
        if (ok) tc_commit(acc_full);
      }
      if (*abort_flag && any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0);
      }
      mbar_arrive(tmem_done);
    }
  } else {
    // --------------------------------------------- warps 2-7 (and 4-7 alone)
    const bool quarter = warp >= 4;   // warps 4-7: one tensor-memory lane quarter each
    const int q = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    bool ok = true;
    if (quarter) {
      // weight scales: column sfa_col + 4 j + g of lane 32 q + l holds the 4
      // scales of row 32 g + l for 64-column block j -- the 16 bytes at 16 l
      // of the block's 512-byte tile (each lane quarter writes the same replica)
      ok = mbar_wait(sfa_full, 0, abort_flag, KID_SMALL_GEMM, 10);
      if (ok) {
        const uint8_t* sa = smem + p.off_sfa + lane * 16;
        for (int j0 = 0; j0 < nk64; j0 += 4) {
          uint32_t v[16];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint4 x = *reinterpret_cast<const uint4*>(sa + (j0 + jj) * 512);
            v[4 * jj] = x.x; v[4 * jj + 1] = x.y; v[4 * jj + 2] = x.z; v[4 * jj + 3] = x.w;
          }
          tmem_st_32x32b_x16(tmem_base + lane_addr + sfa_col + 4u * j0, v);
        }
      }
    }
    // The activation kernel's outputs are complete and visible after this.
    // Its codes go to the B operand (K-major, 128-byte swizzle, TN rows per
    // 256-column block, rows >= M zero) and its scale words to a staging
    // area, by 16-byte cp.async copies of warps 2-7 through the load/store
    // unit (they do not queue behind the weight stream in the TMA engine).
    // 16-byte chunk c of token t in block kb lands at
    // kb TN 128 + (t / 8) 1024 + (t % 8) 128 + (c ^ t % 8) 16.
    pdl_wait();
    {
      const int tid = threadIdx.x - 64;   // 0 .. 191
      const int nchunks = nkb * TN * 8;
      for (int e = tid; e < nchunks; e += 192) {
        const int kb = e / (TN * 8), t = (e / 8) % TN, c = e % 8;
        const uint8_t* src = p.x_codes + static_cast<size_t>(t < p.M ? t : 0) * (p.K / 2) + kb * 128 + c * 16;
        cp_async_16(base + p.off_act + kb * (TN * 128) + (t / 8) * 1024 + (t % 8) * 128 + ((c ^ (t % 8)) * 16), src,
                    t < p.M ? 16u : 0u);
      }
      const int nwords16 = nk64 * SMALL_MAX_TOKENS / 4;
      for (int e = tid; e < nwords16; e += 192) cp_async_16(base + p.off_sfb + e * 16, p.sfb + 4 * e, 16u);
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(act_ready);
    }
    if (quarter) {
      // activation scales: column 32 + 4 j of lane l = token l's 4 scales of
      // block j (the group's other three columns are zero)
      ok = ok && mbar_wait(act_ready, 0, abort_flag, KID_SMALL_GEMM, 12);
      if (ok) {
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(smem + p.off_sfb) + lane;
        for (int j0 = 0; j0 < nk64; j0 += 4) {
          uint32_t v[16];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            v[4 * jj] = sb[(j0 + jj) * SMALL_MAX_TOKENS];
            v[4 * jj + 1] = 0u; v[4 * jj + 2] = 0u; v[4 * jj + 3] = 0u;
          }
          tmem_st_32x32b_x16(tmem_base + lane_addr + SMALL_SFB_COL + 4u * static_cast<uint32_t>(j0), v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_ready);
      }
      if (ok && R_PAD > 0) {
        // D = bf16(sum of the K/256 partials, in slice order), written as the
        // K-major B operand (TN rows x R_PAD, swizzled like the L2^T tile);
        // columns >= r and rows >= M are zero
        uint8_t* dt = smem + p.off_d;
        constexpr int kMaxSlices = SMALL_MAX_K / SMALL_ACT_COLS;
        for (int e = q * 32 + lane; e < TN * R_PAD; e += 128) {
          constexpr int kRp = R_PAD > 0 ? R_PAD : 1;   // (this branch runs only with R_PAD > 0)
          const int t = e / kRp, j = e % kRp;
          float v = 0.0f;
          if (t < p.M && j < p.r) {
            // all slices' partials are loaded first (one round trip), then
            // added in slice order
            float part[kMaxSlices];
#pragma unroll
            for (int s = 0; s < kMaxSlices; ++s)
              part[s] = s < nkb ? __ldcg(p.dpart + (static_cast<size_t>(s) * p.M + t) * p.r + j) : 0.0f;
#pragma unroll
            for (int s = 0; s < kMaxSlices; ++s)
              if (s < nkb) v += part[s];
          }
          *reinterpret_cast<uint16_t*>(dt + swz(static_cast<uint32_t>(t * R_PAD * 2 + j * 2), kLRSwz)) =
              static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(d_ready);
      }
      if (ok) {
        // epilogue: lane = weight row n, columns = tokens
        const int n = n0 + q * 32 + lane;
        const float b = p.bias != nullptr ? bf16_bits_to_f32(p.bias[n]) : 0.0f;
        if (mbar_wait(acc_full, 0, abort_flag, KID_SMALL_GEMM, 11)) {
          tc_fence_after();
          uint32_t v[TN];
          if constexpr (TN == 32) tmem_ld_32x32b_x32(tmem_base + lane_addr + SMALL_ACC_COL, v);
          else tmem_ld_32x32b_x16(tmem_base + lane_addr + SMALL_ACC_COL, v);
          tmem_ld_wait();
          uint16_t* col = p.head_dim == 0
                              ? p.Y + n
                              : p.Y + static_cast<size_t>(n / p.head_dim) * p.M * p.head_dim + n % p.head_dim;
          const size_t stride = p.head_dim == 0 ? static_cast<size_t>(p.N) : static_cast<size_t>(p.head_dim);
#pragma unroll
          for (int t = 0; t < TN; ++t)
            if (t < p.M)
              col[t * stride] = static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[t]) + b, 0.0f) & 0xFFFFu);
        }
      }
      // this warp's tensor-memory accesses are over (each ld / st waited)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_done);
    }
  }

  // Every lane of every warp meets here (a warp whose elected lane worked
  // alone reconverges first), and the allocator frees tensor memory only once
  // the MMAs have completed and the epilogue has read the accumulator.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    mbar_wait_drain(tmem_done, 0, 4 * kWaitLimitNs);
    tc_fence_after();
    tmem_dealloc(tmem_base, SMALL_TMEM_COLS);
  }
}

}  // namespace svdq
