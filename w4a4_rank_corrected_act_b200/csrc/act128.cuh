// act128.cuh -- the activation kernel of the layer's forward for r > 0, with
// the rank-r down-projection on the 5th-generation tensor cores.
//
// It computes what act_quant_kernel computes -- for Xhat = f32(X * inv_lambda)
// the NVFP4 codes and E4M3 block scales (the "A4" of W4A4, aiphreaks.com
// "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers", section
// "Technical Breakdown and Performance Metrics") and D = bf16(bf16(Xhat) . L1),
// the input of the 16-bit low-rank branch (imaginepro.ai practical guide,
// section "Under the Hood") -- with a different split of the work:
//
//   * a CTA owns 128 token rows and one of ks equal K ranges; its 8 quantiser
//     warps (16 rows each) walk the range's 64-column stages together, so
//     one TMA box brings a 128 x 64 bf16 tile and one more the matching
//     R_PAD x 64 slice of L1^T;
//   * each warp quantises its rows of the stage in registers (the same
//     arithmetic as act_quant_kernel) and writes bf16(-Xhat) back in place,
//     which is then exactly the K-major operand of a tcgen05 bf16 MMA
//     (M = 128, N = R_PAD); one thread issues the stage's four K = 16 MMAs
//     into a tensor-memory accumulator, so D costs the quantiser warps no
//     instruction beyond the write-back;
//   * with ks > 1 every CTA of a row block publishes its float32 partial of D
//     (workspace, release flag), waits for the others, and adds the ks
//     partials in K order for its own slice of D's columns.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr int A128_ROWS = 128;
constexpr int A128_QWARPS = 8;                          // quantiser warps, 16 rows each
constexpr int A128_THREADS = (A128_QWARPS + 1) * 32;    // + the TMA / MMA warp
constexpr int A128_STAGES = 4;
constexpr int A128_MAX_KS = 8;
constexpr uint32_t A128_X_BYTES = A128_ROWS * 128;      // 128 rows x 64 bf16
enum : uint32_t { KID_ACT128 = 8 };

template <int R_PAD>
struct A128Cfg {
  static_assert(R_PAD == 16 || R_PAD == 32 || R_PAD == 64, "rank padding");
  static constexpr uint32_t kL1Bytes = R_PAD * 128;              // R_PAD rows x 64 bf16
  static constexpr uint32_t kStage = A128_X_BYTES + kL1Bytes;      // a multiple of 1024
  static constexpr uint32_t kTmemCols = R_PAD <= 32 ? 32 : 64;
  static constexpr uint32_t kTab = 128 * 8;
  static constexpr uint32_t kBars = (3 * A128_STAGES + 3) * 8;
  static constexpr uint32_t kBytes = A128_STAGES * kStage + kTab + kBars + 16 + 1024;
};

struct A128Params {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  uint16_t* D;
  float* dpart;              // [M_pad / 128][ks][r][128] float32 partials of D (ks > 1)
  unsigned long long* flags; // [M_pad / 128][ks]: the epoch once partial (row block, kp) is written
  unsigned long long epoch;  // this call's value of a published flag
  int M, K, r, M_pad, ks;
  float* zero_ptr;           // optional: zero_count floats set to 0 by the grid
  int zero_count;
};

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int R_PAD>
__global__ void __launch_bounds__(A128_THREADS, 2)
    act128_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t,
                  const A128Params p) {
  using Cfg = A128Cfg<R_PAD>;
  constexpr int S = A128_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float2* tab = reinterpret_cast<float2*>(smem + S * Cfg::kStage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStage + Cfg::kTab);
  // bars: [0, S) full, [S, 2S) quantised (8 warps), [2S, 3S) empty (MMA done),
  // 3S acc_full, 3S + 1 tmem_done (the four epilogue warps), 3S + 2 drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t smem_base = smem_u32(smem);
  auto stage = [&](int s) { return smem_base + static_cast<uint32_t>(s) * Cfg::kStage; };
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto quant_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + 2 * S + s); };
  const uint32_t acc_full = smem_u32(bars + 3 * S), tmem_done = smem_u32(bars + 3 * S + 1);
  const uint32_t drain_bar = smem_u32(bars + 3 * S + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x / p.ks, kp = blockIdx.x % p.ks;
  const int row0 = rb * A128_ROWS;
  const int nsub = p.K / 64 / p.ks;     // 64-column stages of this CTA's K range
  const int sub0 = kp * nsub;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(quant_bar(s), A128_QWARPS);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(tmem_done, 4);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int c = threadIdx.x; c < 128; c += A128_THREADS) tab[c] = e4m3_table_entry(c);
  if (warp == A128_QWARPS) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // programmatic dependent launch: nothing in global memory is touched before
  // the previous kernel of the stream has completed; the next may start now
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * A128_THREADS + threadIdx.x; i < p.zero_count; i += gridDim.x * A128_THREADS)
    p.zero_ptr[i] = 0.0f;

  if (warp == A128_QWARPS) {
    // ------------------------------------------------ TMA producer + MMA issuer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_l1t);
      int issued = 0;
      auto load = [&](int j) {
        const int s = j % S;
        mbar_arrive_expect_tx(full_bar(s), Cfg::kStage);
        tma_load_2d(stage(s), &tm_x, full_bar(s), (sub0 + j) * 64, row0);
        tma_load_2d(stage(s) + A128_X_BYTES, &tm_l1t, full_bar(s), (sub0 + j) * 64, 0);
        issued = j + 1;
      };
      for (int j = 0; j < nsub && j < S; ++j) load(j);
      const uint32_t idesc = idesc_bf16(A128_ROWS, R_PAD);
      bool ok = true, any = false;
      for (int j = 0; j < nsub; ++j) {
        const int s = j % S;
        if (!mbar_wait(quant_bar(s), static_cast<uint32_t>(j / S) & 1u, abort_flag, KID_ACT128, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = make_smem_desc(stage(s), LAYOUT_SW128, 1024, 0);
        const uint64_t bd = make_smem_desc(stage(s) + A128_X_BYTES, LAYOUT_SW128, 1024, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem_base, ad + 2 * kk, bd + 2 * kk, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty_bar(s));
        any = true;
        // the stage of the previous sub-tile takes sub-tile j - 1 + S once its MMAs are done
        if (j >= 1 && j - 1 + S < nsub) {
          const int s1 = (j - 1) % S;
          if (!mbar_wait(empty_bar(s1), static_cast<uint32_t>((j - 1) / S) & 1u, abort_flag, KID_ACT128, 2)) {
            ok = false;
            break;
          }
          load(j - 1 + S);
        }
      }
      if (ok && any) tc_commit(acc_full);
      if (*abort_flag) {
        // no MMA still reads shared memory or writes tensor memory, and no
        // copy still lands, when the CTA exits
        if (any) {
          tc_commit(drain_bar);
          mbar_wait_drain(drain_bar, 0);
        }
        for (int j = (issued > S ? issued - S : 0); j < issued; ++j)
          mbar_wait_drain(full_bar(j % S), static_cast<uint32_t>(j / S) & 1u);
      }
    }
  } else {
    // ------------------------------------------------------- quantiser warps
    // Lane l quantises the 16-column block l % 4 of rows l / 4 and l / 4 + 8 of
    // the warp's 16: a whole block per thread, so no lane pair exchanges its
    // maximum.  The block's two 16-byte chunks sit at toff and toff ^ 16 (the
    // 128-byte swizzle keeps them in the same row, next to each other).
    const int blk = lane & 3, rsub = lane >> 2;
    const uint32_t half_k = static_cast<uint32_t>(p.K) >> 1;
    uint32_t toff[2];
    uint8_t* cptr[2];
    uint8_t* sptr[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int row = warp * 16 + i * 8 + rsub, grow = row0 + row;
      toff[i] = swz(static_cast<uint32_t>(row * 128 + blk * 32), 3);
      cptr[i] = grow < p.M ? p.x_codes + static_cast<size_t>(grow) * half_k + 8 * blk : nullptr;
      sptr[i] = p.x_scales + sf_offset(static_cast<uint32_t>(grow), 0, static_cast<uint32_t>(p.K)) + blk;
    }
    float4 ni[4];
    auto load_inv = [&](int j) {
      const float4* src = reinterpret_cast<const float4*>(p.inv_lambda + (sub0 + j) * 64 + 16 * blk);
#pragma unroll
      for (int u = 0; u < 4; ++u) ni[u] = __ldg(src + u);
    };
    if (nsub > 0) load_inv(0);
    const float y6 = tab[0x4C].y;   // E4M3 code 0x4C is 6.0: RN(1/6)
    const uint64_t six = f32x2_pack(6.0f, 6.0f), neg_y6 = f32x2_pack(-y6, -y6);
    for (int j = 0; j < nsub; ++j) {
      const int s = j % S;
      const int col0 = (sub0 + j) * 64;
      uint64_t ninv2[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        ninv2[2 * u] = f32x2_pack(-ni[u].x, -ni[u].y);
        ninv2[2 * u + 1] = f32x2_pack(-ni[u].z, -ni[u].w);
      }
      if (j + 1 < nsub) load_inv(j + 1);
      if (!mbar_wait(full_bar(s), static_cast<uint32_t>(j / S) & 1u, abort_flag, KID_ACT128, 3)) break;
      uint8_t* tile = smem + static_cast<uint32_t>(s) * Cfg::kStage;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 r0 = *reinterpret_cast<const uint4*>(tile + toff[i]);
        const uint4 r1 = *reinterpret_cast<const uint4*>(tile + (toff[i] ^ 16u));
        const uint32_t w8[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        // -Xhat = f32(x * (-1/lambda)), element 2u in the low half of pair u
        uint64_t nxh[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          nxh[u] = f32x2_mul(f32x2_pack(__uint_as_float(w8[u] << 16), __uint_as_float(w8[u] & 0xFFFF0000u)),
                             ninv2[u]);
        uint32_t sc;
        const uint64_t codes = nvfp4_quant_block16_x2(nxh, tab, six, neg_y6, sc);
        if (cptr[i] != nullptr) *reinterpret_cast<uint64_t*>(cptr[i] + (col0 >> 1)) = codes;
        sptr[i][static_cast<size_t>(col0 >> 6) * 512] = static_cast<uint8_t>(sc);
        // bf16(-Xhat) = -bf16(Xhat) in place: the MMA's A operand (negated back at the end)
        uint32_t o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float lo, hi;
          f32x2_unpack(nxh[u], lo, hi);
          o[u] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4*>(tile + toff[i]) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(tile + (toff[i] ^ 16u)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      // the generic-proxy writes of the tile before the tensor core reads it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(quant_bar(s));
    }
  }

  // ------------------------------------------------------------------ D
  // Warps 0-3 read the CTA's accumulator (row 32 w + lane of the block).  With
  // ks == 1 they write D.  Otherwise each CTA publishes its float32 partial
  // ([row block][kp][j][row], rows contiguous) with a release flag, waits for
  // the row block's ks flags, and warps 0-7 add the ks partials in K order for
  // the CTA's slice of D's columns, [kp r / ks, (kp + 1) r / ks).
  bool live = false;
  if (warp < 4) {
    const bool ok = nsub > 0 && mbar_wait(acc_full, 0, abort_flag, KID_ACT128, 4);
    uint32_t acc[R_PAD];
    if (ok) {
      tc_fence_after();
      const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
      for (int c = 0; c < R_PAD / 16; ++c)
        tmem_ld_32x32b_x16(tmem_base + lane_addr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(acc + 16 * c));
      tmem_ld_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tmem_done);
    live = ok && !*abort_flag;
    const int rib = warp * 32 + lane, row = row0 + rib;
    if (p.ks == 1) {
      if (live && row < p.M) {
        uint16_t* dst = p.D + static_cast<size_t>(row) * p.r;
#pragma unroll
        for (int j = 0; j < R_PAD; ++j)
          if (j < p.r) dst[j] = static_cast<uint16_t>(pack_bf16x2(-__uint_as_float(acc[j]), 0.0f) & 0xFFFFu);
      }
    } else if (live) {
      float* dst = p.dpart + static_cast<size_t>(rb * p.ks + kp) * p.r * A128_ROWS + rib;
#pragma unroll
      for (int j = 0; j < R_PAD; ++j)
        if (j < p.r) dst[static_cast<size_t>(j) * A128_ROWS] = -__uint_as_float(acc[j]);
    }
  }
  if (p.ks > 1 && warp < A128_QWARPS) {
    named_barrier_sync(1, A128_QWARPS * 32);   // the CTA's partial is written (warps 0-3)
    unsigned long long* fl = p.flags + static_cast<size_t>(rb) * p.ks;
    if (threadIdx.x == 0) {
      if (!*abort_flag) {
        __threadfence();
        st_release_gpu_u64(fl + kp, p.epoch);
        const unsigned long long t0 = globaltimer();
        for (int k = 0; k < p.ks; ++k) {
          while (ld_acquire_gpu_u64(fl + k) != p.epoch) {
            if (*abort_flag || globaltimer() - t0 > kWaitLimitNs) {
              if (!*abort_flag) report_timeout(KID_ACT128, 5);
              *abort_flag = 1;
              break;
            }
          }
          if (*abort_flag) break;
        }
      }
    }
    named_barrier_sync(1, A128_QWARPS * 32);   // every partial of the row block is published
    if (!*abort_flag) {
      for (int k = 0; k < p.ks; ++k) (void)ld_acquire_gpu_u64(fl + k);
      const int jlo = kp * p.r / p.ks, jhi = (kp + 1) * p.r / p.ks;
      const int npairs = (jhi - jlo) * A128_ROWS;
      const float* part = p.dpart + static_cast<size_t>(rb * p.ks) * p.r * A128_ROWS;
      for (int q = threadIdx.x; q < npairs; q += A128_QWARPS * 32) {
        const int rib = q % A128_ROWS, j = jlo + q / A128_ROWS;
        float t[A128_MAX_KS];
#pragma unroll
        for (int k = 0; k < A128_MAX_KS; ++k)
          t[k] = k < p.ks ? part[(static_cast<size_t>(k) * p.r + j) * A128_ROWS + rib] : 0.0f;
        float v = t[0];
#pragma unroll
        for (int k = 1; k < A128_MAX_KS; ++k)
          if (k < p.ks) v += t[k];
        const int row = row0 + rib;
        if (row < p.M) p.D[static_cast<size_t>(row) * p.r + j] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
      }
    }
  }
  (void)live;

  // tensor memory is freed once every epilogue warp has read it (and with it,
  // every MMA has completed: they waited for acc_full)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == A128_QWARPS) {
    mbar_wait_drain(tmem_done, 0, 4 * kWaitLimitNs);
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace svdq
