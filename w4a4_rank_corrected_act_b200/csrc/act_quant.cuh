// act_quant.cuh -- the activation kernel of the SVDQuant W4A4 linear layer.
//
// One HBM pass over X (M x K bf16) produces, for the smoothed activation
// Xhat = f32(X * inv_lambda):
//   * its NVFP4 codes (M x K/2) and E4M3 block scales (scale-factor tile layout),
//     the "A4" half of W4A4 (aiphreaks.com "Bringing Nunchaku 4-bit Diffusion
//     Inference to Diffusers", section "Technical Breakdown and Performance
//     Metrics": activations quantised to 4 bits after the outliers moved out);
//   * the rank-r down-projection D = bf16(bf16(Xhat) . L1) that feeds the
//     16-bit low-rank branch (same section; imaginepro.ai practical guide,
//     section "Under the Hood": the low-rank correction runs in higher precision).
//
// Design (B200): each CTA owns 32 token rows and streams K in 256-wide chunks
// through a TMA ring (X tile 32 x 256 bf16 as four 128-byte-swizzled boxes, plus
// the matching 256 x r slice of L1).  Eight consumer warps quantise in
// registers (two lanes per 16-element block, one shuffle for the absmax) and
// write bf16(Xhat) back into the swizzled tile in place; the same tile then
// feeds ldmatrix + mma.sync for D, so X is read from HBM exactly once.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr int ACT_BM = 32;          // token rows per CTA
constexpr int ACT_KC = 256;         // K elements per pipeline chunk
constexpr int ACT_CONSUMER_WARPS = 8;
constexpr int ACT_THREADS = (ACT_CONSUMER_WARPS + 1) * 32;
constexpr uint32_t ACT_X_TILE_BYTES = ACT_BM * ACT_KC * 2;   // 16 KB
constexpr uint32_t ACT_X_BOX_BYTES = ACT_BM * 128;           // 32 rows x 64 bf16

struct ActParams {
  const float* inv_lambda;
  uint8_t* x_codes;
  uint8_t* x_scales;
  uint16_t* D;
  int M, K, r, M_pad, stages;
};

template <int R_PAD>
struct ActSmem {
  static constexpr uint32_t kL1Tile = ACT_KC * R_PAD * 2;
  static constexpr uint32_t kStage = ACT_X_TILE_BYTES + kL1Tile;
  static constexpr uint32_t kRed = (R_PAD > 0 ? 4 * ACT_BM * R_PAD * 4 : 0);
  static __host__ __device__ uint32_t bytes(int stages) {
    // stages, reduction buffer, barriers (2 per stage) + abort flag, 1 KB alignment slack
    return stages * kStage + kRed + 2 * stages * 8 + 16 + 1024;
  }
};

template <int R_PAD>
__device__ __forceinline__ void act_zero_pad_rows(const ActParams& p, int row0) {
  // Rows row0..row0+31 lie entirely in [M, M_pad): write their scale entries as 0.
  const int kb64 = p.K / 64;
  for (int idx = threadIdx.x; idx < kb64 * ACT_BM; idx += blockDim.x) {
    const int kb = idx / ACT_BM, i = idx % ACT_BM;
    const uint32_t row = static_cast<uint32_t>(row0 + i);
    *reinterpret_cast<uint32_t*>(p.x_scales + sf_offset(row, kb * 4, p.K)) = 0u;
  }
}

template <int R_PAD>
__global__ void __launch_bounds__(ACT_THREADS, 1)
    act_quant_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_l1, const ActParams p) {
  constexpr uint32_t kL1B = (R_PAD == 64 ? 3 : R_PAD == 32 ? 2 : 1);   // L1 tile swizzle bits
  constexpr uint32_t kStage = ActSmem<R_PAD>::kStage;
  constexpr int kNT = R_PAD / 8;                                        // n8 tiles of D

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  float* red = reinterpret_cast<float*>(smem + stages * kStage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * kStage + ActSmem<R_PAD>::kRed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * stages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * ACT_BM;
  if (row0 >= p.M) {
    act_zero_pad_rows<R_PAD>(p, row0);
    return;
  }
  const int nchunks = p.K / ACT_KC;
  const uint32_t smem_base = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + stages + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), ACT_CONSUMER_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == ACT_CONSUMER_WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (R_PAD > 0) tma_prefetch_desc(&tm_l1);
      const uint32_t tx = ACT_X_TILE_BYTES + (R_PAD > 0 ? ActSmem<R_PAD>::kL1Tile : 0u);
      int c = 0;
      for (; c < nchunks; ++c) {
        const int s = c % stages;
        const uint32_t ph = (c / stages) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1, abort_flag, KID_ACT, 1)) break;
        const uint32_t st = smem_base + s * kStage;
        mbar_arrive_expect_tx(full_bar(s), tx);
#pragma unroll
        for (int b = 0; b < 4; ++b)
          tma_load_2d(st + b * ACT_X_BOX_BYTES, &tm_x, full_bar(s), c * ACT_KC + b * 64, row0);
        if (R_PAD > 0) tma_load_2d(st + ACT_X_TILE_BYTES, &tm_l1, full_bar(s), 0, c * ACT_KC);
      }
      if (*abort_flag) {
        // let copies already issued land before the CTA exits
        const int first = c > stages ? c - stages : 0;
        for (int k = first; k < c; ++k)
          mbar_wait_drain(full_bar(k % stages), (k / stages) & 1);
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    float acc[kNT > 0 ? kNT : 1][4];
#pragma unroll
    for (int t = 0; t < (kNT > 0 ? kNT : 1); ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;
    const int mt = warp & 1, kg = warp >> 1;     // D tiling: m16 tile, quarter of each chunk
    const int box = lane >> 3, chunk16 = lane & 7;
    const uint32_t half_k = static_cast<uint32_t>(p.K) / 2;

    for (int c = 0; c < nchunks; ++c) {
      const int s = c % stages;
      const uint32_t ph = (c / stages) & 1;
      if (!mbar_wait(full_bar(s), ph, abort_flag, KID_ACT, 3)) break;
      uint8_t* xs = smem + s * kStage;
      const int k0 = c * ACT_KC;
      // per-lane smoothing factors for columns k0 + 8*lane .. +7
      const float4 i0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0 + 8 * lane));
      const float4 i1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0 + 8 * lane + 4));
      const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};

#pragma unroll
      for (int rr = 0; rr < ACT_BM / ACT_CONSUMER_WARPS; ++rr) {
        const int row = warp * (ACT_BM / ACT_CONSUMER_WARPS) + rr;
        const int grow = row0 + row;
        const uint32_t off = box * ACT_X_BOX_BYTES + swz(row * 128 + chunk16 * 16, 3);
        const uint4 raw = *reinterpret_cast<const uint4*>(xs + off);
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        float xh[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xh[2 * i] = __fmul_rn(bf16_bits_to_f32(w4[i] & 0xFFFFu), inv[2 * i]);
          xh[2 * i + 1] = __fmul_rn(bf16_bits_to_f32(w4[i] >> 16), inv[2 * i + 1]);
        }
        uint32_t sc;
        const uint32_t codes = nvfp4_quant_half_block(xh, sc);
        if (grow < p.M)
          *reinterpret_cast<uint32_t*>(p.x_codes + static_cast<size_t>(grow) * half_k +
                                       (k0 >> 1) + 4 * lane) = codes;
        // gather the 4 scales of each 64-wide group (lanes 8a, 8a+2, 8a+4, 8a+6)
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 2);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 4);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 6);
        if ((lane & 7) == 0 && grow < p.M_pad) {
          const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
          *reinterpret_cast<uint32_t*>(p.x_scales +
                                       sf_offset(grow, (k0 >> 4) + 4 * box, p.K)) = word;
        }
        if (R_PAD > 0) {
          uint4 o;
          o.x = pack_bf16x2(xh[0], xh[1]);
          o.y = pack_bf16x2(xh[2], xh[3]);
          o.z = pack_bf16x2(xh[4], xh[5]);
          o.w = pack_bf16x2(xh[6], xh[7]);
          *reinterpret_cast<uint4*>(xs + off) = o;
        }
      }

      if (R_PAD > 0) {
        // all bf16(Xhat) rows of the chunk must be in shared memory
        asm volatile("bar.sync 1, %0;" ::"r"(ACT_CONSUMER_WARPS * 32) : "memory");
        const uint32_t xs_u = smem_base + s * kStage;
        const uint32_t l1_u = xs_u + ACT_X_TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const int kk = (kg * 4 + ks) * 16;
          // A fragment: rows mt*16 + (lane & 15), k columns kk + 8*(lane >> 4)
          const int arow = mt * 16 + (lane & 15);
          const int acol = kk + (lane >> 4) * 8;
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(xs_u + (acol >> 6) * ACT_X_BOX_BYTES +
                          swz(arow * 128 + ((acol & 63) >> 3) * 16, 3),
                      a0, a1, a2, a3);
#pragma unroll
          for (int np = 0; np < kNT / 2; ++np) {
            const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int nch = np * 2 + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(l1_u + swz(krow * (R_PAD * 2) + nch * 16, kL1B), b0, b1, b2, b3);
            mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
      // generic-proxy accesses of this stage happen before the TMA refills it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }

    if (R_PAD > 0) {
      asm volatile("bar.sync 1, %0;" ::"r"(ACT_CONSUMER_WARPS * 32) : "memory");
      if (!*abort_flag) {
        // partial D of this warp: rows mt*16 + lane/4 (+8), cols nt*8 + 2*(lane%4) (+1)
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
          const int rlo = mt * 16 + (lane >> 2), col = t * 8 + 2 * (lane & 3);
          float* base = red + (kg * ACT_BM) * R_PAD;
          base[rlo * R_PAD + col] = acc[t][0];
          base[rlo * R_PAD + col + 1] = acc[t][1];
          base[(rlo + 8) * R_PAD + col] = acc[t][2];
          base[(rlo + 8) * R_PAD + col + 1] = acc[t][3];
        }
        asm volatile("bar.sync 1, %0;" ::"r"(ACT_CONSUMER_WARPS * 32) : "memory");
        for (int idx = threadIdx.x; idx < ACT_BM * p.r; idx += ACT_CONSUMER_WARPS * 32) {
          const int row = idx / p.r, col = idx % p.r;
          const int grow = row0 + row;
          if (grow >= p.M) continue;
          const float v = ((red[(0 * ACT_BM + row) * R_PAD + col] +
                            red[(1 * ACT_BM + row) * R_PAD + col]) +
                           red[(2 * ACT_BM + row) * R_PAD + col]) +
                          red[(3 * ACT_BM + row) * R_PAD + col];
          p.D[static_cast<size_t>(grow) * p.r + col] =
              static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace svdq
