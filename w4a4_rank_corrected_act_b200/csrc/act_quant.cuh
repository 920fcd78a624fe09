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
// Design (B200): a CTA owns 16 token rows (one m16 tile); its 8 warps split K
// into 64-column sub-tiles (warp w takes sub-tiles w, w+8, ...).  When there
// are too few rows to fill the GPU, a cluster of ks CTAs shares a row block,
// CTA c taking the c-th of ks equal K ranges; their partial D meet in the
// first CTA's shared memory.  Each warp
// streams its sub-tiles through a private 4-slot TMA ring (16 x 64 bf16 boxes,
// 128-byte swizzle), so no block-wide synchronisation happens until the final
// reduction of D.  In a slot, each lane quantises two whole 16-element blocks
// in registers and writes bf16(Xhat) back in place; ldmatrix then feeds
// mma.sync m16n8k16 with that tile, the B fragments of L1 coming straight from
// L2 in the fragment order the weight stores them in.  X crosses HBM once.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr int ACT_ROWS = 16;          // token rows per CTA
constexpr int ACT_WARPS = 8;
constexpr int ACT_THREADS = ACT_WARPS * 32;
constexpr int ACT_SUB = 64;           // columns per sub-tile
constexpr int ACT_RING = 4;           // slots per warp
constexpr uint32_t ACT_SUB_BYTES = ACT_ROWS * ACT_SUB * 2;   // 2 KB
constexpr int ACT_MAX_KS = 8;         // CTAs per cluster (K split), portable limit

struct ActParams {
  const float* inv_lambda;
  const uint32_t* L1f;     // L1 in mma.m16n8k16 B-fragment order (see l1_fragment_offset)
  uint8_t* x_codes;
  uint8_t* x_scales;
  uint16_t* D;
  int M, K, r, M_pad;
  int ks;                  // CTAs per cluster sharing a row block (K split); K % (64 ks) == 0
  float* zero_ptr;         // optional: zero_count floats set to 0 by the grid (the MLP pair's D
  int zero_count;          // accumulator, which the next kernel of the stream adds into)
};

template <int R_PAD>
struct ActSmem {
  static constexpr uint32_t kRing = ACT_WARPS * ACT_RING * ACT_SUB_BYTES;        // 64 KB
  static constexpr uint32_t kRed = (R_PAD > 0 ? ACT_WARPS * ACT_ROWS * R_PAD * 4 : 0);
  static constexpr uint32_t kTab = 128 * 8;                                     // E4M3 (s, 1/s)
  static constexpr uint32_t kBytes = kRing + kRed + kTab + ACT_WARPS * ACT_RING * 8 + 16 + 1024;
  // with a K split, the partial D of each CTA of a cluster is gathered in the
  // first CTA's ring, [rank][row][col], once every CTA is done with its ring
  static_assert(ACT_MAX_KS * ACT_ROWS * R_PAD * 4 <= kRing, "partial-D gather area");
};

// Position (in 32-bit words) of L1 element pair (k, k+1), column j, in the
// fragment order: for each 16-row k-step g and 8-column n-tile t of L1, the 32
// lanes' B fragments (b0, b1) of mma.m16n8k16 follow each other:
//   word ((g * NT + t) * 32 + lane) * 2 + h  holds  L1[16g + 2(lane%4) + 8h + {0,1}][8t + lane/4]
// with NT = r / 8 and the lower k in the low half.
__host__ __device__ __forceinline__ size_t l1_fragment_word(int k, int j, int r) {
  const int g = k >> 4, kk = k & 15, t = j >> 3, jj = j & 7;
  const int lane = jj * 4 + ((kk & 7) >> 1), h = kk >> 3;
  return ((static_cast<size_t>(g) * (r >> 3) + t) * 32 + lane) * 2 + h;
}

// Two CTAs per SM; at r = 64 one, whose 190 registers hold the 32 D accumulators
// without spilling (128 registers spilled and took 55 instead of 31 us on qkv).
template <int R_PAD>
__global__ void __launch_bounds__(ACT_THREADS, R_PAD > 32 ? 1 : 2)
    act_quant_kernel(const __grid_constant__ CUtensorMap tm_x, const ActParams p) {
  constexpr int kNT = R_PAD / 8;   // n8 tiles (upper bound; the weight holds r/8)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(smem + ActSmem<R_PAD>::kRing);
  float2* tab = reinterpret_cast<float2*>(smem + ActSmem<R_PAD>::kRing + ActSmem<R_PAD>::kRed);
  float* recv = reinterpret_cast<float*>(smem);   // aliases the ring (see ActSmem)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ActSmem<R_PAD>::kRing + ActSmem<R_PAD>::kRed +
                                               ActSmem<R_PAD>::kTab);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + ACT_WARPS * ACT_RING);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t kpart = p.ks > 1 ? cluster_ctarank() : 0u;
  const int row0 = (blockIdx.x / p.ks) * ACT_ROWS;
  const int nsub = p.K / ACT_SUB / p.ks;             // sub-tiles of this CTA's K range
  const int sub0 = static_cast<int>(kpart) * nsub;   // its first sub-tile
  if (threadIdx.x == 0) *abort_flag = 0;
  const uint32_t ring = smem_u32(smem) + warp * ACT_RING * ACT_SUB_BYTES;
  auto bar = [&](int slot) { return smem_u32(bars + warp * ACT_RING + slot); };
  if (lane == 0) {
    for (int sl = 0; sl < ACT_RING; ++sl) mbar_init(bar(sl), 1);
    fence_mbar_init();
  }
  for (int c = threadIdx.x; c < 128; c += ACT_THREADS) tab[c] = e4m3_table_entry(c);
  __syncthreads();   // barriers, the E4M3 table and the abort flag are initialised
  // This grid may be launched while the previous kernel of the stream is still
  // running (programmatic dependent launch): nothing in global memory is read
  // or written before that kernel has completed.  The GEMM that consumes this
  // kernel's output may be launched from now on: it loads weights until its
  // own wait, which waits for this grid to finish.
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * ACT_THREADS + threadIdx.x; i < p.zero_count; i += gridDim.x * ACT_THREADS)
    p.zero_ptr[i] = 0.0f;
  if (row0 >= p.M) {
    // rows entirely in [M, M_pad): their scale entries are written as zero
    // (the whole cluster shares the row block, so every CTA of it leaves here)
    for (int idx = threadIdx.x; idx < nsub * ACT_ROWS; idx += ACT_THREADS) {
      const int g = sub0 + idx / ACT_ROWS, i = idx % ACT_ROWS;
      *reinterpret_cast<uint32_t*>(p.x_scales + sf_offset(row0 + i, g * 4, p.K)) = 0u;
    }
    return;
  }

  const int my_count = nsub > warp ? (nsub - warp + ACT_WARPS - 1) / ACT_WARPS : 0;
  auto issue = [&](int jj) {
    const int slot = jj % ACT_RING;
    mbar_arrive_expect_tx(bar(slot), ACT_SUB_BYTES);
    tma_load_2d(ring + slot * ACT_SUB_BYTES, &tm_x, bar(slot), (sub0 + warp + ACT_WARPS * jj) * ACT_SUB,
                row0);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tm_x);
    for (int jj = 0; jj < my_count && jj < ACT_RING; ++jj) issue(jj);
  }

  const int nt_count = p.r >> 3;
  float acc[kNT > 0 ? kNT : 1][4];
#pragma unroll
  for (int t = 0; t < (kNT > 0 ? kNT : 1); ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;
  const uint32_t half_k = static_cast<uint32_t>(p.K) >> 1;
  // lane l quantises the 16-column block l % 4 of rows l / 4 and l / 4 + 8: a
  // whole block per thread, so no lane pair exchanges its maximum
  const int blk = lane & 3, rsub = lane >> 2;
  const float y6 = tab[0x4C].y;   // E4M3 code 0x4C is 6.0: RN(1/6)
  const uint64_t six = f32x2_pack(6.0f, 6.0f), neg_y6 = f32x2_pack(-y6, -y6);
  // row-dependent addresses, fixed for the whole K range: the block's first
  // 16 bytes in row 8 i + l / 4 of a (swizzled) sub-tile (the second 16 sit at
  // toff ^ 16), its codes (null past M) and its scale byte of column group 0
  uint32_t toff[ACT_ROWS / 8];
  uint8_t* cptr[ACT_ROWS / 8];
  uint8_t* sptr[ACT_ROWS / 8];
#pragma unroll
  for (int i = 0; i < ACT_ROWS / 8; ++i) {
    const int row = i * 8 + rsub, grow = row0 + row;
    toff[i] = swz(static_cast<uint32_t>(row * 128 + blk * 32), 3);
    cptr[i] = grow < p.M ? p.x_codes + static_cast<size_t>(grow) * half_k + 8 * blk : nullptr;
    sptr[i] = p.x_scales + sf_offset(static_cast<uint32_t>(grow), 0, static_cast<uint32_t>(p.K)) + blk;
  }
  int jj = 0;
  for (; jj < my_count; ++jj) {
    const int slot = jj % ACT_RING;
    const int col0 = (sub0 + warp + ACT_WARPS * jj) * ACT_SUB;
    // B fragments of this sub-tile's 4 k-steps (L2-resident), issued early
    uint2 bfr[4][kNT > 0 ? kNT : 1];
    if (R_PAD > 0) {
      const uint2* f = reinterpret_cast<const uint2*>(p.L1f);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int t = 0; t < kNT; ++t)
          if (t < nt_count)
            bfr[ks][t] = __ldg(f + ((static_cast<size_t>(col0 / 16 + ks) * nt_count + t) * 32 + lane));
    }
    // 1/lambda of this lane's 16 columns (L1-resident after the first sub-tiles),
    // in flight while the tile lands; loaded per sub-tile rather than one ahead,
    // which would hold 16 more registers across the loop
    float4 ni[4];
    {
      const float4* src = reinterpret_cast<const float4*>(p.inv_lambda + col0 + 16 * blk);
#pragma unroll
      for (int u = 0; u < 4; ++u) ni[u] = __ldg(src + u);
    }
    if (!mbar_wait(bar(slot), (jj / ACT_RING) & 1, abort_flag, KID_ACT, 1)) break;
    // -1/lambda: the quantiser takes -Xhat (see nvfp4_quant_block16_x2)
    uint64_t ninv2[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ninv2[2 * u] = f32x2_pack(-ni[u].x, -ni[u].y);
      ninv2[2 * u + 1] = f32x2_pack(-ni[u].z, -ni[u].w);
    }
    uint8_t* tile = smem + (ring - smem_u32(smem)) + slot * ACT_SUB_BYTES;

#pragma unroll
    for (int i = 0; i < ACT_ROWS / 8; ++i) {
      const uint32_t off = toff[i];
      const uint4 r0 = *reinterpret_cast<const uint4*>(tile + off);
      const uint4 r1 = *reinterpret_cast<const uint4*>(tile + (off ^ 16u));
      const uint32_t w8[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      // -Xhat = f32(x * (-1/lambda)) (exactly the negated product), element 2u
      // in the low half of pair u
      uint64_t nxh[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        nxh[u] = f32x2_mul(f32x2_pack(__uint_as_float(w8[u] << 16), __uint_as_float(w8[u] & 0xFFFF0000u)),
                           ninv2[u]);
      uint32_t sc;
      const uint64_t codes = nvfp4_quant_block16_x2(nxh, tab, six, neg_y6, sc);
      if (cptr[i] != nullptr) *reinterpret_cast<uint64_t*>(cptr[i] + (col0 >> 1)) = codes;
      sptr[i][static_cast<size_t>(col0 >> 6) * 512] = static_cast<uint8_t>(sc);
      if (R_PAD > 0) {
        // bf16(-Xhat) = -bf16(Xhat): the tile holds the negated operand, and the
        // product with L1 is negated back when D is written
        uint32_t o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float lo, hi;
          f32x2_unpack(nxh[u], lo, hi);
          o[u] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4*>(tile + off) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(tile + (off ^ 16u)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }

    if (R_PAD > 0) {
      __syncwarp();   // the whole 16 x 64 bf16(Xhat) tile is in shared memory
      const uint32_t tile_u = ring + slot * ACT_SUB_BYTES;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(tile_u + swz((lane & 15) * 128 + (ks * 2 + (lane >> 4)) * 16, 3), a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < kNT; ++t)
          if (t < nt_count) mma_bf16_16816(acc[t], a0, a1, a2, a3, bfr[ks][t].x, bfr[ks][t].y);
      }
    }
    // this slot's generic accesses happen before the TMA refills it
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && jj + ACT_RING < my_count) issue(jj + ACT_RING);
  }
  if (*abort_flag && lane == 0) {
    // let copies already issued by this warp land before the CTA exits
    for (int k = jj; k < my_count && k < jj + ACT_RING; ++k)
      mbar_wait_drain(bar(k % ACT_RING), (k / ACT_RING) & 1);
  }

  if (R_PAD > 0) {
    // partial D of this warp: rows lane/4 (+8), cols 8t + 2(lane%4) (+1)
    float* mine = red + warp * ACT_ROWS * R_PAD;
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
      const int rlo = lane >> 2, col = t * 8 + 2 * (lane & 3);
      mine[rlo * R_PAD + col] = acc[t][0];
      mine[rlo * R_PAD + col + 1] = acc[t][1];
      mine[(rlo + 8) * R_PAD + col] = acc[t][2];
      mine[(rlo + 8) * R_PAD + col + 1] = acc[t][3];
    }
    __syncthreads();
    if (p.ks == 1) {
      if (!*abort_flag) {
        for (int idx = threadIdx.x; idx < ACT_ROWS * p.r; idx += ACT_THREADS) {
          const int row = idx / p.r, col = idx % p.r;
          const int grow = row0 + row;
          if (grow >= p.M) continue;
          float v = 0.0f;
#pragma unroll
          for (int w = 0; w < ACT_WARPS; ++w) v += red[(w * ACT_ROWS + row) * R_PAD + col];
          p.D[static_cast<size_t>(grow) * p.r + col] = static_cast<uint16_t>(pack_bf16x2(-v, 0.0f) & 0xFFFFu);
        }
      }
    } else {
      // this CTA's partial (summed over its warps) goes to the first CTA of the
      // cluster, which adds the ks partials in rank order and writes D; the
      // first barrier makes sure that CTA no longer uses its ring
      __syncwarp();
      cluster_sync_all();
      const uint32_t dst0 = mapa_shared(smem_u32(recv), 0) + kpart * (ACT_ROWS * R_PAD * 4);
      for (int idx = threadIdx.x; idx < ACT_ROWS * p.r; idx += ACT_THREADS) {
        const int row = idx / p.r, col = idx % p.r;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < ACT_WARPS; ++w) v += red[(w * ACT_ROWS + row) * R_PAD + col];
        st_shared_cluster_f32(dst0 + static_cast<uint32_t>(row * R_PAD + col) * 4u, v);
      }
      __syncwarp();
      cluster_sync_all();
      if (kpart == 0 && !*abort_flag) {
        for (int idx = threadIdx.x; idx < ACT_ROWS * p.r; idx += ACT_THREADS) {
          const int row = idx / p.r, col = idx % p.r;
          const int grow = row0 + row;
          if (grow >= p.M) continue;
          float v = 0.0f;
          for (int c = 0; c < p.ks; ++c) v += recv[(c * ACT_ROWS + row) * R_PAD + col];
          p.D[static_cast<size_t>(grow) * p.r + col] = static_cast<uint16_t>(pack_bf16x2(-v, 0.0f) & 0xFFFFu);
        }
      }
    }
  }
}

// L1 (K x r, row-major bf16) -> fragment order (see l1_fragment_word).
__global__ void l1_fragment_kernel(const uint16_t* __restrict__ L1, int K, int r,
                                   uint16_t* __restrict__ L1f) {
  const size_t total = static_cast<size_t>(K) * r;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int k = static_cast<int>(i / r), j = static_cast<int>(i % r);
    L1f[l1_fragment_word(k, j, r) * 2 + (k & 1)] = L1[i];
  }
}

// L1 (K x r, row-major bf16) -> L1^T (r x K, row-major): the K-major operand
// of the activation kernel's tensor-core product.
__global__ void l1_transpose_kernel(const uint16_t* __restrict__ L1, int K, int r, uint16_t* __restrict__ L1t) {
  const size_t total = static_cast<size_t>(K) * r;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int j = static_cast<int>(i / K), k = static_cast<int>(i % K);
    L1t[i] = L1[static_cast<size_t>(k) * r + j];
  }
}

}  // namespace svdq
