// int4.cuh -- the INT4 variant of the SVDQuant W4A4 linear layer.
//
// The pages give the layer in two 4-bit formats: NVFP4 on Blackwell and INT4
// on the earlier generations (chaosnode.de "Nunchaku Lite: 4-Bit
// Diffusion-Inferenz direkt in Diffusers", section "Hardware-Support";
// imaginepro.ai "Nunchaku 4-Bit Diffusion Inference in Diffusers: A Practical
// Guide", table of quantisation methods: svdq_w4a4 in INT4).  Format used
// here: signed two's-complement 4-bit codes in [-8, 7], one fp16 scale per
// group of 64 elements along K, s = fp16_RNE(min(f32(amax / 7), 65504)),
// q = clamp(RNE(f32(v / s)), -8, 7) (q = 0 when s == 0); codes packed like
// NVFP4 (element 2j in the low nibble of byte j).  Smoothing, the rank-r
// branch and the residual are those of the NVFP4 layer.
//
// Scale layout ("group-major"): fp16 [K/64][rows_pad], row index fastest, so
// the scales of one group for 128 consecutive rows are 256 contiguous bytes.
// Activations pad rows to a multiple of 128 (padding rows hold zero).
//
// B200 has no 4-bit integer tensor-core MMA and tcgen05 has no per-group
// scaling for integers, so the GEMM runs the exact integer group sums on the
// warp-level 8-bit integer MMA (mma.sync m16n8k32 s8, codes sign-extended in
// registers) and applies the two group scales on the FMA pipe.  The CUDA-core
// work around the MMAs -- the sign extension and this two-scale combine --
// bounds the kernel; the format is served for correctness and portability of
// checkpoints, NVFP4 is the path the hardware is built for.
#pragma once

#include <cuda_fp16.h>

#include "act_quant.cuh"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr uint32_t KID_INT4 = 5;
constexpr int INT4_GROUP = 64;

// ---------------------------------------------------------------------------
// Group quantiser
// ---------------------------------------------------------------------------

// fp16 bits of the scale of a group whose largest magnitude is amax.
__device__ __forceinline__ uint16_t int4_group_scale(float amax) {
  return __half_as_ushort(__float2half_rn(fminf(__fdiv_rn(amax, 7.0f), 65504.0f)));
}

__device__ __forceinline__ float half_bits_to_f32(uint32_t bits) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

// 4-bit two's-complement code of v in a group of scale s (a float holding the
// fp16 value).  Clamping before the rounding gives the same integer as
// clamping after it, because the bounds are integers.
__device__ __forceinline__ uint32_t int4_code(float v, float s) {
  if (s == 0.0f) return 0u;
  const float q = fminf(fmaxf(__fdiv_rn(v, s), -8.0f), 7.0f);
  return static_cast<uint32_t>(__float2int_rn(q)) & 0xFu;
}

// Sign-extend the even (lo) or odd (hi) nibbles of a packed word into four
// int8 lanes: byte b of the result is element 2b (lo) or 2b+1 (hi).  Each
// byte of (v & 0x08..) is 0 or 8, and 8 * 0x1E = 0xF0 sets the upper nibble
// of the negative ones without a carry into the next byte.
__device__ __forceinline__ uint32_t s4_even(uint32_t w) {
  const uint32_t v = w & 0x0F0F0F0Fu;
  return v | ((v & 0x08080808u) * 0x1Eu);
}
__device__ __forceinline__ uint32_t s4_odd(uint32_t w) { return s4_even(w >> 4); }

// D(16x8, s32) += A(16x32, s8) B(32x8, s8), warp-level.
__device__ __forceinline__ void imma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Offline: R = f32(What - (bf16 L1 bf16 L2)^T) (float64, increasing j), then
// INT4 along K.  One CTA per weight row; a warp takes 256-wide chunks, 8 lanes
// form a group of 64.  Scales go to w_scales[k/64][N].
// ---------------------------------------------------------------------------
template <int RMAX>
__global__ void __launch_bounds__(256) prep_residual_int4_kernel(const float* __restrict__ what,
                                                                 const uint16_t* __restrict__ L1,
                                                                 const uint16_t* __restrict__ L2t,
                                                                 int N, int K, int r,
                                                                 uint8_t* __restrict__ w_codes,
                                                                 uint16_t* __restrict__ w_scales) {
  const int nn = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ double l2[RMAX > 0 ? RMAX : 1];
  for (int j = threadIdx.x; j < r; j += blockDim.x)
    l2[j] = static_cast<double>(bf16_bits_to_f32(L2t[static_cast<size_t>(nn) * r + j]));
  __syncthreads();
  for (int c = warp; c < K / 256; c += 8) {
    const int k0 = c * 256 + 8 * lane;
    float v[8];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = k0 + i;
      double acc = 0.0;
      for (int j = 0; j < r; ++j)
        acc = __fma_rn(static_cast<double>(bf16_bits_to_f32(L1[static_cast<size_t>(k) * r + j])),
                       l2[j], acc);
      v[i] = __double2float_rn(__dsub_rn(static_cast<double>(what[static_cast<size_t>(nn) * K + k]), acc));
      am = fmaxf(am, fabsf(v[i]));
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    const uint16_t sb = int4_group_scale(am);
    const float s = half_bits_to_f32(sb);
    uint32_t codes = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) codes |= int4_code(v[i], s) << (4 * i);
    *reinterpret_cast<uint32_t*>(w_codes + static_cast<size_t>(nn) * (K / 2) + k0 / 2) = codes;
    if ((lane & 7) == 0) w_scales[static_cast<size_t>(k0 / INT4_GROUP) * N + nn] = sb;
  }
}

// ---------------------------------------------------------------------------
// Activation kernel (INT4): one HBM pass over X producing the INT4 codes and
// group scales of Xhat = f32(X * inv_lambda) and D = bf16(bf16(Xhat) L1).
// Same structure as the NVFP4 activation kernel: 16 token rows per CTA, 8
// warps taking 64-column sub-tiles -- one quantisation group each -- through
// private 4-slot TMA rings; the 8 lanes that share a row of a sub-tile reduce
// the group maximum with three shuffles.
// ---------------------------------------------------------------------------
struct Int4ActParams {
  const float* inv_lambda;
  const uint32_t* L1f;     // L1 in mma.m16n8k16 B-fragment order (l1_fragment_word)
  uint8_t* x_codes;
  uint16_t* x_scales;      // fp16 [K/64][M_pad]
  uint16_t* D;
  int M, K, r, M_pad;
};

template <int R_PAD>
struct Int4ActSmem {
  static constexpr uint32_t kRing = ACT_WARPS * ACT_RING * ACT_SUB_BYTES;        // 64 KB
  static constexpr uint32_t kRed = (R_PAD > 0 ? ACT_WARPS * ACT_ROWS * R_PAD * 4 : 0);
  static constexpr uint32_t kBytes = kRing + kRed + ACT_WARPS * ACT_RING * 8 + 16 + 1024;
};

template <int R_PAD>
__global__ void __launch_bounds__(ACT_THREADS, 2)
    act_quant_int4_kernel(const __grid_constant__ CUtensorMap tm_x, const Int4ActParams p) {
  constexpr int kNT = R_PAD / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(smem + Int4ActSmem<R_PAD>::kRing);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Int4ActSmem<R_PAD>::kRing + Int4ActSmem<R_PAD>::kRed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + ACT_WARPS * ACT_RING);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * ACT_ROWS;
  const int nsub = p.K / ACT_SUB;
  if (threadIdx.x == 0) *abort_flag = 0;
  const uint32_t ring = smem_u32(smem) + warp * ACT_RING * ACT_SUB_BYTES;
  auto bar = [&](int slot) { return smem_u32(bars + warp * ACT_RING + slot); };
  if (lane == 0) {
    for (int sl = 0; sl < ACT_RING; ++sl) mbar_init(bar(sl), 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  if (row0 >= p.M) {
    // a row block entirely in [M, M_pad): its scales are zero
    for (int idx = threadIdx.x; idx < nsub * ACT_ROWS; idx += ACT_THREADS)
      p.x_scales[static_cast<size_t>(idx / ACT_ROWS) * p.M_pad + row0 + idx % ACT_ROWS] = 0;
    return;
  }

  const int my_count = nsub > warp ? (nsub - warp + ACT_WARPS - 1) / ACT_WARPS : 0;
  auto issue = [&](int jj) {
    const int slot = jj % ACT_RING;
    mbar_arrive_expect_tx(bar(slot), ACT_SUB_BYTES);
    tma_load_2d(ring + slot * ACT_SUB_BYTES, &tm_x, bar(slot), (warp + ACT_WARPS * jj) * ACT_SUB, row0);
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
  const int chunk16 = lane & 7, rsub = lane >> 3;
  float4 ni0 = make_float4(0.f, 0.f, 0.f, 0.f), ni1 = ni0;
  auto load_inv = [&](int j) {
    const float* src = p.inv_lambda + (warp + ACT_WARPS * j) * ACT_SUB + 8 * chunk16;
    ni0 = __ldg(reinterpret_cast<const float4*>(src));
    ni1 = __ldg(reinterpret_cast<const float4*>(src + 4));
  };
  if (my_count > 0) load_inv(0);
  int jj = 0;
  for (; jj < my_count; ++jj) {
    const int slot = jj % ACT_RING;
    const int col0 = (warp + ACT_WARPS * jj) * ACT_SUB;
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
    const uint64_t ninv2[4] = {f32x2_pack(-ni0.x, -ni0.y), f32x2_pack(-ni0.z, -ni0.w),
                               f32x2_pack(-ni1.x, -ni1.y), f32x2_pack(-ni1.z, -ni1.w)};
    if (jj + 1 < my_count) load_inv(jj + 1);
    if (!mbar_wait(bar(slot), (jj / ACT_RING) & 1, abort_flag, KID_INT4, 1)) break;
    uint8_t* tile = smem + (ring - smem_u32(smem)) + slot * ACT_SUB_BYTES;
#pragma unroll
    for (int i = 0; i < ACT_ROWS / 4; ++i) {
      const int row = i * 4 + rsub, grow = row0 + row;
      const uint32_t off = swz(static_cast<uint32_t>(row * 128 + chunk16 * 16), 3);
      const uint4 raw = *reinterpret_cast<const uint4*>(tile + off);
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
      // -Xhat = f32(x * (-1/lambda)), element 2u in the low half of pair u
      uint64_t nxh[4];
      float am = 0.0f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        nxh[u] = f32x2_mul(f32x2_pack(__uint_as_float(w4[u] << 16), __uint_as_float(w4[u] & 0xFFFF0000u)),
                           ninv2[u]);
        float lo, hi;
        f32x2_unpack(nxh[u], lo, hi);
        am = fmaxf(am, fmaxf(fabsf(lo), fabsf(hi)));
      }
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
      const uint16_t sb = int4_group_scale(am);
      const float s = half_bits_to_f32(sb);
      uint32_t codes = 0;
      uint32_t o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float lo, hi;
        f32x2_unpack(nxh[u], lo, hi);
        codes |= int4_code(-lo, s) << (8 * u);
        codes |= int4_code(-hi, s) << (8 * u + 4);
        o[u] = pack_bf16x2(lo, hi);   // bf16(-Xhat) for the low-rank MMA
      }
      if (grow < p.M)
        *reinterpret_cast<uint32_t*>(p.x_codes + static_cast<size_t>(grow) * half_k + (col0 >> 1) + 4 * chunk16) =
            codes;
      if (chunk16 == 0) p.x_scales[static_cast<size_t>(col0 / INT4_GROUP) * p.M_pad + grow] = sb;
      if (R_PAD > 0) *reinterpret_cast<uint4*>(tile + off) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (R_PAD > 0) {
      __syncwarp();
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
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && jj + ACT_RING < my_count) issue(jj + ACT_RING);
  }
  if (*abort_flag && lane == 0) {
    for (int k = jj; k < my_count && k < jj + ACT_RING; ++k)
      mbar_wait_drain(bar(k % ACT_RING), (k / ACT_RING) & 1);
  }
  if (R_PAD > 0) {
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
  }
}

// ---------------------------------------------------------------------------
// GEMM (INT4):  Y = bf16( sum_g sx[m,g] sw[n,g] (sum_{k in g} qx[m,k] qw[n,k])
//                        + D L2 + bias )
// CTA tile 128 x 128, 8 consumer warps in a 2 x 4 grid (warp tile 64 x 32)
// plus one TMA producer warp.  A ring stage holds 256 K-elements (4 groups):
// codes of A and B (128 rows x 128 bytes each, 128-byte swizzle) and the fp16
// scales of the 4 groups for the tile's rows and columns.
//
// Fragments: lane (g8 = lane/4, t4 = lane%4) reads bytes 8 t4 .. 8 t4 + 7 of a
// row's 32 group bytes (16 codes).  Its first word feeds the first of the two
// m16n8k32 MMAs of the group, the second word the second; in each, the even
// codes form the register that the MMA treats as k = 4 t4 .. 4 t4 + 3 and the
// odd codes the one at k + 16.  A and B use the same assignment, so every
// product pairs the same element of the row of X and of the row of R, and the
// two MMAs together cover the 64 elements of the group once.
// The integer group sum c (|c| <= 4096) becomes a float exactly by adding it
// to the bits of 1.5 * 2^23 (M0) and folding -M0 into an FMA with the row
// scale: (c + M0) sx - M0 sx = c sx exactly (at most 24 significant bits);
// a second FMA adds c sx sw to the accumulator.
// ---------------------------------------------------------------------------
constexpr int I4_BM = 128, I4_BN = 128;
constexpr int I4_STAGES = 4;
constexpr int I4_GPS = 4;                          // groups per stage (256 K-elements)
constexpr int I4_CONSUMERS = 8;
constexpr int I4_THREADS = (I4_CONSUMERS + 1) * 32;
constexpr uint32_t I4_A_BYTES = I4_BM * 128;
constexpr uint32_t I4_B_BYTES = I4_BN * 128;
constexpr uint32_t I4_SX_BYTES = I4_GPS * I4_BM * 2;
constexpr uint32_t I4_SW_BYTES = I4_GPS * I4_BN * 2;
constexpr uint32_t I4_STAGE_BYTES = I4_A_BYTES + I4_B_BYTES + I4_SX_BYTES + I4_SW_BYTES;   // 34 KB
constexpr uint32_t I4_SMEM_BYTES = I4_STAGES * I4_STAGE_BYTES + 2 * I4_STAGES * 8 + 16 + 1024;
static_assert(I4_STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of 128-byte swizzle");

struct Int4GemmParams {
  const uint16_t* D;      // M x r bf16 (null when r == 0)
  const uint16_t* L2t;    // N x r bf16
  const uint16_t* bias;   // N bf16 or null
  uint16_t* Y;
  int M, N, K, r;
  int head_dim;           // 0: Y row-major M x N; else head-major [N/head_dim][M][head_dim]
};

__device__ __forceinline__ uint32_t ldg_u32_or0(const uint16_t* p, bool ok) {
  return ok ? __ldg(reinterpret_cast<const unsigned int*>(p)) : 0u;
}

template <int R_PAD>
__global__ void __launch_bounds__(I4_THREADS, 1)
    int4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_sx, const __grid_constant__ CUtensorMap tm_sw,
                     const Int4GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + I4_STAGES * I4_STAGE_BYTES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * I4_STAGES);
  const uint32_t smem0 = smem_u32(smem);
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + I4_STAGES + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * I4_BM, n0 = blockIdx.y * I4_BN;   // grid (M tiles, N tiles)
  const int nst = p.K / (I4_GPS * INT4_GROUP);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < I4_STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), I4_CONSUMERS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();   // codes, scales and D may come from the kernel launched just before

  if (warp == I4_CONSUMERS) {
    // producer: one thread streams the ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_sx);
      tma_prefetch_desc(&tm_sw);
      int issued = 0;
      for (int kt = 0; kt < nst; ++kt) {
        const int s = kt % I4_STAGES;
        if (kt >= I4_STAGES && !mbar_wait(empty(s), ((kt / I4_STAGES) - 1) & 1, abort_flag, KID_INT4, 2)) break;
        const uint32_t base = smem0 + s * I4_STAGE_BYTES;
        mbar_arrive_expect_tx(full(s), I4_STAGE_BYTES);
        tma_load_2d(base, &tm_a, full(s), kt * 128, m0);
        tma_load_2d(base + I4_A_BYTES, &tm_b, full(s), kt * 128, n0);
        tma_load_2d(base + I4_A_BYTES + I4_B_BYTES, &tm_sx, full(s), m0, kt * I4_GPS);
        tma_load_2d(base + I4_A_BYTES + I4_B_BYTES + I4_SX_BYTES, &tm_sw, full(s), n0, kt * I4_GPS);
        issued = kt + 1;
      }
      if (*abort_flag) {
        // copies already issued land before the CTA exits
        for (int kt = issued > I4_STAGES ? issued - I4_STAGES : 0; kt < issued; ++kt)
          mbar_wait_drain(full(kt % I4_STAGES), (kt / I4_STAGES) & 1);
      }
    }
    return;
  }

  const int wm = warp & 1, wn = warp >> 1;
  const int g8 = lane >> 2, t4 = lane & 3;
  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

  // low-rank branch first: acc = D L2 (bf16 operands, fp32), k >= r reads as 0
  if (R_PAD > 0) {
#pragma unroll
    for (int kk = 0; kk < R_PAD / 16; ++kk) {
      const int k = 16 * kk + 2 * t4;
      if (16 * kk >= p.r) break;
      uint32_t b[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint16_t* l2 = p.L2t + static_cast<size_t>(n0 + wn * 32 + j * 8 + g8) * p.r;
        b[j][0] = ldg_u32_or0(l2 + k, k < p.r);
        b[j][1] = ldg_u32_or0(l2 + k + 8, k + 8 < p.r);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r0 = m0 + wm * 64 + i * 16 + g8, r1 = r0 + 8;
        const uint16_t* d0 = p.D + static_cast<size_t>(r0) * p.r;
        const uint16_t* d1 = p.D + static_cast<size_t>(r1) * p.r;
        const uint32_t a0 = ldg_u32_or0(d0 + k, r0 < p.M && k < p.r);
        const uint32_t a1 = ldg_u32_or0(d1 + k, r1 < p.M && k < p.r);
        const uint32_t a2 = ldg_u32_or0(d0 + k + 8, r0 < p.M && k + 8 < p.r);
        const uint32_t a3 = ldg_u32_or0(d1 + k + 8, r1 < p.M && k + 8 < p.r);
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16_16816(acc[i][j], a0, a1, a2, a3, b[j][0], b[j][1]);
      }
    }
  }

  constexpr float kM0 = 12582912.0f;   // 1.5 * 2^23
  constexpr int kM0Bits = 0x4B400000;
  bool ok = true;
  for (int kt = 0; kt < nst; ++kt) {
    const int s = kt % I4_STAGES;
    if (!mbar_wait(full(s), (kt / I4_STAGES) & 1, abort_flag, KID_INT4, 3)) {
      ok = false;
      break;
    }
    const uint8_t* st = smem + s * I4_STAGE_BYTES;
    const uint16_t* sx = reinterpret_cast<const uint16_t*>(st + I4_A_BYTES + I4_B_BYTES);
    const uint16_t* sw = sx + I4_GPS * I4_BM;
#pragma unroll 1
    for (int g = 0; g < I4_GPS; ++g) {
      // B fragments of the group for the warp's 4 n8 tiles, and their scales
      uint32_t bw[4][4];
      uint64_t sw2[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = wn * 32 + j * 8 + g8;
        const uint2 raw =
            *reinterpret_cast<const uint2*>(st + I4_A_BYTES + swz(static_cast<uint32_t>(col * 128 + g * 32 + 8 * t4), 3));
        bw[j][0] = s4_even(raw.x);
        bw[j][1] = s4_odd(raw.x);
        bw[j][2] = s4_even(raw.y);
        bw[j][3] = s4_odd(raw.y);
        const uint32_t sp = *reinterpret_cast<const uint32_t*>(sw + g * I4_BN + wn * 32 + j * 8 + 2 * t4);
        sw2[j] = f32x2_pack(half_bits_to_f32(sp & 0xFFFFu), half_bits_to_f32(sp >> 16));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r0 = wm * 64 + i * 16 + g8;
        const uint2 ra = *reinterpret_cast<const uint2*>(st + swz(static_cast<uint32_t>(r0 * 128 + g * 32 + 8 * t4), 3));
        const uint2 rb =
            *reinterpret_cast<const uint2*>(st + swz(static_cast<uint32_t>((r0 + 8) * 128 + g * 32 + 8 * t4), 3));
        int c[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0;
          imma_16832(c[j], s4_even(ra.x), s4_even(rb.x), s4_odd(ra.x), s4_odd(rb.x), bw[j][0], bw[j][1]);
          imma_16832(c[j], s4_even(ra.y), s4_even(rb.y), s4_odd(ra.y), s4_odd(rb.y), bw[j][2], bw[j][3]);
        }
        const float sx0 = half_bits_to_f32(sx[g * I4_BM + r0]);
        const float sx1 = half_bits_to_f32(sx[g * I4_BM + r0 + 8]);
        const uint64_t sx0_2 = f32x2_pack(sx0, sx0), sx1_2 = f32x2_pack(sx1, sx1);
        const uint64_t nm0_2 = f32x2_pack(-kM0 * sx0, -kM0 * sx0), nm1_2 = f32x2_pack(-kM0 * sx1, -kM0 * sx1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t f01 = f32x2_pack(__int_as_float(c[j][0] + kM0Bits), __int_as_float(c[j][1] + kM0Bits));
          const uint64_t f23 = f32x2_pack(__int_as_float(c[j][2] + kM0Bits), __int_as_float(c[j][3] + kM0Bits));
          const uint64_t t01 = f32x2_fma(f01, sx0_2, nm0_2);   // c sx, exact
          const uint64_t t23 = f32x2_fma(f23, sx1_2, nm1_2);
          uint64_t a01 = f32x2_pack(acc[i][j][0], acc[i][j][1]);
          uint64_t a23 = f32x2_pack(acc[i][j][2], acc[i][j][3]);
          a01 = f32x2_fma(t01, sw2[j], a01);
          a23 = f32x2_fma(t23, sw2[j], a23);
          f32x2_unpack(a01, acc[i][j][0], acc[i][j][1]);
          f32x2_unpack(a23, acc[i][j][2], acc[i][j][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }
  if (!ok || *abort_flag) return;   // nothing is stored after an abort

  float bias0[4], bias1[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = n0 + wn * 32 + j * 8 + 2 * t4;
    bias0[j] = p.bias ? bf16_bits_to_f32(p.bias[col]) : 0.0f;
    bias1[j] = p.bias ? bf16_bits_to_f32(p.bias[col + 1]) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = m0 + wm * 64 + i * 16 + g8 + 8 * h;
      if (row >= p.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = n0 + wn * 32 + j * 8 + 2 * t4;
        const uint32_t v = pack_bf16x2(acc[i][j][2 * h] + bias0[j], acc[i][j][2 * h + 1] + bias1[j]);
        uint16_t* dst = p.head_dim == 0
                            ? p.Y + static_cast<size_t>(row) * p.N + col
                            : p.Y + (static_cast<size_t>(col / p.head_dim) * p.M + row) * p.head_dim +
                                  col % p.head_dim;
        *reinterpret_cast<uint32_t*>(dst) = v;
      }
    }
}

}  // namespace svdq
