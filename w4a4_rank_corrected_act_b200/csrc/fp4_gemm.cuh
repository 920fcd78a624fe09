// fp4_gemm.cuh -- block-scaled NVFP4 GEMM with the low-rank branch fused,
// on the 5th-generation tensor cores (tcgen05) of sm_100a.
//
//   Y = bf16( D . L2  +  deq(Xq) . deq(Rq)^T  +  bias )
//
// "Most operations happen in 4-bit tensor cores, while the low-rank correction
// runs in higher precision" (imaginepro.ai "Nunchaku 4-Bit Diffusion Inference
// in Diffusers: A Practical Guide", section "Under the Hood"); NVFP4 is the
// Blackwell/B200 precision (chaosnode.de "Nunchaku Lite", section
// "Hardware-Support").
//
// Per 128 x BN output tile, an fp32 accumulator lives in tensor memory:
//   1. the low-rank term: R_PAD/16 bf16 MMAs (kind::f16, K = 16) of the D tile
//      (128 x r) against the L2^T tile (BN x r) initialise the accumulator;
//   2. K/64 block-scaled MMAs (kind::mxf4nvf4, K = 64, one UE4M3 scale per 16)
//      accumulate the 4-bit product, reading the scales from tensor memory;
//   3. the epilogue reads the accumulator with tcgen05.ld, adds the bias,
//      rounds to bf16, stages 32 x 32 pieces in shared memory and stores Y
//      with TMA.
// Two accumulator buffers alternate between tiles so the epilogue of tile t
// overlaps the MMAs of tile t+1.  With BN = 256 they cannot both fit next to
// the scale columns (2 x 256 + 96 > 512), so buffer 1 starts at column 160 and
// shares 96 columns with buffer 0; the epilogue reads those shared columns of a
// tile first and releases them before draining the rest.
// Scales reach tensor memory through registers, not through tcgen05.cp on the
// MMA thread (each copy there costs the tensor pipe about as much as an MMA):
// four scale warps read each stage's scale tiles from shared memory and write
// them with tcgen05.st into one of two scale buffers, each lane quarter its own
// replica of the layout the MMA reads; the MMA thread only waits for them.
// Warp roles (384 threads): warp 0 issues TMA / bulk copies into a STAGES-deep
// shared-memory ring, warp 1 issues the MMAs (one thread), warp 2 owns the
// tensor-memory allocation, warps 4-7 run the epilogue and warps 8-11 write
// the scales (warp w accesses lanes 32*(w%4)..+31).  The grid is persistent
// (one CTA per SM, tiles strided).
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 256;                 // fp4 elements per stage = 128 bytes per row
constexpr int GEMM_THREADS = 384;
constexpr uint32_t GEMM_A_TILE = GEMM_BM * 128;   // 16 KB
constexpr uint32_t GEMM_SFA_TILE = 4 * 512;       // 4 scale tiles (4 x 64 K) for 128 rows
constexpr uint32_t GEMM_OUT_PIECE = 32 * 32;      // 32 rows x 16 bf16, 32-byte swizzle
constexpr uint32_t GEMM_STAGE_OUT = 2 * GEMM_OUT_PIECE;   // per epilogue warp: two pieces

struct GemmParams {
  const uint8_t* x_scales;
  const uint8_t* w_scales;
  const uint16_t* bias;
  uint16_t* Y;            // M x N bf16, row-major (the last tile's stores go straight from registers)
  int y_align32;          // Y is 32-byte aligned: one 32-byte store per row piece
  int head_dim;           // 0: Y row-major; else Y head-major, [N / head_dim][M][head_dim]
  int M, N, K, r;
  int m_tiles, n_tiles, num_tiles, kblocks;
  // MLP epilogue only (the up-projection of an MLP pair; N is the hidden width F):
  const float* inv_lambda_next;   // F, 1/lambda of the down-projection
  const uint32_t* L1f_next;       // the down-projection's L1 (F x r_next) in B-fragment order
  int r_next;                     // the down-projection's rank, <= 32
  uint8_t* h_codes;               // M x F/2 NVFP4 codes of the down-projection's smoothed input
  uint8_t* h_scales;              // their E4M3 scales, tile layout (rows padded to 128, padding 0)
  float* d_acc;                   // M x r_next float32, zero on entry: sum of bf16(Hhat) L1_next
  uint16_t* h_out;                // optional M x F bf16: H itself (null: not written)
};

constexpr int GEMM_MLP_PARTS = 2;       // MLP epilogue warps per lane quarter
constexpr int GEMM_MLP_THREADS = 32 * (4 + 4 * GEMM_MLP_PARTS + 4);   // 4 + 8 epilogue + 4 scale warps

template <int BN, bool MLP = false>
struct GemmCfg {
  static constexpr uint32_t kBTile = BN * 128;
  static constexpr uint32_t kSFBTile = (BN / 128) * GEMM_SFA_TILE;
  static constexpr uint32_t kStage = GEMM_A_TILE + kBTile + GEMM_SFA_TILE + kSFBTile;
  // the MLP epilogue, not the mainloop, bounds that kernel: one ring stage
  // fewer leaves room for its per-tile constants
  static constexpr int kStages = (BN == 256 ? 4 : 6) - (MLP ? 1 : 0);
  // MLP epilogue constants of one tile (two slots): 1/lambda of the next layer,
  // the bias (bf16), and the next layer's L1 fragments for the tile's BN / 16 k-steps
  // (r_next <= 32: at most 4 column tiles of 256 bytes each per k-step)
  static constexpr uint32_t kConstInv = BN * 4, kConstBias = BN * 2, kConstL1 = (BN / 16) * 4 * 256;
  static constexpr uint32_t kConstSlot = MLP ? kConstBias + kConstInv + kConstL1 : 0;
  static constexpr uint32_t kTmemCols = 512;
  // tensor-memory columns: two scale buffers in the top 96, accumulators below
  static constexpr uint32_t kSfaCol0 = 416;              // + 16 j: 4 k-blocks x 4 columns
  static constexpr uint32_t kSfbCol0 = 448;              // + 32 j: 4 k-blocks x BN/32 columns
  static constexpr uint32_t kAcc1Col = (BN == 256 ? 160 : 128);
  static constexpr int kOverlapChunks = (BN == 256 ? (256 - 160) / 32 : 0);
  // epilogue staging: 4 warps x two pieces, or 1 KB per MLP epilogue warp
  static constexpr uint32_t kOutBytes = MLP ? 4 * GEMM_MLP_PARTS * 1024 : 4 * GEMM_STAGE_OUT;
  static constexpr uint32_t kTabBytes = MLP ? 128 * 8 : 0;   // E4M3 (s, RN(1/s)) for the MLP epilogue
  static constexpr uint32_t kBarBytes = (2 * kStages + 13) * 8 + 16;
  static constexpr uint32_t kSmemBytes =
      kStages * kStage + kOutBytes + 2 * kConstSlot + kTabBytes + kBarBytes + 1024;
  static_assert(kSfbCol0 + 32 + 4 * (BN / 32) <= kTmemCols, "scale columns");
  static_assert(kAcc1Col + BN <= kSfaCol0, "accumulator buffer 1");
  static_assert(kStage % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 232448, "shared memory");
};


// Bias of columns n0 .. n0 + BN - 1, 16 bytes per lane (lane l holds columns
// n0 + 8 l .. n0 + 8 l + 7); loaded before the accumulator is ready so that its
// latency is hidden, and handed out with shuffles.
template <int BN>
__device__ __forceinline__ uint4 load_tile_bias(const uint16_t* bias, int n0, int lane) {
  uint4 b = make_uint4(0u, 0u, 0u, 0u);
  if (bias != nullptr && lane < BN / 8) b = __ldg(reinterpret_cast<const uint4*>(bias + n0) + lane);
  return b;
}

// One 32-row x 16-column piece of the output for the warp owning the rows
// row0 .. row0 + 31 (lane = row): accumulator bits `v` plus bias, rounded to
// bf16, staged in one of two 32-byte-swizzled 1 KB buffers and stored with
// TMA.  A store may still be reading the other buffer.
__device__ __forceinline__ void store_piece(const uint32_t (&v)[16], int slot, int c, int lane,
                                            bool has_bias, uint4 bias, int n0, int row0,
                                            const CUtensorMap* tm_y, uint8_t* stg, uint32_t stg_u,
                                            int head_dim) {
  float f[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(v[j]);
  if (has_bias) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int src = 2 * c + u;
      const uint32_t bw[4] = {__shfl_sync(0xffffffffu, bias.x, src), __shfl_sync(0xffffffffu, bias.y, src),
                              __shfl_sync(0xffffffffu, bias.z, src), __shfl_sync(0xffffffffu, bias.w, src)};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        f[u * 8 + 2 * h] += bf16_bits_to_f32(bw[h] & 0xFFFFu);
        f[u * 8 + 2 * h + 1] += bf16_bits_to_f32(bw[h] >> 16);
      }
    }
  }
  // the store issued two pieces ago must have finished reading this buffer
  if (lane == 0) bulk_wait_group_read<1>();
  __syncwarp();
  uint8_t* buf = stg + slot * GEMM_OUT_PIECE;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    uint4 o;
    o.x = pack_bf16x2(f[u * 8 + 0], f[u * 8 + 1]);
    o.y = pack_bf16x2(f[u * 8 + 2], f[u * 8 + 3]);
    o.z = pack_bf16x2(f[u * 8 + 4], f[u * 8 + 5]);
    o.w = pack_bf16x2(f[u * 8 + 6], f[u * 8 + 7]);
    *reinterpret_cast<uint4*>(buf + swz(lane * 32 + u * 16, 1)) = o;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    // row-major Y: (column, row); head-major Y: (column in head, row, head)
    const int n = n0 + c * 16;
    if (head_dim == 0) tma_store_2d(tm_y, stg_u + slot * GEMM_OUT_PIECE, n, row0);
    else tma_store_3d(tm_y, stg_u + slot * GEMM_OUT_PIECE, n % head_dim, row0, n / head_dim);
    bulk_commit_group();
  }
}

// Bias added, rounded to bf16 and stored straight from registers: 16 columns
// (32 bytes, one full sector) of one output row per lane, a lane per row.  The
// bias shuffles need every lane, so the row check comes after them.
__device__ __forceinline__ void store_piece_direct(const uint32_t (&v)[16], int c, bool has_bias,
                                                   uint4 bias, uint16_t* dst, bool row_ok,
                                                   bool align32) {
  float f[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(v[j]);
  if (has_bias) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int src = 2 * c + u;
      const uint32_t bw[4] = {__shfl_sync(0xffffffffu, bias.x, src), __shfl_sync(0xffffffffu, bias.y, src),
                              __shfl_sync(0xffffffffu, bias.z, src), __shfl_sync(0xffffffffu, bias.w, src)};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        f[u * 8 + 2 * h] += bf16_bits_to_f32(bw[h] & 0xFFFFu);
        f[u * 8 + 2 * h + 1] += bf16_bits_to_f32(bw[h] >> 16);
      }
    }
  }
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j] = pack_bf16x2(f[2 * j], f[2 * j + 1]);
  if (!row_ok) return;
  if (align32) {
    st_global_v8(dst, o);
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + 8) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Epilogue of one 128 x BN tile for the warp owning tensor-memory lanes
// 32 q .. 32 q + 31 (= tile rows) with stores straight from registers.  Same
// piece order and release rule as epilogue_tile (below); `yrow` is this
// lane's output row at the tile's first column.
template <int BN, int KOV, typename Order, typename Release, typename Dst>
__device__ __forceinline__ void epilogue_tile_direct(uint32_t acc, uint32_t lane_addr, bool has_bias,
                                                     uint4 bias, Dst dst, bool row_ok,
                                                     bool align32, Order order, Release release) {
  constexpr int kPieces = BN / 16;
  static_assert(KOV % 2 == 0 && KOV < kPieces, "shared pieces: an even count below the tile's");
  uint32_t v[2][16];
  if constexpr (KOV > 0) {
    uint32_t ov[KOV][16];
#pragma unroll
    for (int j = 0; j < KOV; ++j) tmem_ld_32x32b_x16(acc + lane_addr + order(j) * 16, ov[j]);
    tmem_ld_wait();
    tc_fence_before();
    release();
    tmem_ld_32x32b_x16(acc + lane_addr + order(KOV) * 16, v[0]);
#pragma unroll
    for (int j = 0; j < KOV; ++j) store_piece_direct(ov[j], order(j), has_bias, bias, dst(order(j)), row_ok, align32);
  } else {
    tc_fence_before();
    release();
    tmem_ld_32x32b_x16(acc + lane_addr + order(0) * 16, v[0]);
  }
  tmem_ld_wait();
#pragma unroll 2
  for (int i = KOV; i < kPieces; ++i) {
    if (i + 1 < kPieces) tmem_ld_32x32b_x16(acc + lane_addr + order(i + 1) * 16, v[(i + 1) & 1]);
    store_piece_direct(v[i & 1], order(i), has_bias, bias, dst(order(i)), row_ok, align32);
    tmem_ld_wait();
  }
}

// Epilogue of one 128 x BN tile for the warp owning tensor-memory lanes
// 32 q .. 32 q + 31 (= tile rows), in 16-column pieces taken in `order`.  The
// first KOV pieces are the columns the next tile's accumulator shares: they
// are read together, `release` runs after that single wait, and only then are
// they converted and stored.  The remaining pieces are read one ahead of the
// one being stored.  `bias` is the tile's bias from load_tile_bias.
template <int BN, int KOV, typename Order, typename Release>
__device__ __forceinline__ void epilogue_tile(uint32_t acc, uint32_t lane_addr, int lane,
                                              bool has_bias, uint4 bias, int n0, int row0,
                                              const CUtensorMap* tm_y, uint8_t* stg, uint32_t stg_u,
                                              Order order, Release release, int head_dim = 0) {
  constexpr int kPieces = BN / 16;
  static_assert(KOV % 2 == 0 && KOV < kPieces, "shared pieces: an even count below the tile's");
  uint32_t v[2][16];
  if constexpr (KOV > 0) {
    uint32_t ov[KOV][16];
#pragma unroll
    for (int j = 0; j < KOV; ++j) tmem_ld_32x32b_x16(acc + lane_addr + order(j) * 16, ov[j]);
    tmem_ld_wait();
    tc_fence_before();
    release();
    tmem_ld_32x32b_x16(acc + lane_addr + order(KOV) * 16, v[0]);
#pragma unroll
    for (int j = 0; j < KOV; ++j)
      store_piece(ov[j], j & 1, order(j), lane, has_bias, bias, n0, row0, tm_y, stg, stg_u, head_dim);
  } else {
    tc_fence_before();
    release();
    tmem_ld_32x32b_x16(acc + lane_addr + order(0) * 16, v[0]);
  }
  tmem_ld_wait();
#pragma unroll 2
  for (int i = KOV; i < kPieces; ++i) {
    if (i + 1 < kPieces) tmem_ld_32x32b_x16(acc + lane_addr + order(i + 1) * 16, v[(i + 1) & 1]);
    store_piece(v[i & 1], i & 1, order(i), lane, has_bias, bias, n0, row0, tm_y, stg, stg_u, head_dim);
    tmem_ld_wait();
  }
}

// GELU, tanh form, y/2 (1 + tanh u) with u = sqrt(2/pi) (y + 0.044715 y^3),
// evaluated without cancellation through 1 + tanh u = 2 / (1 + e^{-2u}):
// with e = e^{-|2u|} <= 1,  GELU(y) = y / (1 + e) for u >= 0 and
// y e / (1 + e) for u < 0.  With t = 2u log2(e), e = 2^-|t|, taken as
// 2^(64 - |t|) 2^-64 with the device's base-2 exponential, so that where it is
// tiny (y below about -10) it becomes a subnormal number instead of being
// flushed, and the result y e keeps its subnormal value.  No branch: one
// exponential and one reciprocal per element.
__device__ __forceinline__ float gelu_tail_f32(float y, float t) {
  float p, rc;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"(64.0f - fabsf(t)));
  const float e = p * 0x1p-64f;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rc) : "f"(1.0f + e));
  return (t < 0.0f ? y * e : y) * rc;
}

// The same for a pair, the polynomial t = 2 sqrt(2/pi) log2(e) (y + 0.044715
// y^3) in packed f32x2; returns the two results packed as bf16 (RNE), lo first.
__device__ __forceinline__ uint32_t gelu_tanh_bf16x2(float y0, float y1) {
  constexpr float kC = 2.302208198144325f;          // 2 sqrt(2/pi) log2(e)
  constexpr float kC3 = 0.1029432395800235f;        // kC * 0.044715
  const uint64_t y = f32x2_pack(y0, y1);
  const uint64_t p = f32x2_fma(f32x2_mul(y, y), f32x2_pack(kC3, kC3), f32x2_pack(kC, kC));
  float t0, t1;
  f32x2_unpack(f32x2_mul(y, p), t0, t1);
  return pack_bf16x2(gelu_tail_f32(y0, t0), gelu_tail_f32(y1, t1));
}

// The MLP epilogue's per-tile constants in shared memory: 1/lambda_next of
// the tile's columns, its bias (bf16; null without bias) and the next layer's
// L1 fragments of its k-steps (piece c: c * nt * 32 + t * 32 + lane); and the
// kernel's table of E4M3 scales (s, RN(1/s)).
struct MlpTileConsts {
  const float* inv;
  const uint16_t* bias;
  const uint2* l1f;
  const float2* tab;
};

// MLP epilogue of one 16-column piece (piece c of the tile: hidden columns
// n .. n + 15) of the up-projection's tile for the warp owning rows row0 ..
// row0 + 31 (lane = row).  For each element: Y_up = bf16(acc + bias);
// H = bf16(GELU(Y_up)); Hhat = f32(H / lambda_next).  The 16 Hhat of the row
// are one NVFP4 block of the down-projection's input: its 8 code bytes and its
// scale go straight to that layer's activation buffers.  bf16(Hhat) goes
// through a per-warp 32 x 16 shared tile into two m16n8k16 A fragments, whose
// bf16 MMAs with the piece's 16 rows of L1_next accumulate the tile's partial
// of D_next in dacc.
template <int NT>
__device__ __forceinline__ void mlp_piece(const uint32_t (&v)[16], int c, int n, int row, const GemmParams& p,
                                          const MlpTileConsts& tc, uint8_t* dstage, uint32_t dstage_u, int lane,
                                          float (&dacc)[2][NT][4], uint64_t six, uint64_t neg_y6) {
  const int F = p.N;
  // bias and 1/lambda_next of the piece: the same 16 values on every lane
  // (shared-memory broadcasts)
  float b[16];
  if (tc.bias != nullptr) {
    const uint4 b0 = reinterpret_cast<const uint4*>(tc.bias + 16 * c)[0];
    const uint4 b1 = reinterpret_cast<const uint4*>(tc.bias + 16 * c)[1];
    const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      b[2 * i] = bf16_bits_to_f32(bw[i] & 0xFFFFu);
      b[2 * i + 1] = bf16_bits_to_f32(bw[i] >> 16);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = 0.0f;
  }
  float inv[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = reinterpret_cast<const float4*>(tc.inv + 16 * c)[i];
    inv[4 * i] = x.x; inv[4 * i + 1] = x.y; inv[4 * i + 2] = x.z; inv[4 * i + 3] = x.w;
  }
  uint32_t hb[8];          // H, packed bf16 pairs
  uint64_t nh[8];          // -Hhat, packed f32 pairs
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t yb = pack_bf16x2(__uint_as_float(v[2 * i]) + b[2 * i], __uint_as_float(v[2 * i + 1]) + b[2 * i + 1]);
    const uint32_t h = gelu_tanh_bf16x2(bf16_bits_to_f32(yb & 0xFFFFu), bf16_bits_to_f32(yb >> 16));
    hb[i] = h;
    nh[i] = f32x2_mul(f32x2_pack(bf16_bits_to_f32(h & 0xFFFFu), bf16_bits_to_f32(h >> 16)),
                      f32x2_pack(-inv[2 * i], -inv[2 * i + 1]));
  }
  uint32_t sc;
  const uint64_t codes = nvfp4_quant_block16_x2(nh, tc.tab, six, neg_y6, sc);
  if (row < p.M) {
    *reinterpret_cast<uint64_t*>(p.h_codes + static_cast<size_t>(row) * (F / 2) + n / 2) = codes;
    if (p.h_out != nullptr) {
      uint4* dst = reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(row) * F + n);
      dst[0] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
      dst[1] = make_uint4(hb[4], hb[5], hb[6], hb[7]);
    }
  }
  // rows of the last row tile at and beyond M get zero scales (padding)
  p.h_scales[sf_offset(static_cast<uint32_t>(row), static_cast<uint32_t>(n / 16), static_cast<uint32_t>(F))] =
      static_cast<uint8_t>(row < p.M ? sc : 0u);
  if (p.r_next == 0) return;
  // the fragments hold bf16(-Hhat) = -bf16(Hhat) (rounding commutes with
  // negation): dacc accumulates the negated partial, negated back when it is
  // added to d_acc
  uint32_t a8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float lo, hi;
    f32x2_unpack(nh[i], lo, hi);
    a8[i] = pack_bf16x2(lo, hi);
  }
  __syncwarp();   // the previous piece's fragments have been read
  *reinterpret_cast<uint4*>(dstage + lane * 32) = make_uint4(a8[0], a8[1], a8[2], a8[3]);
  *reinterpret_cast<uint4*>(dstage + lane * 32 + 16) = make_uint4(a8[4], a8[5], a8[6], a8[7]);
  __syncwarp();
  uint32_t a[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
    ldmatrix_x4(dstage_u + (16 * mt + (lane & 15)) * 32 + (lane >> 4) * 16, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
  const int nt = p.r_next >> 3;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    if (t < nt) {
      const uint2 bf = tc.l1f[(c * nt + t) * 32 + lane];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) mma_bf16_16816(dacc[mt][t], a[mt][0], a[mt][1], a[mt][2], a[mt][3], bf.x, bf.y);
    }
  }
}

// MLP epilogue of one 128 x BN tile for one of the GEMM_MLP_PARTS warps of
// lane quarter q (part h takes the pieces order(h), order(h + PARTS), ...; the
// first KOV pieces are the columns the next tile's accumulator shares,
// released after one batched read), then the tile's partial D_next into d_acc.
template <int BN, int KOV, typename Order, typename Release>
__device__ __forceinline__ void mlp_epilogue_tile(uint32_t acc, uint32_t lane_addr, int lane, int part, int row0,
                                                  int n0, const GemmParams& p, const MlpTileConsts& tc,
                                                  uint8_t* dstage, uint32_t dstage_u, Order order, Release release) {
  constexpr int kPieces = BN / 16, kParts = GEMM_MLP_PARTS, kNT = 4;
  static_assert(KOV % kParts == 0, "every part takes the same number of shared pieces");
  constexpr int kOvMine = KOV / kParts;
  const int row = row0 + lane;
  const uint64_t six = f32x2_pack(6.0f, 6.0f);
  const float y6 = tc.tab[0x4C].y;   // code 0x4C is 6.0: RN(1/6)
  const uint64_t neg_y6 = f32x2_pack(-y6, -y6);
  float dacc[2][kNT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int t = 0; t < kNT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) dacc[mt][t][i] = 0.0f;
  if constexpr (kOvMine > 0) {
    uint32_t ov[kOvMine][16];
#pragma unroll
    for (int j = 0; j < kOvMine; ++j) tmem_ld_32x32b_x16(acc + lane_addr + order(part + kParts * j) * 16, ov[j]);
    tmem_ld_wait();
    tc_fence_before();
    release();
#pragma unroll
    for (int j = 0; j < kOvMine; ++j) {
      const int c = order(part + kParts * j);
      mlp_piece<kNT>(ov[j], c, n0 + 16 * c, row, p, tc, dstage, dstage_u, lane, dacc, six, neg_y6);
    }
  } else {
    tc_fence_before();
    release();
  }
  for (int i = part + KOV; i < kPieces; i += kParts) {
    uint32_t v[16];
    const int c = order(i);
    tmem_ld_32x32b_x16(acc + lane_addr + c * 16, v);
    tmem_ld_wait();
    mlp_piece<kNT>(v, c, n0 + 16 * c, row, p, tc, dstage, dstage_u, lane, dacc, six, neg_y6);
  }
  // the tile's partial D_next: fragment rows lane / 4 (+ 8) of each 16-row
  // block, columns 8 t + 2 (lane % 4) (+ 1)
  const int nt = p.r_next >> 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
      if (t >= nt) continue;
      const int r_lo = row0 + 16 * mt + (lane >> 2), col = 8 * t + 2 * (lane & 3);
      if (r_lo < p.M) {
        atomicAdd(p.d_acc + static_cast<size_t>(r_lo) * p.r_next + col, -dacc[mt][t][0]);
        atomicAdd(p.d_acc + static_cast<size_t>(r_lo) * p.r_next + col + 1, -dacc[mt][t][1]);
      }
      if (r_lo + 8 < p.M) {
        atomicAdd(p.d_acc + static_cast<size_t>(r_lo + 8) * p.r_next + col, -dacc[mt][t][2]);
        atomicAdd(p.d_acc + static_cast<size_t>(r_lo + 8) * p.r_next + col + 1, -dacc[mt][t][3]);
      }
    }
}

template <int BN, int R_PAD, bool MLP = false>
__global__ void __launch_bounds__(MLP ? GEMM_MLP_THREADS : GEMM_THREADS, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_l2,
                    const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using Cfg = GemmCfg<BN, MLP>;
  constexpr int S = Cfg::kStages;
  constexpr uint32_t kLRLayout = (R_PAD == 64 ? LAYOUT_SW128 : R_PAD == 32 ? LAYOUT_SW64 : LAYOUT_SW32);
  constexpr uint32_t kLRSbo = 8 * R_PAD * 2;
  // epilogue warps: 4 (one per lane quarter), or 4 * GEMM_MLP_PARTS for the
  // MLP epilogue (that many per lane quarter, splitting the tile's columns);
  // the scale warps follow
  constexpr int kEpiWarps = MLP ? 4 * GEMM_MLP_PARTS : 4;
  constexpr int kScaleWarp0 = 4 + kEpiWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* out_stage = smem + S * Cfg::kStage;
  uint8_t* const_slots = out_stage + Cfg::kOutBytes;   // MLP epilogue constants, 2 slots
  float2* e4m3_tab = reinterpret_cast<float2*>(const_slots + 2 * Cfg::kConstSlot);   // MLP epilogue only
  uint64_t* bars = reinterpret_cast<uint64_t*>(const_slots + 2 * Cfg::kConstSlot + Cfg::kTabBytes);
  // bars[0..S) full, [S..2S) empty, 2S/2S+1 tmem_full[2], 2S+2 tmem_free, 2S+3 drain,
  // 2S+4/2S+5 sf_ready[2] (scale warps -> MMA), 2S+6/2S+7 sf_free[2] (MMA -> scale warps),
  // 2S+8 tmem_done (tensor memory no longer used: MMA thread + epilogue warps),
  // 2S+9/2S+10 const_full[2], 2S+11/2S+12 const_free[2] (MLP epilogue constants)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t smem_base = smem_u32(smem);
  auto stage_a = [&](int s) { return smem_base + s * Cfg::kStage; };
  auto stage_b = [&](int s) { return smem_base + s * Cfg::kStage + GEMM_A_TILE; };
  auto stage_sfa = [&](int s) { return smem_base + s * Cfg::kStage + GEMM_A_TILE + Cfg::kBTile; };
  auto stage_sfb = [&](int s) {
    return smem_base + s * Cfg::kStage + GEMM_A_TILE + Cfg::kBTile + GEMM_SFA_TILE;
  };
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto tmem_full = [&](int b) { return smem_u32(bars + 2 * S + b); };
  const uint32_t tmem_free = smem_u32(bars + 2 * S + 2);
  const uint32_t drain_bar = smem_u32(bars + 2 * S + 3);
  auto sf_ready = [&](uint32_t b) { return smem_u32(bars + 2 * S + 4 + b); };
  auto sf_free = [&](uint32_t b) { return smem_u32(bars + 2 * S + 6 + b); };
  const uint32_t tmem_done = smem_u32(bars + 2 * S + 8);
  auto const_full = [&](int b) { return smem_u32(bars + 2 * S + 9 + b); };
  auto const_free = [&](int b) { return smem_u32(bars + 2 * S + 11 + b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full(0), 1);
    mbar_init(tmem_full(1), 1);
    mbar_init(tmem_free, kEpiWarps);  // one arrive per epilogue warp
    mbar_init(drain_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sf_ready(b), 4);      // one arrive per scale warp
      mbar_init(sf_free(b), 1);
    }
    mbar_init(tmem_done, kEpiWarps + 1);   // the MMA thread and the epilogue warps
    for (int b = 0; b < 2; ++b) {
      mbar_init(const_full(b), 1);
      mbar_init(const_free(b), kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (MLP) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x) e4m3_tab[c] = e4m3_table_entry(c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the next kernel of the stream may be launched now; it waits for this grid
  // before it touches global memory (see the activation kernel)
  pdl_launch_dependents();

  const int kb_per_tile = p.kblocks;
  const uint32_t k_tiles64 = static_cast<uint32_t>(p.K) >> 6;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      if (R_PAD > 0) {
        tma_prefetch_desc(&tm_d);
        tma_prefetch_desc(&tm_l2);
      }
      int stage = 0;
      uint32_t phase = 0;
      int8_t fill_parity[S];
      for (int s = 0; s < S; ++s) fill_parity[s] = -1;
      const uint32_t tx_main = GEMM_A_TILE + Cfg::kBTile + GEMM_SFA_TILE + Cfg::kSFBTile;
      const uint32_t tx_lr = (GEMM_BM + BN) * R_PAD * 2;
      // Programmatic dependent launch: this grid may start while the kernel
      // that writes the activation codes, scales and D is still running.  The
      // weight half of the first stage is loaded at once; its activation half
      // waits for that kernel (griddepcontrol.wait), as does everything after
      // it.  (Deeper early weight loads compete with that kernel's own reads
      // of X: with the first four stages early the qkv layer took 0.5 us
      // longer back to back.)  The stage barriers count both halves' bytes.
      constexpr int kEarlyStages = 1;
      struct Deferred {
        int stage, kb, m0, mb;   // kb < 0: the low-rank slot (D tile)
      };
      Deferred deferred[S];
      int ndeferred = 0;
      bool dependency_met = false;
      auto load_activation = [&](const Deferred& q) {
        if (q.kb < 0) {
          tma_load_2d(stage_a(q.stage), &tm_d, full_bar(q.stage), 0, q.m0);
        } else {
          tma_load_2d(stage_a(q.stage), &tm_a, full_bar(q.stage), q.kb * 128, q.m0);
          bulk_load(stage_sfa(q.stage), p.x_scales + (static_cast<size_t>(q.mb) * k_tiles64 + q.kb * 4) * 512,
                    GEMM_SFA_TILE, full_bar(q.stage));
        }
      };
      auto meet_dependency = [&]() {
        pdl_wait();
        for (int i = 0; i < ndeferred; ++i) load_activation(deferred[i]);
        ndeferred = 0;
        dependency_met = true;
      };
      // issue the activation half of a stage now, or defer it (first S stages)
      auto activation_half = [&](int st, int kb, int m0, int mb) {
        const Deferred q{st, kb, m0, mb};
        if (dependency_met) {
          load_activation(q);
        } else {
          deferred[ndeferred++] = q;
          if (ndeferred == kEarlyStages) meet_dependency();
        }
      };
      bool ok = true;
      int const_parity[2] = {-1, -1};
      int local_t = 0;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local_t) {
        const int mb = t % p.m_tiles, nb = t / p.m_tiles;
        const int m0 = mb * GEMM_BM, n0 = nb * BN;
        if constexpr (MLP) {
          // the MLP epilogue's constants of this tile into slot local_t % 2,
          // once the epilogue has finished the tile that used it before
          const int cb = local_t & 1;
          if (local_t >= 2 &&
              !mbar_wait(const_free(cb), static_cast<uint32_t>((local_t >> 1) - 1) & 1u, abort_flag, KID_GEMM, 3)) {
            ok = false;
            break;
          }
          const uint32_t slot = smem_u32(const_slots + cb * Cfg::kConstSlot);
          const int nt = p.r_next >> 3;
          const uint32_t l1_bytes = static_cast<uint32_t>(BN / 16) * nt * 256u;
          mbar_arrive_expect_tx(const_full(cb), Cfg::kConstInv + (p.bias != nullptr ? Cfg::kConstBias : 0u) + l1_bytes);
          bulk_load(slot, p.inv_lambda_next + n0, Cfg::kConstInv, const_full(cb));
          if (p.bias != nullptr) bulk_load(slot + Cfg::kConstInv, p.bias + n0, Cfg::kConstBias, const_full(cb));
          if (l1_bytes > 0)
            bulk_load(slot + Cfg::kConstInv + Cfg::kConstBias,
                      reinterpret_cast<const uint8_t*>(p.L1f_next) + static_cast<size_t>(n0 / 16) * nt * 256u, l1_bytes,
                      const_full(cb));
          const_parity[cb] = (local_t >> 1) & 1;
        }
        if (R_PAD > 0) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, KID_GEMM, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), tx_lr);
          tma_load_2d(stage_b(stage), &tm_l2, full_bar(stage), 0, n0);
          activation_half(stage, -1, m0, mb);
          fill_parity[stage] = static_cast<int8_t>(phase);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < kb_per_tile; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, KID_GEMM, 2)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), tx_main);
          tma_load_2d(stage_b(stage), &tm_b, full_bar(stage), kb * 128, n0);
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            bulk_load(stage_sfb(stage) + g * GEMM_SFA_TILE,
                      p.w_scales + (static_cast<size_t>(n0 / 128 + g) * k_tiles64 + kb * 4) * 512,
                      GEMM_SFA_TILE, full_bar(stage));
          activation_half(stage, kb, m0, mb);
          fill_parity[stage] = static_cast<int8_t>(phase);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      // fewer than S stages in all, or an abort: complete the deferred stages
      if (!dependency_met) meet_dependency();
      if (*abort_flag) {
        for (int s = 0; s < S; ++s)
          if (fill_parity[s] >= 0) mbar_wait_drain(full_bar(s), static_cast<uint32_t>(fill_parity[s]));
        for (int b = 0; b < 2; ++b)
          if (const_parity[b] >= 0) mbar_wait_drain(const_full(b), static_cast<uint32_t>(const_parity[b]));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idf = idesc_nvfp4(GEMM_BM, BN);
      const uint32_t idb = idesc_bf16(GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any_issued = false;
      int local = 0;   // tiles issued by this CTA
      uint32_t n = 0;  // k-blocks issued (selects the scale buffer)
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t acc = tmem_base + (buf ? Cfg::kAcc1Col : 0u);
        // the epilogue has drained the previous tile's shared columns (and so
        // everything of the tile before it, which used this buffer)
        if (local > 0) {
          if (!mbar_wait(tmem_free, static_cast<uint32_t>(local - 1) & 1u, abort_flag, KID_GEMM, 4)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        uint32_t accumulate = 0;
        if (R_PAD > 0) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, KID_GEMM, 5)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = make_smem_desc(stage_a(stage), kLRLayout, kLRSbo, 0);
          const uint64_t bd = make_smem_desc(stage_b(stage), kLRLayout, kLRSbo, 0);
#pragma unroll
          for (int kk = 0; kk < R_PAD / 16; ++kk) {
            tc_mma_bf16(acc, ad + 2 * kk, bd + 2 * kk, idb, accumulate);
            accumulate = 1;
          }
          tc_commit(empty_bar(stage));
          any_issued = true;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < kb_per_tile; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, KID_GEMM, 6)) { ok = false; break; }
          const uint32_t sb = n & 1u;
          if (!mbar_wait(sf_ready(sb), (n >> 1) & 1u, abort_flag, KID_GEMM, 9)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa = tmem_base + Cfg::kSfaCol0 + 16 * sb;
          const uint32_t sfb = tmem_base + Cfg::kSfbCol0 + 32 * sb;
          const uint64_t ad = make_smem_desc(stage_a(stage), LAYOUT_SW128, 1024, 0);
          const uint64_t bd = make_smem_desc(stage_b(stage), LAYOUT_SW128, 1024, 0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tc_mma_nvfp4(acc, ad + 2 * i, bd + 2 * i, idf, sfa + 4 * i, sfb + i * (BN / 32), accumulate);
            accumulate = 1;
          }
          tc_commit(empty_bar(stage));
          tc_commit(sf_free(sb));
          ++n;
          any_issued = true;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(tmem_full(buf));
      }
      if (*abort_flag && any_issued) {
        // make sure no MMA still writes tensor memory before it is freed
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0);
      }
      mbar_arrive(tmem_done);
    }
  } else if (MLP && warp >= 4 && warp < kScaleWarp0) {
    // --------------------------------------------------------- MLP epilogue
    const int q = warp & 3, part = (warp - 4) >> 2;
    uint8_t* dstage = out_stage + (warp - 4) * 1024;
    const uint32_t dstage_u = smem_u32(dstage);
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const int mb = t % p.m_tiles, nb = t / p.m_tiles;
      const int m0 = mb * GEMM_BM, n0 = nb * BN;
      const int buf = local & 1;
      const uint32_t acc = tmem_base + (buf ? Cfg::kAcc1Col : 0u);
      if (!mbar_wait(const_full(buf), static_cast<uint32_t>(local >> 1) & 1u, abort_flag, KID_GEMM, 10)) break;
      if (!mbar_wait(tmem_full(buf), static_cast<uint32_t>(local >> 1) & 1u, abort_flag, KID_GEMM, 8)) break;
      tc_fence_after();
      constexpr int kPieces = BN / 16, kOv = 2 * Cfg::kOverlapChunks;
      auto order = [&](int i) { return buf ? i : (i + kPieces - kOv) % kPieces; };
      auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_free);
      };
      const uint8_t* cs = const_slots + buf * Cfg::kConstSlot;
      const MlpTileConsts tc{reinterpret_cast<const float*>(cs),
                             p.bias != nullptr ? reinterpret_cast<const uint16_t*>(cs + Cfg::kConstInv) : nullptr,
                             reinterpret_cast<const uint2*>(cs + Cfg::kConstInv + Cfg::kConstBias), e4m3_tab};
      mlp_epilogue_tile<BN, kOv>(acc, lane_addr, lane, part, m0 + q * 32, n0, p, tc, dstage, dstage_u, order,
                                 release);
      __syncwarp();
      if (lane == 0) mbar_arrive(const_free(buf));
    }
    // this warp's tensor-memory reads are over (every tcgen05.ld waited)
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tmem_done);
  } else if (!MLP && warp >= 4 && warp < kScaleWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    uint8_t* stg = out_stage + q * GEMM_STAGE_OUT;
    const uint32_t stg_u = smem_u32(stg);
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const int mb = t % p.m_tiles, nb = t / p.m_tiles;
      const int m0 = mb * GEMM_BM, n0 = nb * BN;
      const int buf = local & 1;
      const uint32_t acc = tmem_base + (buf ? Cfg::kAcc1Col : 0u);
      const uint4 tile_bias = load_tile_bias<BN>(p.bias, n0, lane);
      if (!mbar_wait(tmem_full(buf), static_cast<uint32_t>(local >> 1) & 1u, abort_flag, KID_GEMM, 8))
        break;
      tc_fence_after();
      // buffer 0 shares its top columns with buffer 1, buffer 1 its bottom
      // columns with buffer 0: those pieces come first
      constexpr int kPieces = BN / 16, kOv = 2 * Cfg::kOverlapChunks;
      auto order = [&](int i) { return buf ? i : (i + kPieces - kOv) % kPieces; };
      auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_free);
      };
      if (t + static_cast<int>(gridDim.x) < p.num_tiles) {
        epilogue_tile<BN, kOv>(acc, lane_addr, lane, p.bias != nullptr, tile_bias, n0, m0 + q * 32, &tm_y,
                               stg, stg_u, order, release, p.head_dim);
      } else {
        // the CTA's last tile: no MMA runs any more, so the stores go straight
        // from registers (shorter per piece than staging + TMA; while the
        // mainloop runs they would compete with it for the load/store unit)
        const int row = m0 + q * 32 + lane;
        auto dst = [&](int c) {
          const int n = n0 + c * 16;
          return p.head_dim == 0
                     ? p.Y + static_cast<size_t>(row) * p.N + n
                     : p.Y + (static_cast<size_t>(n / p.head_dim) * p.M + row) * p.head_dim + n % p.head_dim;
        };
        epilogue_tile_direct<BN, kOv>(acc, lane_addr, p.bias != nullptr, tile_bias, dst, row < p.M,
                                      p.y_align32 != 0, order, release);
      }
    }
    if (lane == 0) bulk_wait_group_all();
    // this warp's tensor-memory reads are over (every tcgen05.ld waited)
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tmem_done);
  } else if (warp >= kScaleWarp0) {
    // ------------------------------------------------------------ scale warps
    // Each lane quarter gets its replica of the layout the MMA reads: for
    // k-block i of a stage, 4 columns of A scales and BN/32 columns of B
    // scales, column (4 i + g) / (BN/32 i + g) of lane 32 q + l holding the 4
    // scales of row 32 g + l -- exactly the 16 bytes at offset 16 l of the
    // 512-byte scale tile in shared memory.
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0, n = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      if (R_PAD > 0) {
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      for (int kb = 0; kb < kb_per_tile; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag, KID_GEMM, 20)) { ok = false; break; }
        const uint8_t* sa = smem + (stage_sfa(stage) - smem_base) + lane * 16;
        const uint8_t* sbp = smem + (stage_sfb(stage) - smem_base) + lane * 16;
        uint32_t va[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 x = *reinterpret_cast<const uint4*>(sa + i * 512);
          va[4 * i] = x.x; va[4 * i + 1] = x.y; va[4 * i + 2] = x.z; va[4 * i + 3] = x.w;
        }
        constexpr int kG = BN / 128;
        uint32_t vb[16 * kG];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int g = 0; g < kG; ++g) {
            const uint4 x = *reinterpret_cast<const uint4*>(sbp + (g * 4 + i) * 512);
            vb[4 * kG * i + 4 * g] = x.x; vb[4 * kG * i + 4 * g + 1] = x.y;
            vb[4 * kG * i + 4 * g + 2] = x.z; vb[4 * kG * i + 4 * g + 3] = x.w;
          }
        const uint32_t sb = n & 1u;
        if (n >= 2 && !mbar_wait(sf_free(sb), ((n >> 1) - 1) & 1u, abort_flag, KID_GEMM, 21)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st_32x32b_x16(tmem_base + lane_addr + Cfg::kSfaCol0 + 16 * sb, va);
        if constexpr (kG == 2) tmem_st_32x32b_x32(tmem_base + lane_addr + Cfg::kSfbCol0 + 32 * sb, vb);
        else tmem_st_32x32b_x16(tmem_base + lane_addr + Cfg::kSfbCol0 + 32 * sb, vb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_ready(sb));
        ++n;
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
  }

  // Every lane of every warp meets here (a warp whose elected lane worked
  // alone reconverges first), and the allocator frees tensor memory only once
  // the MMAs have completed and the epilogue has read the last accumulator.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    mbar_wait_drain(tmem_done, 0, 4 * kWaitLimitNs);
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace svdq
