// svdq.cu -- C ABI of the B200 SVDQuant W4A4 linear layer (host side) and the
// single translation unit that holds every device kernel of the library.
//
// The entry points mirror the statement of the problem on the pages: a
// drop-in replacement of a linear layer whose weights are quantised offline
// (chaosnode.de "Nunchaku Lite: 4-Bit Diffusion-Inferenz direkt in
// Diffusers", section "Nunchaku Lite vs. Original": runtime SVDQ layers in
// place of nn.Linear; watch-ia.com: quantise, package, load and verify) and
// run W4A4 at inference (aiphreaks.com "Bringing Nunchaku 4-bit Diffusion
// Inference to Diffusers", section "Technical Breakdown and Performance
// Metrics").  Argument meaning, layouts and error behaviour: include/svdq.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cusolverDn.h>

#include <algorithm>
#include <atomic>
#include <random>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <string>
#include <vector>

#include "svdq.h"
#include "act_quant.cuh"
#include "act128.cuh"
#include "fp4_gemm.cuh"
#include "int4.cuh"
#include "prepare.cuh"
#include "small_m.cuh"

using namespace svdq;

namespace {

thread_local std::string g_last_error;

svdq_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return SVDQ_ERR_CUDA;
}

#define SVDQ_CUDA(call)                                   \
  do {                                                    \
    cudaError_t e_ = (call);                              \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);   \
  } while (0)

#define SVDQ_CHECK_LAUNCH(name)                           \
  do {                                                    \
    cudaError_t e_ = cudaGetLastError();                  \
    if (e_ != cudaSuccess) return cuda_fail(e_, name);    \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int r_pad_of(int r) { return r == 0 ? 0 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

// Shape check shared by every entry point (see the header for the rules).
svdq_status check_layer_shape(int N, int K, int r) {
  if (N <= 0 || K <= 0 || r < 0 || (K % 16) != 0) return SVDQ_ERR_INVALID_ARG;
  if ((K % 256) != 0 || (N % 128) != 0 || (r % 8) != 0 || r > 64 || r > std::min(N, K))
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  return SVDQ_OK;
}

svdq_status check_weight(const svdq_weight* w) {
  if (w == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (w->format != SVDQ_FORMAT_NVFP4 && w->format != SVDQ_FORMAT_INT4) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(w->N, w->K, w->r);
  if (s != SVDQ_OK) return s;
  if (w->w_codes == nullptr || w->w_scales == nullptr || w->inv_lambda == nullptr)
    return SVDQ_ERR_INVALID_ARG;
  if (w->r > 0 && (w->L1 == nullptr || w->L1f == nullptr || w->L2t == nullptr || w->L1t == nullptr))
    return SVDQ_ERR_INVALID_ARG;
  if (w->has_bias && w->bias == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(w->w_codes) || !aligned16(w->w_scales) || !aligned16(w->inv_lambda) ||
      (w->r > 0 && (!aligned16(w->L1) || !aligned16(w->L1f) || !aligned16(w->L2t) || !aligned16(w->L1t))) ||
      (w->has_bias && !aligned16(w->bias)))
    return SVDQ_ERR_MISALIGNED;
  return SVDQ_OK;
}

int m_pad_of(int M) { return (M + 127) / 128 * 128; }

// Process-wide overrides of automatic launch choices (svdq_set_override);
// 0 = automatic.  Only the explicit ABI call changes them.
std::atomic<int> g_override[SVDQ_OVERRIDE_COUNT];

int override_value(int which) {
  return (which > 0 && which < SVDQ_OVERRIDE_COUNT) ? g_override[which].load(std::memory_order_relaxed) : 0;
}

// Dynamic shared memory above 48 KB has to be enabled for each kernel on each
// device: the attribute applies to the device that is current when it is
// set.  Done once per (device, kernel).
svdq_status opt_in_smem(const void* kernel, uint32_t bytes, const char* what) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  int dev = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({dev, kernel})) return SVDQ_OK;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_fail(e, what);
  done.insert({dev, kernel});
  return SVDQ_OK;
}

// --------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no libcuda link).
// --------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `rows` rows,
// row pitch `pitch_bytes`; box `box_inner` x `box_rows`.
svdq_status make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) {
    g_last_error = "cuTensorMapEncodeTiled entry point unavailable";
    return SVDQ_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    std::snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (%d) inner=%llu rows=%llu box=%ux%u",
                  static_cast<int>(r), static_cast<unsigned long long>(inner),
                  static_cast<unsigned long long>(rows), box_inner, box_rows);
    g_last_error = buf;
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// Head-major output [heads][M][head_dim] bf16, stored in 16-column x 32-row
// pieces through the same 32-byte-swizzled staging as the row-major map.
svdq_status make_tmap_heads(CUtensorMap* m, const void* base, int head_dim, int M, int heads) {
  auto fn = encode_fn();
  if (fn == nullptr) {
    g_last_error = "cuTensorMapEncodeTiled entry point unavailable";
    return SVDQ_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(M),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(head_dim) * 2 * static_cast<cuuint64_t>(M)};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    std::snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled (heads) failed (%d) head_dim=%d M=%d heads=%d",
                  static_cast<int>(r), head_dim, M, heads);
    g_last_error = buf;
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

CUtensorMapSwizzle lr_swizzle(int r_pad) {
  return r_pad == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                     : r_pad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// --------------------------------------------------------------------------
// Launchers
// --------------------------------------------------------------------------
template <int R_PAD>
svdq_status launch_act(const CUtensorMap& tx, const ActParams& p, cudaStream_t st) {
  constexpr uint32_t smem = ActSmem<R_PAD>::kBytes;
  {
    const svdq_status so =
        opt_in_smem(reinterpret_cast<const void*>(act_quant_kernel<R_PAD>), smem, "cudaFuncSetAttribute(act)");
    if (so != SVDQ_OK) return so;
  }
  const int grid = p.M_pad / ACT_ROWS * p.ks;
  // programmatic dependent launch (the kernel waits for its predecessor before
  // touching global memory), and a cluster of ks CTAs per row block when ks > 1
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(ACT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(p.ks);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.ks > 1 ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, act_quant_kernel<R_PAD>, tx, p);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_kernel launch");
  SVDQ_CHECK_LAUNCH("act_quant_kernel");
  return SVDQ_OK;
}

// K split of the activation kernel: with few row blocks of 16 (small M), a
// cluster of ks CTAs shares each block so that more SMs stream X.  The largest
// ks <= 8 with K % (64 ks) == 0, at least one 64-column sub-tile per warp
// (K / ks >= 512) and at most one CTA per SM.  SVDQ_OVERRIDE_ACT_KSPLIT
// (svdq_set_override) replaces it when K % (64 ks) == 0.
int act_k_split(int M, int K) {
  {
    const int v = override_value(SVDQ_OVERRIDE_ACT_KSPLIT);
    if (v >= 1 && v <= ACT_MAX_KS && K % (ACT_SUB * v) == 0) return v;
  }
  const int blocks = (M + ACT_ROWS - 1) / ACT_ROWS;
  int ks = 1;
  for (int c = 2; c <= ACT_MAX_KS; ++c)
    if (K % (ACT_SUB * c) == 0 && K / c >= ACT_SUB * ACT_WARPS && blocks * c <= num_sms()) ks = c;
  return ks;
}

// act128_kernel takes a layer when each CTA walks at least this many 64-column
// stages (measured: at 6 stages, qkv at 1024x1024, the 16-row kernel is 4 us
// faster; at 24, mlp_down and qkv at 18432 tokens, the tensor-core kernel is 6
// and 14 us faster).
constexpr int A128_MIN_STAGES = 12;

// K split of act128_kernel: the largest ks <= A128_MAX_KS with K % (64 ks) == 0
// and at most two CTAs per SM (128-row blocks x ks); SVDQ_OVERRIDE_ACT_KSPLIT
// (svdq_set_override) replaces it when K % (64 ks) == 0.
int a128_k_split(int M, int K) {
  {
    const int v = override_value(SVDQ_OVERRIDE_ACT_KSPLIT);
    if (v >= 1 && v <= A128_MAX_KS && K % (64 * v) == 0) return v;
  }
  const int blocks = m_pad_of(M) / A128_ROWS;
  int ks = 1;
  for (int c = 2; c <= A128_MAX_KS; ++c)
    if (K % (64 * c) == 0 && blocks * c <= 2 * num_sms()) ks = c;
  return ks;
}

// A value no flag of an earlier call (nor, but with probability 2^-64, stale
// workspace contents) holds: a per-process random key mixed with a counter.
unsigned long long next_epoch() {
  static const unsigned long long key = [] {
    std::random_device rd;
    return (static_cast<unsigned long long>(rd()) << 32) ^ rd() ^ 0x5DEECE66Dull;
  }();
  static std::atomic<unsigned long long> counter{0};
  unsigned long long e = 0;
  while (e == 0) e = key ^ ((counter.fetch_add(1) + 1) * 0x9E3779B97F4A7C15ull);
  return e;
}

template <int R_PAD>
svdq_status launch_act128(const CUtensorMap& tx, const CUtensorMap& tl1t, const A128Params& p, cudaStream_t st) {
  constexpr uint32_t smem = A128Cfg<R_PAD>::kBytes;
  {
    const svdq_status so =
        opt_in_smem(reinterpret_cast<const void*>(act128_kernel<R_PAD>), smem, "cudaFuncSetAttribute(act128)");
    if (so != SVDQ_OK) return so;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.M_pad / A128_ROWS * p.ks));
  cfg.blockDim = dim3(A128_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, act128_kernel<R_PAD>, tx, tl1t, p);
  if (e != cudaSuccess) return cuda_fail(e, "act128_kernel launch");
  SVDQ_CHECK_LAUNCH("act128_kernel");
  return SVDQ_OK;
}

template <int BN, int R_PAD, bool MLP = false>
svdq_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                        const CUtensorMap& tl2, const CUtensorMap& ty, const GemmParams& p,
                        cudaStream_t st) {
  using Cfg = GemmCfg<BN, MLP>;
  {
    const svdq_status so = opt_in_smem(reinterpret_cast<const void*>(fp4_gemm_kernel<BN, R_PAD, MLP>),
                                       Cfg::kSmemBytes, "cudaFuncSetAttribute(gemm)");
    if (so != SVDQ_OK) return so;
  }
  const int grid = std::min(p.num_tiles, num_sms());
  // programmatic dependent launch: the kernel may start while the preceding
  // kernel of the stream (the activation kernel) finishes; it waits for it
  // before reading anything that kernel writes
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(MLP ? GEMM_MLP_THREADS : GEMM_THREADS);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fp4_gemm_kernel<BN, R_PAD, MLP>, ta, tb, td, tl2, ty, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_gemm_kernel launch");
  SVDQ_CHECK_LAUNCH("fp4_gemm_kernel");
  return SVDQ_OK;
}

template <int BN, bool MLP = false>
svdq_status dispatch_gemm_r(int r_pad, const CUtensorMap& ta, const CUtensorMap& tb,
                            const CUtensorMap& td, const CUtensorMap& tl2, const CUtensorMap& ty,
                            const GemmParams& p, cudaStream_t st) {
  switch (r_pad) {
    case 0: return launch_gemm<BN, 0, MLP>(ta, tb, td, tl2, ty, p, st);
    case 16: return launch_gemm<BN, 16, MLP>(ta, tb, td, tl2, ty, p, st);
    case 32: return launch_gemm<BN, 32, MLP>(ta, tb, td, tl2, ty, p, st);
    default: return launch_gemm<BN, 64, MLP>(ta, tb, td, tl2, ty, p, st);
  }
}

// ---- INT4 variant -------------------------------------------------------
template <int R_PAD>
svdq_status launch_act_int4(const CUtensorMap& tx, const Int4ActParams& p, cudaStream_t st) {
  constexpr uint32_t smem = Int4ActSmem<R_PAD>::kBytes;
  {
    const svdq_status so = opt_in_smem(reinterpret_cast<const void*>(act_quant_int4_kernel<R_PAD>), smem,
                                       "cudaFuncSetAttribute(act int4)");
    if (so != SVDQ_OK) return so;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.M_pad / ACT_ROWS));
  cfg.blockDim = dim3(ACT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, act_quant_int4_kernel<R_PAD>, tx, p);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_int4_kernel launch");
  SVDQ_CHECK_LAUNCH("act_quant_int4_kernel");
  return SVDQ_OK;
}

svdq_status quantize_act_int4_impl(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                                   uint8_t* x_scales, uint16_t* D, cudaStream_t st) {
  const int K = w->K, r = w->r;
  CUtensorMap tx{};
  svdq_status s = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M,
                            static_cast<uint64_t>(K) * 2, ACT_SUB, ACT_ROWS,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  Int4ActParams p;
  p.inv_lambda = w->inv_lambda;
  p.L1f = reinterpret_cast<const uint32_t*>(w->L1f);
  p.x_codes = x_codes;
  p.x_scales = reinterpret_cast<uint16_t*>(x_scales);
  p.D = D;
  p.M = M;
  p.K = K;
  p.r = r;
  p.M_pad = m_pad_of(M);
  switch (r_pad_of(r)) {
    case 0: return launch_act_int4<0>(tx, p, st);
    case 16: return launch_act_int4<16>(tx, p, st);
    case 32: return launch_act_int4<32>(tx, p, st);
    default: return launch_act_int4<64>(tx, p, st);
  }
}

template <int R_PAD>
svdq_status launch_gemm_int4(const CUtensorMap* maps, const Int4GemmParams& p, cudaStream_t st) {
  {
    const svdq_status so = opt_in_smem(reinterpret_cast<const void*>(int4_gemm_kernel<R_PAD>), I4_SMEM_BYTES,
                                       "cudaFuncSetAttribute(gemm int4)");
    if (so != SVDQ_OK) return so;
  }
  const dim3 grid(static_cast<unsigned>((p.M + I4_BM - 1) / I4_BM), static_cast<unsigned>(p.N / I4_BN));
  int4_gemm_kernel<R_PAD><<<grid, I4_THREADS, I4_SMEM_BYTES, st>>>(maps[0], maps[1], maps[2], maps[3], p);
  SVDQ_CHECK_LAUNCH("int4_gemm_kernel");
  return SVDQ_OK;
}

svdq_status gemm_int4_impl(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                           const svdq_weight* w, uint16_t* Y, cudaStream_t st, int head_dim) {
  const int N = w->N, K = w->K;
  const int m_pad = m_pad_of(M);
  CUtensorMap maps[4] = {};
  svdq_status s = make_tmap(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, K / 2, M, K / 2, 128, I4_BM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  s = make_tmap(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w_codes, K / 2, N, K / 2, 128, I4_BN,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  s = make_tmap(&maps[2], CU_TENSOR_MAP_DATA_TYPE_UINT16, x_scales, m_pad, K / INT4_GROUP,
                static_cast<uint64_t>(m_pad) * 2, I4_BM, I4_GPS, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != SVDQ_OK) return s;
  s = make_tmap(&maps[3], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->w_scales, N, K / INT4_GROUP,
                static_cast<uint64_t>(N) * 2, I4_BN, I4_GPS, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != SVDQ_OK) return s;
  Int4GemmParams p;
  p.D = D;
  p.L2t = w->L2t;
  p.bias = w->has_bias ? w->bias : nullptr;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = w->r;
  p.head_dim = head_dim;
  switch (r_pad_of(w->r)) {
    case 0: return launch_gemm_int4<0>(maps, p, st);
    case 16: return launch_gemm_int4<16>(maps, p, st);
    case 32: return launch_gemm_int4<32>(maps, p, st);
    default: return launch_gemm_int4<64>(maps, p, st);
  }
}

svdq_status quantize_act_impl(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                              uint8_t* x_scales, uint16_t* D, cudaStream_t st, float* zero_ptr = nullptr,
                              int zero_count = 0, float* dpart = nullptr, unsigned long long* flags = nullptr) {
  if (w->format == SVDQ_FORMAT_INT4) return quantize_act_int4_impl(X, M, w, x_codes, x_scales, D, st);
  const int K = w->K, r = w->r, rp = r_pad_of(r);
  const int kernel_choice = override_value(SVDQ_OVERRIDE_ACT_KERNEL);
  if (r > 0 && dpart != nullptr && flags != nullptr &&
      (kernel_choice == 2 || (kernel_choice != 1 && K / (64 * a128_k_split(M, K)) >= A128_MIN_STAGES))) {
    // 128-row CTAs, D on the tensor cores (needs the workspace for its K
    // split), when every CTA has enough stages to amortise the split's
    // cross-CTA reduction; the 16-row kernel otherwise
    CUtensorMap tx{}, tl{};
    svdq_status s = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(K) * 2, 64,
                              A128_ROWS, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != SVDQ_OK) return s;
    s = make_tmap(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L1t, K, r, static_cast<uint64_t>(K) * 2, 64, rp,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != SVDQ_OK) return s;
    A128Params p{};
    p.inv_lambda = w->inv_lambda;
    p.x_codes = x_codes;
    p.x_scales = x_scales;
    p.D = D;
    p.dpart = dpart;
    p.flags = flags;
    p.epoch = next_epoch();
    p.M = M;
    p.K = K;
    p.r = r;
    p.M_pad = m_pad_of(M);
    p.ks = a128_k_split(M, K);
    p.zero_ptr = zero_ptr;
    p.zero_count = zero_count;
    switch (rp) {
      case 16: return launch_act128<16>(tx, tl, p, st);
      case 32: return launch_act128<32>(tx, tl, p, st);
      default: return launch_act128<64>(tx, tl, p, st);
    }
  }
  CUtensorMap tx{};
  svdq_status s = make_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M,
                            static_cast<uint64_t>(K) * 2, ACT_SUB, ACT_ROWS,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  ActParams p;
  p.inv_lambda = w->inv_lambda;
  p.L1f = reinterpret_cast<const uint32_t*>(w->L1f);
  p.x_codes = x_codes;
  p.x_scales = x_scales;
  p.D = D;
  p.M = M;
  p.K = K;
  p.r = r;
  p.M_pad = m_pad_of(M);
  p.ks = act_k_split(M, K);
  p.zero_ptr = zero_ptr;
  p.zero_count = zero_count;
  switch (rp) {
    case 0: return launch_act<0>(tx, p, st);
    case 16: return launch_act<16>(tx, p, st);
    case 32: return launch_act<32>(tx, p, st);
    default: return launch_act<64>(tx, p, st);
  }
}

// head_dim == 0: Y row-major M x N; else Y head-major [N / head_dim][M][head_dim]
// `mlp` (optional): the MLP epilogue's fields (inv_lambda_next ... h_out);
// the kernel then writes the down-projection's input instead of Y.
svdq_status gemm_impl(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                      const svdq_weight* w, uint16_t* Y, cudaStream_t st, int head_dim = 0,
                      const GemmParams* mlp = nullptr) {
  if (w->format == SVDQ_FORMAT_INT4) return gemm_int4_impl(x_codes, x_scales, D, M, w, Y, st, head_dim);
  const int N = w->N, K = w->K, r = w->r, rp = r_pad_of(r);
  const int m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  // 256-wide tiles when N allows it and there are enough of them to fill the GPU
  int BN = (N % 256 == 0) ? 256 : 128;
  if (BN == 256 && m_tiles * (N / 256) < num_sms()) BN = 128;
  {   // tile-width override (svdq_set_override)
    const int v = override_value(SVDQ_OVERRIDE_GEMM_BN);
    if (v == 128 || (v == 256 && N % 256 == 0)) BN = v;
  }
  CUtensorMap ta{}, tb{}, td{}, tl2{}, ty{};
  svdq_status s = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, K / 2, M, K / 2, 128,
                            GEMM_BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  s = make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w_codes, K / 2, N, K / 2, 128, BN,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  if (mlp == nullptr) {
    if (head_dim == 0)
      s = make_tmap(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<uint64_t>(N) * 2, 16, 32,
                    CU_TENSOR_MAP_SWIZZLE_32B);
    else
      s = make_tmap_heads(&ty, Y, head_dim, M, N / head_dim);
    if (s != SVDQ_OK) return s;
  }
  if (r > 0) {
    s = make_tmap(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D, r, M, static_cast<uint64_t>(r) * 2, rp,
                  GEMM_BM, lr_swizzle(rp));
    if (s != SVDQ_OK) return s;
    s = make_tmap(&tl2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L2t, r, N,
                  static_cast<uint64_t>(r) * 2, rp, BN, lr_swizzle(rp));
    if (s != SVDQ_OK) return s;
  }
  GemmParams p{};
  p.x_scales = x_scales;
  p.w_scales = w->w_scales;
  p.bias = w->has_bias ? w->bias : nullptr;
  p.Y = Y;
  p.y_align32 = (reinterpret_cast<uintptr_t>(Y) % 32) == 0;
  p.head_dim = head_dim;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.m_tiles = m_tiles;
  p.n_tiles = N / BN;
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.kblocks = K / GEMM_BK;
  if (mlp != nullptr) {
    p.inv_lambda_next = mlp->inv_lambda_next;
    p.L1f_next = mlp->L1f_next;
    p.r_next = mlp->r_next;
    p.h_codes = mlp->h_codes;
    p.h_scales = mlp->h_scales;
    p.d_acc = mlp->d_acc;
    p.h_out = mlp->h_out;
    return BN == 256 ? dispatch_gemm_r<256, true>(rp, ta, tb, td, tl2, ty, p, st)
                     : dispatch_gemm_r<128, true>(rp, ta, tb, td, tl2, ty, p, st);
  }
  return BN == 256 ? dispatch_gemm_r<256>(rp, ta, tb, td, tl2, ty, p, st)
                   : dispatch_gemm_r<128>(rp, ta, tb, td, tl2, ty, p, st);
}

// D = bf16(acc) for the MLP pair's down-projection (M x r values), launched as
// a programmatic dependent of the up-projection GEMM that accumulates acc.
__global__ void d_round_kernel(const float* __restrict__ acc, uint16_t* __restrict__ D, int n) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    D[i] = static_cast<uint16_t>(pack_bf16x2(__ldcg(acc + i), 0.0f) & 0xFFFFu);
}

svdq_status launch_d_round(const float* acc, uint16_t* D, int n, cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(std::max(1, std::min((n + 255) / 256, num_sms() * 2))));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, d_round_kernel, acc, D, n);
  if (e != cudaSuccess) return cuda_fail(e, "d_round_kernel launch");
  SVDQ_CHECK_LAUNCH("d_round_kernel");
  return SVDQ_OK;
}

// ---- few-token path (small_m.cuh) ----------------------------------------
template <int R_PAD>
svdq_status launch_act_small(const SmallActParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.K / SMALL_ACT_COLS));
  cfg.blockDim = dim3(SMALL_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, act_quant_small_kernel<R_PAD>, p);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_small_kernel launch");
  SVDQ_CHECK_LAUNCH("act_quant_small_kernel");
  return SVDQ_OK;
}

template <int TN, int R_PAD>
svdq_status launch_gemm_small(const CUtensorMap& tw, const CUtensorMap& tl2, SmallGemmParams p, cudaStream_t st) {
  // the deepest weight ring that leaves room (<= 200 KB) for one activation
  // CTA on the same SM
  int stages = SMALL_MAX_STAGES;
  while (stages > 2 && small_gemm_layout(TN, R_PAD, p.K, stages, nullptr) > 200u * 1024u) --stages;
  const uint32_t smem = small_gemm_layout(TN, R_PAD, p.K, stages, &p);
  {
    const svdq_status so = opt_in_smem(reinterpret_cast<const void*>(fp4_gemm_small_m_kernel<TN, R_PAD>),
                                       232448u, "cudaFuncSetAttribute(gemm small M)");
    if (so != SVDQ_OK) return so;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.N / 128));
  cfg.blockDim = dim3(SMALL_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fp4_gemm_small_m_kernel<TN, R_PAD>, tw, tl2, p);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_gemm_small_m_kernel launch");
  SVDQ_CHECK_LAUNCH("fp4_gemm_small_m_kernel");
  return SVDQ_OK;
}

template <int TN>
svdq_status dispatch_gemm_small(int r_pad, const CUtensorMap& tw, const CUtensorMap& tl2, const SmallGemmParams& p,
                                cudaStream_t st) {
  switch (r_pad) {
    case 0: return launch_gemm_small<TN, 0>(tw, tl2, p, st);
    case 16: return launch_gemm_small<TN, 16>(tw, tl2, p, st);
    case 32: return launch_gemm_small<TN, 32>(tw, tl2, p, st);
    default: return launch_gemm_small<TN, 64>(tw, tl2, p, st);
  }
}

struct ActWs {
  uint8_t* codes;
  uint8_t* scales;
  uint16_t* D;
  float* dpart;                 // act128_kernel's K-split partials of D (r > 0)
  unsigned long long* flags;    // and their flags
};

// Bytes of the K-split partials of D ([M_pad / 128][A128_MAX_KS][r][128]
// float32) and of their flags ([M_pad / 128][A128_MAX_KS]), each 256-aligned;
// 0 for r = 0.
size_t act_partials_bytes(int M, int r, size_t* flags_off) {
  if (r == 0) {
    if (flags_off) *flags_off = 0;
    return 0;
  }
  const size_t part = align_up(static_cast<size_t>(A128_MAX_KS) * m_pad_of(M) * r * 4, kAlign);
  const size_t fl = align_up(static_cast<size_t>(m_pad_of(M) / A128_ROWS) * A128_MAX_KS * 8, kAlign);
  if (flags_off) *flags_off = part;
  return part + fl;
}

size_t act_ws_layout(int M, int K, int r, uint8_t* base, ActWs* out) {
  const size_t c = align_up(static_cast<size_t>(M) * (K / 2), kAlign);
  const size_t s = align_up(static_cast<size_t>(m_pad_of(M)) * (K / 16), kAlign);
  const size_t d = align_up(static_cast<size_t>(M) * r * 2, kAlign);
  size_t flags_off = 0;
  const size_t pb = act_partials_bytes(M, r, &flags_off);
  if (out != nullptr) {
    out->codes = base;
    out->scales = base + c;
    out->D = r > 0 ? reinterpret_cast<uint16_t*>(base + c + s) : nullptr;
    out->dpart = r > 0 ? reinterpret_cast<float*>(base + c + s + d) : nullptr;
    out->flags = r > 0 ? reinterpret_cast<unsigned long long*>(base + c + s + d + flags_off) : nullptr;
  }
  return c + s + d + pb;
}

// Workspace of the few-token path (M <= 32): activation codes M x K/2, the
// activation scale words [K/64][32] and the float32 partial down-projections
// [K/256][M][r].
struct SmallWs {
  uint8_t* codes;
  uint32_t* sfb;
  float* dpart;
};

size_t small_ws_layout(int M, int K, int r, uint8_t* base, SmallWs* out) {
  const size_t c = align_up(static_cast<size_t>(M) * (K / 2), kAlign);
  const size_t s = align_up(static_cast<size_t>(K / 64) * SMALL_MAX_TOKENS * 4, kAlign);
  const size_t d = align_up(static_cast<size_t>(K / 256) * M * r * 4, kAlign);
  if (out != nullptr) {
    out->codes = base;
    out->sfb = reinterpret_cast<uint32_t*>(base + c);
    out->dpart = reinterpret_cast<float*>(base + c + s);
  }
  return c + s + d;
}

// The few-token path applies to NVFP4 weights with M <= 32, K <= 4096 and at
// most one 128-row weight tile per SM (SVDQ_OVERRIDE_SMALL_M = 1 turns it off).
bool small_m_path(int M, const svdq_weight* w) {
  if (w->format != SVDQ_FORMAT_NVFP4 || override_value(SVDQ_OVERRIDE_SMALL_M) == 1) return false;
  return M >= 1 && M <= SMALL_MAX_TOKENS && w->K <= SMALL_MAX_K && w->N / 128 <= num_sms();
}

// Workspace bytes of a forward of M rows (either path).
size_t forward_ws_bytes(int M, int K, int r) {
  size_t b = act_ws_layout(M, K, r, nullptr, nullptr);
  if (M <= SMALL_MAX_TOKENS && K <= SMALL_MAX_K) b = std::max(b, small_ws_layout(M, K, r, nullptr, nullptr));
  return b;
}

// Weight buffer layout, each field 256-byte aligned.
size_t weight_layout(int N, int K, int r, int has_bias, uint8_t* base, svdq_weight* out) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, kAlign);
    return base == nullptr ? nullptr : base + o;
  };
  uint8_t* codes = take(static_cast<size_t>(N) * (K / 2));
  uint8_t* scales = take(static_cast<size_t>(N) * (K / 16));
  uint8_t* l1 = take(static_cast<size_t>(K) * r * 2);
  uint8_t* l1f = take(static_cast<size_t>(K) * r * 2);
  uint8_t* l2t = take(static_cast<size_t>(N) * r * 2);
  uint8_t* inv = take(static_cast<size_t>(K) * 4);
  uint8_t* bias = has_bias ? take(static_cast<size_t>(N) * 2) : nullptr;
  uint8_t* l1t = take(static_cast<size_t>(K) * r * 2);
  if (out != nullptr) {
    out->N = N;
    out->K = K;
    out->r = r;
    out->has_bias = has_bias ? 1 : 0;
    out->format = SVDQ_FORMAT_NVFP4;
    out->w_codes = codes;
    out->w_scales = scales;
    out->L1 = r > 0 ? reinterpret_cast<uint16_t*>(l1) : nullptr;
    out->L1f = r > 0 ? reinterpret_cast<uint16_t*>(l1f) : nullptr;
    out->L2t = r > 0 ? reinterpret_cast<uint16_t*>(l2t) : nullptr;
    out->inv_lambda = reinterpret_cast<float*>(inv);
    out->bias = reinterpret_cast<uint16_t*>(bias);
    out->L1t = r > 0 ? reinterpret_cast<uint16_t*>(l1t) : nullptr;
  }
  return off;
}

// The whole layer for M <= 32 tokens on the few-token path: the activation
// kernel (K/256 CTAs) and the swapped-operand GEMM, chained by programmatic
// dependent launch; the workspace holds the small_ws_layout fields.
svdq_status small_forward_impl(const uint16_t* X, int M, const svdq_weight* w, uint16_t* Y, void* ws,
                               cudaStream_t st, int head_dim) {
  const int N = w->N, K = w->K, r = w->r, rp = r_pad_of(r);
  SmallWs a;
  small_ws_layout(M, K, r, static_cast<uint8_t*>(ws), &a);
  SmallActParams ap;
  ap.X = X;
  ap.inv_lambda = w->inv_lambda;
  ap.L1f = reinterpret_cast<const uint32_t*>(w->L1f);
  ap.x_codes = a.codes;
  ap.sfb = a.sfb;
  ap.dpart = a.dpart;
  ap.M = M;
  ap.K = K;
  ap.r = r;
  svdq_status s;
  switch (rp) {
    case 0: s = launch_act_small<0>(ap, st); break;
    case 16: s = launch_act_small<16>(ap, st); break;
    case 32: s = launch_act_small<32>(ap, st); break;
    default: s = launch_act_small<64>(ap, st); break;
  }
  if (s != SVDQ_OK) return s;
  const int TN = M <= 16 ? 16 : 32;
  CUtensorMap tw{}, tl2{};
  s = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w_codes, K / 2, N, K / 2, 128, 128,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  if (r > 0) {
    s = make_tmap(&tl2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L2t, r, N, static_cast<uint64_t>(r) * 2, rp, 128,
                  lr_swizzle(rp));
    if (s != SVDQ_OK) return s;
  }
  SmallGemmParams gp{};
  gp.w_scales = w->w_scales;
  gp.x_codes = a.codes;
  gp.sfb = a.sfb;
  gp.dpart = a.dpart;
  gp.bias = w->has_bias ? w->bias : nullptr;
  gp.Y = Y;
  gp.M = M;
  gp.N = N;
  gp.K = K;
  gp.r = r;
  gp.head_dim = head_dim;
  return TN == 16 ? dispatch_gemm_small<16>(rp, tw, tl2, gp, st) : dispatch_gemm_small<32>(rp, tw, tl2, gp, st);
}

// The whole layer (either path) with its scratch at `ws` (forward_ws_bytes).
svdq_status forward_impl(const uint16_t* X, int M, const svdq_weight* w, uint16_t* Y, void* ws,
                         cudaStream_t st, int head_dim) {
  if (small_m_path(M, w)) return small_forward_impl(X, M, w, Y, ws, st, head_dim);
  ActWs a;
  act_ws_layout(M, w->K, w->r, static_cast<uint8_t*>(ws), &a);
  svdq_status s = quantize_act_impl(X, M, w, a.codes, a.scales, a.D, st, nullptr, 0, a.dpart, a.flags);
  if (s != SVDQ_OK) return s;
  return gemm_impl(a.codes, a.scales, a.D, M, w, Y, st, head_dim);
}

// Workspace of the MLP pair: the up-projection's activation workspace, the
// down-projection's (its codes, scales and D, written by the up-projection's
// epilogue and the rounding kernel), then the float32 accumulator of D.
struct MlpWs {
  ActWs up, down;
  float* d_acc;
};

size_t mlp_ws_layout(int M, int K, int F, int r_up, int r_down, uint8_t* base, MlpWs* out) {
  const size_t a = align_up(forward_ws_bytes(M, K, r_up), kAlign);
  const size_t b = align_up(forward_ws_bytes(M, F, r_down), kAlign);
  const size_t c = align_up(static_cast<size_t>(M) * r_down * 4, kAlign);
  if (out != nullptr) {
    act_ws_layout(M, K, r_up, base, &out->up);
    act_ws_layout(M, F, r_down, base + a, &out->down);
    out->d_acc = reinterpret_cast<float*>(base + a + b);
  }
  return a + b + c;
}

svdq_status mlp_forward_impl(const uint16_t* X, int M, const svdq_weight* up, const svdq_weight* down,
                             uint16_t* Y, uint16_t* H_out, void* ws, cudaStream_t st) {
  MlpWs m;
  mlp_ws_layout(M, up->K, up->N, up->r, down->r, static_cast<uint8_t*>(ws), &m);
  const int nd = M * down->r;
  // the up-projection's activation kernel, which also clears the D accumulator
  svdq_status s = quantize_act_impl(X, M, up, m.up.codes, m.up.scales, m.up.D, st, m.d_acc, nd, m.up.dpart,
                                    m.up.flags);
  if (s != SVDQ_OK) return s;
  GemmParams e{};
  e.inv_lambda_next = down->inv_lambda;
  e.L1f_next = reinterpret_cast<const uint32_t*>(down->L1f);
  e.r_next = down->r;
  e.h_codes = m.down.codes;
  e.h_scales = m.down.scales;
  e.d_acc = m.d_acc;
  e.h_out = H_out;
  s = gemm_impl(m.up.codes, m.up.scales, m.up.D, M, up, nullptr, st, 0, &e);
  if (s != SVDQ_OK) return s;
  if (down->r > 0) {
    s = launch_d_round(m.d_acc, m.down.D, nd, st);
    if (s != SVDQ_OK) return s;
  }
  return gemm_impl(m.down.codes, m.down.scales, m.down.D, M, down, Y, st);
}

struct PrepWs {
  float* what;
  double* G;
  double* ev;
  double* L1f;
  double* L2f;
  double* work;
  int* info;
  int lwork;
};

size_t prep_ws_layout(int N, int K, int r, int lwork, uint8_t* base, PrepWs* out) {
  const int n = std::min(N, K);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, kAlign);
    return base == nullptr ? nullptr : base + o;
  };
  uint8_t* what = take(static_cast<size_t>(N) * K * 4);
  uint8_t* G = take(r > 0 ? static_cast<size_t>(n) * n * 8 : 0);
  uint8_t* ev = take(r > 0 ? static_cast<size_t>(n) * 8 : 0);
  uint8_t* l1 = take(static_cast<size_t>(K) * r * 8);
  uint8_t* l2 = take(static_cast<size_t>(N) * r * 8);
  uint8_t* work = take(r > 0 ? static_cast<size_t>(lwork) * 8 : 0);
  uint8_t* info = take(16);
  if (out != nullptr) {
    out->what = reinterpret_cast<float*>(what);
    out->G = reinterpret_cast<double*>(G);
    out->ev = reinterpret_cast<double*>(ev);
    out->L1f = reinterpret_cast<double*>(l1);
    out->L2f = reinterpret_cast<double*>(l2);
    out->work = reinterpret_cast<double*>(work);
    out->info = reinterpret_cast<int*>(info);
    out->lwork = lwork;
  }
  return off;
}

int syevd_lwork(int n, cusolverDnHandle_t h) {
  int lwork = 0;
  if (cusolverDnDsyevd_bufferSize(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, n, nullptr, n,
                                  nullptr, &lwork) != CUSOLVER_STATUS_SUCCESS)
    return -1;
  return lwork;
}

void to_native(const uint8_t* logical, int rows, int K, uint8_t* native) {
  const int kb = K / 16;
  std::memset(native, 0, static_cast<size_t>(m_pad_of(rows)) * kb);
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < kb; ++j) native[sf_offset(i, j, K)] = logical[static_cast<size_t>(i) * kb + j];
}

void to_logical(const uint8_t* native, int rows, int K, uint8_t* logical) {
  const int kb = K / 16;
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < kb; ++j)
      logical[static_cast<size_t>(i) * kb + j] = native[sf_offset(i, j, K)];
}

// INT4 scales: native fp16 [K/64][rows_pad] (group-major) <-> logical [rows][K/64].
void int4_to_logical(const uint16_t* native, int rows, int rows_pad, int K, uint16_t* logical) {
  const int ng = K / INT4_GROUP;
  for (int i = 0; i < rows; ++i)
    for (int g = 0; g < ng; ++g)
      logical[static_cast<size_t>(i) * ng + g] = native[static_cast<size_t>(g) * rows_pad + i];
}

void int4_to_native(const uint16_t* logical, int rows, int rows_pad, int K, uint16_t* native) {
  const int ng = K / INT4_GROUP;
  std::memset(native, 0, static_cast<size_t>(rows_pad) * ng * 2);
  for (int i = 0; i < rows; ++i)
    for (int g = 0; g < ng; ++g)
      native[static_cast<size_t>(g) * rows_pad + i] = logical[static_cast<size_t>(i) * ng + g];
}

// One bounded wait on an mbarrier that nothing arrives on: the same wait the
// layer's kernels use, made to run out, so the timeout path (status word,
// clean return) can be tested without faulting or hanging the GPU.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), KID_SELFTEST, 1,
              limit_ns);
  __syncthreads();
}

// Exhaustive check of the activation kernel's division-free quotient
// (quotient_f32x2) and of the E2M1 conversion of its signed result.  For every
// positive E4M3 scale s (codes 1..126), both signs, five binades of v around s
// (v / s in [1/8, 8)) and all 2^23 significands of v -- plus zeros, subnormal,
// tiny and huge v for every code including s = 0 -- count quotients that
// differ from IEEE division (counts[0] where the IEEE quotient is a normal
// number or zero, counts[2] where it is subnormal, a range in which the
// correction step is not exact; for s = 0 the defined quotient is a zero with
// v's sign) and codes that differ from E2M1 of the IEEE quotient by the
// format's definition (counts[1]): magnitude thresholds 0.25, 0.75, 1.25,
// 1.75, 2.5, 3.5, 5 with ties to the even code, sign kept.
__device__ unsigned long long g_quotient_mismatch[3];

__device__ void check_quotient(uint32_t c, float v) {
  const float thr[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  const float2 sy = e4m3_table_entry(c);
  const float qr = c == 0 ? __uint_as_float(__float_as_uint(v) & 0x80000000u) : __fdiv_rn(v, sy.x);
  float qt, qt2;
  f32x2_unpack(quotient_f32x2(f32x2_pack(-v, -v), f32x2_pack(sy.x, sy.x), f32x2_pack(-sy.y, -sy.y)), qt,
               qt2);
  if (__float_as_uint(qt) != __float_as_uint(qr) || __float_as_uint(qt2) != __float_as_uint(qr)) {
    const bool subnormal = qr != 0.0f && fabsf(qr) < 0x1p-126f;
    atomicAdd(&g_quotient_mismatch[subnormal ? 2 : 0], 1ull);
  }
  const float a[8] = {qt, qt, qt, qt, qt, qt, qt, qt};
  const uint32_t got = e2m1x8_magnitudes(a) & 15u;
  const float mag = fabsf(qr);
  uint32_t want = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k)
    if (mag > thr[k] || (mag == thr[k] && (k & 1))) want = static_cast<uint32_t>(k + 1);
  want |= (__float_as_uint(qr) >> 31) << 3;
  if (got != want) atomicAdd(&g_quotient_mismatch[1], 1ull);
}

__global__ void selftest_quotient_kernel() {
  const unsigned long long total = 126ull * 5ull * 2ull << 23;
  for (unsigned long long idx = static_cast<unsigned long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < total; idx += static_cast<unsigned long long>(gridDim.x) * blockDim.x) {
    const uint32_t m = static_cast<uint32_t>(idx) & ((1u << 23) - 1u);
    unsigned long long rest = idx >> 23;
    const uint32_t neg = static_cast<uint32_t>(rest & 1ull);
    rest >>= 1;
    const int d = static_cast<int>(rest % 5ull) - 2;
    const uint32_t c = 1u + static_cast<uint32_t>(rest / 5ull);
    const int es = static_cast<int>((__float_as_uint(e4m3_to_f32(c)) >> 23) & 255u);
    check_quotient(c, __uint_as_float((neg << 31) | (static_cast<uint32_t>(es + d) << 23) | m));
  }
  if (blockIdx.x == 0) {
    // zeros, smallest subnormal, smallest normal, tiny, huge, exact ties
    const uint32_t special[10] = {0x00000000u, 0x00000001u, 0x00800000u, 0x0DA24260u, 0x45BB8000u,
                                  0x3E99999Au, 0x40200000u, 0x33D6BF95u, 0x3E800000u, 0x40A00000u};
    for (int t = threadIdx.x; t < 127 * 20; t += blockDim.x) {
      const uint32_t c = static_cast<uint32_t>(t / 20), j = static_cast<uint32_t>(t % 20);
      check_quotient(c, __uint_as_float(special[j >> 1] | ((j & 1u) << 31)));
    }
  }
}

// Exhaustive check of the hardware conversions the kernels round with, for
// every non-negative finite float32 x, against the formats' definitions:
// counts[0] E4M3 (cvt.rn.satfinite.e4m3x2: nearest of the 127 finite E4M3
// values, ties to the even code, saturating at 448), counts[1] E2M1
// (cvt.rn.satfinite.e2m1x2, thresholds as above), counts[2] bf16
// (cvt.rn.bf16x2: round to nearest even on the upper 16 bits).
__device__ unsigned long long g_conversion_mismatch[3];

__global__ void selftest_conversion_kernel() {
  __shared__ float e4m3[127];
  for (int c = threadIdx.x; c < 127; c += blockDim.x) e4m3[c] = e4m3_to_f32(static_cast<uint32_t>(c));
  __syncthreads();
  const float thr[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  unsigned long long bad[3] = {0ull, 0ull, 0ull};
  for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < 0x7F800000u; u += gridDim.x * blockDim.x) {
    const float x = __uint_as_float(u);
    // E4M3: largest code whose value is <= x, then the nearer neighbour
    uint32_t want;
    if (x >= 448.0f) {
      want = 126u;
    } else {
      int lo = 0, hi = 126;   // e4m3[lo] <= x < e4m3[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (e4m3[mid] <= x) lo = mid; else hi = mid;
      }
      const float dl = x - e4m3[lo], dh = e4m3[hi] - x;   // exact: both within a binade of x
      want = static_cast<uint32_t>(dl < dh ? lo : dh < dl ? hi : ((lo & 1) ? hi : lo));
    }
    if (e4m3_rn_satfinite(x) != want) ++bad[0];
    // E2M1
    uint32_t w2 = 0;
#pragma unroll
    for (int k = 0; k < 7; ++k)
      if (x > thr[k] || (x == thr[k] && (k & 1))) w2 = static_cast<uint32_t>(k + 1);
    const float a[8] = {x, x, x, x, x, x, x, x};
    if ((e2m1x8_magnitudes(a) & 15u) != w2) ++bad[1];
    // bf16
    const uint32_t wb = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
    if ((pack_bf16x2(x, 0.0f) & 0xFFFFu) != wb) ++bad[2];
  }
  for (int i = 0; i < 3; ++i)
    if (bad[i]) atomicAdd(&g_conversion_mismatch[i], bad[i]);
}

// --------------------------------------------------------------------------
// Fixed device scratch for svdq_linear_forward_noalloc.  Every GPU that loads
// this library holds it until the process exits.  Host code only ever sees a
// host-side stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress, taken once per device with that device current.
// --------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[SVDQ_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[256] = {};

svdq_status noalloc_scratch_address(void** out) {
  int dev = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) {
    g_last_error = "device ordinal out of range for the no-alloc scratch table";
    return SVDQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    SVDQ_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return SVDQ_OK;
}

}  // namespace

// ==========================================================================
// C ABI
// ==========================================================================
extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "SVDQ_ERR_UNSUPPORTED_SHAPE";
    case SVDQ_ERR_MISALIGNED: return "SVDQ_ERR_MISALIGNED";
    case SVDQ_ERR_WORKSPACE_TOO_SMALL: return "SVDQ_ERR_WORKSPACE_TOO_SMALL";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_SOLVER: return "SVDQ_ERR_SOLVER";
  }
  return "SVDQ_ERR_UNKNOWN";
}

const char* svdq_last_error_detail(void) { return g_last_error.c_str(); }

const char* svdq_version(void) { return "svdq-b200 0.2 (sm_100a)"; }

svdq_status svdq_set_override(int which, int value) {
  if (which <= 0 || which >= SVDQ_OVERRIDE_COUNT || value < 0) return SVDQ_ERR_INVALID_ARG;
  g_override[which].store(value, std::memory_order_relaxed);
  return SVDQ_OK;
}

size_t svdq_weight_bytes(int N, int K, int r, int has_bias) {
  if (check_layer_shape(N, K, r) != SVDQ_OK) return 0;
  return weight_layout(N, K, r, has_bias, nullptr, nullptr);
}

size_t svdq_act_codes_bytes(int M, int K) {
  if (M < 0 || K <= 0 || K % 16) return 0;
  return static_cast<size_t>(M) * (K / 2);
}

size_t svdq_act_scales_bytes(int M, int K) {
  if (M < 0 || K <= 0 || K % 64) return 0;
  return static_cast<size_t>(m_pad_of(M)) * (K / 16);
}

size_t svdq_forward_workspace_bytes(int M, int N, int K, int r) {
  if (M < 0 || check_layer_shape(N, K, r) != SVDQ_OK) return 0;
  return forward_ws_bytes(M, K, r);
}

size_t svdq_prepare_workspace_bytes(int N, int K, int r) {
  if (check_layer_shape(N, K, r) != SVDQ_OK) return 0;
  int lwork = 0;
  if (r > 0) {
    cusolverDnHandle_t h = nullptr;
    if (cusolverDnCreate(&h) != CUSOLVER_STATUS_SUCCESS) return 0;
    lwork = syevd_lwork(std::min(N, K), h);
    cusolverDnDestroy(h);
    if (lwork < 0) return 0;
  }
  return prep_ws_layout(N, K, r, lwork, nullptr, nullptr);
}

svdq_status svdq_weight_bind(void* buf, size_t bytes, int N, int K, int r, int has_bias,
                             svdq_weight* out) {
  if (buf == nullptr || out == nullptr) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_layer_shape(N, K, r);
  if (s != SVDQ_OK) return s;
  if ((reinterpret_cast<uintptr_t>(buf) & (kAlign - 1)) != 0) return SVDQ_ERR_MISALIGNED;
  if (bytes < weight_layout(N, K, r, has_bias, nullptr, nullptr)) return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  weight_layout(N, K, r, has_bias, static_cast<uint8_t*>(buf), out);
  return SVDQ_OK;
}

svdq_status svdq_weight_bind_format(void* buf, size_t bytes, int N, int K, int r, int has_bias, int format,
                                    svdq_weight* out) {
  if (format != SVDQ_FORMAT_NVFP4 && format != SVDQ_FORMAT_INT4) return SVDQ_ERR_INVALID_ARG;
  const svdq_status s = svdq_weight_bind(buf, bytes, N, K, r, has_bias, out);
  if (s == SVDQ_OK) out->format = format;
  return s;
}

svdq_status svdq_prepare_weight(const uint16_t* W, const float* lambda, const uint16_t* bias,
                                const svdq_weight* w, void* ws, size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (W == nullptr || lambda == nullptr || ws == nullptr) return SVDQ_ERR_INVALID_ARG;
  if ((bias != nullptr) != (w->has_bias != 0)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(lambda) || (bias && !aligned16(bias)) || !aligned16(ws))
    return SVDQ_ERR_MISALIGNED;
  const int N = w->N, K = w->K, r = w->r, n = std::min(N, K);
  const int col_gram = K <= N ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  cusolverDnHandle_t h = nullptr;
  int lwork = 0;
  if (r > 0) {
    if (cusolverDnCreate(&h) != CUSOLVER_STATUS_SUCCESS) {
      g_last_error = "cusolverDnCreate failed";
      return SVDQ_ERR_SOLVER;
    }
    lwork = syevd_lwork(n, h);
    if (lwork < 0) {
      cusolverDnDestroy(h);
      g_last_error = "cusolverDnDsyevd_bufferSize failed";
      return SVDQ_ERR_SOLVER;
    }
  }
  PrepWs pw;
  if (ws_bytes < prep_ws_layout(N, K, r, lwork, nullptr, nullptr)) {
    if (h) cusolverDnDestroy(h);
    return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  }
  prep_ws_layout(N, K, r, lwork, static_cast<uint8_t*>(ws), &pw);

  auto fail = [&](svdq_status e) {
    if (h) cusolverDnDestroy(h);
    return e;
  };

  const int nsm = num_sms();
  prep_smooth_kernel<<<nsm * 8, 256, 0, st>>>(W, lambda, bias, N, K, pw.what, w->inv_lambda,
                                              w->has_bias ? w->bias : nullptr);
  {
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return fail(cuda_fail(e0, "prep_smooth_kernel"));
  }
  if (r > 0) {
    dim3 g((n + GRAM_T - 1) / GRAM_T, (n + GRAM_T - 1) / GRAM_T);
    prep_gram_kernel<<<g, 256, 0, st>>>(pw.what, N, K, col_gram, pw.G);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(cuda_fail(e, "prep_gram_kernel"));
    if (cusolverDnSetStream(h, st) != CUSOLVER_STATUS_SUCCESS ||
        cusolverDnDsyevd(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, n, pw.G, n, pw.ev,
                         pw.work, lwork, pw.info) != CUSOLVER_STATUS_SUCCESS) {
      g_last_error = "cusolverDnDsyevd failed";
      return fail(SVDQ_ERR_SOLVER);
    }
    int info = 0;
    e = cudaMemcpyAsync(&info, pw.info, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(cuda_fail(e, "syevd info"));
    if (info != 0) {
      g_last_error = "cusolverDnDsyevd info = " + std::to_string(info);
      return fail(SVDQ_ERR_SOLVER);
    }
    const int dot_grid = col_gram ? N : (K + 31) / 32;
    prep_factor_dot_kernel<<<dot_grid, 256, 0, st>>>(pw.what, N, K, r, col_gram, pw.G, pw.ev, pw.L1f,
                                                     pw.L2f);
    prep_factor_direct_kernel<<<nsm * 4, 256, 0, st>>>(N, K, r, col_gram, pw.G, pw.ev, pw.L1f, pw.L2f);
    prep_sign_kernel<<<r, 256, 0, st>>>(pw.L1f, pw.L2f, N, K, r);
    prep_round_kernel<<<nsm * 4, 256, 0, st>>>(pw.L1f, pw.L2f, N, K, r, w->L1, w->L2t);
    l1_fragment_kernel<<<nsm * 2, 256, 0, st>>>(w->L1, K, r, w->L1f);
    l1_transpose_kernel<<<nsm * 2, 256, 0, st>>>(w->L1, K, r, w->L1t);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(cuda_fail(e, "prepare factor kernels"));
  }
  uint16_t* s16 = reinterpret_cast<uint16_t*>(w->w_scales);
  if (w->format == SVDQ_FORMAT_INT4) {
    switch (r_pad_of(r)) {
      case 0: prep_residual_int4_kernel<0><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, s16); break;
      case 16: prep_residual_int4_kernel<16><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, s16); break;
      case 32: prep_residual_int4_kernel<32><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, s16); break;
      default: prep_residual_int4_kernel<64><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, s16); break;
    }
  } else switch (r_pad_of(r)) {
    case 0: prep_residual_kernel<0><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, w->w_scales); break;
    case 16: prep_residual_kernel<16><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, w->w_scales); break;
    case 32: prep_residual_kernel<32><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, w->w_scales); break;
    default: prep_residual_kernel<64><<<N, 256, 0, st>>>(pw.what, w->L1, w->L2t, N, K, r, w->w_codes, w->w_scales); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(cuda_fail(e, "prep_residual_kernel"));
  if (h) cusolverDnDestroy(h);
  return SVDQ_OK;
}

svdq_status svdq_quantize_act(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                              uint8_t* x_scales, uint16_t* D, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || x_codes == nullptr || x_scales == nullptr || (w->r > 0 && D == nullptr))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(x_codes) || !aligned16(x_scales) || (w->r > 0 && !aligned16(D)))
    return SVDQ_ERR_MISALIGNED;
  return quantize_act_impl(X, M, w, x_codes, x_scales, D, static_cast<cudaStream_t>(stream));
}

size_t svdq_act_workspace_bytes(int M, int K, int r) {
  if (M < 0 || check_layer_shape(128, K, r) != SVDQ_OK) return 0;
  return std::max<size_t>(act_partials_bytes(M, r, nullptr), kAlign);
}

svdq_status svdq_quantize_act_ws(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                                 uint8_t* x_scales, uint16_t* D, void* ws, size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || x_codes == nullptr || x_scales == nullptr || (w->r > 0 && D == nullptr) || ws == nullptr)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(x_codes) || !aligned16(x_scales) || (w->r > 0 && !aligned16(D)) ||
      !aligned16(ws))
    return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < act_partials_bytes(M, w->r, nullptr)) return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  size_t flags_off = 0;
  act_partials_bytes(M, w->r, &flags_off);
  uint8_t* b = static_cast<uint8_t*>(ws);
  return quantize_act_impl(X, M, w, x_codes, x_scales, D, static_cast<cudaStream_t>(stream), nullptr, 0,
                           w->r > 0 ? reinterpret_cast<float*>(b) : nullptr,
                           w->r > 0 ? reinterpret_cast<unsigned long long*>(b + flags_off) : nullptr);
}

svdq_status svdq_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                      const svdq_weight* w, uint16_t* Y, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (x_codes == nullptr || x_scales == nullptr || Y == nullptr || (w->r > 0 && D == nullptr))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(Y) || (w->r > 0 && !aligned16(D)))
    return SVDQ_ERR_MISALIGNED;
  return gemm_impl(x_codes, x_scales, D, M, w, Y, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear_forward(const uint16_t* X, int M, const svdq_weight* w, uint16_t* Y,
                                void* ws, size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || Y == nullptr || ws == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(ws)) return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < forward_ws_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  return forward_impl(X, M, w, Y, ws, static_cast<cudaStream_t>(stream), 0);
}

svdq_status svdq_gemm_heads(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                            const svdq_weight* w, int head_dim, uint16_t* Y, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || head_dim <= 0 || head_dim % 16 != 0 || w->N % head_dim != 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (x_codes == nullptr || x_scales == nullptr || Y == nullptr || (w->r > 0 && D == nullptr))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(Y) || (w->r > 0 && !aligned16(D)))
    return SVDQ_ERR_MISALIGNED;
  return gemm_impl(x_codes, x_scales, D, M, w, Y, static_cast<cudaStream_t>(stream), head_dim);
}

svdq_status svdq_linear_forward_heads(const uint16_t* X, int M, const svdq_weight* w, int head_dim,
                                      uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || head_dim <= 0 || head_dim % 16 != 0 || w->N % head_dim != 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || Y == nullptr || ws == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(ws)) return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < forward_ws_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  return forward_impl(X, M, w, Y, ws, static_cast<cudaStream_t>(stream), head_dim);
}

// Copy-out stream and events of the host-buffer path, created once per device.
struct HostPipe {
  static constexpr int kEvents = 8;
  std::mutex mu;               // one caller at a time enqueues through the pipe
  cudaStream_t out = nullptr;
  cudaEvent_t ev[kEvents] = {};
  cudaEvent_t done = nullptr;
  bool ready = false;
};

svdq_status host_pipe(HostPipe** out) {
  static std::mutex mu;
  static HostPipe pipes[16];
  int dev = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 16) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  std::lock_guard<std::mutex> lock(mu);
  HostPipe& hp = pipes[dev];
  if (!hp.ready) {
    SVDQ_CUDA(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking));
    for (auto& e : hp.ev) SVDQ_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    SVDQ_CUDA(cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming));
    hp.ready = true;
  }
  *out = &hp;
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_host(const uint16_t* X_host, int M, const svdq_weight* w,
                                     uint16_t* Y_host, uint16_t* X_dev, uint16_t* Y_dev, void* ws,
                                     size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X_host == nullptr || Y_host == nullptr || X_dev == nullptr || Y_dev == nullptr || ws == nullptr)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X_dev) || !aligned16(Y_dev) || !aligned16(ws)) return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < forward_ws_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t K = w->K, N = w->N;
  // token rows per pipelined chunk (a multiple of 128); SVDQ_OVERRIDE_HOST_CHUNK_ROWS replaces it
  int kChunk = 1024;
  {
    const int v = override_value(SVDQ_OVERRIDE_HOST_CHUNK_ROWS);
    if (v >= 128 && v % 128 == 0) kChunk = v;
  }
  if (M <= kChunk) {
    SVDQ_CUDA(cudaMemcpyAsync(X_dev, X_host, static_cast<size_t>(M) * K * 2, cudaMemcpyHostToDevice, st));
    s = svdq_linear_forward(X_dev, M, w, Y_dev, ws, ws_bytes, stream);
    if (s != SVDQ_OK) return s;
    SVDQ_CUDA(cudaMemcpyAsync(Y_host, Y_dev, static_cast<size_t>(M) * N * 2, cudaMemcpyDeviceToHost, st));
    return SVDQ_OK;
  }
  // Chunks of rows (rows are independent): X in and the layer run on `stream`,
  // Y out on a second stream, so that chunk i's copy to the host overlaps the
  // copy in and the layer of chunk i + 1.  `stream` finally waits for the last
  // copy out, so the call stays asynchronous and ordered on `stream`.
  HostPipe* hp = nullptr;
  s = host_pipe(&hp);
  if (s != SVDQ_OK) return s;
  // the events and the copy-out stream are shared by every caller on this
  // device: concurrent callers enqueue one after the other
  std::lock_guard<std::mutex> pipe_lock(hp->mu);
  int i = 0;
  for (int r0 = 0; r0 < M; r0 += kChunk, ++i) {
    const int rows = std::min(kChunk, M - r0);
    SVDQ_CUDA(cudaMemcpyAsync(X_dev + r0 * K, X_host + r0 * K, static_cast<size_t>(rows) * K * 2,
                              cudaMemcpyHostToDevice, st));
    s = svdq_linear_forward(X_dev + r0 * K, rows, w, Y_dev + r0 * N, ws, ws_bytes, stream);
    if (s != SVDQ_OK) return s;
    cudaEvent_t ev = hp->ev[i % HostPipe::kEvents];
    SVDQ_CUDA(cudaEventRecord(ev, st));
    SVDQ_CUDA(cudaStreamWaitEvent(hp->out, ev, 0));
    SVDQ_CUDA(cudaMemcpyAsync(Y_host + r0 * N, Y_dev + r0 * N, static_cast<size_t>(rows) * N * 2,
                              cudaMemcpyDeviceToHost, hp->out));
  }
  SVDQ_CUDA(cudaEventRecord(hp->done, hp->out));
  SVDQ_CUDA(cudaStreamWaitEvent(st, hp->done, 0));
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_noalloc(const uint16_t* X, int M, const svdq_weight* w, uint16_t* Y,
                                        void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || Y == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SVDQ_ERR_MISALIGNED;
  const size_t need = forward_ws_bytes(M, w->K, w->r);
  if (need > static_cast<size_t>(SVDQ_NOALLOC_SCRATCH_BYTES)) {
    g_last_error = "svdq_linear_forward_noalloc: this shape needs " + std::to_string(need) +
                   " bytes of scratch; the fixed scratch holds " +
                   std::to_string(static_cast<size_t>(SVDQ_NOALLOC_SCRATCH_BYTES));
    return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  }
  void* scratch = nullptr;
  s = noalloc_scratch_address(&scratch);
  if (s != SVDQ_OK) return s;
  return forward_impl(X, M, w, Y, scratch, static_cast<cudaStream_t>(stream), 0);
}

size_t svdq_mlp_workspace_bytes(int M, int K, int F, int N, int r_up, int r_down) {
  if (M < 0 || check_layer_shape(F, K, r_up) != SVDQ_OK || check_layer_shape(N, F, r_down) != SVDQ_OK ||
      r_down > 32)
    return 0;
  return mlp_ws_layout(M, K, F, r_up, r_down, nullptr, nullptr);
}

svdq_status svdq_mlp_forward(const uint16_t* X, int M, const svdq_weight* up, const svdq_weight* down, uint16_t* Y,
                             uint16_t* H_out, void* ws, size_t ws_bytes, void* stream) {
  svdq_status s = check_weight(up);
  if (s != SVDQ_OK) return s;
  s = check_weight(down);
  if (s != SVDQ_OK) return s;
  if (up->format != SVDQ_FORMAT_NVFP4 || down->format != SVDQ_FORMAT_NVFP4 || down->K != up->N)
    return SVDQ_ERR_INVALID_ARG;
  if (down->r > 32) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || Y == nullptr || ws == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(ws) || (H_out != nullptr && !aligned16(H_out)))
    return SVDQ_ERR_MISALIGNED;
  if (ws_bytes < mlp_ws_layout(M, up->K, up->N, up->r, down->r, nullptr, nullptr))
    return SVDQ_ERR_WORKSPACE_TOO_SMALL;
  return mlp_forward_impl(X, M, up, down, Y, H_out, ws, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_weight_export(const svdq_weight* w, uint8_t* host_codes, uint8_t* host_scales,
                               uint16_t* host_L1, uint16_t* host_L2t, float* host_inv_lambda,
                               void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t N = w->N, K = w->K, r = w->r;
  const bool int4 = w->format == SVDQ_FORMAT_INT4;
  std::vector<uint8_t> native;
  if (host_codes) SVDQ_CUDA(cudaMemcpyAsync(host_codes, w->w_codes, N * K / 2, cudaMemcpyDeviceToHost, st));
  if (host_scales) {
    native.resize(int4 ? N * K / 32 : N * K / 16);
    SVDQ_CUDA(cudaMemcpyAsync(native.data(), w->w_scales, native.size(), cudaMemcpyDeviceToHost, st));
  }
  if (host_L1 && r) SVDQ_CUDA(cudaMemcpyAsync(host_L1, w->L1, K * r * 2, cudaMemcpyDeviceToHost, st));
  if (host_L2t && r) SVDQ_CUDA(cudaMemcpyAsync(host_L2t, w->L2t, N * r * 2, cudaMemcpyDeviceToHost, st));
  if (host_inv_lambda)
    SVDQ_CUDA(cudaMemcpyAsync(host_inv_lambda, w->inv_lambda, K * 4, cudaMemcpyDeviceToHost, st));
  SVDQ_CUDA(cudaStreamSynchronize(st));
  if (host_scales) {
    if (int4)
      int4_to_logical(reinterpret_cast<const uint16_t*>(native.data()), w->N, w->N, w->K,
                      reinterpret_cast<uint16_t*>(host_scales));
    else
      to_logical(native.data(), w->N, w->K, host_scales);
  }
  return SVDQ_OK;
}

svdq_status svdq_weight_import(const svdq_weight* w, const uint8_t* host_codes, const uint8_t* host_scales,
                               const uint16_t* host_L1, const uint16_t* host_L2t,
                               const float* host_inv_lambda, const uint16_t* host_bias, void* stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (host_codes == nullptr || host_scales == nullptr || host_inv_lambda == nullptr ||
      (w->r > 0 && (host_L1 == nullptr || host_L2t == nullptr)) || (w->has_bias != 0) != (host_bias != nullptr))
    return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t N = w->N, K = w->K, r = w->r;
  std::vector<uint8_t> native(w->format == SVDQ_FORMAT_INT4 ? N * K / 32 : N * K / 16);
  if (w->format == SVDQ_FORMAT_INT4)
    int4_to_native(reinterpret_cast<const uint16_t*>(host_scales), w->N, w->N, w->K,
                   reinterpret_cast<uint16_t*>(native.data()));
  else
    to_native(host_scales, w->N, w->K, native.data());
  SVDQ_CUDA(cudaMemcpyAsync(w->w_codes, host_codes, N * K / 2, cudaMemcpyHostToDevice, st));
  SVDQ_CUDA(cudaMemcpyAsync(w->w_scales, native.data(), native.size(), cudaMemcpyHostToDevice, st));
  if (r) {
    SVDQ_CUDA(cudaMemcpyAsync(w->L1, host_L1, K * r * 2, cudaMemcpyHostToDevice, st));
    SVDQ_CUDA(cudaMemcpyAsync(w->L2t, host_L2t, N * r * 2, cudaMemcpyHostToDevice, st));
    l1_fragment_kernel<<<num_sms() * 2, 256, 0, st>>>(w->L1, w->K, w->r, w->L1f);
    SVDQ_CHECK_LAUNCH("l1_fragment_kernel");
    l1_transpose_kernel<<<num_sms() * 2, 256, 0, st>>>(w->L1, w->K, w->r, w->L1t);
    SVDQ_CHECK_LAUNCH("l1_transpose_kernel");
  }
  SVDQ_CUDA(cudaMemcpyAsync(w->inv_lambda, host_inv_lambda, K * 4, cudaMemcpyHostToDevice, st));
  if (host_bias) SVDQ_CUDA(cudaMemcpyAsync(w->bias, host_bias, N * 2, cudaMemcpyHostToDevice, st));
  // the staging copy of the scales must outlive its transfer
  SVDQ_CUDA(cudaStreamSynchronize(st));
  return SVDQ_OK;
}

svdq_status svdq_calib_absmax(const uint16_t* A, int rows, int K, float* colmax, void* stream) {
  if (A == nullptr || colmax == nullptr || rows < 0 || K <= 0 || K % 2) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(colmax)) return SVDQ_ERR_MISALIGNED;
  if (rows == 0) return SVDQ_OK;
  calib_absmax_kernel<<<num_sms() * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      A, rows, K, reinterpret_cast<unsigned int*>(colmax));
  SVDQ_CHECK_LAUNCH("calib_absmax_kernel");
  return SVDQ_OK;
}

svdq_status svdq_calibrate_lambda(const float* x_absmax, const uint16_t* W, int N, int K, float alpha,
                                  float* lambda, void* stream) {
  if (x_absmax == nullptr || W == nullptr || lambda == nullptr || N <= 0 || K <= 0 || K % 2 ||
      !(alpha >= 0.0f && alpha <= 1.0f))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x_absmax) || !aligned16(W) || !aligned16(lambda)) return SVDQ_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // max|W[:, k]| is gathered in lambda itself, then turned into lambda in place
  SVDQ_CUDA(cudaMemsetAsync(lambda, 0, static_cast<size_t>(K) * 4, st));
  calib_absmax_kernel<<<num_sms() * 4, 256, 0, st>>>(W, N, K, reinterpret_cast<unsigned int*>(lambda));
  SVDQ_CHECK_LAUNCH("calib_absmax_kernel");
  calib_lambda_kernel<<<(K + 255) / 256, 256, 0, st>>>(x_absmax, K, static_cast<double>(alpha), lambda);
  SVDQ_CHECK_LAUNCH("calib_lambda_kernel");
  return SVDQ_OK;
}

svdq_status svdq_int4_scales_to_logical(const uint16_t* native, int rows, int rows_pad, int K,
                                        uint16_t* logical) {
  if (native == nullptr || logical == nullptr || rows < 0 || rows_pad < rows || K <= 0 || K % INT4_GROUP)
    return SVDQ_ERR_INVALID_ARG;
  int4_to_logical(native, rows, rows_pad, K, logical);
  return SVDQ_OK;
}

svdq_status svdq_int4_scales_to_native(const uint16_t* logical, int rows, int rows_pad, int K,
                                       uint16_t* native) {
  if (native == nullptr || logical == nullptr || rows < 0 || rows_pad < rows || K <= 0 || K % INT4_GROUP)
    return SVDQ_ERR_INVALID_ARG;
  int4_to_native(logical, rows, rows_pad, K, native);
  return SVDQ_OK;
}

svdq_status svdq_scales_to_logical(const uint8_t* native, int rows, int K, uint8_t* logical) {
  if (native == nullptr || logical == nullptr || rows < 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  to_logical(native, rows, K, logical);
  return SVDQ_OK;
}

svdq_status svdq_act_scales_to_logical(const uint8_t* native, int M, int K, uint8_t* logical) {
  return svdq_scales_to_logical(native, M, K, logical);
}

svdq_status svdq_scales_to_native(const uint8_t* logical, int rows, int K, uint8_t* native) {
  if (native == nullptr || logical == nullptr || rows < 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  to_native(logical, rows, K, native);
  return SVDQ_OK;
}

svdq_status svdq_get_device_status(void* stream, uint32_t* detail) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SVDQ_CUDA(cudaStreamSynchronize(st));
  unsigned int v = 0;
  SVDQ_CUDA(cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)));
  if (detail) *detail = v;
  return v ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

svdq_status svdq_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  const unsigned long long lim =
      std::min<unsigned long long>(std::max<unsigned long long>(limit_ns, 1000ull), 1000000000ull);
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(lim);
  SVDQ_CHECK_LAUNCH("selftest_wait_kernel");
  return SVDQ_OK;
}

svdq_status svdq_selftest_quotient(uint64_t* counts) {
  if (counts == nullptr) return SVDQ_ERR_INVALID_ARG;
  const unsigned long long z[3] = {0ull, 0ull, 0ull};
  SVDQ_CUDA(cudaMemcpyToSymbol(g_quotient_mismatch, z, sizeof(z)));
  selftest_quotient_kernel<<<num_sms() * 8, 256>>>();
  SVDQ_CHECK_LAUNCH("selftest_quotient_kernel");
  SVDQ_CUDA(cudaDeviceSynchronize());
  unsigned long long out[3];
  SVDQ_CUDA(cudaMemcpyFromSymbol(out, g_quotient_mismatch, sizeof(out)));
  for (int i = 0; i < 3; ++i) counts[i] = out[i];
  return SVDQ_OK;
}

svdq_status svdq_selftest_conversions(uint64_t* counts) {
  if (counts == nullptr) return SVDQ_ERR_INVALID_ARG;
  const unsigned long long z[3] = {0ull, 0ull, 0ull};
  SVDQ_CUDA(cudaMemcpyToSymbol(g_conversion_mismatch, z, sizeof(z)));
  selftest_conversion_kernel<<<num_sms() * 8, 256>>>();
  SVDQ_CHECK_LAUNCH("selftest_conversion_kernel");
  SVDQ_CUDA(cudaDeviceSynchronize());
  unsigned long long out[3];
  SVDQ_CUDA(cudaMemcpyFromSymbol(out, g_conversion_mismatch, sizeof(out)));
  for (int i = 0; i < 3; ++i) counts[i] = out[i];
  return SVDQ_OK;
}

svdq_status svdq_clear_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned int z = 0;
  SVDQ_CUDA(cudaMemcpyToSymbolAsync(g_device_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st));
  SVDQ_CUDA(cudaStreamSynchronize(st));
  return SVDQ_OK;
}

}  // extern "C"
