// prepare.cuh -- offline preparation of one SVDQuant linear (device kernels).
//
// The weight is split into a low-rank component and a 4-bit residual
// (imaginepro.ai "Nunchaku 4-Bit Diffusion Inference in Diffusers: A Practical
// Guide", section "Under the Hood"; chaosnode.de "Nunchaku Lite", section
// "Die Technik: SVDQuant": outliers moved from activations into the weights,
// the hard part as a 16-bit low-rank branch, the rest in 4 bit):
//   What = f32(W * lambda) (column k of W scaled by lambda_k),
//   L1 = U_r diag(sigma_r) (K x r), L2 = V_r^T (r x N) of What^T,
//   R = f32(What - (bf16 L1 . bf16 L2)^T), NVFP4 along K.
// The top-r singular pairs come from the float64 Gram matrix of What on its
// smaller side (K x K = What^T What when K <= N, else N x N = What What^T),
// whose eigen-decomposition is done by cuSOLVER (host side); everything else is
// in these kernels.
#pragma once

#include "nvfp4.cuh"
#include "ptx.cuh"

namespace svdq {

// What = f32(W * lambda) per column; inv_lambda = f32(1 / lambda); bias copy.
__global__ void prep_smooth_kernel(const uint16_t* __restrict__ W, const float* __restrict__ lambda,
                                   const uint16_t* __restrict__ bias, int N, int K,
                                   float* __restrict__ what, float* __restrict__ inv_lambda,
                                   uint16_t* __restrict__ bias_out) {
  const size_t total = static_cast<size_t>(N) * K;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int k = static_cast<int>(i % K);
    what[i] = __fmul_rn(bf16_bits_to_f32(W[i]), lambda[k]);
    if (i < static_cast<size_t>(K)) inv_lambda[i] = __fdiv_rn(1.0f, lambda[i]);
    if (bias != nullptr && i < static_cast<size_t>(N)) bias_out[i] = bias[i];
  }
}

// G = What^T What (col_gram, n = K) or What What^T (row gram, n = N), float64.
// 64 x 64 output tile per CTA, 256 threads with 4 x 4 outputs each, the
// summation dimension L staged through shared memory in slices of 16.
constexpr int GRAM_T = 64, GRAM_L = 16;

__global__ void __launch_bounds__(256) prep_gram_kernel(const float* __restrict__ what, int N, int K,
                                                        int col_gram, double* __restrict__ G) {
  const int n = col_gram ? K : N;
  const int L = col_gram ? N : K;
  __shared__ double sa[GRAM_L][GRAM_T + 1];
  __shared__ double sb[GRAM_L][GRAM_T + 1];
  const int a0 = blockIdx.y * GRAM_T, b0 = blockIdx.x * GRAM_T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4] = {};
  // element (i, l) of the n x L operand
  auto elem = [&](int i, int l) -> double {
    if (i >= n || l >= L) return 0.0;
    return col_gram ? static_cast<double>(what[static_cast<size_t>(l) * K + i])
                    : static_cast<double>(what[static_cast<size_t>(i) * K + l]);
  };
  for (int l0 = 0; l0 < L; l0 += GRAM_L) {
    for (int idx = threadIdx.x; idx < GRAM_L * GRAM_T; idx += 256) {
      int ll, ii;
      if (col_gram) {   // coalesced along i (consecutive columns of a What row)
        ll = idx / GRAM_T;
        ii = idx % GRAM_T;
      } else {          // coalesced along l
        ii = idx / GRAM_L;
        ll = idx % GRAM_L;
      }
      sa[ll][ii] = elem(a0 + ii, l0 + ll);
      sb[ll][ii] = elem(b0 + ii, l0 + ll);
    }
    __syncthreads();
#pragma unroll
    for (int ll = 0; ll < GRAM_L; ++ll) {
      double av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        av[u] = sa[ll][ty * 4 + u];
        bv[u] = sb[ll][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(av[u], bv[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int a = a0 + ty * 4 + u, b = b0 + tx * 4 + v;
      if (a < n && b < n) G[static_cast<size_t>(b) * n + a] = acc[u][v];   // column-major
    }
}

// Factors from the eigenpairs (eigenvalues ascending in `ev`, eigenvectors in
// the columns of the column-major n x n matrix `evec`), float64 results,
// L1f K x r and L2f r x N row-major:
//   col_gram (n = K): u_j = evec[:, n-1-j], sigma_j = sqrt(ev[n-1-j]);
//                     L1[:, j] = sigma_j u_j,  L2[j, :] = (What u_j)^T / sigma_j
//   row gram (n = N): v_j = evec[:, n-1-j];  L2[j, :] = v_j^T,  L1[:, j] = What^T v_j
// The dot-product factor: col_gram -> one CTA per weight row nn, warps over j,
// lanes over k; row gram -> one CTA per strip of 32 columns k, warps over j,
// lanes over k, looping over the rows of What (coalesced in both cases).
__global__ void __launch_bounds__(256) prep_factor_dot_kernel(const float* __restrict__ what, int N, int K,
                                                              int r, int col_gram,
                                                              const double* __restrict__ evec,
                                                              const double* __restrict__ ev,
                                                              double* __restrict__ L1f,
                                                              double* __restrict__ L2f) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (col_gram) {
    const int n = K, nn = blockIdx.x;
    for (int j = warp; j < r; j += 8) {
      const double* u = evec + static_cast<size_t>(n - 1 - j) * n;
      double acc = 0.0;
      for (int k = lane; k < K; k += 32)
        acc = fma(static_cast<double>(what[static_cast<size_t>(nn) * K + k]), u[k], acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        const double sig = sqrt(fmax(ev[n - 1 - j], 0.0));
        L2f[static_cast<size_t>(j) * N + nn] = sig > 0.0 ? acc / sig : 0.0;
      }
    }
  } else {
    const int n = N, k = blockIdx.x * 32 + lane;
    double acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.0;
    for (int nn = 0; nn < N; ++nn) {
      const double w = k < K ? static_cast<double>(what[static_cast<size_t>(nn) * K + k]) : 0.0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int j = warp + 8 * t;
        if (j < r) acc[t] = fma(w, evec[static_cast<size_t>(n - 1 - j) * n + nn], acc[t]);
      }
    }
    if (k < K) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int j = warp + 8 * t;
        if (j < r) L1f[static_cast<size_t>(k) * r + j] = acc[t];
      }
    }
  }
}

// The factor read directly off the eigenvectors (grid-strided).
__global__ void prep_factor_direct_kernel(int N, int K, int r, int col_gram,
                                          const double* __restrict__ evec,
                                          const double* __restrict__ ev, double* __restrict__ L1f,
                                          double* __restrict__ L2f) {
  const int n = col_gram ? K : N;
  const size_t total = col_gram ? static_cast<size_t>(K) * r : static_cast<size_t>(r) * N;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += stride) {
    if (col_gram) {
      const int k = static_cast<int>(idx / r), j = static_cast<int>(idx % r);
      const double sig = sqrt(fmax(ev[n - 1 - j], 0.0));
      L1f[idx] = sig * evec[static_cast<size_t>(n - 1 - j) * n + k];
    } else {
      const int j = static_cast<int>(idx / N), nn = static_cast<int>(idx % N);
      L2f[idx] = evec[static_cast<size_t>(n - 1 - j) * n + nn];
    }
  }
}

// Sign convention: flip (u_j, v_j) so the largest-|.| entry of u_j (the
// column j of L1, up to sigma_j > 0) is positive; first index wins ties.
__global__ void __launch_bounds__(256) prep_sign_kernel(double* __restrict__ L1f, double* __restrict__ L2f,
                                                        int N, int K, int r) {
  const int j = blockIdx.x;
  __shared__ double sv[256];
  __shared__ int si[256];
  double best = -1.0;
  int bi = 0x7fffffff;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double a = fabs(L1f[static_cast<size_t>(k) * r + j]);
    if (a > best || (a == best && k < bi)) {
      best = a;
      bi = k;
    }
  }
  sv[threadIdx.x] = best;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      const double a = sv[threadIdx.x + o];
      const int i = si[threadIdx.x + o];
      if (a > sv[threadIdx.x] || (a == sv[threadIdx.x] && i < si[threadIdx.x])) {
        sv[threadIdx.x] = a;
        si[threadIdx.x] = i;
      }
    }
    __syncthreads();
  }
  const bool flip = L1f[static_cast<size_t>(si[0]) * r + j] < 0.0;
  if (!flip) return;
  for (int k = threadIdx.x; k < K; k += blockDim.x) L1f[static_cast<size_t>(k) * r + j] *= -1.0;
  for (int nn = threadIdx.x; nn < N; nn += blockDim.x) L2f[static_cast<size_t>(j) * N + nn] *= -1.0;
}

// bf16 storage of the factors: L1 (K x r) and L2^T (N x r), RNE from float64.
__global__ void prep_round_kernel(const double* __restrict__ L1f, const double* __restrict__ L2f,
                                  int N, int K, int r, uint16_t* __restrict__ L1,
                                  uint16_t* __restrict__ L2t) {
  const size_t tot1 = static_cast<size_t>(K) * r, tot2 = static_cast<size_t>(N) * r;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < tot1 + tot2;
       i += stride) {
    if (i < tot1) {
      L1[i] = f64_to_bf16_rne(L1f[i]);
    } else {
      const size_t t = i - tot1;
      const size_t nn = t / r, j = t % r;
      L2t[t] = f64_to_bf16_rne(L2f[j * N + nn]);
    }
  }
}

// R[n][k] = f32(What[n][k] - sum_j bf16(L1)[k][j] bf16(L2t)[n][j]) (float64,
// increasing j), then NVFP4 along K.  One CTA per weight row; each warp
// handles 256-wide chunks (lane pairs form the 16-element blocks).
template <int RMAX>
__global__ void __launch_bounds__(256) prep_residual_kernel(const float* __restrict__ what,
                                                            const uint16_t* __restrict__ L1,
                                                            const uint16_t* __restrict__ L2t,
                                                            int N, int K, int r,
                                                            uint8_t* __restrict__ w_codes,
                                                            uint8_t* __restrict__ w_scales) {
  const int nn = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ double l2[RMAX > 0 ? RMAX : 1];
  for (int j = threadIdx.x; j < r; j += blockDim.x)
    l2[j] = static_cast<double>(bf16_bits_to_f32(L2t[static_cast<size_t>(nn) * r + j]));
  __syncthreads();
  const int nchunks = K / 256;
  for (int c = warp; c < nchunks; c += 8) {
    const int k0 = c * 256 + 8 * lane;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = k0 + i;
      double acc = 0.0;
      for (int j = 0; j < r; ++j)
        acc = __fma_rn(static_cast<double>(bf16_bits_to_f32(L1[static_cast<size_t>(k) * r + j])),
                       l2[j], acc);
      const double wv = static_cast<double>(what[static_cast<size_t>(nn) * K + k]);
      v[i] = __double2float_rn(__dsub_rn(wv, acc));
    }
    uint32_t sc;
    const uint32_t codes = nvfp4_quant_half_block(v, sc);
    *reinterpret_cast<uint32_t*>(w_codes + static_cast<size_t>(nn) * (K / 2) + k0 / 2) = codes;
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 2);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 4);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 6);
    if ((lane & 7) == 0) {
      const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
      *reinterpret_cast<uint32_t*>(w_scales + sf_offset(nn, k0 / 16, K)) = word;
    }
  }
}

// ---------------------------------------------------------------------------
// Calibration statistics: colmax[k] = max(colmax[k], max_m |A[m][k]|) for a
// row-major rows x K bf16 matrix (activations X, or the weight W).  Thread t
// of the grid owns column pair 2 (t % (K/2)) and a strided slice of the rows;
// the running maximum is kept as float bits, whose integer order matches the
// order of non-negative floats.
__global__ void calib_absmax_kernel(const uint16_t* __restrict__ A, int rows, int K,
                                    unsigned int* __restrict__ colmax_bits) {
  const long long pairs = K / 2;
  const long long T = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long slices = T / pairs > 0 ? T / pairs : 1;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < pairs * slices;
       idx += T) {
    const long long c = idx % pairs, slice = idx / pairs;
    unsigned int m0 = 0u, m1 = 0u;
    for (long long row = slice; row < rows; row += slices) {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(A + row * K + 2 * c);
      m0 = max(m0, (v & 0x7FFFu) << 16);   // |bf16| as float32 bits
      m1 = max(m1, v & 0x7FFF0000u);
    }
    if (m0) atomicMax(colmax_bits + 2 * c, m0);
    if (m1) atomicMax(colmax_bits + 2 * c + 1, m1);
  }
}

// lambda[k] = f32(x^alpha / w^(1 - alpha)) in float64 from the activation and
// weight column maxima (w_in_lambda holds max|W[:, k]| on entry); alpha = 0.5
// is evaluated as f32(sqrt(x / w)); 1 where either maximum is 0.
__global__ void calib_lambda_kernel(const float* __restrict__ x_absmax, int K, double alpha,
                                    float* __restrict__ lambda) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) {
    const double x = x_absmax[k], w = lambda[k];
    double l = 1.0;
    if (x > 0.0 && w > 0.0) l = alpha == 0.5 ? sqrt(x / w) : pow(x, alpha) / pow(w, 1.0 - alpha);
    lambda[k] = static_cast<float>(l);
  }
}

}  // namespace svdq
