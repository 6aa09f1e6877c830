// prep.cuh -- offline weight preparation on the GPU, stages 2 and 3 of
// SVDQuant (Nunchaku README, "Method": migrate the activation outliers into
// the weights with a per-channel factor, split the smoothed weight into a
// 16-bit low-rank part and a residual that is quantized to 4 bits), and the
// AWQ W4A16 weight quantizer (Diffusers blog, quantization_config: awq_w4a16,
// int4, group 64, bf16 scale and zero point). The SVD itself is left to the
// caller's linear-algebra library; everything around it is here:
//
//   column_absmax_kernel   a[k] = max_m |A[m,k]| of a bf16 matrix
//   lowrank_factors_kernel L1 = RN_bf16(V_r sqrt(S_r)), L2 = RN_bf16(sqrt(S_r) U_r^T) from the SVD
//   smoothing_kernel       smooth_inv[k] = RN32(1 / lambda_k),
//                          lambda_k = sqrt(max|X_k| / max|W_k|) in float64 (1 if either is 0)
//   residual_kernel        R[n,k] = RN_bf16(W[n,k] (1 / smooth_inv[k]) - sum_j L1[k,j] L2[j,n]),
//                          every step in float64 with one rounding to bf16 at the end
//   awq_quantize_kernel    per 64-wide group: s = RN_bf16((max - min) / 15) (1 if max == min),
//                          z = clamp(rint(-min / s), 0, 15), q = clamp(rint(w / s + z), 0, 15),
//                          written straight into the fragment order and (s, z) pairs that
//                          awq_w4a16_linear reads
// Rounding to bf16 from float64 is one rounding to 8 significant bits, nearest
// even (frexp, scale by 2^8, rint, scale back: all exact but the rint).
#pragma once

#include "sm100.cuh"

namespace svdq {

// float64 -> the nearest bf16 value with ties to even (normal range), as a bf16 bit pattern
__device__ __forceinline__ uint16_t bf16_bits_from_f64(double v) {
  int e;
  const double f = frexp(v, &e);
  const double r = ldexp(rint(ldexp(f, 8)), e - 8);  // 8 significant bits: exact in float32
  return static_cast<uint16_t>(__float_as_uint(static_cast<float>(r)) >> 16);
}

__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

// absmax[k] |= bits of max_m |A[m, k]| (absmax zeroed by the caller; non-negative
// floats order like their bit patterns, so the integer maximum is exact and
// independent of the order). Thread t always takes the same 8 columns.
__global__ void column_absmax_kernel(const uint16_t* A, int rows, int K, int lda, uint32_t* absmax) {
  const int units = K / 8;
  const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t tid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  // the host launches at least `units` threads, so every column has a thread
  const int c = static_cast<int>(tid % units);
  const size_t row_step = nthreads / units > 0 ? nthreads / units : 1;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  bool any = false;
  for (size_t row = tid / units; row < static_cast<size_t>(rows); row += row_step) {
    const uint4 v = *reinterpret_cast<const uint4*>(A + row * lda + 8 * c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m[2 * j] = fmaxf(m[2 * j], fabsf(__uint_as_float(w[j] << 16)));
      m[2 * j + 1] = fmaxf(m[2 * j + 1], fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
    any = true;
  }
  if (!any) return;
#pragma unroll
  for (int j = 0; j < 8; ++j) atomicMax(absmax + 8 * c + j, __float_as_uint(m[j]));
}

// smooth_inv[k] = RN32(1 / lambda), lambda = sqrt(x_absmax[k] / w_absmax[k]) in
// float64, lambda = 1 where either maximum is 0. w_absmax arrives as float bits
// in smooth_inv's own storage (column_absmax_kernel's output) and is replaced.
__global__ void smoothing_kernel(const float* x_absmax, float* smooth_inv, int K) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const double xm = static_cast<double>(x_absmax[k]);
  const double wm = static_cast<double>(smooth_inv[k]);
  double lam = 1.0;
  if (xm > 0.0 && wm > 0.0) lam = __dsqrt_rn(__ddiv_rn(xm, wm));
  smooth_inv[k] = __double2float_rn(__ddiv_rn(1.0, lam));
}

// The SVD's rank-r factors, each rounded once to bf16: with W_hat = U diag(S) Vh,
// L1[k, j] = RN_bf16(Vh[j, k] sqrt(S[j])) [K, r] and L2[j, n] = RN_bf16(sqrt(S[j]) U[n, j]) [r, N].
__global__ void lowrank_factors_kernel(const double* U, int ldu, const double* S, const double* Vh,
                                       int ldvh, uint16_t* L1, uint16_t* L2, int N, int K, int r) {
  const size_t n1 = static_cast<size_t>(K) * r, total = n1 + static_cast<size_t>(r) * N;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (t < n1) {
      const int k = static_cast<int>(t / r), j = static_cast<int>(t % r);
      L1[t] = bf16_bits_from_f64(__dmul_rn(Vh[static_cast<size_t>(j) * ldvh + k], __dsqrt_rn(S[j])));
    } else {
      const size_t u = t - n1;
      const int j = static_cast<int>(u / N), n = static_cast<int>(u % N);
      L2[u] = bf16_bits_from_f64(__dmul_rn(__dsqrt_rn(S[j]), U[static_cast<size_t>(n) * ldu + j]));
    }
  }
}

// R [N, K] bf16 from W [N, K] bf16, smooth_inv [K], L1 [K, r] bf16, L2 [r, N] bf16.
// A 16 (n) x 16 (k) tile per block; L1 and L2 pass through shared memory in
// chunks of 32 ranks, as float64.
constexpr int kResTile = 16, kResChunk = 32;
__global__ void __launch_bounds__(256) residual_kernel(const uint16_t* W, const float* smooth_inv,
                                                       const uint16_t* L1, const uint16_t* L2, uint16_t* R,
                                                       int N, int K, int r) {
  __shared__ double l1s[kResTile][kResChunk + 1];  // [k][j]
  __shared__ double l2s[kResChunk][kResTile + 1];  // [j][n]
  const int tx = threadIdx.x % kResTile, ty = threadIdx.x / kResTile;  // k, n within the tile
  const int k0 = blockIdx.x * kResTile, n0 = blockIdx.y * kResTile;
  const int k = k0 + tx, n = n0 + ty;
  double acc = 0.0;
  for (int j0 = 0; j0 < r; j0 += kResChunk) {
    // 16 x 32 values of each factor, two per thread
    for (int i = threadIdx.x; i < kResTile * kResChunk; i += blockDim.x) {
      const int a = i / kResChunk, j = i % kResChunk;  // L1: row k0 + a, rank j0 + j
      l1s[a][j] = (k0 + a < K && j0 + j < r) ? bf16_to_f64(L1[static_cast<size_t>(k0 + a) * r + j0 + j]) : 0.0;
      const int jj = i / kResTile, b = i % kResTile;   // L2: rank j0 + jj, column n0 + b
      l2s[jj][b] = (j0 + jj < r && n0 + b < N) ? bf16_to_f64(L2[static_cast<size_t>(j0 + jj) * N + n0 + b]) : 0.0;
    }
    __syncthreads();
    const int nj = r - j0 < kResChunk ? r - j0 : kResChunk;
    for (int j = 0; j < nj; ++j) acc = __fma_rn(l1s[tx][j], l2s[j][ty], acc);
    __syncthreads();
  }
  if (k < K && n < N) {
    const double inv = __ddiv_rn(1.0, static_cast<double>(smooth_inv[k]));
    const double w_hat = __dmul_rn(bf16_to_f64(W[static_cast<size_t>(n) * K + k]), inv);
    R[static_cast<size_t>(n) * K + k] = bf16_bits_from_f64(__dsub_rn(w_hat, acc));
  }
}

// One block per (16-row block, 64-wide group): the 16 rows' (s, z), then the
// 128 fragment words (lane l, word j: rows l / 4 and l / 4 + 8, columns 2 (l % 4)
// + {0, 1, 8, 9} of K step j; nibble slots 0..7 = (row, column) (0, 0), (8, 0),
// (0, 8), (8, 8), (0, 1), (8, 1), (0, 9), (8, 9)) and the 16 (s, z) pairs.
__global__ void __launch_bounds__(128) awq_quantize_kernel(const uint16_t* W, int N, int K,
                                                           uint32_t* qweight, uint32_t* sz) {
  __shared__ double ws[16][65];
  __shared__ double s_s[16], z_s[16];
  const int G = K / 64;
  const int b = blockIdx.x / G, g = blockIdx.x % G;
  for (int i = threadIdx.x; i < 16 * 64; i += blockDim.x) {
    const int rr = i / 64, c = i % 64, n = 16 * b + rr;
    ws[rr][c] = n < N ? bf16_to_f64(W[static_cast<size_t>(n) * K + 64 * g + c]) : 0.0;
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    const int rr = threadIdx.x;
    double mx = ws[rr][0], mn = ws[rr][0];
    for (int c = 1; c < 64; ++c) {
      mx = fmax(mx, ws[rr][c]);
      mn = fmin(mn, ws[rr][c]);
    }
    const double s = mx == mn ? 1.0 : bf16_to_f64(bf16_bits_from_f64(__ddiv_rn(__dsub_rn(mx, mn), 15.0)));
    const double z = fmin(fmax(rint(__ddiv_rn(-mn, s)), 0.0), 15.0) + 0.0;  // an integer: zero is +0
    s_s[rr] = s;
    z_s[rr] = z;
    const int n = 16 * b + rr;
    uint32_t pair = 0;
    if (n < N)
      pair = static_cast<uint32_t>(bf16_bits_from_f64(s)) | (static_cast<uint32_t>(bf16_bits_from_f64(z)) << 16);
    sz[(static_cast<size_t>(b) * G + g) * 16 + rr] = pair;
  }
  __syncthreads();
  const int lane = threadIdx.x / 4, j = threadIdx.x % 4;
  const int r0 = lane / 4, c0 = 2 * (lane % 4);
  uint32_t word = 0;
#pragma unroll
  for (int slot = 0; slot < 8; ++slot) {
    const int rr = r0 + ((slot & 1) ? 8 : 0);
    const int c = 16 * j + c0 + ((slot & 2) ? 8 : 0) + ((slot & 4) ? 1 : 0);
    const double q = fmin(fmax(rint(__dadd_rn(__ddiv_rn(ws[rr][c], s_s[rr]), z_s[rr])), 0.0), 15.0);
    const int n = 16 * b + rr;
    word |= (n < N ? static_cast<uint32_t>(q) : 0u) << (4 * slot);
  }
  qweight[((static_cast<size_t>(b) * G + g) * 32 + lane) * 4 + j] = word;
}

}  // namespace svdq
