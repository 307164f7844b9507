// Weight preparation on the GPU (offline compression, not the layer's hot
// path): calibration maxima and smoothing factors, the matrix products of a
// randomized truncated SVD, and the residual quantisation.
//
// Method: "Nunchaku Lite ... integrated into Diffusers" (axbrief.com),
// section "Hardware Specialization and the Compression Workflow" (inspect the
// model, calibrate the data distribution to find outliers, quantize the
// weights, package; INT4 or NVFP4 precision) and section "The Mechanics of
// 4-Bit Efficiency and SVDQuant" (outliers shifted into the weights, a 16-bit
// low-rank branch from the decomposition, a 4-bit residual); "Problemas do
// Nunchaku Qwen..." (apatero.com), section "O que e Nunchaku..." (the
// low-rank branch comes from a singular value decomposition).
//
// The residual quantiser computes R = lambda_k W[k,n] - sum_j L1[k,j] L2[j,n]
// in fp64 (every product of the bf16 / fp32 inputs is exact in fp64) and
// rounds with the same fp64 operations as the format definitions: a value is
// scaled by a power of two, rounded to an integer (ties to even) and scaled
// back; only the order of the r-term sum can differ from another fp64
// evaluation of R.
#pragma once

#include "ptx.cuh"

namespace svdq {

// ----------------------------------------------------------- calibration
// Largest |x[m, k]| per column k (x bf16 [M x K]): thread per column, a
// slice of rows per block row; maxima of non-negative floats compare as
// their bit patterns.
__global__ void prep_col_amax_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K, int rows_per,
                                     unsigned* __restrict__ out) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * rows_per;
  const int64_t m1 = min(M, m0 + rows_per);
  unsigned a = 0;
  for (int64_t m = m0; m < m1; ++m) a = max(a, static_cast<unsigned>(x[m * K + k] & 0x7FFFu) << 16);
  atomicMax(out + k, a);
}

// Largest |w[k, n]| per row k (w bf16 [K x N]): a block per row.
__global__ void prep_row_amax_kernel(const uint16_t* __restrict__ w, int64_t K, int64_t N,
                                     unsigned* __restrict__ out) {
  const int64_t k = blockIdx.x;
  unsigned a = 0;
  for (int64_t n = threadIdx.x; n < N; n += blockDim.x)
    a = max(a, static_cast<unsigned>(w[k * N + n] & 0x7FFFu) << 16);
  for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
  __shared__ unsigned part[32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned b = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) b = max(b, part[i]);
    out[k] = b;
  }
}

// lambda_k = ax^alpha / aw^(1-alpha) in fp64, 1 where either maximum is 0,
// clamped to [2^-20, 2^20], stored as fp32 (round to nearest).
__global__ void prep_lambda_kernel(const unsigned* __restrict__ ax, const unsigned* __restrict__ aw,
                                   int64_t K, double alpha, float* __restrict__ lam) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const double a = static_cast<double>(__uint_as_float(ax[k]));
  const double b = static_cast<double>(__uint_as_float(aw[k]));
  double l = 1.0;
  if (a > 0.0 && b > 0.0) l = (alpha == 0.5 ? sqrt(a) / sqrt(b) : pow(a, alpha) / pow(b, 1.0 - alpha));
  l = fmin(fmax(l, 0x1p-20), 0x1p20);
  lam[k] = __double2float_rn(l);
}

// W_hat = diag(lambda) W in fp32 (the input of the randomized SVD).
__global__ void prep_smooth_kernel(const uint16_t* __restrict__ w, const float* __restrict__ lam, int64_t K,
                                   int64_t N, float* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= K * N) return;
  out[i] = __fmul_rn(bf16lo(w[i]), lam[i / N]);
}

// ------------------------------------------------------------ fp32 GEMM
// C[i, j] (+)= sum_k A(i, k) B(k, j) over the split-K slice blockIdx.z, with
// A(i, k) = A[i * as0 + k * as1], B(k, j) = B[k * bs0 + j * bs1] (any
// transposition by strides) and C row-major with leading dimension ldc.
// 64 x 64 output tile, 16-deep k-steps staged in shared memory, 256 threads
// with 4 x 4 outputs each; slices accumulate with atomicAdd into a C that
// the caller zeroed.
__global__ void __launch_bounds__(256)
    prep_gemm_f32_kernel(const float* __restrict__ A, int64_t as0, int64_t as1, const float* __restrict__ B,
                         int64_t bs0, int64_t bs1, float* __restrict__ C, int64_t ldc, int64_t Mr, int64_t Nc,
                         int64_t Kd, int64_t kslice) {
  __shared__ float sa[16][68];
  __shared__ float sb[16][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * 64, j0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int64_t k0 = static_cast<int64_t>(blockIdx.z) * kslice;
  const int64_t k1 = min(Kd, k0 + kslice);
  float acc[4][4] = {};
  for (int64_t kk = k0; kk < k1; kk += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int r = e / 64, c = e % 64;  // r: k offset, c: i or j offset
      const int64_t k = kk + r;
      sa[r][c] = (k < k1 && i0 + c < Mr) ? A[(i0 + c) * as0 + k * as1] : 0.f;
      sb[r][c] = (k < k1 && j0 + c < Nc) ? B[k * bs0 + (j0 + c) * bs1] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = sa[r][ty * 4 + u];
        b[u] = sb[r][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = __fmaf_rn(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t i = i0 + ty * 4 + u, j = j0 + tx * 4 + v;
      if (i < Mr && j < Nc) atomicAdd(C + i * ldc + j, acc[u][v]);
    }
}

// G = Y^T Y in fp64 for Y fp32 [rows x l] (row-major): a block per (a, b)
// pair with a <= b; G is symmetric.
__global__ void prep_gram_f64_kernel(const float* __restrict__ Y, int64_t rows, int l, double* __restrict__ G) {
  const int a = blockIdx.y, b = blockIdx.x;
  if (a > b) return;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < rows; i += blockDim.x)
    s = fma(static_cast<double>(Y[i * l + a]), static_cast<double>(Y[i * l + b]), s);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ double part[32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += part[i];
    G[a * l + b] = t;
    G[b * l + a] = t;
  }
}

// Yo[rows x l] = Y . T for a small T [l x l] (fp64, row-major), out of
// place: a thread per output element; T's row a is read by a whole warp at
// once (one broadcast load per step) through the read-only cache.
__global__ void prep_rmul_small_kernel(const float* __restrict__ Y, int64_t rows, int l,
                                       const double* __restrict__ T, float* __restrict__ Yo) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= rows * l) return;
  const int64_t i = e / l;
  const int b = static_cast<int>(e % l);
  double s = 0.0;
  for (int a = 0; a < l; ++a) s = fma(static_cast<double>(Y[i * l + a]), __ldg(T + a * l + b), s);
  Yo[e] = static_cast<float>(s);
}

// --------------------------------------------------- residual quantisation
// v rounded to a binary format with p significant bits, smallest normal
// exponent emin (spacing 2^(emin - p + 1) below it), ties to even, magnitude
// saturated at maxf when satfinite (else returned above it): the value is
// scaled by a power of two, rounded to an integer and scaled back, all exact
// in fp64 except the one rounding.
__device__ __forceinline__ double round_fmt(double v, int p, int emin, double maxf) {
  if (v == 0.0 || !isfinite(v)) return v;
  int ex;
  frexp(v, &ex);                               // |v| = m 2^ex, 0.5 <= m < 1
  const int lead = max(ex - 1, emin);
  const int ue = lead - (p - 1);
  double q = ldexp(rint(ldexp(v, -ue)), ue);
  if (fabs(q) > maxf) q = copysign(maxf, q);
  if (q == 0.0) q = copysign(0.0, v);
  return q;
}

// R[k, n] for one element, fp64: lambda_k w[k,n] - sum_j L1[k,j] L2[j,n].
__device__ __forceinline__ double prep_residual(const uint16_t* __restrict__ w, const float* __restrict__ lam,
                                                const float* __restrict__ l1row, const float* l2col, int r,
                                                int64_t N, int64_t k, int64_t n) {
  double lr = 0.0;
  for (int j = 0; j < r; ++j) lr = fma(static_cast<double>(l1row[j]), static_cast<double>(l2col[j]), lr);
  return static_cast<double>(lam[k]) * static_cast<double>(bf16lo(w[k * N + n])) - lr;
}

// Largest |R| over the whole residual (for the per-tensor scale): a thread
// per (column n, 16-row slice); non-negative doubles compare as bit patterns.
__global__ void prep_residual_amax_kernel(const uint16_t* __restrict__ w, const float* __restrict__ lam,
                                          const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2,
                                          int64_t K, int64_t N, int r, unsigned long long* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * 16;
  if (n >= N) return;
  float l2c[128];
  for (int j = 0; j < r; ++j) l2c[j] = bf16lo(L2[j * N + n]);
  double a = 0.0;
  for (int64_t k = k0; k < min(K, k0 + 16); ++k) {
    float l1r[128];
    for (int j = 0; j < r; ++j) l1r[j] = bf16lo(L1[k * r + j]);
    a = fmax(a, fabs(prep_residual(w, lam, l1r, l2c, r, N, k, n)));
  }
  atomicMax(out, static_cast<unsigned long long>(__double_as_longlong(a)));
}

// Codes and scales of R^T, groups of G along K for each output feature n: a
// thread per (n, group).  INT4: s = bf16(amax / 7), q = clamp(rint(R / s),
// -8, 7).  NVFP4: s = e4m3(amax / 6 * 2^-e) (satfinite), q = e2m1(R / (s 2^e))
// (satfinite, ties to even, sign kept).  s == 0 gives code +0.  Codes go to
// [N x K/2] (element 2j in the low nibble), scales to [N x K/G] (bf16 bits or
// E4M3 bytes).
template <int VARIANT>
__global__ void prep_residual_quant_kernel(const uint16_t* __restrict__ w, const float* __restrict__ lam,
                                           const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2,
                                           int64_t K, int64_t N, int r, int scale_exp,
                                           uint8_t* __restrict__ codes, void* __restrict__ scales) {
  constexpr int G = VARIANT == 0 ? 64 : 16;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t g = blockIdx.y;
  const bool live = n < N;
  const int64_t nn = live ? n : N - 1;  // threads past N compute column N-1 and store nothing
  __shared__ float l1s[G][128];         // the group's L1 rows, shared by the block
  for (int e = threadIdx.x; e < G * r; e += blockDim.x)
    l1s[e / r][e % r] = bf16lo(L1[(g * G + e / r) * r + e % r]);
  __syncthreads();
  float l2c[128];
  for (int j = 0; j < r; ++j) l2c[j] = bf16lo(L2[j * N + nn]);
  double amax = 0.0;
  for (int i = 0; i < G; ++i) amax = fmax(amax, fabs(prep_residual(w, lam, l1s[i], l2c, r, N, g * G + i, nn)));
  double s, sfull;
  if (VARIANT == 0) {
    s = round_fmt(amax / 7.0, 8, -126, 3.3895313892515355e38);
    sfull = s;
    // bf16 bits of s: s is a bf16 value, so its fp32 image has 16 zero low bits
    if (live)
      reinterpret_cast<uint16_t*>(scales)[n * (K / G) + g] =
          static_cast<uint16_t>(__float_as_uint(static_cast<float>(s)) >> 16);
  } else {
    s = round_fmt(ldexp(amax / 6.0, -scale_exp), 4, -6, 448.0);
    sfull = ldexp(s, scale_exp);
    // E4M3 byte of s (non-negative): exponent field 0 for subnormals m 2^-9
    uint32_t code = 0;
    if (s >= 0x1p-6) {
      int ex;
      const double m = frexp(s, &ex);  // s = m 2^ex
      code = (static_cast<uint32_t>(ex - 1 + 7) << 3) | static_cast<uint32_t>(rint((m * 2.0 - 1.0) * 8.0));
    } else if (s > 0.0) {
      code = static_cast<uint32_t>(rint(s * 512.0));
    }
    if (live) reinterpret_cast<uint8_t*>(scales)[n * (K / G) + g] = static_cast<uint8_t>(code);
  }
  if (!live) return;
  uint8_t* crow = codes + n * (K / 2) + g * (G / 2);
  for (int i = 0; i < G; i += 2) {
    uint32_t nib[2];
    for (int h = 0; h < 2; ++h) {
      uint32_t c = 0;
      if (sfull > 0.0) {
        const double v = prep_residual(w, lam, l1s[i + h], l2c, r, N, g * G + i + h, n) / sfull;
        if (VARIANT == 0) {
          const double q = fmin(fmax(rint(v), -8.0), 7.0);
          c = static_cast<uint32_t>(static_cast<int>(q)) & 0xFu;
        } else {
          const double q = round_fmt(v, 2, 0, 6.0);
          const double a = fabs(q);
          // magnitude index in {0, 0.5, 1, 1.5, 2, 3, 4, 6}
          const uint32_t idx = a < 2.0 ? static_cast<uint32_t>(a * 2.0) : (a == 2.0 ? 4u : (a == 3.0 ? 5u : (a == 4.0 ? 6u : 7u)));
          c = idx | (signbit(q) ? 8u : 0u);
        }
      }
      nib[h] = c;
    }
    crow[i / 2] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
  }
}

}  // namespace svdq
