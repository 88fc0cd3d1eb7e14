// OPTQ (sequential column-wise quantisation with error compensation) with the weak columns
// moved to the end of the order.
//
// Pages: "Low-precision quantization" (paper p.4, as summarised on paperlayer.ai): the dense
// weights go through OPTQ's column-by-column quantisation; the weak columns are moved to the end
// of the order, are never quantised, and absorb the compensation of the columns before them, so
// the stored fp16 weak block holds their compensated values.  "Layer-wise Quantization and
// Hessian" (p.3): each row's error is dW H dW^T with H from the calibration inputs (H = X^T X
// here; OPTQ's factor 2 cancels in every update), plus damp * mean(diag H) on the diagonal.
//
// Each step is the optimal-brain-surgeon update: with F the columns not yet quantised (the
// current column first) and M = (H restricted to F)^-1, quantise the current column with the
// (scale, zero) of its group and move the rest of F by -(w - w_hat) / M[0][0] * M[0][1:].
// Written for the GPU, M is not recomputed at each step but kept exact by the Schur-complement
// identity for the inverse of a principal submatrix: removing the first index of F gives
//     M'[i][j] = M[i][j] - M[i][0] M[0][j] / M[0][0]      (i, j in F without its first),
// so the whole run is one Gauss-Jordan inversion of the permuted H followed by one rank-1
// downdate of M and one rank-1 update of the weights per quantised column.  Every number is fp64;
// the code decision is taken in fp32 on the current weight, q = clamp(rint(fp32(w) / s) + z).
// Rows are independent: the weights are kept as an N x K fp64 matrix in the permuted column
// order (dense columns ascending, then the weak columns ascending).
#include "owq_internal.cuh"

namespace owq {
namespace {

constexpr int kOptqThreads = 256;

// A[a][b] = sum_t X[t][perm[a]] X[t][perm[b]] (fp64, t ascending); 32 x 32 tiles
__global__ void k_optq_hessian(const __half* __restrict__ X, int T, int K, const int* __restrict__ perm,
                               double* __restrict__ A) {
  __shared__ double xa[32][33], xb[32][33];
  const int a0 = blockIdx.y * 32, b0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 256 threads: 8 rows of 32
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int t0 = 0; t0 < T; t0 += 32) {
    for (int r = ty; r < 32; r += 8) {
      const int t = t0 + r;
      xa[r][tx] = (t < T && a0 + tx < K) ? (double)__half2float(X[(size_t)t * K + perm[a0 + tx]]) : 0.0;
      xb[r][tx] = (t < T && b0 + tx < K) ? (double)__half2float(X[(size_t)t * K + perm[b0 + tx]]) : 0.0;
    }
    __syncthreads();
    const int tn = min(32, T - t0);
    for (int r = 0; r < tn; ++r) {
      const double vb = xb[r][tx];
      #pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = __fma_rn(xa[r][ty + 8 * q], vb, acc[q]);
    }
    __syncthreads();
  }
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int a = a0 + ty + 8 * q, b = b0 + tx;
    if (a < K && b < K) A[(size_t)a * K + b] = acc[q];
  }
}

// A[a][a] += damp * mean(diag A)  (one CTA)
__global__ void k_optq_damp(double* __restrict__ A, int K, double damp) {
  __shared__ double part[kOptqThreads];
  double s = 0.0;
  for (int a = threadIdx.x; a < K; a += blockDim.x) s += A[(size_t)a * K + a];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double add = damp * (part[0] / K);
  for (int a = threadIdx.x; a < K; a += blockDim.x) A[(size_t)a * K + a] += add;
}

// Gauss-Jordan inversion in place, pivot p: save the pivot row and column ...
__global__ void k_gj_save(const double* __restrict__ A, int K, int p, double* __restrict__ col,
                          double* __restrict__ row) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < K; i += gridDim.x * blockDim.x) {
    col[i] = A[(size_t)i * K + p];
    row[i] = A[(size_t)p * K + i];
  }
}
// ... then eliminate with them (no element reads another one written in the same step)
__global__ void k_gj_update(double* __restrict__ A, int K, int p, const double* __restrict__ col,
                            const double* __restrict__ row) {
  const double inv = 1.0 / col[p];
  for (int i = blockIdx.y; i < K; i += gridDim.y) {
    const double ci = col[i];
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x) {
      double v;
      if (i == p) v = j == p ? inv : row[j] * inv;
      else if (j == p) v = -ci * inv;
      else v = __dsub_rn(A[(size_t)i * K + j], __dmul_rn(ci, __dmul_rn(row[j], inv)));
      A[(size_t)i * K + j] = v;
    }
  }
}

// W64[r][a] = W[r][perm[a]]
__global__ void k_optq_load(const __half* __restrict__ W, int N, int K, const int* __restrict__ perm,
                            double* __restrict__ W64) {
  const size_t n = (size_t)N * K;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t r = e / K;
    const int a = (int)(e % K);
    W64[e] = (double)__half2float(W[r * K + perm[a]]);
  }
}

// step t: quantise column t of every row with its group's (scale, zero); err[r] =
// (w - w_hat) / M[t][t]; the column takes w_hat
__global__ void k_optq_quant(double* __restrict__ W64, int N, int K, int t, const int* __restrict__ perm,
                             const double* __restrict__ M, const __half* __restrict__ scales,
                             const __half* __restrict__ zeros, int group, int bits, uint8_t* __restrict__ codes,
                             double* __restrict__ err) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= N) return;
  const int j = perm[t], G = K / group, g = j / group;
  const float s = __half2float(scales[(size_t)r * G + g]);
  const float z = __half2float(zeros[(size_t)r * G + g]);
  const float qmax = (float)((1 << bits) - 1);
  const double w = W64[(size_t)r * K + t];
  const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(__double2float_rn(w), s)), z), 0.f), qmax);
  const double wh = (double)__half2float(__float2half_rn(__fmul_rn(s, __fsub_rn(q, z))));
  err[r] = __ddiv_rn(__dsub_rn(w, wh), M[(size_t)t * K + t]);
  W64[(size_t)r * K + t] = wh;
  codes[(size_t)r * K + j] = (uint8_t)q;
}

// step t: W64[r][j] -= err[r] M[t][j] and M[i][j] -= M[i][t] M[t][j] / M[t][t] for i, j > t
// (rows 0 .. N-1 of the grid's y range are weight rows, N .. N + K - t - 2 are rows of M)
__global__ void k_optq_update(double* __restrict__ W64, int N, int K, int t, double* __restrict__ M,
                              const double* __restrict__ err) {
  const int rest = K - t - 1;
  const double* mt = M + (size_t)t * K;
  const double inv = 1.0 / mt[t];
  for (int y = blockIdx.y; y < N + rest; y += gridDim.y) {
    double f;
    double* dst;
    if (y < N) {
      f = err[y];
      dst = W64 + (size_t)y * K;
    } else {
      const int i = t + 1 + (y - N);
      dst = M + (size_t)i * K;
      f = __dmul_rn(dst[t], inv);
    }
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < rest; c += gridDim.x * blockDim.x) {
      const int jj = t + 1 + c;
      dst[jj] = __dsub_rn(dst[jj], __dmul_rn(f, mt[jj]));
    }
  }
}

// the weak columns (the last k of the order): fp16 of their compensated values, and their codes
// take the group's zero point
__global__ void k_optq_finish(const double* __restrict__ W64, int N, int K, int k, const int* __restrict__ perm,
                              const __half* __restrict__ zeros, int group, uint8_t* __restrict__ codes,
                              __half* __restrict__ w_weak) {
  const size_t n = (size_t)N * k;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t r = e / k;
    const int s = (int)(e % k);
    const int a = K - k + s, j = perm[a];
    w_weak[e] = __double2half(W64[r * K + a]);   // one rounding, fp64 -> fp16 (round to nearest even)
    codes[r * K + j] = (uint8_t)__half2float(zeros[r * (K / group) + j / group]);
  }
}

}  // namespace

size_t optq_scratch_bytes(int N, int K) {
  return (size_t)K * K * sizeof(double) + (size_t)N * K * sizeof(double) + (size_t)N * sizeof(double) +
         2 * (size_t)K * sizeof(double) + (size_t)K * sizeof(int) + 1024;
}

cudaError_t launch_optq(const __half* W, const __half* X, int N, int K, int T, int bits, int group,
                        const int* perm_host, int k, const __half* scales, const __half* zeros, double damp,
                        uint8_t* codes, __half* w_weak, cudaStream_t s) {
  unsigned char* buf = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&buf, optq_scratch_bytes(N, K), s);
  if (e != cudaSuccess) return e;
  double* M = reinterpret_cast<double*>(buf);
  double* W64 = M + (size_t)K * K;
  double* err = W64 + (size_t)N * K;
  double* col = err + N;
  double* row = col + K;
  int* perm = reinterpret_cast<int*>(row + K);
  e = cudaMemcpyAsync(perm, perm_host, sizeof(int) * K, cudaMemcpyHostToDevice, s);
  const int kt = (K + 31) / 32;
  if (e == cudaSuccess) {
    k_optq_hessian<<<dim3(kt, kt), 256, 0, s>>>(X, T, K, perm, M);
    if (damp != 0.0) k_optq_damp<<<1, kOptqThreads, 0, s>>>(M, K, damp);
    for (int p = 0; p < K && e == cudaSuccess; ++p) {
      k_gj_save<<<(K + kOptqThreads - 1) / kOptqThreads, kOptqThreads, 0, s>>>(M, K, p, col, row);
      k_gj_update<<<dim3((K + kOptqThreads - 1) / kOptqThreads, std::min(K, 4096)), kOptqThreads, 0, s>>>(M, K, p,
                                                                                                      col, row);
      e = cudaGetLastError();
    }
  }
  if (e == cudaSuccess) {
    const size_t NK = (size_t)N * K;
    k_optq_load<<<(unsigned)std::min<size_t>((NK + 255) / 256, 65535), 256, 0, s>>>(W, N, K, perm, W64);
    const int nd = K - k;
    for (int t = 0; t < nd && e == cudaSuccess; ++t) {
      k_optq_quant<<<(N + kOptqThreads - 1) / kOptqThreads, kOptqThreads, 0, s>>>(W64, N, K, t, perm, M, scales,
                                                                                zeros, group, bits, codes, err);
      const int rest = K - t - 1;
      if (rest > 0)
        k_optq_update<<<dim3((rest + kOptqThreads - 1) / kOptqThreads, std::min(N + rest, 8192)), kOptqThreads, 0,
                        s>>>(W64, N, K, t, M, err);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess && k > 0) {
      const size_t Nk = (size_t)N * k;
      k_optq_finish<<<(unsigned)std::min<size_t>((Nk + 255) / 256, 65535), 256, 0, s>>>(W64, N, K, k, perm, zeros,
                                                                                        group, codes, w_weak);
      e = cudaGetLastError();
    }
  }
  cudaError_t e2 = cudaFreeAsync(buf, s);
  return e != cudaSuccess ? e : e2;
}

}  // namespace owq
