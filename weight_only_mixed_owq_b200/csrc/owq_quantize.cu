// OWQ quantiser on the GPU: Hessian diagonal, all-column RTN pre-quantisation, column
// sensitivity, top-k weak-column selection, then min-max RTN of the dense columns.
//
// Pages: "OWQ: Outlier-Aware Weight Quantization for Efficient Fine-Tuning and Inference
// of Large Language Models" (paperlayer.ai), "Weak-column selection" (paper p.4: the score
// of a column combines its perturbation norm with its Hessian diagonal element; the top-k
// columns stay in fp16 and are excluded from quantisation), "Error Analysis" / appendix
// §1 Eq. (10) (second-order error dW H dW^T); min-max RTN is the simple quantiser named in
// "OWQ -- paper by Lee et al. (2023) -- summary and ideas", Key points.
//
// Determinism: every fp64 sum runs over its index in ascending order with separate
// multiply and add (no fused multiply-add), so the selection is a pure function of the
// inputs.  Every float-to-integer decision uses IEEE fp32 division and round-half-to-even.
#include <mutex>

#include "owq_internal.cuh"

namespace owq {
namespace {

// min-max RTN parameters of one (row, group) from its range; returns s (fp16) and z.
__device__ __forceinline__ void rtn_from_range(float mn, float mx, int qmax, __half* s_out,
                                               float* s32_out, float* z32_out) {
  if (mn == mx) { mn = -1.f; mx = 1.f; }
  __half s = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)qmax));
  if (__half2float(s) == 0.f) {            // range below fp16 resolution
    mn = -1.f; mx = 1.f;
    s = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)qmax));
  }
  float s32 = __half2float(s);
  float z = rintf(__fdiv_rn(-mn, s32));
  z = fminf(fmaxf(z, 0.f), (float)qmax);
  z = __fadd_rn(z, 0.f);                   // canonical +0
  *s_out = s; *s32_out = s32; *z32_out = z;
}

__device__ __forceinline__ float rtn_code(float w, float s32, float z32, int qmax) {
  float q = __fadd_rn(rintf(__fdiv_rn(w, s32)), z32);
  return fminf(fmaxf(q, 0.f), (float)qmax);
}

// lambda_j = sum_t X[t, j]^2, t ascending.  One thread per column.
__global__ void k_hessian_diag(const __half* __restrict__ X, int T, int K, double* __restrict__ lam) {
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  double acc = 0.0;
  const __half* p = X + j;
  #pragma unroll 4
  for (int t = 0; t < T; ++t) {
    double v = (double)__half2float(p[(size_t)t * K]);
    acc = __dadd_rn(acc, __dmul_rn(v, v));
  }
  lam[j] = acc;
}

// One warp per (row, group): range over the group's dense columns (weak ones read as 0,
// which the range always contains), then s and z.
__global__ void k_rtn_params(const __half* __restrict__ W, int N, int K, int group, int bits,
                             const uint8_t* __restrict__ weak_mask,
                             __half* __restrict__ scales, __half* __restrict__ zeros) {
  const int G = K / group;
  long long item = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (item >= (long long)N * G) return;
  int lane = threadIdx.x & 31;
  int i = (int)(item / G), g = (int)(item % G);
  const __half* row = W + (size_t)i * K + (size_t)g * group;
  float mn = 0.f, mx = 0.f;
  for (int j = lane; j < group; j += 32) {
    float v = __half2float(row[j]);
    if (weak_mask && weak_mask[g * group + j]) v = 0.f;
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  #pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    __half s; float s32, z32;
    rtn_from_range(mn, mx, (1 << bits) - 1, &s, &s32, &z32);
    scales[item] = s;
    zeros[item] = __float2half_rn(z32);
  }
}

// colsum_j = sum_i (W[i,j] - W_hat0[i,j])^2, i ascending; W_hat0 = fp16_rn(s (q - z)) of the
// all-column RTN (scales/zeros hold that quantisation here).  The squares are independent, only
// each column's sum is ordered: a CTA owns 32 columns; its 256 threads form the squared
// differences of a 64-row chunk into shared memory (the next chunk's weights and (scale, zero)
// pairs already in registers), then warp 0 adds each column's 64 values in row order to its
// running fp64 sum -- the same __dmul_rn / __dadd_rn sequence as one thread walking the column.
constexpr int kCsCols = 32, kCsRows = 64, kCsThreads = 256, kCsPer = kCsRows * kCsCols / kCsThreads;
__global__ void __launch_bounds__(kCsThreads) k_colsum_dw2(const __half* __restrict__ W, int N, int K, int group,
                                                            int bits, const __half* __restrict__ scales,
                                                            const __half* __restrict__ zeros,
                                                            double* __restrict__ colsum) {
  __shared__ double s_d2[2][kCsRows][kCsCols];
  const int tid = threadIdx.x, j0 = blockIdx.x * kCsCols;
  const int G = K / group, qmax = (1 << bits) - 1;
  const int nch = (N + kCsRows - 1) / kCsRows;
  // this thread's elements of a chunk: row (tid + u 256) / 32, column (tid % 32)
  const int c = tid % kCsCols, j = j0 + c, g = j / group;
  __half wv[kCsPer], sv[kCsPer], zv[kCsPer];
  auto load = [&](int ch) {
    #pragma unroll
    for (int u = 0; u < kCsPer; ++u) {
      const int i = ch * kCsRows + (tid + u * kCsThreads) / kCsCols;
      const bool ok = i < N && j < K;
      wv[u] = ok ? W[(size_t)i * K + j] : __float2half_rn(0.f);
      sv[u] = ok ? scales[(size_t)i * G + g] : __float2half_rn(0.f);
      zv[u] = ok ? zeros[(size_t)i * G + g] : __float2half_rn(0.f);
    }
  };
  double acc = 0.0;   // warp 0, lane c: column j0 + c
  if (nch > 0) load(0);
  for (int ch = 0; ch < nch; ++ch) {
    const int buf = ch & 1;
    double d2[kCsPer];
    #pragma unroll
    for (int u = 0; u < kCsPer; ++u) {
      const float w = __half2float(wv[u]), s32 = __half2float(sv[u]), z32 = __half2float(zv[u]);
      const float q = rtn_code(w, s32, z32, qmax);
      const float wh = __half2float(__float2half_rn(__fmul_rn(s32, __fsub_rn(q, z32))));
      const double d = __dsub_rn((double)w, (double)wh);
      d2[u] = __dmul_rn(d, d);
    }
    if (ch + 1 < nch) load(ch + 1);   // in flight while the sums below run
    #pragma unroll
    for (int u = 0; u < kCsPer; ++u) s_d2[buf][(tid + u * kCsThreads) / kCsCols][c] = d2[u];
    __syncthreads();   // (also: warp 0 finished the sums of chunk ch - 1, which used the other buffer)
    if (tid < kCsCols) {
      const int rows = min(kCsRows, N - ch * kCsRows);
      for (int r = 0; r < rows; ++r) acc = __dadd_rn(acc, s_d2[buf][r][tid]);
    }
  }
  if (tid < kCsCols && j0 + tid < K) colsum[j0 + tid] = acc;
}

struct Cand { double v; int j; };

__device__ __forceinline__ bool better(double av, int aj, double bv, int bj) {
  return av > bv || (av == bv && aj < bj);
}

// sens_j = lambda_j * colsum_j; the k best (descending, ties to the lower index), written
// ascending to idx; weak_mask[j] = 1 for those.  One block of 1024 threads.
__global__ void __launch_bounds__(1024) k_topk(const double* __restrict__ lam, const double* __restrict__ colsum,
                                               double* __restrict__ sens, int K, int k,
                                               int32_t* __restrict__ idx, uint8_t* __restrict__ weak_mask) {
  __shared__ double sv[32];
  __shared__ int sj[32];
  __shared__ int chosen[kMaxWeak];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  for (int j = tid; j < K; j += blockDim.x) {
    sens[j] = __dmul_rn(lam[j], colsum[j]);
    weak_mask[j] = 0;
  }
  __syncthreads();
  for (int r = 0; r < k; ++r) {
    double bv = -1.0; int bj = 0x7fffffff;
    for (int j = tid; j < K; j += blockDim.x) {
      double v = sens[j];
      if (v >= 0.0 && better(v, j, bv, bj)) { bv = v; bj = j; }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
      double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (better(ov, oj, bv, bj)) { bv = ov; bj = oj; }
    }
    if (lane == 0) { sv[wid] = bv; sj[wid] = bj; }
    __syncthreads();
    if (wid == 0) {
      bv = lane < nw ? sv[lane] : -1.0;
      bj = lane < nw ? sj[lane] : 0x7fffffff;
      #pragma unroll
      for (int o = 16; o; o >>= 1) {
        double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (better(ov, oj, bv, bj)) { bv = ov; bj = oj; }
      }
      if (lane == 0) {
        if (bj >= K) bj = 0;           // unreachable for finite inputs (every sens >= 0)
        chosen[r] = bj;
        sens[bj] = -1.0;
      }
    }
    __syncthreads();
  }
  // ascending order by rank
  for (int t = tid; t < k; t += blockDim.x) {
    int v = chosen[t], rank = 0;
    for (int u = 0; u < k; ++u) rank += chosen[u] < v;
    idx[rank] = v;
    weak_mask[v] = 1;
  }
}

__global__ void k_codes(const __half* __restrict__ W, int N, int K, int group, int bits,
                        const __half* __restrict__ scales, const __half* __restrict__ zeros,
                        const uint8_t* __restrict__ weak_mask, uint8_t* __restrict__ codes) {
  size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)N * K) return;
  int i = (int)(e / K), j = (int)(e % K), G = K / group, g = j / group;
  float s32 = __half2float(scales[(size_t)i * G + g]);
  float z32 = __half2float(zeros[(size_t)i * G + g]);
  float q = weak_mask[j] ? z32 : rtn_code(__half2float(W[e]), s32, z32, (1 << bits) - 1);
  codes[e] = (uint8_t)q;
}

__global__ void k_gather_weak(const __half* __restrict__ W, int N, int K,
                              const int32_t* __restrict__ idx, int k, __half* __restrict__ w_weak, int* status) {
  size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)N * k) return;
  int i = (int)(e / k), t = (int)(e % k);
  w_weak[e] = in_range(idx[t], K, status) ? W[(size_t)i * K + idx[t]] : __float2half_rn(0.f);
}

}  // namespace

cudaError_t launch_quantize(const __half* W, const __half* X, int N, int K, int T, int bits,
                            int group, int k, uint8_t* codes, __half* scales, __half* zeros,
                            int32_t* idx, __half* w_weak, cudaStream_t s) {
  const size_t scratch = (size_t)K * (3 * sizeof(double)) + (size_t)K;
  char* buf = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&buf, scratch, s);
  if (e != cudaSuccess) return e;
  double* lam = (double*)buf;
  double* colsum = lam + K;
  double* sens = colsum + K;
  uint8_t* mask = (uint8_t*)(sens + K);
  const int G = K / group;
  const long long items = (long long)N * G;

  k_hessian_diag<<<(K + 255) / 256, 256, 0, s>>>(X, T, K, lam);
  // all-column RTN into the output scale/zero buffers (overwritten below)
  k_rtn_params<<<(unsigned)((items + 7) / 8), 256, 0, s>>>(W, N, K, group, bits, nullptr, scales, zeros);
  k_colsum_dw2<<<(K + kCsCols - 1) / kCsCols, kCsThreads, 0, s>>>(W, N, K, group, bits, scales, zeros, colsum);
  k_topk<<<1, 1024, 0, s>>>(lam, colsum, sens, K, k, idx, mask);
  k_rtn_params<<<(unsigned)((items + 7) / 8), 256, 0, s>>>(W, N, K, group, bits, mask, scales, zeros);
  const size_t NK = (size_t)N * K;
  k_codes<<<(unsigned)((NK + 255) / 256), 256, 0, s>>>(W, N, K, group, bits, scales, zeros, mask, codes);
  if (k > 0) {
    const size_t Nk = (size_t)N * k;
    k_gather_weak<<<(unsigned)((Nk + 255) / 256), 256, 0, s>>>(W, N, K, idx, k, w_weak, device_status_ptr());
  }
  e = cudaGetLastError();
  cudaError_t e2 = cudaFreeAsync(buf, s);
  return e != cudaSuccess ? e : e2;
}

}  // namespace owq

// ---------------------------------------------------------------------------------------
// owq_quantize_noalloc: the same quantiser with its scratch in a fixed device array.
//
// Some callers cannot let a library allocate device memory: serving processes that reserve
// (almost) all of the GPU's memory up front for their own pool, where a library-side
// cudaMalloc fails or fragments that pool, and processes that forbid any allocation after
// start-up.  This entry point therefore takes its scratch (lambda, column sums and scores in
// fp64, plus a byte mask: 25 bytes per input column) from a file-scope device array of
// OWQ_NOALLOC_MAX_K columns (1 MB), which every GPU that loads the library holds until the
// process exits.  The array is shared by all calls: calls whose work overlaps on the GPU
// (different streams, no ordering between them) race on it and must be serialised by the
// caller.  Nothing in it has to start at zero: every kernel fully writes the part it reads
// later (the mask is cleared by the selection kernel itself).
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char owq_noalloc_scratch[(size_t)OWQ_NOALLOC_MAX_K * (3 * sizeof(double) + 1)];

namespace owq {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned char* g_noalloc_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device.  In host code the array's name
// is only a host-side stand-in, never a device address, so the address is looked up with the
// device current: on every call made outside a stream capture (so a context created anew, e.g.
// after cudaDeviceReset, gets its own address), and taken from the per-device cache during a
// capture (a lookup there could load the module, which a capture does not allow; the first
// call on a device must therefore come before any capture).
cudaError_t noalloc_scratch(cudaStream_t s, unsigned char** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, owq_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = static_cast<unsigned char*>(p);
  } else if (!g_noalloc_addr[dev]) {
    return cudaErrorStreamCaptureUnsupported;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

cudaError_t launch_quantize_static(const __half* W, const __half* X, int N, int K, int T, int bits,
                                   int group, int k, uint8_t* codes, __half* scales, __half* zeros,
                                   int32_t* idx, __half* w_weak, cudaStream_t s) {
  unsigned char* buf = nullptr;
  cudaError_t e = noalloc_scratch(s, &buf);
  if (e != cudaSuccess) return e;
  double* lam = reinterpret_cast<double*>(buf);
  double* colsum = lam + K;
  double* sens = colsum + K;
  uint8_t* mask = reinterpret_cast<uint8_t*>(sens + K);
  const int G = K / group;
  const long long items = (long long)N * G;
  k_hessian_diag<<<(K + 255) / 256, 256, 0, s>>>(X, T, K, lam);
  k_rtn_params<<<(unsigned)((items + 7) / 8), 256, 0, s>>>(W, N, K, group, bits, nullptr, scales, zeros);
  k_colsum_dw2<<<(K + kCsCols - 1) / kCsCols, kCsThreads, 0, s>>>(W, N, K, group, bits, scales, zeros, colsum);
  k_topk<<<1, 1024, 0, s>>>(lam, colsum, sens, K, k, idx, mask);
  k_rtn_params<<<(unsigned)((items + 7) / 8), 256, 0, s>>>(W, N, K, group, bits, mask, scales, zeros);
  const size_t NK = (size_t)N * K;
  k_codes<<<(unsigned)((NK + 255) / 256), 256, 0, s>>>(W, N, K, group, bits, scales, zeros, mask, codes);
  if (k > 0) {
    const size_t Nk = (size_t)N * k;
    k_gather_weak<<<(unsigned)((Nk + 255) / 256), 256, 0, s>>>(W, N, K, idx, k, w_weak, device_status_ptr());
  }
  return cudaGetLastError();
}

}  // namespace
}  // namespace owq

extern "C" owq_status_t owq_quantize_noalloc(const uint16_t* W, const uint16_t* X, int N, int K, int T,
                                             int bits, int group, int k, uint8_t* codes, uint16_t* scales,
                                             uint16_t* zeros, int32_t* idx, uint16_t* w_weak,
                                             owq_stream_t stream) {
  using namespace owq;
  if (!W || !X || !codes || !scales || !zeros) return OWQ_ERR_NULL;
  if (k > 0 && (!idx || !w_weak)) return OWQ_ERR_NULL;
  if (bits != 3 && bits != 4) return OWQ_ERR_BITS;
  if (N < 1 || N > (1 << 20) || K < kBlockCodes || K > 65536 || K % kBlockCodes) return OWQ_ERR_SHAPE;
  if (group != K && group != 128) return OWQ_ERR_GROUP;
  if (k < 0 || k > K || k > kMaxWeak) return OWQ_ERR_SHAPE;
  if (T < 1 || T > (1 << 20)) return OWQ_ERR_SHAPE;
  if (K > OWQ_NOALLOC_MAX_K) return OWQ_ERR_SHAPE;   // beyond the static scratch
  if (!aligned16(W) || !aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros) ||
      (k > 0 && (!aligned16(idx) || !aligned16(w_weak))))
    return OWQ_ERR_ALIGN;
  int dev = -1, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return OWQ_ERR_DEVICE;
  }
  cudaError_t e = launch_quantize_static(reinterpret_cast<const __half*>(W), reinterpret_cast<const __half*>(X),
                                         N, K, T, bits, group, k, codes, reinterpret_cast<__half*>(scales),
                                         reinterpret_cast<__half*>(zeros), idx, reinterpret_cast<__half*>(w_weak),
                                         reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { cudaGetLastError(); return OWQ_ERR_CUDA; }
  return OWQ_OK;
}
