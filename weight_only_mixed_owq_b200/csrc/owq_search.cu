// Truncation-aware 2-D grid search of the quantisation parameters (step size, zero point) per
// (output row, group).
//
// Pages: "Low-precision quantization" (paper "Quantization Configuration Search", pp.4-5, as
// summarised on paperlayer.ai): before OPTQ, OWQ searches a grid over the step size and the zero
// point with nearest rounding and truncation (clamping to the code range), so that the range may
// shrink below min-max when that lowers the reconstruction error.  The pages give no grid; the
// reading taken: step = fp16_rn((mx - mn) * alpha / (2^b - 1)) for the min-max range of the
// group's dense columns (always containing 0; [-1, 1] when it is a single point) and alpha in
// {1.00, 0.98, ..., 0.50}; zero point = every integer in [0, 2^b - 1]; error = sum over the
// group's dense columns, ascending, of (w - fp16_rn(s (q - z)))^2 in fp64 (each square rounded
// before it is added), q = clamp(rint(w / s) + z, 0, 2^b - 1) in fp32; the first minimum in
// the order (alpha descending, z ascending) wins.  Weak columns take no part.
//
// One CTA per (row, group); one thread per (alpha, z) candidate, each summing its own error in
// column order (so the sums are the same operations in the same order as the definition); then
// a lexicographic (error, candidate) minimum over the CTA.
#include "owq_internal.cuh"

namespace owq {
namespace {

constexpr int kAlphas = 26;
constexpr int kSearchThreads = kAlphas * 16;   // candidates of 4-bit codes (3-bit: 208 used)

struct SearchArgs {
  const __half* W;
  const int32_t* idx;
  __half* scales;
  __half* zeros;
  int N, K, bits, group, k;
  float alpha[kAlphas];
};

__global__ void __launch_bounds__(kSearchThreads)
k_search_params(const __grid_constant__ SearchArgs a) {
  extern __shared__ uint32_t weak_bits[];        // one bit per column of the group
  __shared__ float red_mn[kSearchThreads / 32], red_mx[kSearchThreads / 32];
  __shared__ double red_e[kSearchThreads / 32];
  __shared__ int red_c[kSearchThreads / 32];
  const int G = a.K / a.group;
  const int row = blockIdx.x / G, gi = blockIdx.x % G;
  const int g0 = gi * a.group;
  const int nw = (a.group + 31) / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) weak_bits[i] = 0u;
  __syncthreads();
  for (int t = threadIdx.x; t < a.k; t += blockDim.x) {
    const int j = a.idx[t] - g0;
    if (j >= 0 && j < a.group) atomicOr(&weak_bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  const __half* w = a.W + (size_t)row * a.K + g0;
  auto weak = [&](int j) { return (weak_bits[j >> 5] >> (j & 31)) & 1u; };

  // min-max range of the dense columns, always containing 0 (exact in fp32)
  float mn = 0.f, mx = 0.f;
  for (int j = threadIdx.x; j < a.group; j += blockDim.x)
    if (!weak(j)) {
      const float v = __half2float(w[j]);
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
  #pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) { red_mn[warp] = mn; red_mx[warp] = mx; }
  __syncthreads();
  mn = red_mn[0];
  mx = red_mx[0];
  for (int i = 1; i < (int)blockDim.x / 32; ++i) { mn = fminf(mn, red_mn[i]); mx = fmaxf(mx, red_mx[i]); }
  if (mn == mx) { mn = -1.f; mx = 1.f; }

  // this thread's candidate
  const int qmax = (1 << a.bits) - 1;
  const int nc = kAlphas * (qmax + 1);
  const int c = threadIdx.x;
  double err = __longlong_as_double(0x7ff0000000000000LL);   // +inf: not a candidate
  __half s16 = __float2half_rn(0.f);
  if (c < nc) {
    const int ai = c / (qmax + 1), z = c % (qmax + 1);
    s16 = __float2half_rn(__fdiv_rn(__fmul_rn(__fsub_rn(mx, mn), a.alpha[ai]), (float)qmax));
    const float s32 = __half2float(s16);
    if (s32 != 0.f) {
      const float zf = (float)z, qf = (float)qmax;
      double acc = 0.0;
      #pragma unroll 4
      for (int j = 0; j < a.group; ++j) {
        if (weak(j)) continue;
        const float v = __half2float(w[j]);
        const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(v, s32)), zf), 0.f), qf);
        const float wh = __half2float(__float2half_rn(__fmul_rn(s32, __fsub_rn(q, zf))));
        const double e = __dsub_rn((double)v, (double)wh);
        acc = __dadd_rn(acc, __dmul_rn(e, e));
      }
      err = acc;
    }
  }
  // first minimum in candidate order: smallest error, then smallest index
  int best = c;
  #pragma unroll
  for (int o = 16; o; o >>= 1) {
    const double e2 = __shfl_xor_sync(0xffffffffu, err, o);
    const int c2 = __shfl_xor_sync(0xffffffffu, best, o);
    if (e2 < err || (e2 == err && c2 < best)) { err = e2; best = c2; }
  }
  if (lane == 0) { red_e[warp] = err; red_c[warp] = best; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double e = red_e[0];
    int b = red_c[0];
    for (int i = 1; i < (int)blockDim.x / 32; ++i)
      if (red_e[i] < e || (red_e[i] == e && red_c[i] < b)) { e = red_e[i]; b = red_c[i]; }
    __half s_out, z_out;
    if (e == __longlong_as_double(0x7ff0000000000000LL)) {
      // every step rounded to 0 in fp16 (a range below fp16 resolution): fall back to [-1, 1]
      s_out = __float2half_rn(__fdiv_rn(2.f, (float)qmax));
      z_out = __float2half_rn((float)((qmax + 1) / 2));
    } else {
      const int ai = b / (qmax + 1), z = b % (qmax + 1);
      s_out = __float2half_rn(__fdiv_rn(__fmul_rn(__fsub_rn(mx, mn), a.alpha[ai]), (float)qmax));
      z_out = __float2half_rn((float)z);
    }
    a.scales[(size_t)row * G + gi] = s_out;
    a.zeros[(size_t)row * G + gi] = z_out;
  }
}

}  // namespace

cudaError_t launch_search_params(const __half* W, int N, int K, int bits, int group, const int32_t* idx, int k,
                                 __half* scales, __half* zeros, cudaStream_t s) {
  SearchArgs a;
  a.W = W; a.idx = idx; a.scales = scales; a.zeros = zeros;
  a.N = N; a.K = K; a.bits = bits; a.group = group; a.k = k;
  for (int i = 0; i < kAlphas; ++i) a.alpha[i] = (float)(1.0 - 0.02 * i);   // 1.00, 0.98, ..., 0.50
  const size_t smem = (size_t)((group + 31) / 32) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_search_params, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const long long ctas = (long long)N * (K / group);
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  k_search_params<<<(unsigned)ctas, kSearchThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace owq
