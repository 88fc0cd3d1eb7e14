// The storage-favoured form of the low-precision matrix and its repack into the latency layout.
//
// Pages: "Storage Methods" (appendix §2 of the OWQ paper, pp.10-11, as summarised on
// paperlayer.ai).  The latency-favoured form keeps the full N x K low-precision matrix with the
// weak columns zero-filled (b + 16 k / K bits per weight); the storage-favoured form drops the
// weak columns from it (b + (16 - b) k / K bits per weight) and needs an index remap when the
// matrix is used.  The pages give only the bit counts; the stream here is, per row, the codes of
// the K - k dense columns in column order as one LSB-first stream of `bits` bits per code
// (code p at bits [p b, p b + b)), padded with zero bits to whole uint32 words.  The kernels
// convert between that stream and the full code matrix, so a layer stored compactly is repacked
// into the latency layout once, at load time.
//
// Both kernels map a dense stream position p to its column j (or back) with the weak index list
// in shared memory: for a dense column j, p = j - #{t : idx[t] < j}; the p-th dense column is
// the fixed point of j = p + #{t : idx[t] <= j} (reached from j = p in at most k + 1 steps,
// since the count only grows and is at most k).
#include "owq_internal.cuh"

namespace owq {
namespace {

constexpr int kStoreThreads = 256;

// #{t : idx[t] < j} over a sorted list in shared memory
__device__ __forceinline__ int count_below(const int* idx, int k, int j) {
  int lo = 0, hi = k;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (idx[mid] < j) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// the p-th dense (non-weak) column
__device__ __forceinline__ int dense_col(const int* idx, int k, int p) {
  int j = p;
  #pragma unroll 1
  for (int it = 0; it <= k; ++it) {
    const int jn = p + count_below(idx, k, j + 1);   // #{idx <= j}
    if (jn == j) break;
    j = jn;
  }
  return j;
}

// is column j weak (binary search)
__device__ __forceinline__ bool is_weak(const int* idx, int k, int j) {
  const int c = count_below(idx, k, j);
  return c < k && idx[c] == j;
}

// grid (ceil(Ws / 256), rows): thread = one word w of the stream, for rows blockIdx.y,
// blockIdx.y + gridDim.y, ...
__global__ void k_storage_pack(const uint8_t* __restrict__ codes, int N, int K, int bits,
                               const int32_t* __restrict__ idx_g, int k, int Ws, uint32_t* __restrict__ words,
                               int* status) {
  __shared__ int idx[kMaxWeak];
  for (int t = threadIdx.x; t < k; t += blockDim.x) idx[t] = idx_g[t];
  __syncthreads();
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= Ws) return;
  const int nd = K - k;
  const long long b0 = 32LL * w;                      // first bit of this word
  const int p0 = (int)(b0 / bits);                    // first code touching the word
  const int p_end = min(nd, (int)((b0 + 31) / bits) + 1);
  const int j0 = p0 < p_end ? dense_col(idx, k, p0) : 0;
  for (int row = blockIdx.y; row < N; row += gridDim.y) {
    const uint8_t* c = codes + (size_t)row * K;
    uint32_t out = 0u;
    int j = j0;
    for (int p = p0; p < p_end; ++p) {
      const uint32_t v = in_range(j, K, status) ? c[j] : 0u;   // the p-th dense column
      const long long o = (long long)p * bits - b0;   // bit offset of code p in this word (may be < 0)
      out |= o >= 0 ? (v << o) : (v >> -o);
      ++j;                                            // the next dense column
      while (j < K && is_weak(idx, k, j)) ++j;
    }
    words[(size_t)row * Ws + w] = out;
  }
}

// grid (ceil(K / 256), rows): thread = one column j, for rows blockIdx.y, blockIdx.y +
// gridDim.y, ...
__global__ void k_storage_unpack(const uint32_t* __restrict__ words, int N, int K, int bits, int group,
                                 const int32_t* __restrict__ idx_g, int k, int Ws,
                                 const __half* __restrict__ zeros, uint8_t* __restrict__ codes, int* status) {
  __shared__ int idx[kMaxWeak];
  for (int t = threadIdx.x; t < k; t += blockDim.x) idx[t] = idx_g[t];
  __syncthreads();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const int below = count_below(idx, k, j);
  const bool weak = below < k && idx[below] == j;
  const long long bit = (long long)(j - below) * bits;
  const int w = (int)(bit >> 5), o = (int)(bit & 31);
  const int G = K / group;
  for (int row = blockIdx.y; row < N; row += gridDim.y) {
    uint32_t v;
    if (weak) {
      // a weak column holds its group's zero point (the zero-filled code of the latency layout)
      v = (uint32_t)__half2float(zeros[(size_t)row * G + j / group]);
    } else {
      const uint32_t* r = words + (size_t)row * Ws;
      v = in_range(w, Ws, status) ? r[w] >> o : 0u;   // the column's position in the dense stream
      if (o + bits > 32 && in_range(w + 1, Ws, status)) v |= r[w + 1] << (32 - o);
      v &= (1u << bits) - 1u;
    }
    codes[(size_t)row * K + j] = (uint8_t)v;
  }
}

}  // namespace

int storage_words_per_row(int K, int bits, int k) { return ((K - k) * bits + 31) / 32; }

cudaError_t launch_storage_pack(const uint8_t* codes, int N, int K, int bits, const int32_t* idx, int k,
                                uint32_t* words, cudaStream_t s) {
  const int Ws = storage_words_per_row(K, bits, k);
  if (Ws == 0) return cudaSuccess;
  dim3 grid((Ws + kStoreThreads - 1) / kStoreThreads, std::min(N, 65535));
  k_storage_pack<<<grid, kStoreThreads, 0, s>>>(codes, N, K, bits, idx, k, Ws, words, device_status_ptr());
  return cudaGetLastError();
}

cudaError_t launch_storage_unpack(const uint32_t* words, int N, int K, int bits, int group, const int32_t* idx,
                                  int k, const __half* zeros, uint8_t* codes, cudaStream_t s) {
  const int Ws = storage_words_per_row(K, bits, k);
  dim3 grid((K + kStoreThreads - 1) / kStoreThreads, std::min(N, 65535));
  k_storage_unpack<<<grid, kStoreThreads, 0, s>>>(words, N, K, bits, group, idx, k, Ws, zeros, codes,
                                                 device_status_ptr());
  return cudaGetLastError();
}

}  // namespace owq
