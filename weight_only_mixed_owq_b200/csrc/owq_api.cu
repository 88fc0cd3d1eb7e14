// C ABI of the library (declared in include/owq.h): argument validation, layer handles,
// launches.  Every argument is validated on the host before anything is launched.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>
#include <vector>

#include "owq_internal.cuh"

namespace owq {

__device__ int g_device_status;

int* device_status_ptr() {
  int* p = nullptr;
  if (cudaGetSymbolAddress((void**)&p, g_device_status) != cudaSuccess) return nullptr;
  return p;
}

namespace {

std::mutex g_mu;
std::unordered_set<Layer*>& registry() {
  static std::unordered_set<Layer*> s;
  return s;
}

Layer* lookup(owq_layer_t h) {
  Layer* L = reinterpret_cast<Layer*>(h);
  if (!L) return nullptr;
  std::lock_guard<std::mutex> g(g_mu);
  return registry().count(L) ? L : nullptr;
}

owq_status_t check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return OWQ_ERR_DEVICE; }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return OWQ_ERR_DEVICE;
  }
  return major == 10 ? OWQ_OK : OWQ_ERR_DEVICE;
}

owq_status_t check_shape(int N, int K, int bits, int group, int k) {
  if (bits != 3 && bits != 4) return OWQ_ERR_BITS;
  if (N < 1 || N > (1 << 20) || K < kBlockCodes || K > 65536 || K % kBlockCodes) return OWQ_ERR_SHAPE;
  if (group != K && group != 128) return OWQ_ERR_GROUP;
  if (k < 0 || k > K || k > kMaxWeak) return OWQ_ERR_SHAPE;
  return OWQ_OK;
}

// idx (k device ints) copied to the host on `s` (synchronised) and checked: strictly
// ascending in [0, K)
owq_status_t check_idx_on_host(const int32_t* idx, int k, int K, cudaStream_t s) {
  if (k == 0) return OWQ_OK;
  std::vector<int32_t> h(k);
  if (cudaMemcpyAsync(h.data(), idx, sizeof(int32_t) * k, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return OWQ_ERR_CUDA;
  }
  for (int t = 0; t < k; ++t) {
    if (h[t] < 0 || h[t] >= K) return OWQ_ERR_INDEX;
    if (t > 0 && h[t] <= h[t - 1]) return OWQ_ERR_INDEX;
  }
  return OWQ_OK;
}

owq_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return OWQ_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? OWQ_ERR_NOMEM : OWQ_ERR_CUDA;
}

void release(Layer* L) {
  if (!L) return;
  cudaFree(L->packed);
  cudaFree(L->scales);
  cudaFree(L->zeros);
  cudaFree(L->w_weak);
  cudaFree(L->idx);
  cudaFree(L->w_weak_t);
  cudaFree(L->sz_t);
  cudaFree(L->xfrag);
  cudaFree(L->gemm_ws);
  cudaFree(L->gemm_xw);
  cudaFree(L->wg_ws);
  cudaFree(L->part);
  L->magic = 0;
  delete L;
}

}  // namespace
}  // namespace owq

using namespace owq;

extern "C" {

const char* owq_status_string(owq_status_t s) {
  switch (s) {
    case OWQ_OK: return "OWQ_OK";
    case OWQ_ERR_NULL: return "OWQ_ERR_NULL: a required pointer is NULL";
    case OWQ_ERR_SHAPE: return "OWQ_ERR_SHAPE: N, K, M, T or k out of range";
    case OWQ_ERR_BITS: return "OWQ_ERR_BITS: bits must be 3 or 4";
    case OWQ_ERR_GROUP: return "OWQ_ERR_GROUP: group must be K or 128";
    case OWQ_ERR_INDEX: return "OWQ_ERR_INDEX: idx must be strictly ascending in [0, K)";
    case OWQ_ERR_ALIGN: return "OWQ_ERR_ALIGN: device pointers must be 16-byte aligned";
    case OWQ_ERR_CUDA: return "OWQ_ERR_CUDA: a CUDA call or launch failed";
    case OWQ_ERR_TIMEOUT: return "OWQ_ERR_TIMEOUT: a bounded device wait gave up";
    case OWQ_ERR_NOMEM: return "OWQ_ERR_NOMEM: allocation failed";
    case OWQ_ERR_HANDLE: return "OWQ_ERR_HANDLE: not a live layer handle";
    case OWQ_ERR_DEVICE: return "OWQ_ERR_DEVICE: no sm_100 CUDA device";
    case OWQ_ERR_ARG: return "OWQ_ERR_ARG: argument outside its documented set";
    case OWQ_ERR_BOUNDS: return "OWQ_ERR_BOUNDS: a debug-bounds index check failed on the device";
    default: return "OWQ: unknown status";
  }
}

const char* owq_version(void) { return kDebugBounds ? "0.1.0+debug-bounds" : "0.1.0"; }

owq_status_t owq_quantize(const uint16_t* W, const uint16_t* X, int N, int K, int T, int bits,
                          int group, int k, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                          int32_t* idx, uint16_t* w_weak, owq_stream_t stream) {
  if (!W || !X || !codes || !scales || !zeros) return OWQ_ERR_NULL;
  if (k > 0 && (!idx || !w_weak)) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (T < 1 || T > (1 << 20)) return OWQ_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros) ||
      (k > 0 && (!aligned16(idx) || !aligned16(w_weak))))
    return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  return cuda_status(launch_quantize(reinterpret_cast<const __half*>(W), reinterpret_cast<const __half*>(X),
                                     N, K, T, bits, group, k, codes, reinterpret_cast<__half*>(scales),
                                     reinterpret_cast<__half*>(zeros), idx, reinterpret_cast<__half*>(w_weak),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

owq_status_t owq_pack(const uint8_t* codes, int N, int K, int bits, int group, const uint16_t* scales,
                      const uint16_t* zeros, const int32_t* idx, int k, const uint16_t* w_weak,
                      owq_stream_t stream, owq_layer_t* out) {
  if (!out) return OWQ_ERR_NULL;
  *out = nullptr;
  if (!codes || !scales || !zeros) return OWQ_ERR_NULL;
  if (k > 0 && (!idx || !w_weak)) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(zeros) ||
      (k > 0 && (!aligned16(idx) || !aligned16(w_weak))))
    return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // idx: copy to the host and validate before anything is allocated or launched
  std::vector<int32_t> hidx(k);
  if (k > 0) {
    if (cudaMemcpyAsync(hidx.data(), idx, sizeof(int32_t) * k, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return OWQ_ERR_CUDA;
    }
    for (int t = 0; t < k; ++t) {
      if (hidx[t] < 0 || hidx[t] >= K) return OWQ_ERR_INDEX;
      if (t > 0 && hidx[t] <= hidx[t - 1]) return OWQ_ERR_INDEX;
    }
  }

  Layer* L = new (std::nothrow) Layer();
  if (!L) return OWQ_ERR_NOMEM;
  L->magic = kLayerMagic;
  cudaGetDevice(&L->device);
  L->N = N; L->K = K; L->bits = bits; L->group = group; L->G = K / group; L->k = k;
  L->k_ld = std::max(16, (k + 15) & ~15);   // 16-wide tensor-core k slices
  L->stream = s;
  L->maps_ready = false;
  const size_t packed_bytes = (size_t)((N + 15) & ~15) * K * bits / 8;   // 16-row tiles
  const size_t sz_bytes = (size_t)N * L->G * sizeof(__half);
  const size_t weak_bytes = (size_t)N * L->k_ld * sizeof(__half);

  cudaError_t e = cudaSuccess;
  auto alloc = [&](void** p, size_t n) { if (e == cudaSuccess) e = cudaMalloc(p, std::max<size_t>(n, 16)); };
  alloc((void**)&L->packed, packed_bytes);
  alloc((void**)&L->scales, sz_bytes);
  alloc((void**)&L->zeros, sz_bytes);
  alloc((void**)&L->w_weak, weak_bytes);
  alloc((void**)&L->idx, sizeof(int32_t) * std::max(k, 1));
  const size_t RT = (size_t)(N + 15) / 16;
  const size_t weak_t_bytes = RT * 16 * L->k_ld * sizeof(__half);
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, L->device) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  L->cta_slots = gemv_cta_slots(N, K, sms);
  const size_t part_bytes = RT * L->cta_slots * 16 * 16 * sizeof(unsigned long long);
  L->epoch = 0;
  alloc((void**)&L->w_weak_t, weak_t_bytes);
  alloc((void**)&L->sz_t, RT * L->G * 16 * sizeof(__half2));
  alloc((void**)&L->xfrag, (size_t)16 * K * sizeof(__half));
  alloc((void**)&L->part, part_bytes);
  uint32_t* mask_dev = nullptr;
  alloc((void**)&mask_dev, sizeof(uint32_t) * (K / 32));
  if (e != cudaSuccess) { cudaFree(mask_dev); release(L); return cuda_status(e); }

  // host-side tables: weak bitmask per 32-code chunk; first weak slot and count per block
  std::vector<uint32_t> mask(K / 32, 0u);
  for (int t = 0; t < k; ++t) mask[hidx[t] / 32] |= 1u << (hidx[t] % 32);
  for (int b = 0; b < K / kBlockCodes; ++b) L->blk_weak[b] = 0u;
  for (int t = k - 1; t >= 0; --t) {   // descending: the first slot of each block wins
    const int b = hidx[t] / kBlockCodes;
    L->blk_weak[b] = ((uint32_t)t << 16) | ((L->blk_weak[b] & 0xFFFFu) + 1u);
  }

  if (e == cudaSuccess) e = cudaMemsetAsync(L->packed, 0, packed_bytes, s);   // padding rows of the last tile
  if (e == cudaSuccess) e = cudaMemcpyAsync(L->scales, scales, sz_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(L->zeros, zeros, sz_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(L->w_weak, 0, weak_bytes, s);
  if (e == cudaSuccess && k > 0)
    e = cudaMemcpy2DAsync(L->w_weak, (size_t)L->k_ld * sizeof(__half), w_weak, (size_t)k * sizeof(__half),
                          (size_t)k * sizeof(__half), N, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && k > 0) e = cudaMemcpyAsync(L->idx, idx, sizeof(int32_t) * k, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(mask_dev, mask.data(), sizeof(uint32_t) * (K / 32), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(L->part, 0, part_bytes, s);   // epoch 0: never a live tag
  if (e == cudaSuccess)
    e = launch_pack(codes, reinterpret_cast<const __half*>(zeros), mask_dev, N, K, bits, group, L->packed, s);
  if (e == cudaSuccess) e = launch_weak_tiles(L->w_weak, N, L->k_ld, L->w_weak_t, s);
  if (e == cudaSuccess) e = launch_sz_tiles(L->scales, L->zeros, N, L->G, L->sz_t, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // host tables above must outlive the copies
  cudaFree(mask_dev);
  if (e != cudaSuccess) { release(L); return cuda_status(e); }
  {
    std::lock_guard<std::mutex> g(g_mu);
    registry().insert(L);
  }
  *out = reinterpret_cast<owq_layer_t>(L);
  return OWQ_OK;
}

owq_status_t owq_search_params(const uint16_t* W, int N, int K, int bits, int group, const int32_t* idx, int k,
                               uint16_t* scales, uint16_t* zeros, owq_stream_t stream) {
  if (!W || !scales || !zeros || (k > 0 && !idx)) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (!aligned16(W) || !aligned16(scales) || !aligned16(zeros) || (k > 0 && !aligned16(idx))) return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = check_idx_on_host(idx, k, K, s))) return st;
  return cuda_status(launch_search_params(reinterpret_cast<const __half*>(W), N, K, bits, group, idx, k,
                                          reinterpret_cast<__half*>(scales), reinterpret_cast<__half*>(zeros), s));
}

owq_status_t owq_optq(const uint16_t* W, const uint16_t* X, int N, int K, int T, int bits, int group,
                      const int32_t* idx, int k, const uint16_t* scales, const uint16_t* zeros, double damp,
                      uint8_t* codes, uint16_t* w_weak, owq_stream_t stream) {
  if (!W || !X || !scales || !zeros || !codes || (k > 0 && (!idx || !w_weak))) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (T < 1 || T > (1 << 20)) return OWQ_ERR_SHAPE;
  if (!(damp >= 0.0) || !(damp <= 1e6)) return OWQ_ERR_ARG;
  if (!aligned16(W) || !aligned16(X) || !aligned16(scales) || !aligned16(zeros) || !aligned16(codes) ||
      (k > 0 && (!aligned16(idx) || !aligned16(w_weak))))
    return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<int32_t> h(k);
  if (k > 0) {
    if (cudaMemcpyAsync(h.data(), idx, sizeof(int32_t) * k, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return OWQ_ERR_CUDA;
    }
    for (int t = 0; t < k; ++t) {
      if (h[t] < 0 || h[t] >= K) return OWQ_ERR_INDEX;
      if (t > 0 && h[t] <= h[t - 1]) return OWQ_ERR_INDEX;
    }
  }
  // the order of the columns: the dense ones ascending, then the weak ones ascending
  std::vector<int> perm;
  perm.reserve(K);
  std::vector<char> weak(K, 0);
  for (int t = 0; t < k; ++t) weak[h[t]] = 1;
  for (int j = 0; j < K; ++j)
    if (!weak[j]) perm.push_back(j);
  for (int t = 0; t < k; ++t) perm.push_back(h[t]);
  return cuda_status(launch_optq(reinterpret_cast<const __half*>(W), reinterpret_cast<const __half*>(X), N, K, T,
                                 bits, group, perm.data(), k, reinterpret_cast<const __half*>(scales),
                                 reinterpret_cast<const __half*>(zeros), damp, codes,
                                 reinterpret_cast<__half*>(w_weak), s));
}

owq_status_t owq_quantize_optq(const uint16_t* W, const uint16_t* X, int N, int K, int T, int bits, int group,
                               int k, double damp, uint8_t* codes, uint16_t* scales, uint16_t* zeros, int32_t* idx,
                               uint16_t* w_weak, owq_stream_t stream) {
  if (!(damp >= 0.0) || !(damp <= 1e6)) return OWQ_ERR_ARG;
  // 1. the weak columns (the selection of owq_quantize; its RTN outputs are overwritten below)
  owq_status_t st = owq_quantize(W, X, N, K, T, bits, group, k, codes, scales, zeros, idx, w_weak, stream);
  if (st) return st;
  // 2. the (step, zero) search over the dense columns, 3. OPTQ with the weak columns last
  st = owq_search_params(W, N, K, bits, group, k > 0 ? idx : nullptr, k, scales, zeros, stream);
  if (st) return st;
  return owq_optq(W, X, N, K, T, bits, group, k > 0 ? idx : nullptr, k, scales, zeros, damp, codes,
                  k > 0 ? w_weak : nullptr, stream);
}

owq_status_t owq_storage_words(int K, int bits, int k, int* words_per_row) {
  if (!words_per_row) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(1, K, bits, K, k);
  if (st) return st;
  *words_per_row = storage_words_per_row(K, bits, k);
  return OWQ_OK;
}

owq_status_t owq_storage_pack(const uint8_t* codes, int N, int K, int bits, const int32_t* idx, int k,
                              uint32_t* words, owq_stream_t stream) {
  if (!codes || !words || (k > 0 && !idx)) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, K, k);
  if (st) return st;
  if (!aligned16(codes) || !aligned16(words) || (k > 0 && !aligned16(idx))) return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = check_idx_on_host(idx, k, K, s))) return st;
  return cuda_status(launch_storage_pack(codes, N, K, bits, idx, k, words, s));
}

owq_status_t owq_storage_unpack(const uint32_t* words, int N, int K, int bits, int group, const int32_t* idx,
                                int k, const uint16_t* zeros, uint8_t* codes, owq_stream_t stream) {
  if (!words || !zeros || !codes || (k > 0 && !idx)) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (!aligned16(words) || !aligned16(zeros) || !aligned16(codes) || (k > 0 && !aligned16(idx))) return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = check_idx_on_host(idx, k, K, s))) return st;
  return cuda_status(launch_storage_unpack(words, N, K, bits, group, idx, k,
                                           reinterpret_cast<const __half*>(zeros), codes, s));
}

owq_status_t owq_pack_storage(const uint32_t* words, int N, int K, int bits, int group, const uint16_t* scales,
                              const uint16_t* zeros, const int32_t* idx, int k, const uint16_t* w_weak,
                              owq_stream_t stream, owq_layer_t* out) {
  if (!out) return OWQ_ERR_NULL;
  *out = nullptr;
  if (!words || !scales || !zeros || (k > 0 && (!idx || !w_weak))) return OWQ_ERR_NULL;
  owq_status_t st = check_shape(N, K, bits, group, k);
  if (st) return st;
  if (!aligned16(words) || !aligned16(scales) || !aligned16(zeros) ||
      (k > 0 && (!aligned16(idx) || !aligned16(w_weak))))
    return OWQ_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = check_idx_on_host(idx, k, K, s))) return st;
  // the full code matrix, for the time of the repack
  uint8_t* codes = nullptr;
  if (cudaMalloc(&codes, (size_t)N * K) != cudaSuccess) {
    cudaGetLastError();
    return OWQ_ERR_NOMEM;
  }
  cudaError_t e = launch_storage_unpack(words, N, K, bits, group, idx, k, reinterpret_cast<const __half*>(zeros),
                                        codes, s);
  st = e == cudaSuccess ? owq_pack(codes, N, K, bits, group, scales, zeros, idx, k, w_weak, stream, out)
                        : cuda_status(e);
  if (cudaStreamSynchronize(s) != cudaSuccess && st == OWQ_OK) st = OWQ_ERR_CUDA;
  cudaGetLastError();
  cudaFree(codes);
  if (st != OWQ_OK && *out) {
    owq_layer_free(*out);
    *out = nullptr;
  }
  return st;
}

// one armed test failure (owq_debug_inject), taken by the next call of its kind
static int g_inject = OWQ_INJECT_NONE;
static long long g_inject_wait = kDefaultWaitLimit;

// wait bound of this call; true if the armed failure is of kind `what` (then disarmed)
static bool take_inject(int what, long long* wait_limit) {
  *wait_limit = kDefaultWaitLimit;
  if (g_inject != what) return false;
  *wait_limit = g_inject_wait;
  g_inject = OWQ_INJECT_NONE;
  return true;
}

owq_status_t owq_debug_inject(int what, long long wait_cycles) {
  if (what == OWQ_INJECT_NONE) { g_inject = what; return OWQ_OK; }
  if (what == OWQ_INJECT_BOUNDS) {   // the debug-bounds build only
    if (!kDebugBounds) return OWQ_ERR_ARG;
    g_inject = what;
    return OWQ_OK;
  }
  if ((what != OWQ_INJECT_GEMV_TAG && what != OWQ_INJECT_GEMM_ARRIVE) || wait_cycles < 1) return OWQ_ERR_ARG;
  g_inject = what;
  g_inject_wait = wait_cycles;
  return OWQ_OK;
}

static owq_status_t make_problem(Layer* L, const uint16_t* x, uint16_t* y, GemvProblem* P) {
  if (!x || !y) return OWQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(y)) return OWQ_ERR_ALIGN;
  P->packed = L->packed;
  P->scales = L->scales;
  P->zeros = L->zeros;
  P->w_weak = L->w_weak;
  P->idx = L->idx;
  P->x = reinterpret_cast<const __half*>(x);
  P->y = reinterpret_cast<__half*>(y);
  P->N = L->N; P->K = L->K; P->G = L->G; P->k = L->k; P->k_ld = L->k_ld;
  P->w_weak_t = L->w_weak_t; P->sz_t = L->sz_t; P->xfrag = L->xfrag; P->part = L->part; P->cta_slots = L->cta_slots;
  if (++L->epoch == 0) ++L->epoch;   // 0 marks the zeroed workspace
  P->epoch = L->epoch;
  P->wtag = L->epoch;
  P->row_groups = 0; P->cta_base = 0; P->ncta = 0; P->chunk = 0; P->lt_cap = 0;
  return OWQ_OK;
}

owq_status_t owq_gemv(owq_layer_t layer, const uint16_t* x, uint16_t* y, int M, owq_stream_t stream) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (M < 1 || M > kMaxGemvM) return OWQ_ERR_SHAPE;
  GemvProblem P;
  owq_status_t st = make_problem(L, x, y, &P);
  if (st) return st;
  long long wl;
  if (take_inject(OWQ_INJECT_GEMV_TAG, &wl)) P.wtag = 0;
  return cuda_status(launch_gemv(&P, 1, L->bits, M, wl, reinterpret_cast<cudaStream_t>(stream)));
}

owq_status_t owq_gemv_multi(const owq_layer_t* layers, const uint16_t* const* xs, uint16_t* const* ys,
                            int count, int M, owq_stream_t stream) {
  if (!layers || !xs || !ys) return OWQ_ERR_NULL;
  if (count < 1 || count > 16 || M < 1 || M > kMaxGemvM) return OWQ_ERR_SHAPE;
  GemvProblem P[16];
  int bits = 0;
  for (int q = 0; q < count; ++q) {
    Layer* L = lookup(layers[q]);
    if (!L) return OWQ_ERR_HANDLE;
    for (int j = 0; j < q; ++j)   // each layer's split-tile workspace serves one product
      if (layers[j] == layers[q]) return OWQ_ERR_HANDLE;
    if (q == 0) bits = L->bits;
    else if (L->bits != bits) return OWQ_ERR_BITS;
    owq_status_t st = make_problem(L, xs[q], ys[q], &P[q]);
    if (st) return st;
  }
  long long wl;
  if (take_inject(OWQ_INJECT_GEMV_TAG, &wl))
    for (int q = 0; q < count; ++q) P[q].wtag = 0;
  return cuda_status(launch_gemv(P, count, bits, M, wl, reinterpret_cast<cudaStream_t>(stream)));
}

owq_status_t owq_gemm(owq_layer_t layer, const uint16_t* x, uint16_t* y, int M, owq_stream_t stream) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (M < 1 || M > 65536) return OWQ_ERR_SHAPE;
  if (!x || !y) return OWQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(y)) return OWQ_ERR_ALIGN;
  long long wl;
  const bool skip = take_inject(OWQ_INJECT_GEMM_ARRIVE, &wl);
  return gemm_sm100(*L, reinterpret_cast<const __half*>(x), reinterpret_cast<__half*>(y), M, wl, skip,
                    reinterpret_cast<cudaStream_t>(stream));
}

owq_status_t owq_gemm_plan(int N, int K, int M, int sms, int plan[4]) {
  if (!plan) return OWQ_ERR_NULL;
  if (N < 1 || N > (1 << 20) || K < kBlockCodes || K > 65536 || K % kBlockCodes || M < 1 || M > 65536)
    return OWQ_ERR_SHAPE;
  if (sms < 1) return OWQ_ERR_ARG;
  const GemmPlan g = gemm_plan(N, K, M, sms);
  plan[0] = g.tile_tokens;
  plan[1] = g.splits;
  plan[2] = g.tail_tt;
  plan[3] = g.tail_sp;
  return OWQ_OK;
}

owq_status_t owq_weak_grad(owq_layer_t layer, const uint16_t* x, const uint16_t* dy, float* dw_weak,
                           int M, owq_stream_t stream) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (M < 1 || M > 65536) return OWQ_ERR_SHAPE;
  if (!x || !dy || (L->k > 0 && !dw_weak)) return OWQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(dy) || (dw_weak && !aligned16(dw_weak))) return OWQ_ERR_ALIGN;
  return cuda_status(launch_weak_grad(*L, reinterpret_cast<const __half*>(x),
                                      reinterpret_cast<const __half*>(dy), dw_weak, M,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

owq_status_t owq_input_grad(owq_layer_t layer, const uint16_t* dy, uint16_t* dx, int M,
                            owq_stream_t stream) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (M < 1 || M > 65536) return OWQ_ERR_SHAPE;
  if (!dy || !dx) return OWQ_ERR_NULL;
  if (!aligned16(dy) || !aligned16(dx)) return OWQ_ERR_ALIGN;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const __half* dyh = reinterpret_cast<const __half*>(dy);
  __half* dxh = reinterpret_cast<__half*>(dx);
  if (M > kIgGemmMinM && L->N % 8 == 0) {   // dY rows must be 16-byte strided for its tensor map
    const owq_status_t st = igemm_sm100(*L, dyh, dxh, M, kDefaultWaitLimit, s);
    if (st) return st;
    long long wl;
    const bool inject = L->k > 0 && take_inject(OWQ_INJECT_BOUNDS, &wl);
    return cuda_status(launch_input_grad_weak(*L, dyh, dxh, M, inject, s));
  }
  return cuda_status(launch_input_grad(*L, dyh, dxh, M, s));
}

owq_status_t owq_dequant(owq_layer_t layer, uint16_t* w_hat, uint8_t* codes, owq_stream_t stream) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (!w_hat) return OWQ_ERR_NULL;
  if (!aligned16(w_hat) || (codes && !aligned16(codes))) return OWQ_ERR_ALIGN;
  return cuda_status(launch_dequant(*L, reinterpret_cast<__half*>(w_hat), codes,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

owq_status_t owq_layer_info(owq_layer_t layer, int* N, int* K, int* bits, int* group, int* k) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (N) *N = L->N;
  if (K) *K = L->K;
  if (bits) *bits = L->bits;
  if (group) *group = L->group;
  if (k) *k = L->k;
  return OWQ_OK;
}

owq_status_t owq_layer_bytes(owq_layer_t layer, size_t* packed, size_t* scales_zeros, size_t* weak,
                             size_t* index) {
  Layer* L = lookup(layer);
  if (!L) return OWQ_ERR_HANDLE;
  if (packed) *packed = (size_t)L->N * L->K * L->bits / 8;
  if (scales_zeros) *scales_zeros = (size_t)L->N * L->G * 4;
  if (weak) *weak = (size_t)L->N * L->k * 2;
  if (index) *index = (size_t)L->k * 4;
  return OWQ_OK;
}

owq_status_t owq_layer_free(owq_layer_t layer) {
  if (!layer) return OWQ_OK;
  Layer* L = reinterpret_cast<Layer*>(layer);
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!registry().erase(L)) return OWQ_ERR_HANDLE;
  }
  release(L);
  return OWQ_OK;
}

owq_status_t owq_device_status(void) {
  owq_status_t st = check_device();
  if (st) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return OWQ_ERR_CUDA; }
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) { cudaGetLastError(); return OWQ_ERR_CUDA; }
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) { cudaGetLastError(); return OWQ_ERR_CUDA; }
  return (v & kStatusBounds) ? OWQ_ERR_BOUNDS : v ? OWQ_ERR_TIMEOUT : OWQ_OK;
}

}  // extern "C"
