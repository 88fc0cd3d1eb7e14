// Internal declarations shared by the library's translation units (not installed).
#pragma once

#include <cstddef>
#include <cstdint>
#include <algorithm>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda.h>

#include "../../include/owq.h"

namespace owq {

constexpr uint32_t kLayerMagic = 0x4f575131u;  // "OWQ1"
constexpr int kBlockCodes = 128;               // codes per packed block (16 * bits bytes)
constexpr int kChunkCodes = 32;                // codes per chunk (bits words)
constexpr int kMaxWeak = 1024;
constexpr int kMaxBlocks = 512;                // K <= 65536
constexpr int kMaxGemvM = 16;

struct Layer {
  uint32_t magic;
  int device;
  int N, K, bits, group, G, k, k_ld;   // k_ld: row stride of w_weak (k rounded up to 16)
  uint32_t* packed;     // N x (K*bits/32) words
  __half* scales;       // N x G
  __half* zeros;        // N x G
  __half* w_weak;       // N x k_ld (zero padded)
  int32_t* idx;         // k (device)
  __half* w_weak_t;     // the weak block tile-major: [N/16 tiles][k_ld/16 slices][16 rows][16]
  __half2* sz_t;        // (scale, zero) pairs tile-major: [N/16 tiles][G][16 rows] (rows >= N: (0, 0))
  uint32_t* xfrag;      // decode scratch: up to 16 activation rows in fragment order (see owq_gemv.cu)
  // decode workspace: the partial sums a CTA publishes for a row tile shared with higher CTAs,
  // [N/16 tiles][cta_slots][16 rows][16 tokens], each a 64-bit word (fp32 value | call epoch
  // << 32); zero at pack time
  unsigned long long* part;
  // per 128-column block: its first weak slot << 16 | its weak-column count (the slots of a
  // block are consecutive, the index list being increasing); host copy, made at pack time
  uint32_t blk_weak[kMaxBlocks];
  int cta_slots;        // most CTAs below the one finishing a row tile in the decode product
  uint32_t epoch;       // decode calls made on this handle (tags the partial sums of each call)
  cudaStream_t stream;  // stream of owq_pack (used to order the release)
  float* gemm_ws;       // prefill split-K partial sums (grown on first need, outside capture)
  size_t gemm_ws_bytes;
  __half* gemm_xw;      // prefill weak activations [M][k_ld] (grown on first need, outside capture)
  size_t gemm_xw_bytes;
  void* wg_ws;          // weak-gradient scratch: gathered weak activations [M][k rounded up to
  size_t wg_ws_bytes;   // 32] fp16, then per-token-split fp32 partials (grown on first need)
  // tcgen05 GEMM tensor maps, encoded lazily on first use
  bool maps_ready;
  alignas(64) CUtensorMap map_packed;
  alignas(64) CUtensorMap map_sz;      // (scale, zero) pairs of per-group layers
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device status word (owq_device_status reads and clears it): bit 0 a bounded wait gave up,
// bit 1 a debug-bounds check failed.
int* device_status_ptr();
constexpr int kStatusTimeout = 1, kStatusBounds = 2;

// Debug-bounds build (-DOWQ_DEBUG_BOUNDS): the kernels check their data-dependent indices (the
// weak index list and the positions derived from it) before an access; a failed check sets
// kStatusBounds in the status word and the access is skipped, so an indexing fault reports as
// OWQ_ERR_BOUNDS instead of faulting.  In the default build in_range is constant true.
#ifdef OWQ_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool in_range(long long i, long long n, int* status) {
  if constexpr (kDebugBounds) {
    if (i >= 0 && i < n) return true;
    if (status) atomicOr(status, kStatusBounds);
    return false;
  } else {
    (void)i; (void)n; (void)status;
    return true;
  }
}
// Bound of a device wait when no test shortens it: about 2 s at the B200's clock.
constexpr long long kDefaultWaitLimit = 4000000000LL;

// ---- launchers (return cudaError_t of the launch) ----
cudaError_t launch_pack(const uint8_t* codes, const __half* zeros, const uint32_t* weak_mask,
                        int N, int K, int bits, int group, uint32_t* packed, cudaStream_t s);
cudaError_t launch_dequant(const Layer& L, __half* w_hat, uint8_t* codes, cudaStream_t s);
cudaError_t launch_weak_tiles(const __half* w_weak, int N, int k_ld, __half* w_weak_t, cudaStream_t s);
cudaError_t launch_sz_tiles(const __half* scales, const __half* zeros, int N, int G, __half2* sz_t, cudaStream_t s);

struct GemvProblem {
  const uint32_t* packed;
  const __half* scales;
  const __half* zeros;
  const __half* w_weak;
  const int32_t* idx;
  const __half* x;
  __half* y;
  int N, K, G, k, k_ld;
  const __half* w_weak_t;   // tile-major weak block
  const __half2* sz_t;      // tile-major (scale, zero) pairs
  uint32_t* xfrag;          // activations in fragment order (when they do not fit in shared memory)
  unsigned long long* part;  // tagged partial sums of split row tiles
  int cta_slots;             // partial-sum slots per row tile (CTAs that may share a tile, minus 1)
  uint32_t epoch;            // tag of this call's partial sums (never 0)
  uint32_t wtag;             // tag the partial sums are published under: epoch (0 only when a
                             // test injects a lost hand-off)
  int row_groups;     // 16-row tiles
  int cta_base;       // first CTA of this problem
  int ncta;           // CTAs serving this problem
  int chunk;          // (row tile, block) units per warp
  int lt_cap;         // row tiles one CTA's chunks touch (segment counters in shared memory)
};
// Decode work split: each warp of the grid (kGemvWarps per SM) takes an equal contiguous chunk
// of the (16-row tile, 128-code block) units, never fewer than kGemvMinChunk.  A CTA (at least
// kGemvMinWarps warps) then spans at least kGemvMinWarps * cmin units, so a row tile of K/128
// units meets at most gemv_cta_slots + 1 CTAs; the slots size the layer's partial-sum workspace.
constexpr int kGemvWarps = 16;
constexpr int kGemvMinWarps = 8;
constexpr int kGemvMinChunk = 4;
inline int gemv_min_chunk(int N, int K, int sm_count) {
  const long long units = (long long)((N + 15) / 16) * (K / kBlockCodes);
  const long long warps = (long long)sm_count * kGemvWarps;
  return (int)std::max<long long>(kGemvMinChunk, (units + warps - 1) / warps);
}
inline int gemv_cta_slots(int N, int K, int sm_count) {
  const int span = kGemvMinWarps * gemv_min_chunk(N, K, sm_count);
  return std::max(1, (K / kBlockCodes - 1 + span - 1) / span);
}
cudaError_t launch_gemv(const GemvProblem* probs, int count, int bits, int M, long long wait_limit,
                        cudaStream_t s);

cudaError_t launch_quantize(const __half* W, const __half* X, int N, int K, int T, int bits,
                            int group, int k, uint8_t* codes, __half* scales, __half* zeros,
                            int32_t* idx, __half* w_weak, cudaStream_t s);

// truncation-aware (step, zero) grid search per (row, group) over the dense columns
cudaError_t launch_search_params(const __half* W, int N, int K, int bits, int group, const int32_t* idx, int k,
                                 __half* scales, __half* zeros, cudaStream_t s);

// OPTQ with the weak columns last: perm (host, K entries) = dense columns ascending, then the
// weak columns ascending; scratch K*K + N*K doubles (stream-ordered)
size_t optq_scratch_bytes(int N, int K);
cudaError_t launch_optq(const __half* W, const __half* X, int N, int K, int T, int bits, int group,
                        const int* perm_host, int k, const __half* scales, const __half* zeros, double damp,
                        uint8_t* codes, __half* w_weak, cudaStream_t s);

// storage-favoured dense stream (words per row = ceil((K - k) bits / 32)) <-> full code matrix
int storage_words_per_row(int K, int bits, int k);
cudaError_t launch_storage_pack(const uint8_t* codes, int N, int K, int bits, const int32_t* idx, int k,
                                uint32_t* words, cudaStream_t s);
cudaError_t launch_storage_unpack(const uint32_t* words, int N, int K, int bits, int group, const int32_t* idx,
                                  int k, const __half* zeros, uint8_t* codes, cudaStream_t s);

// weak column tuning: dW_weak = dY^T x[:, idx] (fp32 N x k) and dX = dY W_eff (fp16 M x K)
cudaError_t launch_weak_grad(const Layer& L, const __half* x, const __half* dy, float* dw, int M,
                             cudaStream_t s);
cudaError_t launch_input_grad(Layer& L, const __half* dy, __half* dx, int M, cudaStream_t s);
// many tokens: the packed product on the 5th-generation tensor cores (weak columns left at
// exactly 0), then the weak columns dx[:, idx] = dY W_weak (overwritten)
// the tensor-memory pipeline above this many tokens (N % 8 == 0): measured on the OPT-6.7B
// shapes, 17-32 tokens run 1.4-2.4x faster there than two 16-token passes
constexpr int kIgGemmMinM = 16;
owq_status_t igemm_sm100(Layer& L, const __half* dy, __half* dx, int M, long long wait_limit, cudaStream_t s);
// inject (debug-bounds build tests): token 0 of slot 0 is stored one row of K too far, which
// the bounds check must catch
cudaError_t launch_input_grad_weak(Layer& L, const __half* dy, __half* dx, int M, bool inject, cudaStream_t s);

// Launch shape of one prefill product: tile width in tokens; K splits of every tile (fewer
// tiles than SMs; `ksteps` 128-code steps each); or a split tail: the row tiles of the last
// tail_tt token tiles split tail_sp ways over K (tail_ksteps steps each).  Host only.
struct GemmPlan {
  int tile_tokens, splits, ksteps, tail_tt, tail_sp, tail_ksteps;
};
int gemm_tile_tokens(int M);
GemmPlan gemm_plan(int N, int K, int M, int sms);

// skip_arrive: a test-injected lost arrival (one dequantisation thread per CTA skips its first
// arrival), so that the bounded waits run out
owq_status_t gemm_sm100(Layer& L, const __half* x, __half* y, int M, long long wait_limit,
                        bool skip_arrive, cudaStream_t s);

}  // namespace owq
