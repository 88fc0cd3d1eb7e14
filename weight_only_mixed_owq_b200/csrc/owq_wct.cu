// Weak column tuning (WCT) kernels: the two products a frozen OWQ layer needs in a backward
// pass when only its fp16 weak columns are trained ("PEFT with Weak Column Tuning", p.5 of the
// OWQ paper as summarised on paperlayer.ai; "WCT-based fine-tuning", p.7).
//
//   weak-block gradient   dW_weak[i, t] = sum_m dY[m, i] x[m, idx[t]]          (fp32 N x k)
//   input gradient        dX[m, j]      = sum_i dY[m, i] W_eff[i, j]            (fp16 M x K)
//
// where W_eff is the dequantised matrix fp16_rn(s (q - z)) with the weak columns' fp16 values
// in place of their zero-filled codes.  Both accumulate in fp32.
#include "owq_internal.cuh"
#include "owq_format.cuh"
#include "owq_sm100.cuh"

namespace owq {
namespace {
using namespace sm100;

// ---------------------------------------------------------------- weak-block gradient
// A CTA computes a 32-row x 32-weak-column tile of dW_weak; its 256 threads own one weak column
// and four rows each.  Tokens are staged 32 at a time: dY rows (coalesced along the output
// rows) and the gathered activation columns x[:, idx[t]].
constexpr int kWgRows = 32, kWgCols = 32, kWgTok = 32, kWgThreads = 256;

__global__ void __launch_bounds__(kWgThreads)
k_weak_grad(const __half* __restrict__ x, const __half* __restrict__ dy,
            const int32_t* __restrict__ idx, float* __restrict__ dw, int N, int K, int k, int M, int* status) {
  __shared__ float s_dy[kWgTok][kWgRows];
  __shared__ float s_xw[kWgTok][kWgCols];
  __shared__ int s_idx[kWgCols];
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  const int i0 = blockIdx.x * kWgRows, t0 = blockIdx.y * kWgCols;
  if (tid < kWgCols) s_idx[tid] = (t0 + tid < k) ? idx[t0 + tid] : -1;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int m0 = 0; m0 < M; m0 += kWgTok) {
    __syncthreads();   // s_idx written / previous chunk consumed
    #pragma unroll
    for (int u = 0; u < (kWgTok * kWgRows) / kWgThreads; ++u) {
      const int e = tid + u * kWgThreads, m = e / kWgRows, r = e % kWgRows;
      const int mm = m0 + m, row = i0 + r;
      s_dy[m][r] = (mm < M && row < N) ? __half2float(dy[(size_t)mm * N + row]) : 0.f;
      const int col = s_idx[r];   // r doubles as the weak-column slot (kWgRows == kWgCols)
      s_xw[m][r] = (mm < M && col >= 0 && in_range(col, K, status)) ? __half2float(x[(size_t)mm * K + col]) : 0.f;
    }
    __syncthreads();
    #pragma unroll 8
    for (int m = 0; m < kWgTok; ++m) {
      const float xv = s_xw[m][tx];
      #pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fmaf(s_dy[m][ty * 4 + r], xv, acc[r]);
    }
  }
  const int t = t0 + tx;
  if (t < k) {
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = i0 + ty * 4 + r;
      if (row < N) dw[(size_t)row * k + t] = acc[r];
    }
  }
}

// ---------------------------------------------------------------- weak-block gradient on the tensor cores
// dW_weak = dY^T xw as mma.sync m16n8k16 (fp16 x fp16 -> fp32): MMA rows = output rows i, MMA K =
// tokens, MMA N = weak columns t.  A CTA of 4 warps computes a 64-row x 32-column tile of one
// token split; tokens stream 32 at a time through a 4-stage cp.async ring holding the dY tile
// [32 tokens][64 rows] (rows contiguous, as dY stores them) and the gathered activations
// [32 tokens][32 columns].  Both operands reach their fragments through ldmatrix.trans, so dY
// is never transposed in memory.  Rows are padded by 16 bytes against bank conflicts.  Each split
// writes its fp32 tile (to dW directly when there is one split); the splits are then added in
// split order, so repeated calls give the same bits.
constexpr int kWmRows = 64, kWmCols = 32, kWmTok = 32, kWmThreads = 128, kWmStages = 4;
constexpr int kWmDyLd = kWmRows + 8, kWmXLd = kWmCols + 8;   // padded row strides (halves)

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const int n = valid ? 16 : 0;   // 0: the 16 bytes are filled with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
               "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// xw[m][t] = x[m][idx[t]] for t < k, 0 for k <= t < kp
__global__ void k_wg_gather(const __half* __restrict__ x, int M, int K, const int32_t* __restrict__ idx, int k,
                            int kp, __half* __restrict__ xw, int* status) {
  const size_t n = (size_t)M * kp;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t m = e / kp;
    const int t = (int)(e % kp);
    xw[e] = t < k && in_range(idx[t], K, status) ? x[m * K + idx[t]] : __float2half_rn(0.f);
  }
}

// grid (N / 64, kp / 32, token splits); out = dW (one split) or the split's partial [N][k]
__global__ void __launch_bounds__(kWmThreads)
k_weak_grad_mma(const __half* __restrict__ dy, const __half* __restrict__ xw, float* __restrict__ out, int N,
                int k, int kp, int M, int per) {
  __shared__ __align__(128) __half s_dy[kWmStages][kWmTok][kWmDyLd];
  __shared__ __align__(128) __half s_x[kWmStages][kWmTok][kWmXLd];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * kWmRows, t0 = blockIdx.y * kWmCols;
  const int m_lo = blockIdx.z * per, m_hi = min(M, m_lo + per);
  const int nchunk = (m_hi - m_lo + kWmTok - 1) / kWmTok;
  auto load = [&](int c, int st) {   // chunk c of this split into stage st
    const int mb = m_lo + c * kWmTok;
    #pragma unroll
    for (int u = 0; u < 2; ++u) {    // dY: 32 tokens x 8 pieces of 8 rows
      const int e = tid + u * kWmThreads, m = e >> 3, pc = e & 7;
      const int mm = mb + m, row = i0 + pc * 8;
      const bool ok = mm < m_hi && row < N;
      cp_async16(&s_dy[st][m][pc * 8], dy + (ok ? (size_t)mm * N + row : 0), ok);
    }
    {                                // xw: 32 tokens x 4 pieces of 8 columns
      const int m = tid >> 2, pc = tid & 3, mm = mb + m;
      const bool ok = mm < m_hi;
      cp_async16(&s_x[st][m][pc * 8], xw + (ok ? (size_t)mm * kp + t0 + pc * 8 : 0), ok);
    }
  };
  float d[4][4];
  #pragma unroll
  for (int n = 0; n < 4; ++n)
    #pragma unroll
    for (int i = 0; i < 4; ++i) d[n][i] = 0.f;
  #pragma unroll
  for (int st = 0; st < kWmStages - 1; ++st) {
    if (st < nchunk) load(st, st);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int q = lane >> 3, r8 = lane & 7;   // ldmatrix: matrix q, row r8
  for (int c = 0; c < nchunk; ++c) {
    asm volatile("cp.async.wait_group %0;" :: "n"(kWmStages - 2) : "memory");
    __syncthreads();   // chunk c landed for every thread; the stage refilled below is free
    if (c + kWmStages - 1 < nchunk) load(c + kWmStages - 1, (c + kWmStages - 1) % kWmStages);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int st = c % kWmStages;
    #pragma unroll
    for (int ks = 0; ks < kWmTok / 16; ++ks) {
      const int mk = ks * 16;
      uint32_t a[4];
      // A = dY^T rows 16 warp + 0..15, tokens mk..mk+15: matrices (m 0-7, i 0-7), (m 0-7, i 8-15),
      // (m 8-15, i 0-7), (m 8-15, i 8-15), each read transposed
      ldsm_x4_t(a, &s_dy[st][mk + (q >> 1) * 8 + r8][warp * 16 + (q & 1) * 8]);
      #pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        uint32_t b[4];   // B = xw, tokens mk..mk+15 x columns 16 nh .. 16 nh + 15 (two n8 tiles)
        ldsm_x4_t(b, &s_x[st][mk + (q & 1) * 8 + r8][nh * 16 + (q >> 1) * 8]);
        mma_16816(d[2 * nh], a, b[0], b[1]);
        mma_16816(d[2 * nh + 1], a, b[2], b[3]);
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  const int g = lane >> 2, c4 = lane & 3;
  #pragma unroll
  for (int n = 0; n < 4; ++n)
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = i0 + warp * 16 + g + 8 * (i >> 1), t = t0 + n * 8 + 2 * c4 + (i & 1);
      if (row < N && t < k) out[((size_t)blockIdx.z * N + row) * k + t] = d[n][i];
    }
}

// dW = sum of the splits' partials in split order
__global__ void k_wg_reduce(const float* __restrict__ part, int splits, size_t n, float* __restrict__ dw) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    float v = part[e];
    for (int z = 1; z < splits; ++z) v += part[(size_t)z * n + e];
    dw[e] = v;
  }
}

// ---------------------------------------------------------------- input gradient, weak columns
// dx[m][idx[t]] = fp16_rn(sum_i dY[m][i] W_weak[i][t]) for many tokens.  The packed product runs
// first and leaves exactly 0 in the weak columns (their codes hold q = z), so this pass simply
// writes them.  mma.sync m16n8k16: MMA rows = tokens, MMA K = rows i, MMA N = weak slots.  A CTA
// of 4 warps computes 64 tokens x 32 slots over one split of the rows, 32 rows at a time
// through a 4-stage cp.async ring ([64 tokens][32 rows] of dY, [32 rows][32 slots] of the weak
// block); A through ldmatrix, B through ldmatrix.trans.  One split writes dx directly; several
// write fp32 partials that a second kernel adds in split order (repeat calls: identical bits).
constexpr int kIwTok = 64, kIwCols = 32, kIwRows = 32, kIwThreads = 128, kIwStages = 4;
constexpr int kIwDyLd = kIwRows + 8, kIwWLd = kIwCols + 8;   // padded row strides (halves)

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}

// grid (M / 64, k_ld / 32, row splits of `per` rows, a multiple of 32); N % 8 == 0
__global__ void __launch_bounds__(kIwThreads)
k_igw_mma(const __half* __restrict__ dy, const __half* __restrict__ w, const int32_t* __restrict__ idx,
          __half* __restrict__ dx, float* __restrict__ part, int N, int K, int M, int k, int k_ld, int per,
          int* status, int inject) {
  __shared__ __align__(128) __half s_dy[kIwStages][kIwTok][kIwDyLd];
  __shared__ __align__(128) __half s_w[kIwStages][kIwRows][kIwWLd];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mb = blockIdx.x * kIwTok, t0 = blockIdx.y * kIwCols;
  const int i_lo = blockIdx.z * per, i_hi = min(N, i_lo + per);
  const int nchunk = (i_hi - i_lo + kIwRows - 1) / kIwRows;
  auto load = [&](int c, int st) {   // rows i_lo + 32 c .. of this split into stage st
    const int ib = i_lo + c * kIwRows;
    #pragma unroll
    for (int u = 0; u < 2; ++u) {    // dY: 64 tokens x 4 pieces of 8 rows
      const int e = tid + u * kIwThreads, m = e >> 2, pc = e & 3;
      const int mm = mb + m, row = ib + pc * 8;
      const bool ok = mm < M && row < i_hi;
      cp_async16(&s_dy[st][m][pc * 8], dy + (ok ? (size_t)mm * N + row : 0), ok);
    }
    {                                // weak block: 32 rows x 4 pieces of 8 slots
      const int r = tid >> 2, pc = tid & 3, row = ib + r, col = t0 + pc * 8;
      const bool ok = row < i_hi && col < k_ld;
      cp_async16(&s_w[st][r][pc * 8], w + (ok ? (size_t)row * k_ld + col : 0), ok);
    }
  };
  float d[4][4];
  #pragma unroll
  for (int n = 0; n < 4; ++n)
    #pragma unroll
    for (int i = 0; i < 4; ++i) d[n][i] = 0.f;
  #pragma unroll
  for (int st = 0; st < kIwStages - 1; ++st) {
    if (st < nchunk) load(st, st);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int q = lane >> 3, r8 = lane & 7;   // ldmatrix: matrix q, row r8
  for (int c = 0; c < nchunk; ++c) {
    asm volatile("cp.async.wait_group %0;" :: "n"(kIwStages - 2) : "memory");
    __syncthreads();   // chunk c landed for every thread; the stage refilled below is free
    if (c + kIwStages - 1 < nchunk) load(c + kIwStages - 1, (c + kIwStages - 1) % kIwStages);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int st = c % kIwStages;
    #pragma unroll
    for (int ks = 0; ks < kIwRows / 16; ++ks) {
      const int mk = ks * 16;
      uint32_t a[4];   // tokens 16 warp + 0..15 x rows mk..mk+15: (t 0-7, i 0-7), (t 8-15, i 0-7), (t 0-7, i 8-15), (t 8-15, i 8-15)
      ldsm_x4(a, &s_dy[st][warp * 16 + (q & 1) * 8 + r8][mk + (q >> 1) * 8]);
      #pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        uint32_t bb[4];   // rows mk..mk+15 x slots 16 nh..16 nh+15, read transposed (two n8 tiles)
        ldsm_x4_t(bb, &s_w[st][mk + (q & 1) * 8 + r8][nh * 16 + (q >> 1) * 8]);
        mma_16816(d[2 * nh], a, bb[0], bb[1]);
        mma_16816(d[2 * nh + 1], a, bb[2], bb[3]);
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  const int g = lane >> 2, c4 = lane & 3;
  #pragma unroll
  for (int n = 0; n < 4; ++n)
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = mb + warp * 16 + g + 8 * (i >> 1), t = t0 + n * 8 + 2 * c4 + (i & 1);
      if (m < M && t < k) {
        if (part) {
          part[((size_t)blockIdx.z * M + m) * k + t] = d[n][i];
        } else {
          // (inject: the debug-bounds test's planted index, token 0 of slot 0 one row of K too far)
          const int col = idx[t] + (kDebugBounds && inject && m == 0 && t == 0 ? K : 0);
          if (in_range(col, K, status)) dx[(size_t)m * K + col] = __float2half_rn(d[n][i]);
        }
      }
    }
}

// dx[m][idx[t]] = fp16 of the sum of the splits' partials, in split order
__global__ void k_igw_reduce(const float* __restrict__ part, int splits, int M, int k, int K,
                             const int32_t* __restrict__ idx, __half* __restrict__ dx, int* status, int inject) {
  const size_t n = (size_t)M * k;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    float v = part[e];
    for (int z = 1; z < splits; ++z) v += part[(size_t)z * n + e];
    const int col = idx[e % k] + (kDebugBounds && inject && e == 0 ? K : 0);
    if (in_range(col, K, status)) dx[(e / k) * K + col] = __float2half_rn(v);
  }
}

// ---------------------------------------------------------------- input gradient
constexpr int kIgThreads = 256, kIgMaxTok = 16, kIgStages = 4, kIgMaxSlices = 8;
constexpr int kIgWeakBytes = 32 * 1024;   // shared memory for a column block's weak values

struct IgArgs {
  const uint32_t* packed;
  const __half2* sz_t;    // (scale, zero) pairs, tile-major [N/16][G][16]
  const __half* w_weak;   // N x k_ld
  const int32_t* idx;     // k, strictly increasing
  const __half* dy;       // M x N (this pass's first token)
  __half* dx;             // M x K
  int* status;            // device status word (bounded waits)
  long long wait_limit;
  int N, K, G, group, k, k_ld, M, tiles_per_slice;
  uint32_t blk[kMaxBlocks];   // per column block: first weak slot << 16 | weak-column count
};

// ---------------------------------------------------------------- input gradient on the tensor cores
// dX^T = W_eff^T dY^T per (16-row tile, 128-code block) unit as mma.sync m16n8k16: MMA rows =
// 16 input columns j, MMA K = the tile's 16 rows i, MMA N = 8 tokens.  Grid: (K / 128 column
// blocks) x (row slices); a CTA of 8 warps covers one column block and one slice of the row
// tiles, warp w taking tiles w, w + 8, ... of the slice.  Each warp streams its tiles' packed
// block (one contiguous 16 x 16 * bits byte run of the tiled storage) and the tile's (scale,
// zero) pairs through a private 4-stage ring of bulk copies; the block's weak values over the
// slice's rows are staged in shared memory once (their slots are consecutive, the index list
// being increasing).
//
// The scale varies along the contraction here (row i), so it goes with dY: the A operand is the
// exact integer q - z, the B operand dY s split into an fp16 high part and the fp16 residual
// (dY s - hi, exact in fp16 unless it falls below the normal range), both multiplied by the same
// A; every product is exact and the sums are fp32.  This evaluates dY (s (q - z)) with the unrounded dequantised weights, like the
// decode product, instead of fp16_rn(s (q - z)): each weight differs by at most half an fp16
// spacing; with one nonzero dY per token the output is fp16_rn(s (q - z)) exactly.
//
// The transposed operand is built straight from the staged block.  Lane (g, t) holds, for MMA
// row g (column 16 s + g of slice s) and g + 8, the rows 2t, 2t + 1 and 2t + 8, 2t + 9; all its
// codes lie in chunk g / 2 of those four rows (pairs 2 s and 2 s + 1, the even code for even g,
// the odd one for odd g).  One byte permute puts the same half of two rows' words side by side
// (shifted down a byte where the code sits at bit 8 or above), an AND with OR leaves
// 1024 + q 2^o in each fp16 half and one fp16x2 fma with the row pair's constants leaves q - z
// exactly.  The weak columns' codes give exactly 0 (they hold the integral zero point); their
// fp16 values enter through one more product with the unscaled dY per 16-column slice that
// holds any.  The warps' partial sums meet in shared memory in a fixed tree.  The slices of a
// column block form one thread-block cluster: each CTA then adds, for its share of the block's
// outputs, the CTAs' sums in slice order through distributed shared memory, so repeated calls
// give identical bits and no workspace is needed.  Every ring wait is bounded (on expiry: the
// status word, no further products, the copies in flight waited for).
__device__ __forceinline__ uint32_t ig_h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ __half2 u32_h2(uint32_t u) { return *reinterpret_cast<const __half2*>(&u); }
__device__ __forceinline__ uint32_t h2_u32(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }
__device__ __forceinline__ uint32_t ig_h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Bit offset of pair j's codes in each half after extraction (codes at bit 8 or above are
// moved down a byte by the permute), and the classes of those offsets.
template <int BITS>
__host__ __device__ constexpr int ig_off(int j) {
  if (BITS == 3 && j == 11) return 6;   // the spread pair, rebuilt at offset 6
  const int o = BITS == 3 ? slot3(j).off : slot4(j).off;
  return o >= 8 ? o - 8 : o;
}
template <int BITS>
__host__ __device__ constexpr int ig_ncls() { return BITS == 3 ? 5 : 2; }
template <int BITS>
__host__ __device__ constexpr int ig_cls_off(int c) {   // 3-bit: 0, 3, 6, 1, 4; 4-bit: 0, 4
  return BITS == 3 ? (c == 0 ? 0 : c == 1 ? 3 : c == 2 ? 6 : c == 3 ? 1 : 4) : 4 * c;
}
template <int BITS>
__host__ __device__ constexpr int ig_cls(int off) {
  return BITS == 3 ? (off == 0 ? 0 : off == 3 ? 1 : off == 6 ? 2 : off == 1 ? 3 : 4) : off / 4;
}

// Codes of pair j (the half `sel` picks) of rows a (low fp16 half) and b (high half), as
// 1024 + q 2^o in each half (the bits 0x6400 with the code at offset o = ig_off(j)).
template <int BITS>
__device__ __forceinline__ uint32_t ig_tpair(const uint32_t* wa, const uint32_t* wb, int j, uint32_t sel,
                                             uint32_t sel8) {
  constexpr uint32_t kMagic = 0x64006400u;
  if constexpr (BITS == 3) {
    if (j == 11) {   // bit e of each code at bit 15 of word e: to bits 6, 7, 8
      const uint32_t t0 = __byte_perm(wa[0], wb[0], sel), t1 = __byte_perm(wa[1], wb[1], sel);
      const uint32_t t2 = __byte_perm(wa[2], wb[2], sel);
      return ((t0 >> 9) & 0x00400040u) | ((t1 >> 8) & 0x00800080u) | ((t2 >> 7) & 0x01000100u) | kMagic;
    }
    const Slot sl = slot3(j);
    const uint32_t v = __byte_perm(wa[sl.word], wb[sl.word], sl.off >= 8 ? sel8 : sel);
    return (v & (0x00070007u << ig_off<3>(j))) | kMagic;
  } else {
    const Slot sl = slot4(j);
    const uint32_t v = __byte_perm(wa[sl.word], wb[sl.word], sl.off >= 8 ? sel8 : sel);
    return (v & (0x000F000Fu << ig_off<4>(j))) | kMagic;
  }
}

template <int BITS>
__host__ __device__ constexpr int ig_stage_bytes() { return 256 * BITS + 64; }   // one tile's block + its 16 (s, z) pairs
template <int BITS>
__host__ __device__ constexpr int ig_smem_bytes() {   // the warps' rings, their barriers, the staged weak values
  return (kIgThreads / 32) * kIgStages * (ig_stage_bytes<BITS>() + 8) + kIgWeakBytes;
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kIgThreads, 2)
k_input_grad_mma(const __grid_constant__ IgArgs a) {
  constexpr int NCL = ig_ncls<BITS>();
  constexpr int kBlkB = 16 * BITS;                 // one row's block, bytes
  constexpr int kTileBlkB = 16 * kBlkB;            // one tile's block, bytes
  constexpr int kStage = ig_stage_bytes<BITS>();
  constexpr int kTok = 8 * NT;
  extern __shared__ __align__(128) unsigned char ig_smem[];
  __shared__ float s_red[4][kTok][kBlockCodes];
  __shared__ int s_slot[kBlockCodes];              // weak slot of column c of the block, or -1
  __shared__ int s_wsl;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  const int b = blockIdx.x, slice = blockIdx.y, S = gridDim.y;
  const int Kb = a.K / kBlockCodes, tiles = (a.N + 15) / 16;
  const int grp = (b * kBlockCodes) / a.group;   // the block's group (per-channel: 0)
  unsigned char* ring = ig_smem + warp * kIgStages * kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ig_smem + (kIgThreads / 32) * kIgStages * kStage) + warp * kIgStages;
  __half* s_wv = reinterpret_cast<__half*>(ig_smem + (kIgThreads / 32) * kIgStages * (kStage + 8));

  const int t_lo = slice * a.tiles_per_slice, t_hi = min(tiles, t_lo + a.tiles_per_slice);
  const int rows = max(0, t_hi - t_lo) * 16;
  const int nmine = t_hi > t_lo + warp ? (t_hi - t_lo - warp + 7) / 8 : 0;   // this warp's tiles
  int issued = 0;
  // lane 0: the warp's next tile (block b of 16 rows, then its (scale, zero) pairs) into its stage
  const unsigned char* src_blk = reinterpret_cast<const unsigned char*>(a.packed) + ((size_t)(t_lo + warp) * Kb + b) * kTileBlkB;
  const __half2* src_sz = a.sz_t + ((size_t)(t_lo + warp) * a.G + grp) * 16;
  auto issue = [&]() {
    const int st = issued % kIgStages;
    mbar_arrive_expect_tx(&bars[st], (uint32_t)kStage);
    bulk_load(ring + st * kStage, src_blk, (uint32_t)kTileBlkB, &bars[st]);
    bulk_load(ring + st * kStage + kTileBlkB, src_sz, 64u, &bars[st]);
    src_blk += (size_t)8 * Kb * kTileBlkB;
    src_sz += (size_t)8 * a.G * 16;
    ++issued;
  };
  if (lane == 0) {
    for (int st = 0; st < kIgStages; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
    while (issued < min(nmine, kIgStages)) issue();
  }

  // the block's weak slots t0 .. t0 + nweak - 1 (from the pack-time table): their columns and,
  // staged, their values over the slice's rows are loaded in one round trip
  const int t0 = (int)(a.blk[b] >> 16), nweak = (int)(a.blk[b] & 0xFFFFu);
  if (tid < kBlockCodes) s_slot[tid] = -1;
  if (tid == 0) s_wsl = 0;
  const int my_t = tid < nweak ? t0 + tid : -1;
  const int my_col = my_t >= 0 ? a.idx[my_t] - b * kBlockCodes : -1;
  // s_wv[(slot - t0) * rows + r] (rows >= N: 0), staged for up to 8 weak columns, 4 rows x 8
  // columns of loads in flight per thread per pass
  const bool staged = nweak > 0 && nweak <= 8 && nweak * rows * (int)sizeof(__half) <= kIgWeakBytes;
  const int passes = staged ? (rows + 4 * kIgThreads - 1) / (4 * kIgThreads) : 0;
  uint16_t v[4][8];
  auto stage_load = [&](int r0) {
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = r0 + u * kIgThreads, row = t_lo * 16 + r;
      const __half* src = a.w_weak + (size_t)row * a.k_ld + t0;
      #pragma unroll
      for (int wi = 0; wi < 8; ++wi)
        v[u][wi] = wi < nweak && r < rows && row < a.N ? __half_as_ushort(src[wi]) : (uint16_t)0;
    }
  };
  auto stage_store = [&](int r0) {
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = r0 + u * kIgThreads;
      #pragma unroll
      for (int wi = 0; wi < 8; ++wi)
        if (wi < nweak && r < rows) s_wv[wi * rows + r] = __ushort_as_half(v[u][wi]);
    }
  };
  if (passes > 0) stage_load(tid);
  __syncthreads();   // s_slot cleared
  if (my_col >= 0 && my_col < kBlockCodes) {
    s_slot[my_col] = my_t;
    atomicOr(&s_wsl, 1 << (my_col >> 4));
  }
  if (passes > 0) {
    stage_store(tid);
    for (int pz = 1; pz < passes; ++pz) {
      stage_load(tid + pz * 4 * kIgThreads);
      stage_store(tid + pz * 4 * kIgThreads);
    }
  }
  __syncthreads();
  const int wsl = s_wsl;   // slices (16 columns) of the block holding weak columns
  // the lane's weak columns: bit 2 s for column 16 s + g, bit 2 s + 1 for column 16 s + g + 8
  uint32_t wmask = 0;
  if (nweak > 0) {
    #pragma unroll
    for (int sl = 0; sl < 8; ++sl) {
      wmask |= (s_slot[16 * sl + g] >= 0 ? 1u : 0u) << (2 * sl);
      wmask |= (s_slot[16 * sl + g + 8] >= 0 ? 2u : 0u) << (2 * sl);
    }
  }

  // byte permutes taking half g % 2 of two words (sel), the same one byte lower (sel8)
  const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u, sel8 = (g & 1) ? 0x7733u : 0x5511u;

  float D[8][NT][4];
  #pragma unroll
  for (int sl = 0; sl < 8; ++sl)
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i) D[sl][nt][i] = 0.f;

  // dY fragments of a tile (rows 16 tile + 2 tg (+1, +8, +9), token 8 nt + g), loaded two tiles
  // ahead (one with two token blocks): two 32-bit loads per token block where the tile is whole and N even, else by halves
  const bool n_even = (a.N & 1) == 0;
  auto load_dy = [&](int tile, uint32_t (&yy)[NT][2]) {
    const int i0 = tile * 16 + 2 * tg;
    const bool whole = n_even && tile * 16 + 16 <= a.N;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = 8 * nt + g;
      yy[nt][0] = yy[nt][1] = 0u;
      if (m >= a.M) continue;
      const __half* p = a.dy + (size_t)m * a.N + i0;
      if (whole) {
        yy[nt][0] = *reinterpret_cast<const uint32_t*>(p);
        yy[nt][1] = *reinterpret_cast<const uint32_t*>(p + 8);
      } else {
        uint16_t v[4];
        #pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int du = (u & 1) + 8 * (u >> 1);
          v[u] = i0 + du < a.N ? __half_as_ushort(p[du]) : (uint16_t)0;
        }
        yy[nt][0] = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
        yy[nt][1] = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
      }
    }
  };
  constexpr int PD = NT == 1 ? 2 : 1;   // prefetch distance, in the warp's tiles
  uint32_t yq[PD + 1][NT][2];           // dY of the warp's tiles j .. j + PD
  #pragma unroll
  for (int p = 0; p < PD; ++p)
    if (p < nmine) load_dy(t_lo + warp + 8 * p, yq[p]);
  bool ok = true;
  int failed_at = -1;
  for (int j = 0; j < nmine; ++j) {
    const int tile = t_lo + warp + 8 * j, st = j % kIgStages;
    if (j + PD < nmine) load_dy(tile + 8 * PD, yq[PD]);
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[st], (uint32_t)((j / kIgStages) & 1), a.status, a.wait_limit));
      if (!ok) failed_at = j;
    }
    if (ok) {
      const unsigned char* stg = ring + st * kStage;
      // chunk g / 2 of rows 2 tg, 2 tg + 1, 2 tg + 8, 2 tg + 9, and their (scale, zero) pairs
      uint32_t w0[BITS], w1[BITS], w2[BITS], w3[BITS];
      #pragma unroll
      for (int jj = 0; jj < BITS; ++jj) {
        const unsigned char* c0 = stg + (g >> 1) * 4 * BITS + 4 * jj;
        w0[jj] = *reinterpret_cast<const uint32_t*>(c0 + (2 * tg) * kBlkB);
        w1[jj] = *reinterpret_cast<const uint32_t*>(c0 + (2 * tg + 1) * kBlkB);
        w2[jj] = *reinterpret_cast<const uint32_t*>(c0 + (2 * tg + 8) * kBlkB);
        w3[jj] = *reinterpret_cast<const uint32_t*>(c0 + (2 * tg + 9) * kBlkB);
      }
      const uint32_t* szs = reinterpret_cast<const uint32_t*>(stg + kTileBlkB);
      const uint32_t sz0 = szs[2 * tg], sz1 = szs[2 * tg + 1], sz2 = szs[2 * tg + 8], sz3 = szs[2 * tg + 9];
      __syncwarp();   // every lane has read the stage
      if (lane == 0 && issued < nmine) {
        fence_proxy_async_smem();
        issue();      // into the stage just read
      }
      // row pairs (2 tg, 2 tg + 1) and (2 tg + 8, 2 tg + 9): scales, and -(1024 2^-o + z) per class
      const uint32_t S2[2] = {__byte_perm(sz0, sz1, 0x5410), __byte_perm(sz2, sz3, 0x5410)};
      const uint32_t Z2[2] = {__byte_perm(sz0, sz1, 0x7632), __byte_perm(sz2, sz3, 0x7632)};
      uint32_t NZ[2][NCL];
      #pragma unroll
      for (int c = 0; c < NCL; ++c) {
        const uint32_t neg_o = 0x8000u | ((uint32_t)(25 - ig_cls_off<BITS>(c)) << 10);   // -2^(10 - o)
        NZ[0][c] = ig_h2_sub(neg_o | (neg_o << 16), Z2[0]);
        NZ[1][c] = ig_h2_sub(neg_o | (neg_o << 16), Z2[1]);
      }
      // B operands: dY s as fp16 hi + lo, rows (2 tg, 2 tg + 1) and (2 tg + 8, 2 tg + 9)
      uint32_t bh[NT][2], bl[NT][2];
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
          const __half2 y = u32_h2(yq[0][nt][h]), sc2 = u32_h2(S2[h]);
          const __half2 hi = __hmul2(y, sc2);
          bh[nt][h] = h2_u32(hi);
          bl[nt][h] = h2_u32(__hfma2(y, sc2, __hneg2(hi)));
        }
      const int ra = (tile - t_lo) * 16 + 2 * tg;   // row 2 tg of the tile, within the slice
      #pragma unroll
      for (int sl = 0; sl < 8; ++sl) {
        uint32_t at[4];
        #pragma unroll
        for (int r = 0; r < 4; ++r) {   // r: (rows 2 tg.. | 2 tg + 8..) x (column g | g + 8)
          const int jp = 2 * sl + (r & 1), rp = r >> 1;
          const int cls = ig_cls<BITS>(ig_off<BITS>(jp));
          const uint32_t sc = (uint32_t)(15 - ig_cls_off<BITS>(cls)) << 10;   // 2^-o
          const uint32_t v = rp == 0 ? ig_tpair<BITS>(w0, w1, jp, sel, sel8) : ig_tpair<BITS>(w2, w3, jp, sel, sel8);
          at[r] = ig_h2_fma(v, sc | (sc << 16), NZ[rp][cls]);   // q - z, exact
        }
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816(D[sl][nt], at, bh[nt][0], bh[nt][1]);
          mma_16816(D[sl][nt], at, bl[nt][0], bl[nt][1]);
        }
      }
      // the weak columns (their codes gave exactly 0): one more product per slice holding any,
      // with their fp16 values for this lane's columns and zeros elsewhere
      if (wsl) {
        #pragma unroll
        for (int sl = 0; sl < 8; ++sl) {
          if (!((wsl >> sl) & 1)) continue;
          uint32_t aw[4] = {0u, 0u, 0u, 0u};
          #pragma unroll
          for (int u = 0; u < 2; ++u) {   // u: column 16 sl + g (+ 8 u) -> registers u, u + 2
            if (!((wmask >> (2 * sl + u)) & 1u)) continue;
            const int wi = s_slot[16 * sl + g + 8 * u] - t0;
            if (staged) {
              aw[u] = *reinterpret_cast<const uint32_t*>(s_wv + wi * rows + ra);
              aw[u + 2] = *reinterpret_cast<const uint32_t*>(s_wv + wi * rows + ra + 8);
            } else {
              uint16_t v[4];
              #pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int gr = t_lo * 16 + ra + (e & 1) + 8 * (e >> 1);
                v[e] = gr < a.N ? __half_as_ushort(a.w_weak[(size_t)gr * a.k_ld + t0 + wi]) : (uint16_t)0;
              }
              aw[u] = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
              aw[u + 2] = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
            }
          }
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816(D[sl][nt], aw, yq[0][nt][0], yq[0][nt][1]);
        }
      }
    }
    #pragma unroll
    for (int p = 0; p < PD; ++p)
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt) { yq[p][nt][0] = yq[p + 1][nt][0]; yq[p][nt][1] = yq[p + 1][nt][1]; }
  }
  // after a timeout: never leave with bulk copies still writing into this CTA's memory
  if (failed_at >= 0 && lane == 0)
    for (int j = failed_at; j < issued; ++j)
      mbar_wait(&bars[j % kIgStages], (uint32_t)((j / kIgStages) & 1), a.status, a.wait_limit);

  // the 8 warps' sums in a fixed tree: (w, w + 4), then (w, w + 2), then (0, 1)
  // D[sl][nt][i]: column 16 sl + g + 8 (i >> 1), token 8 nt + 2 tg + (i & 1)
  #pragma unroll
  for (int half = 4; half >= 1; half >>= 1) {
    if (warp >= half && warp < 2 * half) {
      #pragma unroll
      for (int sl = 0; sl < 8; ++sl)
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            s_red[warp - half][8 * nt + 2 * tg + (i & 1)][16 * sl + g + 8 * (i >> 1)] = D[sl][nt][i];
    }
    __syncthreads();
    if (warp < half) {
      #pragma unroll
      for (int sl = 0; sl < 8; ++sl)
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            D[sl][nt][i] += s_red[warp][8 * nt + 2 * tg + (i & 1)][16 * sl + g + 8 * (i >> 1)];
    }
    __syncthreads();
  }
  if (S == 1) {   // one slice: the CTA's sums are the outputs
    if (warp == 0) {
      #pragma unroll
      for (int sl = 0; sl < 8; ++sl)
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = 8 * nt + 2 * tg + (i & 1), c = b * kBlockCodes + 16 * sl + g + 8 * (i >> 1);
            if (m < a.M) a.dx[(size_t)m * a.K + c] = __float2half_rn(D[sl][nt][i]);
          }
    }
    return;
  }
  // the cluster of the column block's S slices: publish, then add in slice order
  if (warp == 0) {
    #pragma unroll
    for (int sl = 0; sl < 8; ++sl)
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i)
          s_red[0][8 * nt + 2 * tg + (i & 1)][16 * sl + g + 8 * (i >> 1)] = D[sl][nt][i];
  }
  cluster_sync();
  {
    constexpr int ne = kTok * kBlockCodes;
    const int share = (ne + S - 1) / S, rank = (int)cluster_ctarank();
    const int e_hi = min(ne, (rank + 1) * share);
    for (int e = rank * share + tid; e < e_hi; e += kIgThreads) {
      const int m = e / kBlockCodes, c = e % kBlockCodes;
      if (m >= a.M) continue;
      float sum = 0.f;
      for (int r = 0; r < S; ++r) sum += ld_dsmem_f32(&s_red[0][m][c], (uint32_t)r);
      a.dx[(size_t)m * a.K + b * kBlockCodes + c] = __float2half_rn(sum);
    }
  }
  cluster_sync();   // no CTA leaves while its sums may still be read
}

// SM count of device `dev` (cached per device ordinal)
int wct_sm_count(int dev) {
  constexpr int kMaxDev = 64;
  static int n[kMaxDev] = {};
  if (dev < 0 || dev >= kMaxDev) return 148;
  if (!n[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    n[dev] = v;
  }
  return n[dev];
}

template <int BITS, int NT>
cudaError_t launch_ig(const IgArgs& a, int dev, int Kb, int slices, cudaStream_t s) {
  constexpr int smem = ig_smem_bytes<BITS>();
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  if (dev < 0 || dev >= kMaxDev || !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_input_grad_mma<BITS, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)Kb, (unsigned)slices, 1);
  cfg.blockDim = dim3(kIgThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)slices;   // the slices of a column block: one cluster
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_input_grad_mma<BITS, NT>, a);
}

}  // namespace

cudaError_t launch_weak_grad(const Layer& L, const __half* x, const __half* dy, float* dw, int M,
                             cudaStream_t s) {
  if (L.k == 0) return cudaSuccess;
  // tensor-core kernel: needs 16-byte rows of dY (N % 8 == 0) and the gathered activations
  // (and, with several token splits, the partials) in the handle's scratch, which grows only
  // outside a stream capture; otherwise the CUDA-core kernel, which needs no scratch
  const int kp = (L.k + kWmCols - 1) / kWmCols * kWmCols;
  const int R = (L.N + kWmRows - 1) / kWmRows, C = kp / kWmCols;
  const int sms = wct_sm_count(L.device);
  int splits = std::max(1, std::min((2 * sms + R * C - 1) / (R * C), (M + 255) / 256));
  int per = (M + splits - 1) / splits;
  per = (per + kWmTok - 1) / kWmTok * kWmTok;
  splits = (M + per - 1) / per;
  const size_t xw_bytes = ((size_t)M * kp * sizeof(__half) + 255) / 256 * 256;
  const size_t need = xw_bytes + (splits > 1 ? (size_t)splits * L.N * L.k * sizeof(float) : 0);
  Layer& Lm = const_cast<Layer&>(L);
  bool mma = L.N % 8 == 0;
  if (mma && need > L.wg_ws_bytes) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
      cudaGetLastError();
      mma = false;
    } else {
      cudaFree(Lm.wg_ws);
      Lm.wg_ws = nullptr;
      Lm.wg_ws_bytes = 0;
      if (cudaMalloc(&Lm.wg_ws, need) != cudaSuccess) {
        cudaGetLastError();
        Lm.wg_ws = nullptr;
        mma = false;
      } else {
        Lm.wg_ws_bytes = need;
      }
    }
  }
  if (!mma) {
    const dim3 grid((L.N + kWgRows - 1) / kWgRows, (L.k + kWgCols - 1) / kWgCols);
    k_weak_grad<<<grid, kWgThreads, 0, s>>>(x, dy, L.idx, dw, L.N, L.K, L.k, M, device_status_ptr());
    return cudaGetLastError();
  }
  __half* xw = reinterpret_cast<__half*>(L.wg_ws);
  float* part = splits > 1 ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(L.wg_ws) + xw_bytes) : nullptr;
  const size_t nxw = (size_t)M * kp;
  k_wg_gather<<<(unsigned)std::min<size_t>((nxw + 255) / 256, 4096), 256, 0, s>>>(x, M, L.K, L.idx, L.k, kp, xw,
                                                                                       device_status_ptr());
  k_weak_grad_mma<<<dim3(R, C, splits), kWmThreads, 0, s>>>(dy, xw, splits > 1 ? part : dw, L.N, L.k, kp, M, per);
  if (splits > 1) {
    const size_t n = (size_t)L.N * L.k;
    k_wg_reduce<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, s>>>(part, splits, n, dw);
  }
  return cudaGetLastError();
}

cudaError_t launch_input_grad(Layer& L, const __half* dy, __half* dx, int M, cudaStream_t s) {
  const int Kb = L.K / kBlockCodes;
  const int tiles = (L.N + 15) / 16;
  // two CTAs per SM over the column blocks and row slices (about one wave), each slice at least
  // one tile per warp, the slices of a column block one cluster (at most 8 CTAs)
  int slices = std::max(1, std::min({(tiles + 7) / 8, (2 * wct_sm_count(L.device)) / Kb, kIgMaxSlices}));
  const int per = (tiles + slices - 1) / slices;
  slices = (tiles + per - 1) / per;
  IgArgs a;
  a.packed = L.packed;
  a.sz_t = L.sz_t;
  a.w_weak = L.w_weak;
  a.idx = L.idx;
  a.status = device_status_ptr();
  a.wait_limit = kDefaultWaitLimit;
  a.N = L.N;
  a.K = L.K;
  a.G = L.G;
  a.group = L.group;
  a.k = L.k;
  a.k_ld = L.k_ld;
  a.tiles_per_slice = per;
  for (int i = 0; i < Kb; ++i) a.blk[i] = L.blk_weak[i];
  if (!a.status) return cudaErrorInvalidDevicePointer;
  for (int m0 = 0; m0 < M; m0 += kIgMaxTok) {
    a.dy = dy + (size_t)m0 * L.N;
    a.dx = dx + (size_t)m0 * L.K;
    a.M = std::min(kIgMaxTok, M - m0);
    const cudaError_t e =
        L.bits == 3 ? (a.M <= 8 ? launch_ig<3, 1>(a, L.device, Kb, slices, s) : launch_ig<3, 2>(a, L.device, Kb, slices, s))
                    : (a.M <= 8 ? launch_ig<4, 1>(a, L.device, Kb, slices, s) : launch_ig<4, 2>(a, L.device, Kb, slices, s));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_input_grad_weak(Layer& L, const __half* dy, __half* dx, int M, bool inject, cudaStream_t s) {
  if (L.k == 0) return cudaSuccess;
  const int R = (M + kIwTok - 1) / kIwTok, C = (L.k + kIwCols - 1) / kIwCols;
  const int nch = (L.N + kIwRows - 1) / kIwRows;
  // split the rows so that about two CTAs per SM run, at least 4 chunks each
  int splits = std::max(1, std::min((2 * wct_sm_count(L.device) + R * C - 1) / (R * C), nch / 4));
  int per = (nch + splits - 1) / splits;
  splits = (nch + per - 1) / per;
  per *= kIwRows;
  float* part = nullptr;
  if (splits > 1) {
    const size_t need = (size_t)splits * M * L.k * sizeof(float);
    bool have = need <= L.wg_ws_bytes;
    if (!have) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone) {
        cudaFree(L.wg_ws);
        L.wg_ws = nullptr;
        L.wg_ws_bytes = 0;
        if (cudaMalloc(&L.wg_ws, need) == cudaSuccess) {
          L.wg_ws_bytes = need;
          have = true;
        }
      }
      cudaGetLastError();
    }
    if (have) {
      part = reinterpret_cast<float*>(L.wg_ws);
    } else {   // inside a capture without scratch: one split
      splits = 1;
      per = nch * kIwRows;
    }
  }
  int* status = device_status_ptr();
  k_igw_mma<<<dim3(R, C, splits), kIwThreads, 0, s>>>(dy, L.w_weak, L.idx, dx, part, L.N, L.K, M, L.k, L.k_ld, per,
                                                      status, inject ? 1 : 0);
  if (splits > 1) {
    const size_t n = (size_t)M * L.k;
    k_igw_reduce<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, s>>>(part, splits, M, L.k, L.K, L.idx, dx,
                                                                                          status, inject ? 1 : 0);
  }
  return cudaGetLastError();
}

}  // namespace owq
