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

namespace owq {
namespace {

// ---------------------------------------------------------------- weak-block gradient
// A CTA computes a 32-row x 32-weak-column tile of dW_weak; its 256 threads own one weak column
// and four rows each.  Tokens are staged 32 at a time: dY rows (coalesced along the output
// rows) and the gathered activation columns x[:, idx[t]].
constexpr int kWgRows = 32, kWgCols = 32, kWgTok = 32, kWgThreads = 256;

__global__ void __launch_bounds__(kWgThreads)
k_weak_grad(const __half* __restrict__ x, const __half* __restrict__ dy,
            const int32_t* __restrict__ idx, float* __restrict__ dw, int N, int K, int k, int M) {
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
      s_xw[m][r] = (mm < M && col >= 0) ? __half2float(x[(size_t)mm * K + col]) : 0.f;
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
                            int kp, __half* __restrict__ xw) {
  const size_t n = (size_t)M * kp;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t m = e / kp;
    const int t = (int)(e % kp);
    xw[e] = t < k ? x[m * K + idx[t]] : __float2half_rn(0.f);
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

// ---------------------------------------------------------------- input gradient
// Grid: (K / 128 column blocks) x (row slices).  A CTA walks its slice of one column block in
// stages of 64 rows (four 16-row tiles, whose blocks are contiguous in the tiled storage); each
// of its 256 threads owns one code pair (two adjacent columns) and 16 rows of every stage.
//
// Dequantisation in fp16x2: the pair's two codes sit at the same bit offset of the two halves
// of one word, so one shift-and-mask gives (q_even, q_odd) as 16-bit integers; OR-ing 0x6400
// (1024.0) into each half makes the exact halves 1024 + q, subtracting (1024 + z) leaves q - z
// exactly, and one fp16x2 multiply by the scale rounds s (q - z) once, i.e. fp16_rn(s (q - z)).
//
// The four row quarters of a pair are summed in shared memory in a fixed order.  With more
// than one slice, each CTA stores its fp32 partial sums to the layer's workspace; the last CTA
// of a column block to finish (a counter per block) adds the slices in slice order and writes
// the fp16 result, so repeated calls give identical bits.  Nothing waits on another CTA.
constexpr int kIgThreads = 256, kIgStageRows = 64, kIgMaxTok = 16;

struct IgArgs {
  const uint32_t* packed;
  const __half* scales;
  const __half* zeros;
  const __half* w_weak;
  const int32_t* idx;
  const __half* dy;   // M x N (this pass's first token)
  __half* dx;         // M x K
  float* part;        // [slices][16 tokens][K] (slices > 1)
  unsigned int* count;  // [K / 128], zero between calls
  int N, K, G, group, k, k_ld, M, stages_per_slice;
};

template <int BITS>
__device__ __forceinline__ uint32_t pair_codes(const uint32_t* w, int word, int shift, bool spread) {
  if (BITS == 3 && spread)   // bit e of the even / odd code is bit 15 / 31 of word e
    return ((w[word] >> 15) & 0x00010001u) | ((w[word + 1] >> 14) & 0x00020002u) |
           ((w[word + 2] >> 13) & 0x00040004u);
  return (w[word] >> shift) & (((1u << BITS) - 1u) * 0x00010001u);
}

template <int BITS, int TOK>
__global__ void __launch_bounds__(kIgThreads)
k_input_grad(const IgArgs a) {
  constexpr int kStageWords4 = 4 * 16 * BITS;   // uint4 per stage: 4 tiles x 16 blocks x BITS
  __shared__ uint4 s_words[2][kStageWords4];
  __shared__ __half2 s_scale[2][kIgStageRows];
  __shared__ __half2 s_zb[2][kIgStageRows];       // (1024 + z, 1024 + z)
  __shared__ __align__(16) float s_dy[2][kIgStageRows][TOK];
  __shared__ float2 s_red[3][TOK][64];
  __shared__ int s_last;
  __shared__ int s_slot[kBlockCodes];

  const int tid = threadIdx.x, p = tid & 63, h = tid >> 6;
  const int b = blockIdx.x, slice = blockIdx.y, S = gridDim.y;
  const int Kb = a.K / kBlockCodes, tiles = (a.N + 15) / 16;
  const int g = (b * kBlockCodes) / a.group;
  const int col = b * kBlockCodes + 2 * p;

  // the pair's slot in a block: chunk p % 4, pair p / 4 of the chunk
  const int chunk = p & 3, jj = p >> 2;
  const Slot sl = BITS == 3 ? slot3(jj) : slot4(jj);
  const bool spread = sl.word < 0;
  const int word = chunk * BITS + (spread ? 0 : sl.word);
  const int shift = spread ? 0 : sl.off;

  // weak slots of the block's columns: one parallel pass over idx into a shared table
  if (tid < kBlockCodes) s_slot[tid] = -1;
  __syncthreads();
  for (int t = tid; t < a.k; t += kIgThreads) {
    const int c = a.idx[t] - b * kBlockCodes;
    if (c >= 0 && c < kBlockCodes) s_slot[c] = t;
  }
  __syncthreads();
  const int tw0 = s_slot[2 * p], tw1 = s_slot[2 * p + 1];
  const bool weak = tw0 >= 0 || tw1 >= 0;

  const int nstages = (tiles + 3) / 4;
  const int st0 = slice * a.stages_per_slice;
  const int st1 = min(nstages, st0 + a.stages_per_slice);

  // staged loads of one stage into registers
  uint4 r_words = make_uint4(0, 0, 0, 0);
  __half r_s = __float2half(0.f), r_z = __float2half(0.f);
  __half r_dy[(TOK * kIgStageRows + kIgThreads - 1) / kIgThreads];
  // weak values of this thread's rows, one stage ahead (threads with a weak column only)
  __half2 wk_next[16], wk_cur[16];
  auto load = [&](int st) {
    if (weak) {
      #pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        const int row = st * kIgStageRows + h * 16 + rr;
        const __half* wr = a.w_weak + (size_t)row * a.k_ld;
        wk_next[rr] = __halves2half2(tw0 >= 0 && row < a.N ? wr[tw0] : __float2half(0.f),
                                     tw1 >= 0 && row < a.N ? wr[tw1] : __float2half(0.f));
      }
    }
    if (tid < kStageWords4) {
      const int tile = st * 4 + tid / (16 * BITS);
      r_words = make_uint4(0, 0, 0, 0);
      if (tile < tiles)
        r_words = reinterpret_cast<const uint4*>(a.packed + ((size_t)tile * Kb + b) * 16 * 4 * BITS)[tid % (16 * BITS)];
    }
    if (tid < kIgStageRows) {
      const int row = st * kIgStageRows + tid;
      r_s = row < a.N ? a.scales[(size_t)row * a.G + g] : __float2half(0.f);
      r_z = row < a.N ? a.zeros[(size_t)row * a.G + g] : __float2half(0.f);
    }
    #pragma unroll
    for (int u = 0; u < (int)(sizeof(r_dy) / sizeof(r_dy[0])); ++u) {
      const int e = tid + u * kIgThreads, m = e / kIgStageRows, rr = e % kIgStageRows;
      const int row = st * kIgStageRows + rr;
      r_dy[u] = (e < TOK * kIgStageRows && m < a.M && row < a.N) ? a.dy[(size_t)m * a.N + row] : __float2half(0.f);
    }
  };
  auto store = [&](int buf) {
    if (weak) {
      #pragma unroll
      for (int rr = 0; rr < 16; ++rr) wk_cur[rr] = wk_next[rr];
    }
    if (tid < kStageWords4) s_words[buf][tid] = r_words;
    if (tid < kIgStageRows) {
      s_scale[buf][tid] = __halves2half2(r_s, r_s);
      const __half zb = __hadd(r_z, __float2half(1024.f));   // exact: z is a small integer
      s_zb[buf][tid] = __halves2half2(zb, zb);
    }
    #pragma unroll
    for (int u = 0; u < (int)(sizeof(r_dy) / sizeof(r_dy[0])); ++u) {
      const int e = tid + u * kIgThreads;
      if (e < TOK * kIgStageRows) s_dy[buf][e % kIgStageRows][e / kIgStageRows] = __half2float(r_dy[u]);
    }
  };

  float2 acc[TOK];
  #pragma unroll
  for (int m = 0; m < TOK; ++m) acc[m] = make_float2(0.f, 0.f);

  if (st0 < st1) {
    load(st0);
    store(0);
  }
  __syncthreads();
  for (int st = st0; st < st1; ++st) {
    const int buf = (st - st0) & 1;
    if (st + 1 < st1) load(st + 1);
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(s_words[buf]);
    #pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      const int r = h * 16 + rr;               // row within the stage
      // row r of the stage is row r % 16 of tile r / 16: block (r / 16) * 16 + r % 16 = r
      const uint32_t v = pair_codes<BITS>(sw + r * 4 * BITS, word, shift, spread) | 0x64006400u;
      const __half2 qz = __hsub2(*reinterpret_cast<const __half2*>(&v), s_zb[buf][r]);
      float2 wv = __half22float2(__hmul2(s_scale[buf][r], qz));
      if (weak) {
        const float2 wk = __half22float2(wk_cur[rr]);
        if (tw0 >= 0) wv.x = wk.x;
        if (tw1 >= 0) wv.y = wk.y;
      }
      const float* d = s_dy[buf][r];
      #pragma unroll
      for (int m = 0; m < TOK; ++m) {
        acc[m].x = fmaf(wv.x, d[m], acc[m].x);
        acc[m].y = fmaf(wv.y, d[m], acc[m].y);
      }
    }
    if (st + 1 < st1) store(buf ^ 1);
    __syncthreads();
  }

  // the four row quarters, summed in the order 0, 1, 2, 3
  if (h > 0) {
    #pragma unroll
    for (int m = 0; m < TOK; ++m) s_red[h - 1][m][p] = acc[m];
  }
  __syncthreads();
  if (h == 0) {
    #pragma unroll
    for (int m = 0; m < TOK; ++m) {
      #pragma unroll
      for (int q = 0; q < 3; ++q) {
        acc[m].x += s_red[q][m][p].x;
        acc[m].y += s_red[q][m][p].y;
      }
    }
    if (S == 1) {
      #pragma unroll
      for (int m = 0; m < TOK; ++m)
        if (m < a.M)
          *reinterpret_cast<__half2*>(a.dx + (size_t)m * a.K + col) = __floats2half2_rn(acc[m].x, acc[m].y);
    } else {
      #pragma unroll
      for (int m = 0; m < TOK; ++m)
        *reinterpret_cast<float2*>(a.part + ((size_t)slice * kIgMaxTok + m) * a.K + col) = acc[m];
    }
  }
  if (S == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(a.count + b, 1u) == (unsigned)(S - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int e = tid; e < TOK * kBlockCodes; e += kIgThreads) {
    const int m = e / kBlockCodes, c = b * kBlockCodes + e % kBlockCodes;
    const float* src = a.part + (size_t)m * a.K + c;
    const size_t step = (size_t)kIgMaxTok * a.K;
    float sum = 0.f;
    int s = 0;
    for (; s + 4 <= S; s += 4) {   // four loads in flight, added in slice order
      const float v0 = __ldcg(src + s * step), v1 = __ldcg(src + (s + 1) * step);
      const float v2 = __ldcg(src + (s + 2) * step), v3 = __ldcg(src + (s + 3) * step);
      sum += v0;
      sum += v1;
      sum += v2;
      sum += v3;
    }
    for (; s < S; ++s) sum += __ldcg(src + s * step);
    if (m < a.M) a.dx[(size_t)m * a.K + c] = __float2half_rn(sum);
  }
  if (tid == 0) a.count[b] = 0u;   // ready for the next call on this stream
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

template <int BITS, int TOK>
cudaError_t launch_ig(const IgArgs& a, int slices, cudaStream_t s) {
  k_input_grad<BITS, TOK><<<dim3(a.K / kBlockCodes, slices), kIgThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_ig_tok(const IgArgs& a, int slices, cudaStream_t s) {
  if (a.M <= 1) return launch_ig<BITS, 1>(a, slices, s);
  if (a.M <= 2) return launch_ig<BITS, 2>(a, slices, s);
  if (a.M <= 4) return launch_ig<BITS, 4>(a, slices, s);
  if (a.M <= 8) return launch_ig<BITS, 8>(a, slices, s);
  return launch_ig<BITS, 16>(a, slices, s);
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
    k_weak_grad<<<grid, kWgThreads, 0, s>>>(x, dy, L.idx, dw, L.N, L.K, L.k, M);
    return cudaGetLastError();
  }
  __half* xw = reinterpret_cast<__half*>(L.wg_ws);
  float* part = splits > 1 ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(L.wg_ws) + xw_bytes) : nullptr;
  const size_t nxw = (size_t)M * kp;
  k_wg_gather<<<(unsigned)std::min<size_t>((nxw + 255) / 256, 4096), 256, 0, s>>>(x, M, L.K, L.idx, L.k, kp, xw);
  k_weak_grad_mma<<<dim3(R, C, splits), kWmThreads, 0, s>>>(dy, xw, splits > 1 ? part : dw, L.N, L.k, kp, M, per);
  if (splits > 1) {
    const size_t n = (size_t)L.N * L.k;
    k_wg_reduce<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, s>>>(part, splits, n, dw);
  }
  return cudaGetLastError();
}

cudaError_t launch_input_grad(Layer& L, const __half* dy, __half* dx, int M, cudaStream_t s) {
  const int Kb = L.K / kBlockCodes;
  const int nstages = ((L.N + 15) / 16 + 3) / 4;
  // two CTAs per SM (what the registers allow) over the column blocks and row slices, rounded
  // down so that the grid is one wave
  int slices = std::max(1, std::min(nstages, (2 * wct_sm_count(L.device)) / Kb));
  int per = (nstages + slices - 1) / slices;
  slices = (nstages + per - 1) / per;
  // workspace: one arrival counter per column block (zero between calls), then the partial sums
  const size_t cnt_bytes = ((size_t)Kb * sizeof(unsigned int) + 255) / 256 * 256;
  if (slices > 1) {
    const size_t need = cnt_bytes + (size_t)slices * kIgMaxTok * L.K * sizeof(float);
    if (need > L.ig_ws_bytes) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        slices = 1;   // no allocation inside a capture: one slice needs no workspace
      } else {
        cudaFree(L.ig_ws);
        L.ig_ws = nullptr;
        L.ig_ws_bytes = 0;
        if (cudaMalloc(&L.ig_ws, need) != cudaSuccess) {
          cudaGetLastError();
          L.ig_ws = nullptr;
          slices = 1;
        } else if (cudaMemsetAsync(L.ig_ws, 0, cnt_bytes, s) != cudaSuccess) {
          return cudaGetLastError();
        } else {
          L.ig_ws_bytes = need;
        }
      }
    }
  }
  if (slices == 1) per = nstages;
  IgArgs a;
  a.packed = L.packed;
  a.scales = L.scales;
  a.zeros = L.zeros;
  a.w_weak = L.w_weak;
  a.idx = L.idx;
  a.count = slices > 1 ? reinterpret_cast<unsigned int*>(L.ig_ws) : nullptr;
  a.part = slices > 1 ? reinterpret_cast<float*>(reinterpret_cast<char*>(L.ig_ws) + cnt_bytes) : nullptr;
  a.N = L.N;
  a.K = L.K;
  a.G = L.G;
  a.group = L.group;
  a.k = L.k;
  a.k_ld = L.k_ld;
  a.stages_per_slice = per;
  for (int m0 = 0; m0 < M; m0 += kIgMaxTok) {
    a.dy = dy + (size_t)m0 * L.N;
    a.dx = dx + (size_t)m0 * L.K;
    a.M = std::min(kIgMaxTok, M - m0);
    const cudaError_t e = L.bits == 3 ? launch_ig_tok<3>(a, slices, s) : launch_ig_tok<4>(a, slices, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace owq
