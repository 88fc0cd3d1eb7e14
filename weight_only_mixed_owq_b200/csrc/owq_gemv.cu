// Decode product y = W_hat x + W_weak x[idx] for 1 <= M <= 16 tokens, one launch.
//
// Pages: "Real-device acceleration" (OWQ paper "Acceleration on Real Device", p.6, as
// summarised on paperlayer.ai): a low-bit weight times fp16 activation product whose
// kernel also picks the weak-column activation channels on the fly; "Storage Methods"
// (appendix §2): the dense matrix is zero-filled at the weak columns, so the dense and
// weak terms simply add.
//
// Design (B200, HBM-bound at small M):
//  * A warp owns R consecutive output rows; its lanes split K in 128-code blocks
//    (bits x 16 bytes per row: `bits` 128-bit loads).  Warp-shuffle reduction at the end.
//  * Dequantisation never builds W_hat.  For a block with scale s and zero z,
//        sum_j W_hat_ij x_j  ~  s * (sum_j q_j x_j - z * sum_j x_j),
//    and q_j x_j is computed exactly: one AND lifts a code pair into an fp16x2 whose
//    halves equal q * 2^(o-24) (see owq_format.cuh), and fma.rn.f32.f16 multiplies
//    two fp16 values exactly into an fp32 accumulator (one accumulator per offset class,
//    rescaled by a power of two at the end of the block).  The per-block activation sums
//    are computed once per CTA into shared memory.
//  * The weak columns: the CTA gathers x[m, idx[t]] into shared memory once; each warp
//    then streams its rows of the fp16 weak block (128-bit loads) and adds the products
//    into the same fp32 sums before the reduction.  No second kernel.
#include "owq_internal.cuh"

namespace owq {
namespace {

constexpr int kMaxProblems = 16;
constexpr int kRowsPerCta = 16;  // a CTA covers 16 rows: R rows per warp x (16 / R) warps

struct GemvArgs {
  GemvProblem p[kMaxProblems];
  int count;
  int M;
};

__device__ __forceinline__ void fma_pair(float& acc, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc) : "r"(a), "r"(b));
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Accumulate one 32-code chunk (words w[0..BITS)) times the 16 activation pairs xp.
// Classes: 3-bit offsets {0,3,6} -> acc[0..2]; 4-bit offsets {0,4} -> acc[0..1].
template <int BITS>
__device__ __forceinline__ void chunk_fma(const uint32_t* w, const uint32_t* xp, float* acc) {
  if constexpr (BITS == 3) {
    #pragma unroll
    for (int j = 0; j < 3; ++j) {
      const uint32_t v = w[j], u = v >> 9;
      fma_pair(acc[0], v & 0x00070007u, xp[5 * j + 0]);
      fma_pair(acc[1], v & 0x00380038u, xp[5 * j + 1]);
      fma_pair(acc[2], v & 0x01C001C0u, xp[5 * j + 2]);
      fma_pair(acc[0], u & 0x00070007u, xp[5 * j + 3]);
      fma_pair(acc[1], u & 0x00380038u, xp[5 * j + 4]);
    }
    const uint32_t p15 = ((w[0] >> 15) & 0x00010001u) | ((w[1] >> 14) & 0x00020002u) |
                         ((w[2] >> 13) & 0x00040004u);
    fma_pair(acc[0], p15, xp[15]);
  } else {
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t v = w[j], u = v >> 8;
      fma_pair(acc[0], v & 0x000F000Fu, xp[4 * j + 0]);
      fma_pair(acc[1], v & 0x00F000F0u, xp[4 * j + 1]);
      fma_pair(acc[0], u & 0x000F000Fu, xp[4 * j + 2]);
      fma_pair(acc[1], u & 0x00F000F0u, xp[4 * j + 3]);
    }
  }
}

// sum_j q_j x_j of a block from the class accumulators (exact power-of-two rescales).
template <int BITS>
__device__ __forceinline__ float class_combine(const float* a) {
  if constexpr (BITS == 3) return 16777216.f * a[0] + 2097152.f * a[1] + 262144.f * a[2];
  else return 16777216.f * a[0] + 1048576.f * a[1];
}

template <int BITS, int R>
__device__ __forceinline__ void load_block(uint32_t (&w)[R][4 * BITS], const uint32_t* packed,
                                           const int* rows, size_t row_words, int b) {
  #pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint4* src = reinterpret_cast<const uint4*>(packed + (size_t)rows[r] * row_words) + (size_t)b * BITS;
    #pragma unroll
    for (int v = 0; v < BITS; ++v) {
      uint4 q = ldg_stream(src + v);
      w[r][4 * v] = q.x; w[r][4 * v + 1] = q.y; w[r][4 * v + 2] = q.z; w[r][4 * v + 3] = q.w;
    }
  }
}

template <int BITS, int MT, int R>
__global__ void __launch_bounds__(kRowsPerCta / R * 32)
k_gemv(const __grid_constant__ GemvArgs args) {
  constexpr int kWarps = kRowsPerCta / R;
  constexpr int NC = BITS == 3 ? 3 : 2;          // offset classes
  constexpr bool HOIST = MT <= 4;                // keep the x chunk of every token in registers
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int M = args.M;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // ---- which problem does this CTA serve (a CTA never spans two problems) ----
  int pi = 0;
  const int cta_group0 = blockIdx.x * kWarps;
  #pragma unroll 1
  for (int q = 1; q < args.count; ++q)
    if (cta_group0 >= args.p[q].group_base) pi = q;
  const GemvProblem& P = args.p[pi];
  const int K = P.K, Kb = K / kBlockCodes, G = P.G, k = P.k;
  const int groups_per_block = kBlockCodes * G / K;  // 1 if group == 128, else 0 (per-channel)

  // ---- this warp's rows; issue the first block's loads before the prologue ----
  const int rg = cta_group0 + warp - P.group_base;
  const bool active = rg < P.row_groups;
  const int row0 = rg * R;
  const size_t row_words = (size_t)K * BITS / 32;
  int rows[R];
  #pragma unroll
  for (int r = 0; r < R; ++r) rows[r] = min(row0 + r, P.N - 1);
  uint32_t w[R][4 * BITS];
  if (active && lane < Kb) load_block<BITS, R>(w, P.packed, rows, row_words, lane);

  // ---- CTA prologue: per-block activation sums and the weak-column gather ----
  float* sx = reinterpret_cast<float*>(smem_raw);               // [MT][Kb]
  __half* xw = reinterpret_cast<__half*>(sx + ((MT * Kb + 3) & ~3));  // [MT][k_ld], 16-B aligned
  for (int e = threadIdx.x; e < MT * Kb; e += blockDim.x) {
    const int m = e / Kb, b = e % Kb;
    float s = 0.f;
    if (m < M) {
      const uint4* xb = reinterpret_cast<const uint4*>(P.x + (size_t)m * K + (size_t)b * kBlockCodes);
      #pragma unroll 4
      for (int v = 0; v < kBlockCodes / 8; ++v) {
        uint4 q = ldg_nc(xb + v);
        const uint32_t h[4] = {q.x, q.y, q.z, q.w};
        #pragma unroll
        for (int u = 0; u < 4; ++u) {
          __half2 hh = *reinterpret_cast<const __half2*>(&h[u]);
          float2 f = __half22float2(hh);
          s += f.x;
          s += f.y;
        }
      }
    }
    sx[e] = s;
  }
  for (int e = threadIdx.x; e < MT * P.k_ld; e += blockDim.x) {
    const int m = e / P.k_ld, t = e % P.k_ld;
    xw[e] = (m < M && t < k) ? P.x[(size_t)m * K + P.idx[t]] : __float2half_rn(0.f);
  }
  __syncthreads();
  if (!active) return;

  float y[R][MT];
  #pragma unroll
  for (int r = 0; r < R; ++r)
    #pragma unroll
    for (int m = 0; m < MT; ++m) y[r][m] = 0.f;

  #pragma unroll 1
  for (int b = lane; b < Kb; b += 32) {
    // prefetch the next block of this lane while this one is computed
    uint32_t wn[R][4 * BITS];
    if (b + 32 < Kb) load_block<BITS, R>(wn, P.packed, rows, row_words, b + 32);
    float acc[R][MT][NC];
    #pragma unroll
    for (int r = 0; r < R; ++r)
      #pragma unroll
      for (int m = 0; m < MT; ++m)
        #pragma unroll
        for (int c = 0; c < NC; ++c) acc[r][m][c] = 0.f;

    #pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      if constexpr (HOIST) {
        uint32_t xp[MT][16];
        #pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int mm = min(m, M - 1);
          const uint4* xs = reinterpret_cast<const uint4*>(P.x + (size_t)mm * K + (size_t)b * kBlockCodes + ch * 32);
          #pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 q = ldg_nc(xs + v);
            xp[m][4 * v] = q.x; xp[m][4 * v + 1] = q.y; xp[m][4 * v + 2] = q.z; xp[m][4 * v + 3] = q.w;
          }
        }
        #pragma unroll
        for (int r = 0; r < R; ++r)
          #pragma unroll
          for (int m = 0; m < MT; ++m) chunk_fma<BITS>(&w[r][ch * BITS], xp[m], acc[r][m]);
      } else {
        #pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int mm = min(m, M - 1);
          const uint4* xs = reinterpret_cast<const uint4*>(P.x + (size_t)mm * K + (size_t)b * kBlockCodes + ch * 32);
          uint32_t xp[16];
          #pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 q = ldg_nc(xs + v);
            xp[4 * v] = q.x; xp[4 * v + 1] = q.y; xp[4 * v + 2] = q.z; xp[4 * v + 3] = q.w;
          }
          #pragma unroll
          for (int r = 0; r < R; ++r) chunk_fma<BITS>(&w[r][ch * BITS], xp, acc[r][m]);
        }
      }
    }
    // fold the block: s * (sum q x - z * sum x)
    const int gi = groups_per_block ? b : 0;
    #pragma unroll
    for (int r = 0; r < R; ++r) {
      const float s = __half2float(P.scales[(size_t)rows[r] * G + gi]);
      const float z = __half2float(P.zeros[(size_t)rows[r] * G + gi]);
      #pragma unroll
      for (int m = 0; m < MT; ++m)
        y[r][m] = fmaf(s, class_combine<BITS>(acc[r][m]) - z * sx[m * Kb + b], y[r][m]);
    }
    #pragma unroll
    for (int r = 0; r < R; ++r)
      #pragma unroll
      for (int v = 0; v < 4 * BITS; ++v) w[r][v] = wn[r][v];
  }

  // ---- weak columns: fp16 W_weak rows times the gathered activations ----
  #pragma unroll 1
  for (int t8 = lane; t8 * 8 < k; t8 += 32) {
    #pragma unroll
    for (int r = 0; r < R; ++r) {
      uint4 q = ldg_nc(P.w_weak + (size_t)rows[r] * P.k_ld + t8 * 8);
      const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
      #pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 xv4 = *reinterpret_cast<const uint4*>(xw + m * P.k_ld + t8 * 8);
        const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
        #pragma unroll
        for (int u = 0; u < 4; ++u) fma_pair(y[r][m], wv[u], xv[u]);
      }
    }
  }

  // ---- reduce over the lanes and store ----
  #pragma unroll
  for (int r = 0; r < R; ++r)
    #pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = y[r][m];
      #pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      y[r][m] = v;
    }
  if (lane == 0) {
    #pragma unroll
    for (int r = 0; r < R; ++r)
      if (row0 + r < P.N)
        #pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < M) P.y[(size_t)m * P.N + row0 + r] = __float2half_rn(y[r][m]);
  }
}

template <int MT> constexpr int rows_per_warp() { return MT <= 4 ? 4 : 2; }

template <int BITS, int MT>
cudaError_t launch_t(GemvArgs& a, cudaStream_t s) {
  constexpr int R = rows_per_warp<MT>();
  constexpr int kWarps = kRowsPerCta / R;
  int total_groups = 0;
  size_t smem = 0;
  for (int q = 0; q < a.count; ++q) {
    GemvProblem& P = a.p[q];
    P.row_groups = (P.N + R - 1) / R;
    // each problem starts on a CTA boundary so that a CTA serves one problem
    P.group_base = total_groups;
    total_groups += ((P.row_groups + kWarps - 1) / kWarps) * kWarps;
    size_t need = (size_t)((MT * (P.K / kBlockCodes) + 3) & ~3) * sizeof(float) +
                  (size_t)MT * P.k_ld * sizeof(__half);
    if (need > smem) smem = need;
  }
  smem = (smem + 15) & ~size_t(15);
  auto kern = k_gemv<BITS, MT, R>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)(total_groups / kWarps);
  kern<<<grid, kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(GemvArgs& a, cudaStream_t s) {
  const int M = a.M;
  if (M <= 1) return launch_t<BITS, 1>(a, s);
  if (M <= 2) return launch_t<BITS, 2>(a, s);
  if (M <= 4) return launch_t<BITS, 4>(a, s);
  if (M <= 8) return launch_t<BITS, 8>(a, s);
  return launch_t<BITS, 16>(a, s);
}

}  // namespace

cudaError_t launch_gemv(const GemvProblem* probs, int count, int bits, int M, cudaStream_t s) {
  if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
  GemvArgs a{};
  for (int q = 0; q < count; ++q) a.p[q] = probs[q];
  a.count = count;
  a.M = M;
  return bits == 3 ? launch_bits<3>(a, s) : launch_bits<4>(a, s);
}

}  // namespace owq
