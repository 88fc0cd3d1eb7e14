// Decode product y = W_hat x + W_weak x[idx] for 1 <= M <= 16 tokens, one launch.
//
// Pages: "Real-device acceleration" (OWQ paper "Acceleration on Real Device", p.6, as
// summarised on paperlayer.ai): a low-bit weight x fp16 activation product whose kernel also
// picks the weak-column activation channels on the fly; "Storage Methods" (appendix §2): the
// dense matrix is zero-filled at the weak columns, so the dense and weak terms simply add.
//
// Design (B200, HBM-bound):
//  * Persistent CTAs, one per SM, 8 warps.  A CTA walks 16-row tiles of W; its warps split
//    K into 8 contiguous ranges of 128-code blocks.  Each warp streams its (16 rows x up to
//    kSub blocks) sub-tiles through a private S-stage shared-memory ring filled by
//    cp.async.bulk (one copy per row, completion counted on the stage's mbarrier), so about
//    150 KB per SM is in flight without costing registers.
//  * The contraction runs on the tensor cores (mma.sync m16n8k16, fp16 x fp16 -> fp32): with
//    the packed layout of owq_format.cuh a lane's chunk of a block is exactly its A fragment,
//    and one AND per code pair makes each A register (the codes as exact fp16 values
//    q * 2^(o - 24), o the bit offset; one accumulator per offset class).  Activations are
//    the B fragment (up to 8 tokens per n8 tile, two tiles for M > 8).  This keeps the issued
//    work below one instruction per code, which CUDA-core FMAs cannot reach.
//  * Scale and zero point: for a group with scale s and zero z,
//        sum_j s (q_j - z) x_j = s * (sum_j q_j x_j - z * sum_j x_j);
//    the per-block activation sums are computed once per CTA.  Per-channel layers fold once
//    per row tile, per-group layers once per block.  (The exact fp16 rounding of each
//    s (q - z) is not applied; the difference is far inside the output tolerance.)
//  * Weak columns: the fp16 weak block is the A operand of extra k slices (exact fp16
//    products) against the activations gathered once per CTA into shared memory.
//  * The 8 warps' partial sums of a row tile are added in shared memory; one fp16 rounding
//    per output.
#include "owq_format.cuh"
#include "owq_internal.cuh"
#include "owq_sm100.cuh"

namespace owq {
namespace {

using namespace sm100;

constexpr int kMaxProblems = 16;
constexpr int kWarps = 8;
constexpr long long kWaitLimit = 4000000000LL;   // ~2 s

struct GemvArgs {
  GemvProblem p[kMaxProblems];
  int count;
  int M;
  int* status;   // device status word (bounded waits)
};

template <int BITS>
struct Geo {
  static constexpr int kBlk = 16 * BITS;                       // bytes of one block of one row
  static constexpr int kSub = BITS == 3 ? 8 : 4;               // blocks per ring stage
  // padded row stride: the 32 lanes' fragment loads of one stage hit 32 distinct banks
  static constexpr int kRowStride = BITS == 3 ? 400 : 320;
  static constexpr int kStage = 16 * kRowStride;
  static constexpr int kS = BITS == 3 ? 3 : 4;                 // stages per warp
  static constexpr int kRing = kWarps * kS * kStage;
  static constexpr int kBars = kWarps * kS * 8;
};

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ldg_u128(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// D = A * B + C, m16n8k16, f16 inputs, f32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                         const float (&c)[4]) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
               "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
               : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
                 "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// sum_j q_j x_j from the class accumulators (exact power-of-two rescales)
template <int BITS>
__device__ __forceinline__ float combine(float a0, float a1, float a2) {
  if constexpr (BITS == 3) return 16777216.f * a0 + 2097152.f * a1 + 262144.f * a2;
  else return 16777216.f * a0 + 1048576.f * a1;
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kWarps * 32, 1)
k_gemv_mma(const __grid_constant__ GemvArgs args) {
  using G_ = Geo<BITS>;
  constexpr int S = G_::kS;
  constexpr int NC = BITS == 3 ? 3 : 2;      // offset classes
  constexpr int MT = 8 * NT;                 // token capacity
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int M = args.M;

  int pi = 0;
  #pragma unroll 1
  for (int q = 1; q < args.count; ++q)
    if ((int)blockIdx.x >= args.p[q].cta_base) pi = q;
  const GemvProblem& P = args.p[pi];
  const int K = P.K, Kb = K / kBlockCodes, Gn = P.G, k = P.k, N = P.N;
  const bool per_group = Gn > 1;
  const size_t row_bytes = (size_t)K * BITS / 8;

  unsigned char* ring = smem + warp * S * G_::kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G_::kRing) + warp * S;
  float* red = reinterpret_cast<float*>(smem + G_::kRing + G_::kBars);          // [2][warps][16][MT]
  float* sx = red + 2 * kWarps * 16 * MT;                                        // [MT][Kb]
  __half* xw = reinterpret_cast<__half*>(sx + ((MT * Kb + 3) & ~3));           // [MT][k_ld]

  // this CTA's row tiles and this warp's block range
  const int c = (int)blockIdx.x - P.cta_base;
  const int RT = (N + 15) / 16;
  const int n_rt = c < RT ? (RT - c + P.ncta - 1) / P.ncta : 0;
  const int b_lo = warp * Kb / kWarps, b_hi = (warp + 1) * Kb / kWarps;
  const int nb = b_hi - b_lo;
  const int n_sub = nb > 0 ? (nb + G_::kSub - 1) / G_::kSub : 1;   // an empty range still takes one empty item
  const int T = n_rt * n_sub;

  auto issue = [&](int it) {   // called by the whole warp
    const int st = it % S, rt = c + (it / n_sub) * P.ncta, sub = it % n_sub;
    const int b0 = b_lo + sub * G_::kSub;
    const int nbs = max(0, min(G_::kSub, b_hi - b0));
    const int nrows = min(16, N - rt * 16);
    const uint32_t bytes = (uint32_t)(nbs * G_::kBlk);
    if (lane == 0) mbar_arrive_expect_tx(&bars[st], bytes * (uint32_t)nrows);
    __syncwarp();
    if (lane < nrows && bytes > 0) {
      const unsigned char* src = reinterpret_cast<const unsigned char*>(P.packed) +
                                 (size_t)(rt * 16 + lane) * row_bytes + (size_t)b0 * G_::kBlk;
      bulk_load(ring + st * G_::kStage + lane * G_::kRowStride, src, bytes, &bars[st]);
    }
  };
  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  int issued = 0;
  for (; issued < min(S, T); ++issued) issue(issued);

  // ---- CTA prologue: per-block activation sums (16 lanes per block) and the weak gather ----
  const int pieces = MT * Kb * 16;
  for (int p0 = 0; p0 < pieces; p0 += blockDim.x) {
    const int p = p0 + threadIdx.x;
    float v = 0.f;
    const int m = p / (Kb * 16), rem = p % (Kb * 16);
    if (p < pieces && m < M) {
      const uint4 q = ldg_u128(P.x + (size_t)m * K + (size_t)rem * 8);
      const uint32_t h[4] = {q.x, q.y, q.z, q.w};
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[u]));
        v += f.x;
        v += f.y;
      }
    }
    #pragma unroll
    for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (p < pieces && (p & 15) == 0) sx[p >> 4] = v;
  }
  for (int e = threadIdx.x; e < MT * P.k_ld; e += blockDim.x) {
    const int m = e / P.k_ld, t = e % P.k_ld;
    xw[e] = (m < M && t < k) ? P.x[(size_t)m * K + P.idx[t]] : __float2half_rn(0.f);
  }
  __syncthreads();

  // activation sums over this warp's block range (per-channel fold), tokens 2tig, 2tig+1 (+8)
  float sxw[NT][2];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    #pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = 8 * nt + 2 * tig + e;
      float v = 0.f;
      for (int b = b_lo; b < b_hi; ++b) v += sx[tok * Kb + b];
      sxw[nt][e] = v;
    }

  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
  float D[NC][NT][4];
  float y[NT][4];
  int it = 0, fail_it = -1;
  bool ok = true;
  #pragma unroll 1
  for (int rti = 0; rti < n_rt; ++rti) {
    const int rt = c + rti * P.ncta;
    const int row_a = min(rt * 16 + g, N - 1), row_b = min(rt * 16 + g + 8, N - 1);
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        y[nt][i] = 0.f;
        #pragma unroll
        for (int cl = 0; cl < NC; ++cl) D[cl][nt][i] = 0.f;
      }
    #pragma unroll 1
    for (int sub = 0; sub < n_sub; ++sub, ++it) {
      const int st = it % S;
      if (ok) {
        const bool ok_lane = mbar_wait(&bars[st], (uint32_t)((it / S) & 1), args.status, kWaitLimit);
        ok = __all_sync(0xffffffffu, ok_lane);
        if (!ok) fail_it = it;
      }
      const int b0 = b_lo + sub * G_::kSub;
      const int nbs = ok ? max(0, min(G_::kSub, b_hi - b0)) : 0;
      const unsigned char* stage = ring + st * G_::kStage;
      #pragma unroll 1
      for (int bb = 0; bb < nbs; ++bb) {
        const int b = b0 + bb;
        // A fragments: chunk tig of rows g and g + 8
        uint32_t wa[BITS], wb[BITS];
        {
          const unsigned char* ra = stage + g * G_::kRowStride + bb * G_::kBlk + tig * 4 * BITS;
          const unsigned char* rb = ra + 8 * G_::kRowStride;
          if constexpr (BITS == 4) {
            const uint4 qa = *reinterpret_cast<const uint4*>(ra);
            const uint4 qb = *reinterpret_cast<const uint4*>(rb);
            wa[0] = qa.x; wa[1] = qa.y; wa[2] = qa.z; wa[3] = qa.w;
            wb[0] = qb.x; wb[1] = qb.y; wb[2] = qb.z; wb[3] = qb.w;
          } else {
            #pragma unroll
            for (int j = 0; j < BITS; ++j) {
              wa[j] = reinterpret_cast<const uint32_t*>(ra)[j];
              wb[j] = reinterpret_cast<const uint32_t*>(rb)[j];
            }
          }
        }
        // B fragments: activation pairs p = 4j + tig of block b, token 8nt + g
        uint32_t xb[NT][16];
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tok = 8 * nt + g;
          if (tok < M) {
            const __half* xr = P.x + (size_t)tok * K + (size_t)b * kBlockCodes + 2 * tig;
            #pragma unroll
            for (int j = 0; j < 16; ++j) xb[nt][j] = ldg_u32(xr + 8 * j);
          } else {
            #pragma unroll
            for (int j = 0; j < 16; ++j) xb[nt][j] = 0u;
          }
        }
        #pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int cl = pair_class<BITS>(2 * s);
          // the first k slice of each offset class in a block restarts its accumulator
          // when the layer has one scale per block (per-group)
          const bool first = BITS == 3 ? (s < 3) : (s < 2);
          const uint32_t a[4] = {pair_bits<BITS>(wa, 2 * s), pair_bits<BITS>(wb, 2 * s),
                                 pair_bits<BITS>(wa, 2 * s + 1), pair_bits<BITS>(wb, 2 * s + 1)};
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (per_group && first) mma16816(D[cl][nt], a, xb[nt][2 * s], xb[nt][2 * s + 1], zero4);
            else mma16816(D[cl][nt], a, xb[nt][2 * s], xb[nt][2 * s + 1], D[cl][nt]);
          }
        }
        if (per_group) {
          const float sa = __half2float(P.scales[(size_t)row_a * Gn + b]);
          const float za = __half2float(P.zeros[(size_t)row_a * Gn + b]);
          const float sb = __half2float(P.scales[(size_t)row_b * Gn + b]);
          const float zb = __half2float(P.zeros[(size_t)row_b * Gn + b]);
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float sxv = sx[(8 * nt + 2 * tig + (i & 1)) * Kb + b];
              const float v = combine<BITS>(D[0][nt][i], D[1][nt][i], D[NC - 1][nt][i]);
              const float sc = i < 2 ? sa : sb, z = i < 2 ? za : zb;
              y[nt][i] = fmaf(sc, fmaf(-z, sxv, v), y[nt][i]);
            }
        }
      }
      __syncwarp();
      if (ok && it + S < T) {
        if (lane == 0) fence_proxy_async_smem();
        issue(it + S);
        ++issued;
      }
    }

    // ---- this warp's part of the row tile is done: fold, weak columns, reduction ----
    if (!per_group) {
      const float sa = __half2float(P.scales[row_a]), za = __half2float(P.zeros[row_a]);
      const float sb = __half2float(P.scales[row_b]), zb = __half2float(P.zeros[row_b]);
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float v = combine<BITS>(D[0][nt][i], D[1][nt][i], D[NC - 1][nt][i]);
          const float sc = i < 2 ? sa : sb, z = i < 2 ? za : zb;
          y[nt][i] = sc * fmaf(-z, sxw[nt][i & 1], v);
        }
    }
    #pragma unroll 1
    for (int ws = warp; ws * 16 < k; ws += kWarps) {
      const __half* wr_a = P.w_weak + (size_t)row_a * P.k_ld + 16 * ws + 2 * tig;
      const __half* wr_b = P.w_weak + (size_t)row_b * P.k_ld + 16 * ws + 2 * tig;
      const uint32_t a[4] = {ldg_u32(wr_a), ldg_u32(wr_b), ldg_u32(wr_a + 8), ldg_u32(wr_b + 8)};
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const __half* xr = xw + (8 * nt + g) * P.k_ld + 16 * ws + 2 * tig;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(xr + 8);
        float dw[4];
        mma16816(dw, a, b0, b1, zero4);
        #pragma unroll
        for (int i = 0; i < 4; ++i) y[nt][i] += dw[i];
      }
    }
    float* rbuf = red + (size_t)(rti & 1) * kWarps * 16 * MT + (size_t)warp * 16 * MT;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        rbuf[(g + 8 * (i >> 1)) * MT + 8 * nt + 2 * tig + (i & 1)] = y[nt][i];
    __syncthreads();
    if ((int)threadIdx.x < 16 * MT) {
      const int r = threadIdx.x / MT, tok = threadIdx.x % MT;
      const float* rs = red + (size_t)(rti & 1) * kWarps * 16 * MT + r * MT + tok;
      float v = 0.f;
      #pragma unroll
      for (int w = 0; w < kWarps; ++w) v += rs[w * 16 * MT];
      const int row = rt * 16 + r;
      if (ok && row < N && tok < M) P.y[(size_t)tok * N + row] = __float2half_rn(v);
    }
  }
  // after a timeout: never exit with bulk copies still writing into this CTA's memory
  if (fail_it >= 0 && lane == 0)
    for (int j = fail_it; j < issued; ++j)
      mbar_wait(&bars[j % S], (uint32_t)((j / S) & 1), args.status, kWaitLimit);
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
  }
  return n;
}

template <int BITS, int NT>
cudaError_t launch_t(GemvArgs& a, cudaStream_t s) {
  using G_ = Geo<BITS>;
  constexpr int MT = 8 * NT;
  const int C = sm_count();
  long long work[kMaxProblems], total = 0;
  size_t extra = 0;
  for (int q = 0; q < a.count; ++q) {
    GemvProblem& P = a.p[q];
    const int Kb = P.K / kBlockCodes;
    P.row_groups = (P.N + 15) / 16;
    work[q] = (long long)P.row_groups * Kb;
    total += work[q];
    const size_t need = (size_t)((MT * Kb + 3) & ~3) * sizeof(float) + (size_t)MT * P.k_ld * sizeof(__half);
    if (need > extra) extra = need;
  }
  // CTAs per problem in proportion to its work, at least one each, one resident wave in total
  int n[kMaxProblems], used = 0, big = 0;
  for (int q = 0; q < a.count; ++q) {
    n[q] = max(1, min(a.p[q].row_groups, (int)(work[q] * C / total)));
    used += n[q];
    if (work[q] > work[big]) big = q;
  }
  while (used > C) {
    int q = 0;
    for (int j = 1; j < a.count; ++j) if (n[j] > n[q]) q = j;
    if (n[q] == 1) break;
    --n[q];
    --used;
  }
  if (used < C) {
    const int add = min(C - used, a.p[big].row_groups - n[big]);
    if (add > 0) { n[big] += add; used += add; }
  }
  int base = 0;
  for (int q = 0; q < a.count; ++q) {
    a.p[q].cta_base = base;
    a.p[q].ncta = n[q];
    base += n[q];
  }
  const size_t smem = (size_t)G_::kRing + G_::kBars + (size_t)2 * kWarps * 16 * MT * sizeof(float) +
                      ((extra + 15) & ~size_t(15));
  if (smem > 232448) return cudaErrorInvalidValue;
  auto kern = k_gemv_mma<BITS, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<base, kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(GemvArgs& a, cudaStream_t s) {
  return a.M <= 8 ? launch_t<BITS, 1>(a, s) : launch_t<BITS, 2>(a, s);
}

}  // namespace

cudaError_t launch_gemv(const GemvProblem* probs, int count, int bits, int M, cudaStream_t s) {
  if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
  GemvArgs a{};
  for (int q = 0; q < count; ++q) a.p[q] = probs[q];
  a.count = count;
  a.M = M;
  a.status = device_status_ptr();
  if (!a.status) return cudaErrorInvalidDevicePointer;
  return bits == 3 ? launch_bits<3>(a, s) : launch_bits<4>(a, s);
}

}  // namespace owq
