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
//    8 blocks) items through a private S-stage shared-memory ring: the layer stores every
//    16-row tile block-major, so an item is one contiguous range and one cp.async.bulk,
//    completion counted on the stage's mbarrier.  About 150 KB per SM is in flight without
//    costing registers.
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
constexpr int kWarps = 16;
constexpr long long kWaitLimit = 4000000000LL;   // ~2 s

struct GemvArgs {
  GemvProblem p[kMaxProblems];
  int count;
  int M;
  int* status;   // device status word (bounded waits)
};

template <int BITS, int S>
struct Geo {
  static constexpr int kBlk = 16 * BITS;                       // bytes of one block of one row
  static constexpr int kTileBlk = 16 * kBlk;                   // one block of a 16-row tile (contiguous)
  static constexpr int kSub = 4;                               // blocks per ring stage
  static constexpr int kStage = kSub * kTileBlk;               // 3 KB (3-bit) / 4 KB (4-bit)
  static constexpr int kRing = kWarps * S * kStage;
  static constexpr int kBars = kWarps * S * 8;
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

// D += A * B, m16n8k16, f16 inputs, f32 accumulators (in place)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
               "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// sum_j q_j x_j from the class accumulators (exact power-of-two rescales)
template <int BITS>
__device__ __forceinline__ float combine(float a0, float a1, float a2) {
  if constexpr (BITS == 3) return 16777216.f * a0 + 2097152.f * a1 + 262144.f * a2;
  else return 16777216.f * a0 + 1048576.f * a1;
}

// Activations in fragment order: pair p = 4j + t of block b of token m is word
// (m * xstride + b * 64 + t * 16 + 4 ((j / 4) ^ t) + j % 4) -- lane t's sixteen pairs of a block
// are four 16-byte units, XOR-swizzled so that the four lanes t of a load hit four bank groups.
__device__ __forceinline__ int xi_word(int b, int t, int v) { return b * 64 + t * 16 + 4 * (v ^ t); }

// Per-block work of one warp: A fragments of rows g, g+8 from the staged tile, B fragments
// from the staged activations (xr: this lane's 64-byte unit row of block 0, xo: the four
// swizzled unit offsets), 8 k slices of m16n8k16 into the class accumulators.
template <int BITS, int NT, bool XSMEM>
__device__ __forceinline__ void block_mma(const unsigned char* frag, const uint32_t* const* xr, const int* xo,
                                          const __half* const* xg, int b, float (&D)[BITS == 3 ? 3 : 2][NT][4]) {
  constexpr int kBlk = 16 * BITS;
  uint32_t wa[BITS], wb[BITS];
  if constexpr (BITS == 4) {
    const uint4 qa = *reinterpret_cast<const uint4*>(frag);
    const uint4 qb = *reinterpret_cast<const uint4*>(frag + 8 * kBlk);
    wa[0] = qa.x; wa[1] = qa.y; wa[2] = qa.z; wa[3] = qa.w;
    wb[0] = qb.x; wb[1] = qb.y; wb[2] = qb.z; wb[3] = qb.w;
  } else {
    #pragma unroll
    for (int j = 0; j < BITS; ++j) {
      wa[j] = reinterpret_cast<const uint32_t*>(frag)[j];
      wb[j] = reinterpret_cast<const uint32_t*>(frag + 8 * kBlk)[j];
    }
  }
  uint32_t xb[NT][16];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if constexpr (XSMEM) {
      const uint32_t* base = xr[nt] + b * 64;
      #pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 q = *reinterpret_cast<const uint4*>(base + xo[v]);
        xb[nt][4 * v] = q.x; xb[nt][4 * v + 1] = q.y; xb[nt][4 * v + 2] = q.z; xb[nt][4 * v + 3] = q.w;
      }
    } else {
      const __half* base = xg[nt] + (size_t)b * kBlockCodes;
      #pragma unroll
      for (int j = 0; j < 16; ++j) xb[nt][j] = ldg_u32(base + 8 * j);
    }
  }
  #pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int cl = pair_class<BITS>(2 * s);
    const uint32_t a[4] = {pair_bits<BITS>(wa, 2 * s), pair_bits<BITS>(wb, 2 * s),
                           pair_bits<BITS>(wa, 2 * s + 1), pair_bits<BITS>(wb, 2 * s + 1)};
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma16816(D[cl][nt], a, xb[nt][2 * s], xb[nt][2 * s + 1]);
  }
}

template <int BITS, int NT>
__device__ __forceinline__ void zero_acc(float (&D)[BITS == 3 ? 3 : 2][NT][4]) {
  #pragma unroll
  for (int cl = 0; cl < (BITS == 3 ? 3 : 2); ++cl)
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i) D[cl][nt][i] = 0.f;
}

// P warps share a 16-row tile (each owns Kb / P consecutive blocks); the CTA's warps work on
// kWarps / P row tiles at a time (a "round").
template <int BITS, int NT, int S, int P, bool XSMEM, bool PG>
__global__ void __launch_bounds__(kWarps * 32, 1)
k_gemv_mma(const __grid_constant__ GemvArgs args) {
  using G_ = Geo<BITS, S>;
  constexpr int NC = BITS == 3 ? 3 : 2;      // offset classes
  constexpr int MT = 8 * NT;                 // token capacity
  constexpr int G8 = kWarps / P;             // row tiles per round
  constexpr int UNR = NT == 1 ? 2 : 1;       // blocks per loop iteration (independent accumulators)
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int M = args.M;
  const int gw = warp / P, pw = warp % P;    // row tile of the round, part of K

  int pi = 0;
  #pragma unroll 1
  for (int q = 1; q < args.count; ++q)
    if ((int)blockIdx.x >= args.p[q].cta_base) pi = q;
  const GemvProblem& Pb = args.p[pi];
  const int K = Pb.K, Kb = K / kBlockCodes, Gn = Pb.G, k = Pb.k, N = Pb.N, k_ld = Pb.k_ld;
  constexpr bool per_group = PG;             // one scale / zero per 128-code block
  const int xstride = K / 2 + 4;             // words per staged token row

  // shared memory carve-up (sizes computed identically on the host)
  unsigned char* ring = smem + warp * S * G_::kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G_::kRing) + warp * S;
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + G_::kRing) + kWarps * S;   // activations
  uint64_t* wbar = xbar + 1;                                                      // [2] weak rows per round
  float* red = reinterpret_cast<float*>(smem + G_::kRing + G_::kBars + 32);      // [2][warps][16][MT]
  float* sx = red + 2 * kWarps * 16 * MT;                                         // [MT][Kb]
  __half* xw = reinterpret_cast<__half*>(sx + ((MT * Kb + 3) & ~3));            // [MT][k_ld]
  __half* wk = xw + MT * k_ld;                                                    // [2][G8*16][k_ld]
  uint32_t* xs = reinterpret_cast<uint32_t*>(wk + 2 * G8 * 16 * k_ld);          // [M][xstride]

  // rounds of this CTA, this warp's block range
  const int c = (int)blockIdx.x - Pb.cta_base;
  const int RT = (N + 15) / 16;
  const int units = (RT + G8 - 1) / G8;
  const int n_rnd = c < units ? (units - c + Pb.ncta - 1) / Pb.ncta : 0;
  const int b_lo = pw * Kb / P, b_hi = (pw + 1) * Kb / P;
  const int nb = b_hi - b_lo;
  const int n_sub = nb > 0 ? (nb + G_::kSub - 1) / G_::kSub : 1;   // an empty range still takes one empty item
  const int T = n_rnd * n_sub;

  // the layer stores each 16-row tile block-major (owq_pack.cu), so an item -- 16 rows x nbs
  // consecutive blocks -- is one contiguous range: one bulk copy issued by lane 0
  auto issue = [&](int it) {
    const int st = it % S, rt = (c + (it / n_sub) * Pb.ncta) * G8 + gw, sub = it % n_sub;
    const int b0 = b_lo + sub * G_::kSub;
    const int nbs = rt < RT ? max(0, min(G_::kSub, b_hi - b0)) : 0;
    const uint32_t bytes = (uint32_t)(nbs * G_::kTileBlk);
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[st], bytes);
      if (bytes > 0) {
        const unsigned char* src = reinterpret_cast<const unsigned char*>(Pb.packed) +
                                   ((size_t)rt * Kb + b0) * G_::kTileBlk;
        bulk_load(ring + st * G_::kStage, src, bytes, &bars[st]);
      }
    }
  };
  // weak rows of the round's row tiles (consecutive rows of W_weak): one copy by thread 0
  auto issue_weak = [&](int rnd) {
    if (threadIdx.x != 0 || k == 0) return;
    const int row0 = (c + rnd * Pb.ncta) * G8 * 16;
    const int nrows = max(0, min(G8 * 16, N - row0));
    const uint32_t bytes = (uint32_t)(nrows * k_ld * 2);
    mbar_arrive_expect_tx(&wbar[rnd & 1], bytes);
    if (bytes > 0) bulk_load(wk + (rnd & 1) * G8 * 16 * k_ld, Pb.w_weak + (size_t)row0 * k_ld, bytes, &wbar[rnd & 1]);
  };
  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&bars[st], 1);
    if (warp == 0) { mbar_init(xbar, 1); mbar_init(&wbar[0], 1); mbar_init(&wbar[1], 1); }
    fence_mbar_init();
  }
  __syncthreads();   // every barrier initialised before any thread waits on one
  int issued = 0;
  for (; issued < min(S, T); ++issued) issue(issued);
  if (n_rnd > 0) issue_weak(0);
  if (n_rnd > 1) issue_weak(1);
  // the weights do not depend on the previous kernel in the stream: let the next one start
  // and only now wait for the previous one before touching activations or outputs
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- CTA prologue: activations into shared memory (one bulk copy per token row), the
  //      per-block activation sums, the weak-column gather, then the activations are permuted
  //      in place into fragment order ----
  if constexpr (XSMEM) {
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(xbar, (uint32_t)(M * K * 2));
      for (int m = 0; m < M; ++m) bulk_load(xs + m * xstride, Pb.x + (size_t)m * K, (uint32_t)(K * 2), xbar);
    }
    mbar_wait(xbar, 0, args.status, kWaitLimit);
  }
  {
    const int pieces = M * Kb * 16;
    for (int p0 = 0; p0 < pieces; p0 += blockDim.x) {
      const int p = p0 + threadIdx.x;
      float v = 0.f;
      if (p < pieces) {
        const int m = p / (Kb * 16), rem = p % (Kb * 16);
        uint4 q;
        if constexpr (XSMEM) q = *reinterpret_cast<const uint4*>(xs + m * xstride + rem * 4);
        else q = ldg_u128(Pb.x + (size_t)m * K + (size_t)rem * 8);
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
  }
  for (int e = threadIdx.x; e < MT * k_ld; e += blockDim.x) {
    const int m = e / k_ld, t = e % k_ld;
    __half v = __float2half_rn(0.f);
    if (m < M && t < k) {
      const int col = Pb.idx[t];
      if constexpr (XSMEM) v = reinterpret_cast<const __half*>(xs + m * xstride)[col];
      else v = Pb.x[(size_t)m * K + col];
    }
    xw[e] = v;
  }
  if constexpr (XSMEM) {
    __syncthreads();   // sums and gather read the natural order
    for (int e = threadIdx.x; e < M * Kb; e += blockDim.x) {
      uint32_t* blk = xs + (e / Kb) * xstride + (e % Kb) * 64;
      uint32_t w[64];
      #pragma unroll
      for (int v = 0; v < 16; ++v) {
        const uint4 q = reinterpret_cast<const uint4*>(blk)[v];
        w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
      }
      #pragma unroll
      for (int t = 0; t < 4; ++t)
        #pragma unroll
        for (int v = 0; v < 4; ++v)   // pairs j = 4v .. 4v+3 of lane t: p = 4j + t
          *reinterpret_cast<uint4*>(blk + t * 16 + 4 * (v ^ t)) =
              make_uint4(w[4 * (4 * v) + t], w[4 * (4 * v + 1) + t], w[4 * (4 * v + 2) + t], w[4 * (4 * v + 3) + t]);
    }
  }
  __syncthreads();

  // activation sums over this warp's block range (per-channel fold), tokens 2tig, 2tig+1 (+8);
  // tokens >= M only feed outputs that are never stored
  float sxw[NT][2];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    #pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = min(8 * nt + 2 * tig + e, M - 1);
      float v = 0.f;
      for (int b = b_lo; b < b_hi; ++b) v += sx[tok * Kb + b];
      sxw[nt][e] = v;
    }
  // per-lane operand pointers (tokens >= M are clamped: their columns are discarded)
  const uint32_t* xr[NT];
  const __half* xg[NT];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = min(8 * nt + g, M - 1);
    xr[nt] = xs + tok * xstride + tig * 16;
    xg[nt] = Pb.x + (size_t)tok * K + 2 * tig;
  }
  int xo[4];
  #pragma unroll
  for (int v = 0; v < 4; ++v) xo[v] = 4 * (v ^ tig);
  const int frag_lane = g * G_::kBlk + tig * 4 * BITS;

  float y[NT][4];
  int it = 0, fail_it = -1;
  bool ok = true;
  #pragma unroll 1
  for (int rnd = 0; rnd < n_rnd; ++rnd) {
    const int rt = (c + rnd * Pb.ncta) * G8 + gw;
    const bool live = rt < RT;
    const int row_a = min(rt * 16 + g, N - 1), row_b = min(rt * 16 + g + 8, N - 1);
    float sa = 0.f, za = 0.f, sb = 0.f, zb = 0.f;    // per-channel scale / zero, used at the end
    if (!per_group && live) {
      sa = __half2float(Pb.scales[row_a]); za = __half2float(Pb.zeros[row_a]);
      sb = __half2float(Pb.scales[row_b]); zb = __half2float(Pb.zeros[row_b]);
    }
    float D[UNR][NC][NT][4];
    #pragma unroll
    for (int u = 0; u < UNR; ++u) zero_acc<BITS, NT>(D[u]);
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i) y[nt][i] = 0.f;

    // per-group fold of one block's accumulators
    auto fold = [&](float (&Du)[NC][NT][4], int b) {
      const float gsa = __half2float(Pb.scales[(size_t)row_a * Gn + b]);
      const float gza = __half2float(Pb.zeros[(size_t)row_a * Gn + b]);
      const float gsb = __half2float(Pb.scales[(size_t)row_b * Gn + b]);
      const float gzb = __half2float(Pb.zeros[(size_t)row_b * Gn + b]);
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = min(8 * nt + 2 * tig + (i & 1), M - 1);
          const float v = combine<BITS>(Du[0][nt][i], Du[1][nt][i], Du[NC - 1][nt][i]);
          const float sc = i < 2 ? gsa : gsb, z = i < 2 ? gza : gzb;
          y[nt][i] = fmaf(sc, fmaf(-z, sx[tok * Kb + b], v), y[nt][i]);
        }
    };

    #pragma unroll 1
    for (int sub = 0; sub < n_sub; ++sub, ++it) {
      const int st = it % S;
      if (ok) {
        const bool ok_lane = mbar_wait(&bars[st], (uint32_t)((it / S) & 1), args.status, kWaitLimit);
        ok = __all_sync(0xffffffffu, ok_lane);
        if (!ok) fail_it = it;
      }
      const int b0 = b_lo + sub * G_::kSub;
      const int nbs = (ok && live) ? max(0, min(G_::kSub, b_hi - b0)) : 0;
      const unsigned char* frag = ring + st * G_::kStage + frag_lane;
      if (nbs == G_::kSub) {
        // full item: all kSub blocks unrolled, UNR independent accumulator sets
        #pragma unroll
        for (int bb = 0; bb < G_::kSub; ++bb) {
          if (per_group) zero_acc<BITS, NT>(D[bb % UNR]);
          block_mma<BITS, NT, XSMEM>(frag + bb * G_::kTileBlk, xr, xo, xg, b0 + bb, D[bb % UNR]);
          if (per_group) fold(D[bb % UNR], b0 + bb);
        }
      } else {
        #pragma unroll 1
        for (int bb = 0; bb < nbs; ++bb) {
          if (per_group) zero_acc<BITS, NT>(D[0]);
          block_mma<BITS, NT, XSMEM>(frag + bb * G_::kTileBlk, xr, xo, xg, b0 + bb, D[0]);
          if (per_group) fold(D[0], b0 + bb);
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
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = combine<BITS>(D[0][0][nt][i], D[0][1][nt][i], D[0][NC - 1][nt][i]);
          if constexpr (UNR == 2) v += combine<BITS>(D[1][0][nt][i], D[1][1][nt][i], D[1][NC - 1][nt][i]);
          const float sc = i < 2 ? sa : sb, z = i < 2 ? za : zb;
          y[nt][i] = sc * fmaf(-z, sxw[nt][i & 1], v);
        }
    }
    if (k > 0) {
      const bool ok_w = mbar_wait(&wbar[rnd & 1], (uint32_t)((rnd >> 1) & 1), args.status, kWaitLimit);
      if (live && ok_w) {
        const __half* wr = wk + (size_t)((rnd & 1) * G8 * 16 + gw * 16 + g) * k_ld + 2 * tig;
        #pragma unroll 1
        for (int ws = pw; ws * 16 < k; ws += P) {
          const uint32_t a[4] = {*reinterpret_cast<const uint32_t*>(wr + 16 * ws),
                                 *reinterpret_cast<const uint32_t*>(wr + 8 * k_ld + 16 * ws),
                                 *reinterpret_cast<const uint32_t*>(wr + 16 * ws + 8),
                                 *reinterpret_cast<const uint32_t*>(wr + 8 * k_ld + 16 * ws + 8)};
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const __half* xr = xw + (8 * nt + g) * k_ld + 16 * ws + 2 * tig;
            mma16816(y[nt], a, *reinterpret_cast<const uint32_t*>(xr), *reinterpret_cast<const uint32_t*>(xr + 8));
          }
        }
      }
    }
    float* rbuf = red + (size_t)(rnd & 1) * kWarps * 16 * MT + (size_t)warp * 16 * MT;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        rbuf[(g + 8 * (i >> 1)) * MT + 8 * nt + 2 * tig + (i & 1)] = y[nt][i];
    __syncthreads();
    // the weak buffer of this round is free again: fetch the round after next into it
    if (rnd + 2 < n_rnd) {
      if (threadIdx.x == 0) fence_proxy_async_smem();
      issue_weak(rnd + 2);
    }
    // reduce: thread -> (row tile of the round, row, token), sum over the P warps of that tile
    for (int e = threadIdx.x; e < G8 * 16 * MT; e += blockDim.x) {
      const int tg = e / (16 * MT), r = (e / MT) % 16, tok = e % MT;
      const int rtile = (c + rnd * Pb.ncta) * G8 + tg;
      const float* rs = red + (size_t)(rnd & 1) * kWarps * 16 * MT + (size_t)(tg * P) * 16 * MT + r * MT + tok;
      float v = 0.f;
      #pragma unroll
      for (int w = 0; w < P; ++w) v += rs[w * 16 * MT];
      const int row = rtile * 16 + r;
      if (ok && rtile < RT && row < N && tok < M) Pb.y[(size_t)tok * N + row] = __float2half_rn(v);
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

template <int BITS, int NT, int S, int P, bool XSMEM>
cudaError_t launch_k(GemvArgs& a, size_t smem, cudaStream_t s) {
  auto kern = a.p[0].G > 1 ? k_gemv_mma<BITS, NT, S, P, XSMEM, true> : k_gemv_mma<BITS, NT, S, P, XSMEM, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int base = 0;
  for (int q = 0; q < a.count; ++q) base += a.p[q].ncta;
  // programmatic dependent launch: this kernel may start while the previous one in the stream
  // drains; it waits (griddepcontrol.wait) before reading activations or writing outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(base);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int BITS, int NT, int P>
cudaError_t launch_p(GemvArgs& a, cudaStream_t s) {
  constexpr int MT = 8 * NT;
  constexpr int G8 = kWarps / P;
  constexpr size_t kMaxSmem = 232448;
  const int C = sm_count();
  long long work[kMaxProblems], total = 0;
  size_t extra = 0, xbytes = 0;
  for (int q = 0; q < a.count; ++q) {
    GemvProblem& Pq = a.p[q];
    const int Kb = Pq.K / kBlockCodes;
    Pq.row_groups = ((Pq.N + 15) / 16 + G8 - 1) / G8;        // CTA rounds of work
    work[q] = (long long)Pq.row_groups * Kb;
    total += work[q];
    const size_t need = (size_t)((MT * Kb + 3) & ~3) * sizeof(float) + (size_t)MT * Pq.k_ld * sizeof(__half) +
                        (size_t)2 * G8 * 16 * Pq.k_ld * sizeof(__half);
    if (need > extra) extra = need;
    const size_t xb = (size_t)a.M * (Pq.K / 2 + 4) * sizeof(uint32_t);
    if (xb > xbytes) xbytes = xb;
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
  // shared memory: ring + barriers + reduction + sums / gather / weak rows (+ staged activations)
  auto smem_for = [&](int S, bool xs) {
    const size_t ring = (size_t)kWarps * S * Geo<BITS, 1>::kStage;
    return ring + (size_t)kWarps * S * 8 + 32 + (size_t)2 * kWarps * 16 * MT * sizeof(float) +
           ((extra + 15) & ~size_t(15)) + (xs ? xbytes : 0);
  };
  if (smem_for(3, true) <= kMaxSmem) return launch_k<BITS, NT, 3, P, true>(a, smem_for(3, true), s);
  if (smem_for(2, true) <= kMaxSmem) return launch_k<BITS, NT, 2, P, true>(a, smem_for(2, true), s);
  if (smem_for(3, false) <= kMaxSmem) return launch_k<BITS, NT, 3, P, false>(a, smem_for(3, false), s);
  if (smem_for(2, false) <= kMaxSmem) return launch_k<BITS, NT, 2, P, false>(a, smem_for(2, false), s);
  return cudaErrorInvalidValue;
}

template <int BITS, int NT>
cudaError_t launch_t(GemvArgs& a, cudaStream_t s) {
  // warps per 16-row tile: as few as possible (more K per warp) while the rounds still cover
  // every SM once
  int rt_total = 0;
  for (int q = 0; q < a.count; ++q) rt_total += (a.p[q].N + 15) / 16;
  const int C = sm_count();
  if (rt_total >= 4 * C) return launch_p<BITS, NT, 4>(a, s);
  if (rt_total >= 2 * C) return launch_p<BITS, NT, 8>(a, s);
  return launch_p<BITS, NT, 16>(a, s);
}

template <int BITS>
cudaError_t launch_bits(GemvArgs& a, cudaStream_t s) {
  return a.M <= 8 ? launch_t<BITS, 1>(a, s) : launch_t<BITS, 2>(a, s);
}

}  // namespace

cudaError_t launch_gemv(const GemvProblem* probs, int count, int bits, int M, cudaStream_t s) {
  if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
  // one launch serves layers of one kind (per-channel or per-group scales)
  for (int q = 1; q < count; ++q)
    if ((probs[q].G > 1) != (probs[0].G > 1)) {
      for (int j = 0; j < count; ++j) {
        cudaError_t e = launch_gemv(probs + j, 1, bits, M, s);
        if (e != cudaSuccess) return e;
      }
      return cudaSuccess;
    }
  GemvArgs a{};
  for (int q = 0; q < count; ++q) a.p[q] = probs[q];
  a.count = count;
  a.M = M;
  a.status = device_status_ptr();
  if (!a.status) return cudaErrorInvalidDevicePointer;
  return bits == 3 ? launch_bits<3>(a, s) : launch_bits<4>(a, s);
}

}  // namespace owq
