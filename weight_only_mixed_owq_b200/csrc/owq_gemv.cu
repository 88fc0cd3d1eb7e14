// Decode product y = W_hat x + W_weak x[idx] for 1 <= M <= 16 tokens, one launch.
//
// Pages: "Real-device acceleration" (OWQ paper "Acceleration on Real Device", p.6, as
// summarised on paperlayer.ai): a low-bit weight x fp16 activation product whose kernel also
// picks the weak-column activation channels on the fly; "Storage Methods" (appendix §2): the
// dense matrix is zero-filled at the weak columns, so the dense and weak terms simply add.
//
// Design (B200, HBM-bound):
//  * Work is the list of (16-row tile, 128-code block) units in row-tile order.  Every warp of
//    a persistent grid (one CTA of 16 warps per SM) takes one equal contiguous chunk of it
//    (stream-K), so no SM idles while another finishes and no warp waits for another: there
//    is no barrier after the prologue.
//  * A warp streams its chunk through a private S-stage shared-memory ring filled by
//    cp.async.bulk: the layer stores each 16-row tile block-major, so an item (16 rows x up to
//    4 or 8 blocks of one tile) is one contiguous copy; the weak block, stored tile-major too,
//    is streamed the same way at the start of each tile.  Every weight copy carries an
//    evict-first L2 hint: the weights are read once per call, the activations are not.
//  * The contraction runs on the tensor cores (mma.sync m16n8k16, fp16 x fp16 -> fp32): with
//    the packed layout of owq_format.cuh a lane's chunk of a block is exactly its A fragment,
//    and one AND per code pair makes each A register (the codes as exact fp16 values
//    q * 2^(o - 24), o the bit offset; one accumulator per offset class).  Activations are the
//    B fragment (up to 8 tokens per n8 tile, two tiles for M > 8), staged once per CTA in
//    fragment order.  This keeps the issued work per code low enough for the HBM rate.
//  * Scale and zero point, 1-8 tokens: for a group with scale s and zero z,
//        sum_j s (q_j - z) x_j = s * (sum_j q_j x_j - z * sum_j x_j);
//    the activation sums come from per-block prefix sums computed once per CTA (the product
//    of the unrounded dequantised weights).  9-16 tokens, and per-group layers from 4 tokens:
//    each code pair is dequantised in registers to fp16_rn(s (q - z)), the oracle's W_hat bit
//    for bit (two fp16x2 operations per pair, shared by the tokens), into one accumulator.
//  * A row tile split between warps: the segments inside one CTA leave their partial sums in
//    shared memory and the last to arrive (a CTA-scope counter) adds them in unit order; across
//    CTAs, each CTA's sum is published as 64-bit words tagged with the call's epoch (no counter
//    or fence) and the CTA holding the tile's last units adds them in CTA order.  Every sum
//    runs in a fixed order: the output is the same bit for bit on every call.
#include "owq_format.cuh"
#include "owq_internal.cuh"
#include "owq_sm100.cuh"

namespace owq {
namespace {

using namespace sm100;

constexpr int kMaxProblems = 16;
constexpr int kAhead = 2;                        // items in flight per warp (see GemvArgs::ahead)

struct GemvArgs {
  GemvProblem p[kMaxProblems];
  int count;
  int M;
  int ahead;     // ring items a warp keeps in flight beyond the one it is reading (1 .. S)
  uint32_t k2, k4;   // 2 and 4 (run-time values: see pair_bits)
  int* status;   // device status word (bounded waits)
  long long wait_limit;   // bound of every device wait, in SM clock cycles
};

template <int BITS, int SUB>   // SUB: blocks per ring item
struct Geo {
  static constexpr int kBlk = 16 * BITS;                       // bytes of one block of one row
  static constexpr int kTileBlk = 16 * kBlk;                   // one block of a 16-row tile
  static constexpr int kStageW = SUB * kTileBlk;               // weights of an item
  static constexpr int kWs = kStageW / 512;                    // weak k slices per item
  // a stage: the item's weights, then (per-group layers) its (scale, zero) pairs, 16 per block
  static constexpr int stage_bytes(bool pg) { return kStageW + (pg ? SUB * 64 : 0); }
};

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

template <int NCA, int NT>
__device__ __forceinline__ void zero_acc(float (&D)[NCA][NT][4]) {
  #pragma unroll
  for (int cl = 0; cl < NCA; ++cl)
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      #pragma unroll
      for (int i = 0; i < 4; ++i) D[cl][nt][i] = 0.f;
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_splat(__half h) {
  const uint32_t u = __half_as_ushort(h);
  return u | (u << 16);
}

// Dequantisation constants of the two rows (g, g + 8) a lane holds: the scale splat s and,
// per offset class c, -(1024 / 2^o_c + z) splat.  A code pair at offset o lifted as
// (bits | 0x6400) = 1024 + q 2^o per half gives (1024 + q 2^o) 2^-o - (1024 2^-o + z) = q - z
// exactly (one fma.rn.f16x2), then * s rounds once: W_hat = fp16_rn(s (q - z)) bit for bit.
template <int BITS>
struct RowDq {
  static constexpr int NC = BITS == 3 ? 3 : 2;
  uint32_t s2[2], nz[2][NC];
  __device__ __forceinline__ void set(int h, __half2 sz) {   // h: 0 = row g, 1 = row g + 8
    s2[h] = h2_splat(__low2half(sz));
    const float z = __half2float(__high2half(sz));
    #pragma unroll
    for (int c = 0; c < NC; ++c)
      nz[h][c] = h2_splat(__float2half_rn(-(1024.f / (float)(1 << class_off<BITS>(c)) + z)));
  }
};
template <int BITS>
__device__ __forceinline__ uint32_t class_scale(int c) {   // 2^-o_c splat (exact)
  return h2_splat(__float2half_rn(1.f / (float)(1 << class_off<BITS>(c))));
}


// One unit (one 128-code block of a 16-row tile) of one warp: A fragments of rows g, g+8
// from the staged tile (byte offset fa in shared memory: this lane's chunk), B fragments from
// the staged activations (byte offsets xv: this lane's four 16-byte fragment pieces of block 0,
// plus xoff for the block) or from global memory (xg, block b), then 8 k slices of m16n8k16
// into the offset-class accumulators (EXACT: each code pair first dequantised to
// fp16_rn(s (q - z)), one accumulator).  Shared memory is addressed as the kernel's shared
// array plus 32-bit offsets, so each load is one shared load at register + immediate.
template <int BITS, int NT, bool XSMEM, bool EXACT>
__device__ __forceinline__ void unit_mma(const unsigned char* sm, int fa, const int (&xv)[NT][4], int xoff,
                                         const uint4* const (&xg)[NT], int b, uint32_t k2, uint32_t k4,
                                         const RowDq<BITS>& dq, float (&D)[EXACT ? 1 : (BITS == 3 ? 3 : 2)][NT][4]) {
  constexpr int kBlk = 16 * BITS;
  uint32_t wa[BITS], wb[BITS];
  if constexpr (BITS == 4) {
    const uint4 qa = *reinterpret_cast<const uint4*>(sm + fa);
    const uint4 qb = *reinterpret_cast<const uint4*>(sm + fa + 8 * kBlk);
    wa[0] = qa.x; wa[1] = qa.y; wa[2] = qa.z; wa[3] = qa.w;
    wb[0] = qb.x; wb[1] = qb.y; wb[2] = qb.z; wb[3] = qb.w;
  } else {
    #pragma unroll
    for (int j = 0; j < BITS; ++j) {
      wa[j] = *reinterpret_cast<const uint32_t*>(sm + fa + 4 * j);
      wb[j] = *reinterpret_cast<const uint32_t*>(sm + fa + 8 * kBlk + 4 * j);
    }
  }
  uint32_t xb[NT][16];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if constexpr (XSMEM) {
      #pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 q = *reinterpret_cast<const uint4*>(sm + xv[nt][v] + xoff);
        xb[nt][4 * v] = q.x; xb[nt][4 * v + 1] = q.y; xb[nt][4 * v + 2] = q.z; xb[nt][4 * v + 3] = q.w;
      }
    } else {
      // fragment-ordered activations in global memory: this lane's 16 words of block b
      const uint4* base = xg[nt] + (size_t)b * 16;
      #pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 q = ldg_u128(base + v);
        xb[nt][4 * v] = q.x; xb[nt][4 * v + 1] = q.y; xb[nt][4 * v + 2] = q.z; xb[nt][4 * v + 3] = q.w;
      }
    }
  }
  constexpr uint32_t kMagic = 0x64006400u;
  #pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int cl = pair_class<BITS>(2 * s);   // (pairs 2s and 2s + 1 share the class)
    if constexpr (EXACT) {
      const uint32_t sc = class_scale<BITS>(cl);
      const uint32_t a[4] = {h2_mul(h2_fma(pair_bits<BITS>(wa, 2 * s, k2, k4) | kMagic, sc, dq.nz[0][cl]), dq.s2[0]),
                             h2_mul(h2_fma(pair_bits<BITS>(wb, 2 * s, k2, k4) | kMagic, sc, dq.nz[1][cl]), dq.s2[1]),
                             h2_mul(h2_fma(pair_bits<BITS>(wa, 2 * s + 1, k2, k4) | kMagic, sc, dq.nz[0][cl]), dq.s2[0]),
                             h2_mul(h2_fma(pair_bits<BITS>(wb, 2 * s + 1, k2, k4) | kMagic, sc, dq.nz[1][cl]), dq.s2[1])};
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma16816(D[0][nt], a, xb[nt][2 * s], xb[nt][2 * s + 1]);
    } else {
      (void)kMagic;
      const uint32_t a[4] = {pair_bits<BITS>(wa, 2 * s, k2, k4), pair_bits<BITS>(wb, 2 * s, k2, k4),
                             pair_bits<BITS>(wa, 2 * s + 1, k2, k4), pair_bits<BITS>(wb, 2 * s + 1, k2, k4)};
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma16816(D[cl][nt], a, xb[nt][2 * s], xb[nt][2 * s + 1]);
    }
  }
}

// Partial sums of split row tiles travel as 64-bit words (fp32 value in the low half, the
// call's epoch in the high half): a 64-bit access is single-copy atomic, so a reader sees
// either an older word or this call's complete value, and needs no fence or counter.
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, uint32_t epoch) {
  const unsigned long long w = (unsigned long long)__float_as_uint(v) | ((unsigned long long)epoch << 32);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" :: "l"(p), "l"(w) : "memory");
}
// Segments still expected by a row tile whose segments are all in this CTA: count down one,
// acquire-release at CTA scope (the segment's accumulator adds are released with it; the
// segment that reaches 0 acquires all of them).
__device__ __forceinline__ int count_down_cta(int* c) {
  int old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.s32 %0, [%1], -1;" : "=r"(old) : "r"(smem_u32(c)) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long ld_tagged(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

// The sequence of ring items of one warp's chunk [lo, hi) of (tile, block) units, walked from
// the top down: for every tile segment that contains the tile's block 0, first the weak k
// slices of the tile (kWs per item), then its blocks (up to `sub` per item, never crossing a
// tile).  Walking down, the top segment of a chunk (the lower part of a tile the next warp
// finishes) is published first and the bottom segment (the part that finishes a tile whose
// lower part the previous warp published first) comes last.  Producer and consumer each run
// their own copy, so they agree item by item.
struct ItemGen {
  int rt, bh, rem, wpos, nsl, Kb, wsi, sub;
  bool seg_end;   // the last item returned closes its tile segment
  __device__ void init(int hi, int units, int Kb_, int nsl_, int wsi_, int sub_) {
    Kb = Kb_; nsl = nsl_; wsi = wsi_; sub = sub_; rem = units; seg_end = false;
    rt = units > 0 ? (hi - 1) / Kb : 0;
    bh = hi - rt * Kb;
    wpos = (units > 0 && rem >= bh) ? 0 : nsl;   // the segment reaches block 0
  }
  // kind 0: weak slices [first, first + cnt) of tile rt_; kind 1: blocks [first, first + cnt)
  __device__ __forceinline__ bool next(int& kind, int& rt_, int& first, int& cnt) {
    if (rem <= 0) return false;
    rt_ = rt;
    seg_end = false;
    if (wpos < nsl) {
      kind = 0; first = wpos; cnt = min(wsi, nsl - wpos); wpos += cnt;
      return true;
    }
    kind = 1; cnt = min(sub, min(bh, rem)); first = bh - cnt;
    bh -= cnt; rem -= cnt;
    if (rem <= 0 || bh == 0) {
      seg_end = true;
      if (rem > 0) { --rt; bh = Kb; wpos = rem >= Kb ? 0 : nsl; }
    }
    return true;
  }
  __device__ __forceinline__ bool segment_done() const { return seg_end; }
};

// Activations too large for shared memory are written once per call, before the product, in
// fragment order: for token m, block b and lane t, the 16 words 4j + t (j = 0..15) of the
// block, contiguous ([m][b][t][16 words]), so a lane fetches its B fragments of a block with
// four 16-byte loads.
__global__ void k_x_frag(const __half* __restrict__ x, int M, int K, uint32_t* __restrict__ xf) {
  const int Kb = K / kBlockCodes;
  const size_t n = (size_t)M * Kb * 64;   // words
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t mb = e / 64;             // (token, block)
    const int w = (int)(e % 64), t = w / 16, j = w % 16;
    xf[e] = reinterpret_cast<const uint32_t*>(x)[mb * 64 + 4 * j + t];
  }
}

template <int BITS, int NT, int WARPS, int SUB, int S, bool XSMEM, bool PG, bool EXACT>
__global__ void __launch_bounds__(WARPS * 32, 1)
k_gemv_mma(const __grid_constant__ GemvArgs args) {
  constexpr int kWarps = WARPS;
  using G_ = Geo<BITS, SUB>;
  constexpr int NC = BITS == 3 ? 3 : 2;      // offset classes
  // EXACT (9-16 tokens; per-group layers from 4 tokens): each code pair is dequantised to
  // fp16_rn(s (q - z)) in registers, one accumulator, the cost shared by the tokens.
  // Otherwise the codes are multiplied as exact q 2^(o - 24) values into offset-class
  // accumulators and the scale and zero point are applied to the sums (fewer instructions
  // per code at 1 token).
  constexpr int NCA = EXACT ? 1 : NC;
  constexpr int MT = 8 * NT;                 // token capacity
  constexpr int kStage = G_::stage_bytes(PG);
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int M = args.M;

  int pi = 0;
  #pragma unroll 1
  for (int q = 1; q < args.count; ++q)
    if ((int)blockIdx.x >= args.p[q].cta_base) pi = q;
  const GemvProblem& Pb = args.p[pi];
  const int K = Pb.K, Kb = K / kBlockCodes, k = Pb.k, N = Pb.N, k_ld = Pb.k_ld;
  const int nsl = k > 0 ? k_ld / 16 : 0;     // weak k slices of a tile
  const int xstride = K / 2 + 4;             // words per staged token row
  const int RT = (N + 15) / 16;              // row tiles
  const int W = RT * Kb;                     // (tile, block) units
  const int c = Pb.chunk;
  const int ahead = min(args.ahead, S);
  const uint32_t k2 = args.k2, k4 = args.k4;

  // shared memory carve-up (sizes computed identically on the host)
  unsigned char* ring = smem + warp * S * kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * S * kStage) + warp * S;
  float* psx = reinterpret_cast<float*>(smem + kWarps * S * kStage + kWarps * S * 8 + 16);   // [MT][Kb+1] (!EXACT)
  __half* xw = reinterpret_cast<__half*>(psx + (EXACT ? 0 : ((MT * (Kb + 1) + 3) & ~3)));        // [MT][k_ld]
  uint32_t* xs = reinterpret_cast<uint32_t*>(xw + MT * k_ld);                                      // [M][xstride]
  // row tiles whose segments are all in this CTA: accumulators [lt][16][MT] and segment counts
  // split row tiles: early slots [min(lt_cap, warps)][16][MT] (indexed by tile, or by warp when
  // the CTA touches more tiles than it has warps: a warp walks at most one early segment) and
  // the segment counts of the tiles the CTA touches
  const int lcap = Pb.lt_cap;
  const bool by_tile = lcap <= kWarps;
  float* lacc = reinterpret_cast<float*>(xs + (XSMEM ? M * xstride : 0));
  int* lcnt = reinterpret_cast<int*>(lacc + (by_tile ? lcap : kWarps) * 16 * MT);
  const int cta_c0 = ((int)blockIdx.x - Pb.cta_base) * kWarps;   // first chunk of this CTA
  const int t_lo = min(cta_c0 * c, W) / Kb;                        // first tile it touches

  // this warp's chunk of units
  const int wi = ((int)blockIdx.x - Pb.cta_base) * kWarps + warp;
  const int lo = min(wi * c, W), hi = min(lo + c, W);
  const int b_top = hi > lo ? hi - ((hi - 1) / Kb) * Kb : 0;   // block end of the top segment
  ItemGen prod, cons;
  prod.init(hi, hi - lo, Kb, nsl, G_::kWs, SUB);
  cons.init(hi, hi - lo, Kb, nsl, G_::kWs, SUB);
  int issued = 0;
  uint64_t pol;   // the weights are read once per call: evict them from L2 first
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  // lane 0 only: the next item of the chunk into the next stage (false once the chunk is exhausted)
  auto issue = [&]() -> bool {
    int kind, rt, first, cnt;
    if (!prod.next(kind, rt, first, cnt)) return false;
    const int st = issued % S;
    const unsigned char* src;
    uint32_t bytes;
    if (kind == 0) {
      src = reinterpret_cast<const unsigned char*>(Pb.w_weak_t) + ((size_t)rt * nsl + first) * 512;
      bytes = (uint32_t)(cnt * 512);
    } else {
      src = reinterpret_cast<const unsigned char*>(Pb.packed) + ((size_t)rt * Kb + first) * G_::kTileBlk;
      bytes = (uint32_t)(cnt * G_::kTileBlk);
      if constexpr (PG) {
        mbar_arrive_expect_tx(&bars[st], bytes + (uint32_t)(cnt * 64));
        bulk_load_hint(ring + st * kStage + G_::kStageW, Pb.sz_t + ((size_t)rt * Kb + first) * 16, (uint32_t)(cnt * 64),
                       &bars[st], pol);
        bulk_load_hint(ring + st * kStage, src, bytes, &bars[st], pol);
        ++issued;
        return true;
      }
    }
    mbar_arrive_expect_tx(&bars[st], bytes);
    bulk_load_hint(ring + st * kStage, src, bytes, &bars[st], pol);
    ++issued;
    return true;
  };

  if (lane == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  for (int lt = threadIdx.x; lt < lcap; lt += blockDim.x) {   // segments of each split tile in this CTA
    const int t = t_lo + lt, cf = (t * Kb) / c, cl = ((t + 1) * Kb - 1) / c;
    lcnt[lt] = (t < RT && cl > cf) ? max(0, min(cl, cta_c0 + kWarps - 1) - max(cf, cta_c0) + 1) : 0;
  }
  // the weak-column indices are static: fetch this thread's before waiting for the previous
  // kernel (gather elements e = threadIdx.x + it * blockDim.x, it < 2, of [MT][k_ld])
  int gidx[2];
  #pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int e = it * blockDim.x + threadIdx.x;
    const int m = e / k_ld, t = e - m * k_ld;
    gidx[it] = (e < MT * k_ld && m < M && t < k) ? Pb.idx[t] : -1;
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the weights do not depend on the previous kernel: each warp's first item streams while this
  // CTA waits for it (the rest follow the activation loads)
  if (lane == 0) issue();
  // activations (and outputs) belong to the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- CTA prologue ----
  if constexpr (XSMEM) {
    // The activations: every 16-byte piece of the rows is loaded at once (so the whole load is
    // one round trip), the weight stream is issued behind these loads, then the pieces are
    // stored in fragment order: word 4j + t of a block, for lane t, goes to t*16 + 4((j/4) ^ t)
    // + j%4 (16-byte fragment loads spread over all banks).  The same pass forms the per-block
    // activation sums; the weak-column activations are gathered alongside.
    const int pieces = K / 8;   // 16-byte pieces of one token row; 16 per block
    const int total = M * pieces;
    constexpr int kPer = 16;    // pieces per thread per pass
    #pragma unroll 1
    for (int p0 = 0; p0 < total; p0 += kPer * (int)blockDim.x) {
      uint4 q[kPer];
      #pragma unroll
      for (int it = 0; it < kPer; ++it) {
        const int p = p0 + it * blockDim.x + threadIdx.x;
        if (p < total) q[it] = ldg_u128(Pb.x + (size_t)p * 8);
      }
      __half gx[2];
      if (p0 == 0) {
        #pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int e = it * blockDim.x + threadIdx.x;
          gx[it] = gidx[it] >= 0 && in_range(gidx[it], K, args.status) ? Pb.x[(size_t)(e / k_ld) * K + gidx[it]]
                                                                         : __float2half_rn(0.f);
        }
        if (lane == 0)
          for (int j = 1; j < ahead; ++j)
            if (!issue()) break;
        #pragma unroll
        for (int it = 0; it < 2; ++it) {
          const int e = it * blockDim.x + threadIdx.x;
          if (e < MT * k_ld) xw[e] = gx[it];
        }
      }
      #pragma unroll
      for (int it = 0; it < kPer; ++it) {
        if (p0 + it * (int)blockDim.x >= total) break;   // uniform: whole passes of the CTA
        const int p = p0 + it * blockDim.x + threadIdx.x;
        float v = 0.f;
        int m = 0, pp = 0;
        if (p < total) {
          m = p / pieces;
          pp = p - m * pieces;
          const uint32_t h[4] = {q[it].x, q[it].y, q[it].z, q[it].w};
          if constexpr (!EXACT) {
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[u]));
              v += f.x;
              v += f.y;
            }
          }
          uint32_t* blk = xs + m * xstride + (pp >> 4) * 64;
          const int j = pp & 15;
          #pragma unroll
          for (int t = 0; t < 4; ++t) blk[t * 16 + 4 * ((j >> 2) ^ t) + (j & 3)] = h[t];
        }
        if constexpr (!EXACT) {
          #pragma unroll
          for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (p < total && (pp & 15) == 0) psx[m * (Kb + 1) + (pp >> 4) + 1] = v;
        }
      }
    }
    #pragma unroll 1
    for (int e = 2 * blockDim.x + threadIdx.x; e < MT * k_ld; e += blockDim.x) {
      const int m = e / k_ld, t = e - m * k_ld;
      xw[e] = (m < M && t < k && in_range(Pb.idx[t], K, args.status)) ? Pb.x[(size_t)m * K + Pb.idx[t]]
                                                                       : __float2half_rn(0.f);
    }
  } else {
    // activations stay in global memory (fragment-ordered by k_x_frag): per-block sums (for
    // the offset-class products) and the weak-column gather only
    const int pieces = K / 8;
    const int total = EXACT ? 0 : M * pieces;
    if (EXACT && lane == 0)
      for (int j = 1; j < ahead; ++j)
        if (!issue()) break;
    #pragma unroll 4
    for (int p0 = 0; p0 < total; p0 += blockDim.x) {
      const int p = p0 + threadIdx.x;
      float v = 0.f;
      int m = 0, pp = 0;
      if (p < total) {
        m = p / pieces;
        pp = p - m * pieces;
        const uint4 q = ldg_u128(Pb.x + (size_t)p * 8);
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
      if (p < total && (pp & 15) == 0) psx[m * (Kb + 1) + (pp >> 4) + 1] = v;
      if (p0 == 0 && lane == 0)
        for (int j = 1; j < ahead; ++j)
          if (!issue()) break;
    }
    #pragma unroll 1
    for (int e = threadIdx.x; e < MT * k_ld; e += blockDim.x) {
      const int m = e / k_ld, t = e - m * k_ld;
      const int col = e < (int)blockDim.x ? gidx[0] : e < 2 * (int)blockDim.x ? gidx[1] : ((m < M && t < k) ? Pb.idx[t] : -1);
      xw[e] = col >= 0 && in_range(col, K, args.status) ? Pb.x[(size_t)m * K + col] : __float2half_rn(0.f);
    }
  }
  __syncthreads();
  #pragma unroll 1
  for (int tw = warp; tw < (EXACT ? 0 : MT); tw += kWarps) {   // prefix sums of the block sums, a warp per token (tokens >= M: zeros)
    float* row = psx + tw * (Kb + 1);
    const int per = (Kb + 31) / 32, b_lo = lane * per, b_hi = min(b_lo + per, Kb);
    float run = 0.f;
    for (int b = b_lo; b < b_hi; ++b) run += tw < M ? row[b + 1] : 0.f;
    float incl = run;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    float acc = incl - run;
    __syncwarp();
    for (int b = b_lo; b < b_hi; ++b) {
      acc += tw < M ? row[b + 1] : 0.f;
      row[b + 1] = acc;
    }
    if (lane == 0) row[0] = 0.f;
  }
  if constexpr (!EXACT) __syncthreads();
  if (lo >= hi) return;   // no work for this warp (no barrier follows)

  // per-lane operand offsets in shared memory (tokens >= M are clamped: their columns are
  // discarded)
  const int xs_off = (int)(reinterpret_cast<const unsigned char*>(xs) - smem);
  int xv[NT][4];
  const uint4* xg[NT];
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = min(8 * nt + g, M - 1);
    #pragma unroll
    for (int v = 0; v < 4; ++v) xv[nt][v] = xs_off + 4 * (tok * xstride + tig * 16 + 4 * (v ^ tig));
    xg[nt] = reinterpret_cast<const uint4*>(Pb.xfrag) + ((size_t)tok * Kb * 4 + tig) * 4;
  }
  const int fa0 = warp * S * kStage + g * G_::kBlk + tig * 4 * BITS;   // this lane's chunk in stage 0

  float D[NCA][NT][4], Dw[NT][4], y[NT][4];
  zero_acc<NCA, NT>(D);
  RowDq<BITS> dq;
  #pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    #pragma unroll
    for (int i = 0; i < 4; ++i) { Dw[nt][i] = 0.f; y[nt][i] = 0.f; }
  int seg_b1 = b_top;              // block end of the current tile segment (walking down)
  int sz_rt = -1;                  // tile whose (scale, zero) pairs are in szA / szB
  __half2 szA = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f)), szB = szA;
  int st = 0;                      // stage being consumed
  uint32_t phase = 0;              // its barrier phase
  int consumed = 0;
  int failed_at = -1;              // item whose wait timed out
  bool ok = true;
  int kind, rt, first, cnt;
  #pragma unroll 1
  while (cons.next(kind, rt, first, cnt)) {
    if constexpr (!PG) {
      if (rt != sz_rt) {   // per-channel pairs of a new tile (EXACT: before its units; else at its segment end)
        sz_rt = rt;
        szA = Pb.sz_t[(size_t)rt * 16 + g];
        szB = Pb.sz_t[(size_t)rt * 16 + g + 8];
        if constexpr (EXACT) { dq.set(0, szA); dq.set(1, szB); }
      }
    }
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[st], phase, args.status, args.wait_limit));
      if (!ok) failed_at = consumed;
    }
    const int fa = fa0 + st * kStage;
    if (ok && kind == 0) {
      // weak k slices: A = the fp16 weak rows (tile-major slice: [16 rows][16]), B = gathered x
      #pragma unroll 1
      for (int i = 0; i < cnt; ++i) {
        const uint32_t* ws = reinterpret_cast<const uint32_t*>(ring + st * kStage + i * 512);
        const uint32_t a[4] = {ws[g * 8 + tig], ws[(g + 8) * 8 + tig], ws[g * 8 + 4 + tig], ws[(g + 8) * 8 + 4 + tig]};
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const __half* xr2 = xw + (8 * nt + g) * k_ld + 16 * (first + i) + 2 * tig;
          mma16816(Dw[nt], a, *reinterpret_cast<const uint32_t*>(xr2), *reinterpret_cast<const uint32_t*>(xr2 + 8));
        }
      }
    } else if (ok) {
      const __half2* szs = reinterpret_cast<const __half2*>(ring + st * kStage + G_::kStageW);
      auto fold_block = [&](int bb, int b) {   // per-group layers: one (scale, zero) pair per block
        const float2 fa_ = __half22float2(szs[bb * 16 + g]);
        const float2 fb_ = __half22float2(szs[bb * 16 + g + 8]);
        const float gsa = fa_.x, gza = fa_.y, gsb = fb_.x, gzb = fb_.y;
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tok = 8 * nt + 2 * tig + (i & 1);
            const float sxv = psx[tok * (Kb + 1) + b + 1] - psx[tok * (Kb + 1) + b];
            const float v = combine<BITS>(D[0][nt][i], D[NCA > 1 ? 1 : 0][nt][i], D[NCA - 1][nt][i]);
            const float sc = i < 2 ? gsa : gsb, z = i < 2 ? gza : gzb;
            y[nt][i] = fmaf(sc, fmaf(-z, sxv, v), y[nt][i]);
          }
        zero_acc<NCA, NT>(D);
      };
      const int xoff = first * 256;
      if (cnt == SUB) {
        #pragma unroll 4
        for (int bb = 0; bb < SUB; ++bb) {
          if constexpr (PG && EXACT) { dq.set(0, szs[bb * 16 + g]); dq.set(1, szs[bb * 16 + g + 8]); }
          unit_mma<BITS, NT, XSMEM, EXACT>(smem, fa + bb * G_::kTileBlk, xv, xoff + bb * 256, xg, first + bb, k2, k4, dq, D);
          if constexpr (PG && !EXACT) fold_block(bb, first + bb);
        }
      } else {
        #pragma unroll 1
        for (int bb = 0; bb < cnt; ++bb) {
          if constexpr (PG && EXACT) { dq.set(0, szs[bb * 16 + g]); dq.set(1, szs[bb * 16 + g + 8]); }
          unit_mma<BITS, NT, XSMEM, EXACT>(smem, fa + bb * G_::kTileBlk, xv, xoff + bb * 256, xg, first + bb, k2, k4, dq, D);
          if constexpr (PG && !EXACT) fold_block(bb, first + bb);
        }
      }
    }
    __syncwarp();
    ++consumed;
    if (lane == 0 && ok && issued < consumed + ahead) {   // keep `ahead` items in flight
      fence_proxy_async_smem();
      issue();
    }
    if (++st == S) { st = 0; phase ^= 1u; }

    // end of a tile segment: fold, then store (whole tile) or hand over (split tile)
    if (kind == 1 && cons.segment_done()) {
      const int seg_b0 = first;
      if constexpr (EXACT) {   // the sums are already scaled
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i) { y[nt][i] = D[0][nt][i]; D[0][nt][i] = 0.f; }
      } else if constexpr (!PG) {
        const float2 fa_ = __half22float2(szA), fb_ = __half22float2(szB);
        const float sa = fa_.x, za = fa_.y, sb = fb_.x, zb = fb_.y;
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tok = 8 * nt + 2 * tig + (i & 1);
            const float sxv = psx[tok * (Kb + 1) + seg_b1] - psx[tok * (Kb + 1) + seg_b0];
            const float v = combine<BITS>(D[0][nt][i], D[NCA > 1 ? 1 : 0][nt][i], D[NCA - 1][nt][i]);
            const float sc = i < 2 ? sa : sb, z = i < 2 ? za : zb;
            y[nt][i] = sc * fmaf(-z, sxv, v);
          }
        zero_acc<NCA, NT>(D);
      }
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) { y[nt][i] += Dw[nt][i]; Dw[nt][i] = 0.f; }

      const int t0 = rt * Kb;
      if ((t0 + Kb - 1) / c == t0 / c) {   // the whole tile is in this chunk
        if (ok) {
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = rt * 16 + g + 8 * (i >> 1), tok = 8 * nt + 2 * tig + (i & 1);
              if (row < N && tok < M) Pb.y[(size_t)tok * N + row] = __float2half_rn(y[nt][i]);
            }
        }
      } else if (lo < t0 && wi == cta_c0 + kWarps - 1) {
        // the top segment of the CTA's top warp (walked first): all this CTA holds of a tile
        // that a higher CTA finishes, so it is published at once, long before that CTA reaches
        // the tile's lowest units (it walks down too)
        unsigned long long* pt = Pb.part + ((size_t)rt * Pb.cta_slots + cta_c0 / kWarps - (t0 / c) / kWarps) * 256;
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            st_tagged(pt + (g + 8 * (i >> 1)) * 16 + 8 * nt + 2 * tig + (i & 1), y[nt][i], Pb.wtag);
      } else {
        // split tile, two-level hand-off.  Each segment in this CTA leaves its partial in shared
        // memory: the tile's lowest segment, when its warp walks it first (the warp's chunk
        // reaches below the tile), in an early slot; every other segment is the last one its
        // warp walks, so in that warp's ring, idle from then on.  The last segment to arrive
        // adds them in unit order (the same order every call), then stores the tile (all its
        // segments are here), publishes this CTA's sum (a higher CTA holds the tile's last
        // units), or adds the lower CTAs' sums (bounded wait on the tag, CTA order).
        const int c_first = t0 / c, c_last = (t0 + Kb - 1) / c;
        const bool early = c_first * c < t0;   // the tile's lowest segment is walked first
        float* eslot = lacc + (by_tile ? rt - t_lo : c_first - cta_c0) * 16 * MT;
        if (lo < t0 || failed_at < 0) {       // (after a timeout, copies may still reach the ring)
          float* mine = lo < t0 ? eslot : reinterpret_cast<float*>(ring);
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            #pragma unroll
            for (int i = 0; i < 4; ++i) mine[(g + 8 * (i >> 1)) * MT + 8 * nt + 2 * tig + (i & 1)] = y[nt][i];
        }
        __syncwarp();   // the warp's stores precede lane 0's release
        int old = 0;
        if (lane == 0) old = count_down_cta(&lcnt[rt - t_lo]);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == 1) {
          __syncwarp();
          float v[NT][4];
          #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            #pragma unroll
            for (int i = 0; i < 4; ++i) v[nt][i] = 0.f;
          const int cw0 = max(c_first, cta_c0), cw1 = min(c_last, cta_c0 + kWarps - 1);
          #pragma unroll 1
          for (int cw = cw0; cw <= cw1; ++cw) {
            const float* src = (cw == c_first && early)
                                   ? eslot : reinterpret_cast<const float*>(smem + (cw - cta_c0) * S * kStage);
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              #pragma unroll
              for (int i = 0; i < 4; ++i) v[nt][i] += src[(g + 8 * (i >> 1)) * MT + 8 * nt + 2 * tig + (i & 1)];
          }
          const int jf = c_first / kWarps, jl = c_last / kWarps, j = cta_c0 / kWarps;
          const unsigned long long* pt = Pb.part + (size_t)rt * Pb.cta_slots * 256;
          if (j < jl) {
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              #pragma unroll
              for (int i = 0; i < 4; ++i)
                st_tagged(const_cast<unsigned long long*>(pt) + (j - jf) * 256 + (g + 8 * (i >> 1)) * 16 + 8 * nt + 2 * tig + (i & 1),
                          v[nt][i], Pb.wtag);
          } else {
            float tot[NT][4];
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              #pragma unroll
              for (int i = 0; i < 4; ++i) tot[nt][i] = 0.f;
            bool good = ok;
            #pragma unroll 1
            for (int s2 = 0; s2 < j - jf && good; ++s2) {
              unsigned long long w[NT][4];
              #pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                #pragma unroll
                for (int i = 0; i < 4; ++i) w[nt][i] = ld_tagged(pt + s2 * 256 + (g + 8 * (i >> 1)) * 16 + 8 * nt + 2 * tig + (i & 1));
              const long long t_start = clock64();
              #pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                  while ((uint32_t)(w[nt][i] >> 32) != Pb.epoch) {
                    if (clock64() - t_start > args.wait_limit) {
                      atomicOr(args.status, 1);
                      good = false;
                      break;
                    }
                    w[nt][i] = ld_tagged(pt + s2 * 256 + (g + 8 * (i >> 1)) * 16 + 8 * nt + 2 * tig + (i & 1));
                  }
                  tot[nt][i] += __uint_as_float((uint32_t)w[nt][i]);
                }
            }
            if (good) {
              #pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int row = rt * 16 + g + 8 * (i >> 1), tok = 8 * nt + 2 * tig + (i & 1);
                  if (row < N && tok < M) Pb.y[(size_t)tok * N + row] = __float2half_rn(tot[nt][i] + v[nt][i]);
                }
            }
          }
        }
      }
      #pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int i = 0; i < 4; ++i) y[nt][i] = 0.f;
      seg_b1 = Kb;
    }
  }
  // after a timeout: never exit with bulk copies still writing into this CTA's memory
  if (failed_at >= 0 && lane == 0)
    for (int j = failed_at; j < issued; ++j)
      mbar_wait(&bars[j % S], (uint32_t)((j / S) & 1), args.status, args.wait_limit);
}

// SM count of the current device (cached per device ordinal)
int sm_count() {
  constexpr int kMaxDev = 64;
  static int n[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    return 148;
  }
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

// Exact per-pair dequantisation (see the kernel) for two token tiles, and for per-group layers
// from 4 tokens (their per-block scale fold costs more than the exact form there)
inline bool gemv_exact(int NT, bool pg, int M) { return NT == 2 || (pg && M >= 4); }

template <int BITS, int NT, int WARPS, int SUB, int S, bool XSMEM>
cudaError_t launch_k(GemvArgs& a, size_t smem, cudaStream_t s) {
  if constexpr (!XSMEM) {
    for (int q = 0; q < a.count; ++q) {
      const size_t n = (size_t)a.M * a.p[q].K / 2;
      k_x_frag<<<(unsigned)std::min<size_t>((n + 255) / 256, 2048), 256, 0, s>>>(a.p[q].x, a.M, a.p[q].K, a.p[q].xfrag);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  void (*kern)(GemvArgs);
  const bool pg = a.p[0].G > 1;
  if constexpr (NT == 2) {
    kern = pg ? k_gemv_mma<BITS, NT, WARPS, SUB, S, XSMEM, true, true>
              : k_gemv_mma<BITS, NT, WARPS, SUB, S, XSMEM, false, true>;
  } else {
    kern = pg ? (gemv_exact(NT, true, a.M) ? k_gemv_mma<BITS, NT, WARPS, SUB, S, XSMEM, true, true>
                                           : k_gemv_mma<BITS, NT, WARPS, SUB, S, XSMEM, true, false>)
              : k_gemv_mma<BITS, NT, WARPS, SUB, S, XSMEM, false, false>;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int base = 0;
  for (int q = 0; q < a.count; ++q) base += a.p[q].ncta;
  // programmatic dependent launch: this kernel may start while the previous one in the stream
  // drains; it waits (griddepcontrol.wait) before reading activations or writing outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(base);
  cfg.blockDim = dim3(WARPS * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// CTAs per problem in proportion to its work (one resident wave in total), then an equal
// chunk of (tile, block) units per warp: at least kGemvMinChunk, and large enough that a row
// tile meets at most cta_slots + 1 CTAs (the size of the layer's partial-sum workspace)
void plan(GemvArgs& a, int warps_per_cta) {
  const int C = sm_count();
  long long work[kMaxProblems], total = 0;
  for (int q = 0; q < a.count; ++q) {
    GemvProblem& Pq = a.p[q];
    Pq.row_groups = (Pq.N + 15) / 16;
    work[q] = (long long)Pq.row_groups * (Pq.K / kBlockCodes);
    total += work[q];
  }
  int n[kMaxProblems], used = 0, big = 0;
  for (int q = 0; q < a.count; ++q) {
    n[q] = max(1, (int)(work[q] * C / total));
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
  if (used < C) n[big] += C - used;
  int base = 0;
  for (int q = 0; q < a.count; ++q) {
    GemvProblem& Pq = a.p[q];
    const int Kb = Pq.K / kBlockCodes;
    const long long warps = (long long)n[q] * warps_per_cta;
    int chunk = (int)((work[q] + warps - 1) / warps);
    // at least kGemvMinChunk units, and a CTA span large enough that a tile meets at most
    // cta_slots + 1 CTAs (the layer's workspace; the minimum already guarantees it)
    const int span = (Kb - 1 + Pq.cta_slots - 1) / Pq.cta_slots;
    chunk = max(chunk, max(kGemvMinChunk, (span + warps_per_cta - 1) / warps_per_cta));
    const int nchunks = (int)((work[q] + chunk - 1) / chunk);
    Pq.chunk = chunk;
    Pq.lt_cap = (warps_per_cta * chunk - 1) / Kb + 2;
    Pq.ncta = min(n[q], (nchunks + warps_per_cta - 1) / warps_per_cta);
    Pq.cta_base = base;
    base += Pq.ncta;
  }
}

template <int BITS, int NT>
cudaError_t launch_t(GemvArgs& a, cudaStream_t s) {
  constexpr int MT = 8 * NT;
  constexpr size_t kMaxSmem = 232448;
  size_t extra = 0, xbytes = 0;
  for (int q = 0; q < a.count; ++q) {
    const GemvProblem& Pq = a.p[q];
    const int Kb = Pq.K / kBlockCodes;
    const size_t need = (gemv_exact(NT, Pq.G > 1, a.M) ? 0 : (size_t)((MT * (Kb + 1) + 3) & ~3) * sizeof(float)) +
                        (size_t)MT * Pq.k_ld * sizeof(__half);
    if (need > extra) extra = need;
    const size_t xb = (size_t)a.M * (Pq.K / 2 + 4) * sizeof(uint32_t);
    if (xb > xbytes) xbytes = xb;
  }
  const bool pg = a.p[0].G > 1;
  auto smem_for = [&](int warps, int sub, int S, bool xs) {
    const size_t stage = sub == 8 ? Geo<BITS, 8>::stage_bytes(pg) : Geo<BITS, 4>::stage_bytes(pg);
    return (size_t)warps * S * stage + (size_t)warps * S * 8 + 16 + ((extra + 15) & ~size_t(15)) + (xs ? xbytes : 0);
  };
  // the split-tile hand-off area: early slots and segment counters (see the kernel)
  auto local_bytes = [&](int warps) {
    size_t b = 0;
    for (int q = 0; q < a.count; ++q) {
      const int lt = a.p[q].lt_cap;
      b = std::max(b, (size_t)std::min(lt, warps) * 16 * MT * sizeof(float) + (size_t)((lt + 3) & ~3) * sizeof(int));
    }
    return b;
  };
#define OWQ_TRY(W, SUB, S, XS)                                                           \
  if (smem_for(W, SUB, S, XS) <= kMaxSmem) {                                             \
    plan(a, W);                                                                          \
    const size_t sm = smem_for(W, SUB, S, XS) + local_bytes(W);                          \
    if (sm <= kMaxSmem) return launch_k<BITS, NT, W, SUB, S, XS>(a, sm, s);              \
  }
  // 16 warps with the activations in shared memory: larger items first, then deeper rings
  OWQ_TRY(16, 8, 2, true)
  OWQ_TRY(16, 4, 4, true)
  OWQ_TRY(16, 4, 3, true)
  OWQ_TRY(16, 4, 2, true)
  if constexpr (NT == 2) {
    // more tokens than fit beside a 16-warp ring: 8 warps keep them in shared memory, or read
    // them fragment-ordered from global memory with the register room of 8-warp CTAs
    OWQ_TRY(8, 4, 4, true)
    OWQ_TRY(8, 4, 3, true)
    OWQ_TRY(8, 4, 2, true)
    OWQ_TRY(8, 4, 4, false)
  }
  OWQ_TRY(16, 4, 3, false)
  OWQ_TRY(16, 4, 2, false)
#undef OWQ_TRY
  return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t launch_bits(GemvArgs& a, cudaStream_t s) {
  return a.M <= 8 ? launch_t<BITS, 1>(a, s) : launch_t<BITS, 2>(a, s);
}

}  // namespace

cudaError_t launch_gemv(const GemvProblem* probs, int count, int bits, int M, long long wait_limit,
                        cudaStream_t s) {
  if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
  // one launch serves layers of one kind (per-channel or per-group scales)
  for (int q = 1; q < count; ++q)
    if ((probs[q].G > 1) != (probs[0].G > 1)) {
      for (int j = 0; j < count; ++j) {
        cudaError_t e = launch_gemv(probs + j, 1, bits, M, wait_limit, s);
        if (e != cudaSuccess) return e;
      }
      return cudaSuccess;
    }
  GemvArgs a{};
  for (int q = 0; q < count; ++q) a.p[q] = probs[q];
  a.count = count;
  a.M = M;
  a.status = device_status_ptr();
  a.wait_limit = wait_limit;
  a.ahead = kAhead;
  a.k2 = 2u;
  a.k4 = 4u;
  if (!a.status) return cudaErrorInvalidDevicePointer;
  return bits == 3 ? launch_bits<3>(a, s) : launch_bits<4>(a, s);
}

}  // namespace owq
