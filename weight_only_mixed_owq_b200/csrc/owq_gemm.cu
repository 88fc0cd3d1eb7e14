// Prefill product y = W_tilde x^T for many tokens on the 5th-generation tensor cores.
//
// Pages: "Real-device acceleration" (OWQ paper "Acceleration on Real Device", p.6, as
// summarised on paperlayer.ai: a 3-bit weight x fp16 activation product with the weak-
// column activations picked on the fly) and "Storage Methods" (appendix §2: the dense
// low-precision matrix is zero-filled at the weak columns, the weak columns are a separate
// fp16 block).  W_tilde is the dequantised dense matrix with its weak columns replaced by
// their fp16 values, so y = W_hat x + W_weak x[idx] exactly as the method defines it.
//
// One CTA computes a 128-weight-row x BN-token tile of y^T (MMA M = weight rows,
// MMA N = tokens), looping over K in 128-code steps through an S-stage ring:
//   warp 0      TMA producer.  Dense step: the packed 128 x (16*bits) byte tile (a 3-D box over
//               the layer's 16-row-tile storage), for per-group layers the step's (scale, zero)
//               pairs of the 8 tiles, and two 128B-swizzled BN x 64 fp16 activation boxes.
//               Weak step (after the dense ones): two boxes of the gathered weak activations.
//   warp 1      TMEM allocation and the single MMA-issuing thread (tcgen05.mma kind::f16 with
//               the A operand in tensor memory, B from shared memory, fp32 accumulator BN
//               columns wide in tensor memory).
//   warps 2-9   the A operand: each thread owns one weight row (its warp's TMEM lane quarter)
//               and one 64-code slab of each step.  Dense step: unpack in registers, form
//               fp16_rn(s (q - z)) with exact fp16x2 arithmetic, tcgen05.st into the step's A
//               stage in tensor memory (no shared-memory A tile, so the ring holds more
//               stages).  The weak columns hold q = z, so their dequantised value is exactly 0;
//               the weak steps load the fp16 weak block rows instead, adding W_weak x[idx] into
//               the same accumulator.  The same warps run the epilogue (tcgen05.ld, fp16
//               rounding, coalesced stores).
// Every mbarrier wait is bounded (clock64 limit): on expiry the thread records the device
// status word and leaves its loop, so a broken pipeline ends the kernel instead of hanging.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "owq_format.cuh"
#include "owq_internal.cuh"
#include "owq_sm100.cuh"

namespace owq {
namespace {

using namespace sm100;

constexpr int kBM = 128;               // weight rows per tile (MMA M)
constexpr int kStepCodes = 128;        // K per pipeline step
// tensor-memory columns of a CTA: the accumulator (BN) + S A stages of 64, as a power of two;
// 256 lets two CTAs share an SM
template <int BN, int S>
constexpr uint32_t tmem_cols() { return BN + 64 * S <= 256 ? 256u : 512u; }

template <int BITS, int BN>
struct Smem {
  static constexpr int kX = 2 * BN * 128;           // two 64-column swizzled activation boxes
  static constexpr int kP = kBM * 16 * BITS;        // packed tile
  static constexpr int kSZ = kBM * 4;               // (scale, zero) pairs of the step (per-group layers)
  static constexpr int kStage = ((kX + kP + kSZ) + 1023) & ~1023;
};

template <int BITS, int BN, int S>
constexpr int smem_bytes() { return S * Smem<BITS, BN>::kStage + 1024 /*barriers*/ + 1024 /*align slack*/; }

struct GemmParams {
  const __half* scales;   // per-channel layers: read once per row (per-group: staged by TMA)
  const __half* zeros;
  const __half* w_weak;   // the weak block [N][k_ld] (read by the A-operand warps in weak steps)
  int k_ld;
  __half* y;
  float* ws;        // split-K partial sums: split sp, token t, row n at sp * ws_stride + (t - ws_t0) N + n
  size_t ws_stride;
  int ws_t0;
  int* status;
  int N, K, M, G;
  int ksteps;       // dense 128-code steps per split (blockIdx.z)
  // short last wave: grid.y = tail_y0 whole token tiles, then tail_sp CTAs (K splits of
  // tail_ksteps steps) for each further token tile (tail_y0 = grid.y: no tail)
  int tail_y0, tail_sp, tail_ksteps;
  int nw;           // weak steps: 128 columns of the weak block each (run by the last split)
  long long wait_limit;   // bound of every mbarrier wait, in SM clock cycles
  int skip_arrive;  // test-injected lost arrival: dequantisation thread 0 skips its first one
};

// fp16x2 helpers (exact integer arithmetic on small values)
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
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_splat(float v) {
  __half h = __float2half_rn(v);
  uint32_t u = __half_as_ushort(h);
  return u | (u << 16);
}

// fp16_rn(s (q - z)) of pair j of a chunk (both halves).  The pair is lifted as
// (bits | 0x6400) = 1024 + q 2^o per half, then (1024 + q 2^o) * 2^-o - (1024 2^-o + z) = q - z
// exactly (one fma.rn.f16x2), then * s rounds once: bit-exact with the definition.
template <int BITS>
__device__ __forceinline__ uint32_t dequant_pair(const uint32_t* w, int j, uint32_t s2, const uint32_t* scl,
                                                 const uint32_t* nz) {
  constexpr uint32_t kMagic = 0x64006400u;
  const int c = pair_class<BITS>(j);
  return h2_mul(h2_fma(pair_bits<BITS>(w, j) | kMagic, scl[c], nz[c]), s2);
}

// TAIL: the grid holds a split tail (GemmParams::tail_*); without it the CTA's token tile and
// K split are blockIdx.y and blockIdx.z, and none of the tail arithmetic is compiled in (it
// cost the 64-token tiles 5% where it was always present)
template <int BITS, int BN, int S, int DW, bool TAIL>
__global__ void __launch_bounds__(32 * (2 + DW), 1)
k_gemm_sm100(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_p,
             const __grid_constant__ CUtensorMap map_xw, const __grid_constant__ CUtensorMap map_sz,
             const __grid_constant__ GemmParams p) {
  using L = Smem<BITS, BN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * L::kStage);
  uint64_t* full = bars;            // [S] TMA landed
  uint64_t* empty = bars + S;       // [S] MMAs of the stage done
  uint64_t* afull = bars + 2 * S;   // [S] A tile written to tensor memory
  uint64_t* accf = bars + 3 * S;    // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // (row tile, token tile, K split) of this CTA
  int ty = 0, sp = 0, nsp = 1, ksteps = 0;
  if constexpr (TAIL) {
    ty = blockIdx.y; sp = blockIdx.z; nsp = gridDim.z; ksteps = p.ksteps;
    if (ty >= p.tail_y0) {
      const int u = ty - p.tail_y0;
      ty = p.tail_y0 + u / p.tail_sp;
      sp = u % p.tail_sp;
      nsp = p.tail_sp;
      ksteps = p.tail_ksteps;
    }
  }
  const int n0 = blockIdx.x * kBM;                     // first weight row
  const int m0 = (TAIL ? ty : (int)blockIdx.y) * BN;   // first token
  const int kb0 = TAIL ? sp * ksteps : (int)blockIdx.z * p.ksteps;                  // first dense step of this split
  const int nD = max(0, min(TAIL ? ksteps : p.ksteps, p.K / kStepCodes - kb0));     // dense steps of this split
  const int nK = nD + ((TAIL ? sp == nsp - 1 : blockIdx.z == gridDim.z - 1) ? p.nw : 0);   // + the weak steps (last split)
  const bool per_group = p.G > 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], 32 * DW);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_p);
  }
  // tensor memory: the accumulator (BN columns) then S A stages of 64 columns (128 rows x 128
  // fp16 codes, two per 32-bit column)
  if (warp == 1) tmem_alloc(tmem_slot, tmem_cols<BN, S>());
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      // dense step: the packed block of the 8 16-row tiles of this CTA (tile-major storage),
      // their (scale, zero) pairs (per-group layers) and two activation boxes; weak step: two
      // boxes of the gathered weak activations
      const uint32_t kDense = L::kX + L::kP + (per_group ? L::kSZ : 0);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nK && ok; ++i) {
        const int s = i % S, u = i / S;
        if (u > 0) ok = mbar_wait(&empty[s], (u - 1) & 1, p.status, p.wait_limit);
        if (!ok) break;
        unsigned char* st = smem + s * L::kStage;
        if (i < nD) {
          const int kb = kb0 + i;
          mbar_arrive_expect_tx(&full[s], kDense);
          tma_load_3d(st + L::kX, &map_p, &full[s], 0, kb, n0 / 16);
          if (per_group) tma_load_3d(st + L::kX + L::kP, &map_sz, &full[s], 0, kb, n0 / 16);
          tma_load_2d(st, &map_x, &full[s], kb * kStepCodes, m0);
          tma_load_2d(st + BN * 128, &map_x, &full[s], kb * kStepCodes + 64, m0);
        } else {
          const int c0 = (i - nD) * kStepCodes;
          mbar_arrive_expect_tx(&full[s], L::kX);
          tma_load_2d(st, &map_xw, &full[s], c0, m0);
          tma_load_2d(st + BN * 128, &map_xw, &full[s], c0 + 64, m0);
        }
        issued = i + 1;
      }
      // never leave with copies in flight: wait for the last issued use of every stage
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait(&full[i % S], (i / S) & 1, p.status, p.wait_limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // This one thread paces the CTA at small M, so its loop is kept short: the shared-memory
      // descriptor is linear in its 16-byte-granular start address (shared addresses stay below
      // 2^18, so the 14-bit field never carries), hence one base descriptor plus per-stage and
      // per-slice constants; and it waits only for the A stage: the dequantisation threads
      // arrive there after waiting for the same stage's TMA barrier, so the activation tile
      // the MMA reads has landed too.
      constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
      const uint64_t dbase = desc_sw128_kmajor(smem_u32(smem));
      bool ok = true;
      for (int i = 0; i < nK && ok; ++i) {
        const int s = i % S, u = i / S;
        ok = mbar_wait(&afull[s], u & 1, p.status, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ds = dbase + (uint64_t)((s * L::kStage) >> 4);
        const uint32_t at = tmem + BN + 64 * s;
        mma_f16_ts(tmem, at, ds, idesc, i != 0);
        #pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          mma_f16_ts(tmem, at + 8 * kk, ds + (uint64_t)((((kk >> 2) * BN * 128) + (kk & 3) * 32) >> 4), idesc, 1u);
        mma_commit(&empty[s]);
      }
      mma_commit(accf);
    }
  } else {
    // ---------------- A operand ----------------
    // DW warps, NSL = DW / 4 per lane quarter: warp w owns the lane quarter w % 4 of tensor
    // memory and slab sl = (w - 2) / 4 of each step.  Thread (row r = 32 (w % 4) + lane, sl)
    // writes codes 8U sl .. 8U sl + 8U - 1 of its row (U = 16 / NSL units of 8 codes), columns
    // 4U sl .. 4U sl + 4U - 1 of the step's A stage.  For unit j the four chunks' pair j are
    // the codes 8j .. 8j + 7.
    constexpr int NSL = DW / 4, U = 16 / NSL;
    const int quarter = warp & 3, jh = (warp - 2) >> 2;
    const int r = 32 * quarter + lane;
    const int row = min(n0 + r, p.N - 1);
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    uint32_t s2 = 0, scl[3], nz[3];
    constexpr float kOff[3] = {1.f, BITS == 3 ? 8.f : 16.f, 64.f};
    scl[0] = h2_splat(1.f);
    scl[1] = h2_splat(1.f / kOff[1]);
    scl[2] = h2_splat(1.f / kOff[2]);
    auto set_sz = [&](__half sh, __half zh) {
      const uint32_t su = __half_as_ushort(sh);
      const float z = __half2float(zh);
      s2 = su | (su << 16);
      #pragma unroll
      for (int c = 0; c < 3; ++c) nz[c] = h2_splat(-(1024.f / kOff[c] + z));
    };
    if (!per_group) set_sz(p.scales[row], p.zeros[row]);   // per-channel: one pair per row
    bool ok = true;
    for (int i = 0; i < nK && ok; ++i) {
      const int s = i % S, u = i / S;
      ok = mbar_wait(&full[s], u & 1, p.status, p.wait_limit);   // (also: the stage's previous MMAs are done)
      if (!ok) break;
      tc_fence_after();
      const unsigned char* st = smem + s * L::kStage;
      const uint32_t at = tmem + lane_base + BN + 64 * s + 4 * U * jh;
      uint32_t d[U / 4][16];
      if (i < nD) {
        if (per_group) {   // this step's pair, staged with the packed tile ([8 tiles][16 rows])
          const __half2 sz = *reinterpret_cast<const __half2*>(st + L::kX + L::kP + r * 4);
          set_sz(__low2half(sz), __high2half(sz));
        }
        // (plain loads: a same-box A/B against explicit ld.shared measured them 2-4% faster here,
        // where each thread reads only BITS 16-byte words per step)
        const uint4* pw = reinterpret_cast<const uint4*>(st + L::kX + r * 16 * BITS);
        uint32_t w[4 * BITS];
        #pragma unroll
        for (int v = 0; v < BITS; ++v) {
          const uint4 q = pw[v];
          w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
        }
        // the slab is uniform per warp: each branch sees compile-time pair indices.  The weak
        // columns hold q = z: their value is exactly 0 (the weak steps add them).
        auto units = [&](auto sl_c) {
          constexpr int SL = decltype(sl_c)::value;
          #pragma unroll
          for (int ju = 0; ju < U; ++ju)
            #pragma unroll
            for (int q = 0; q < 4; ++q)   // codes 8j + 2q, 8j + 2q + 1 -> column 4 ju + q of the slab
              d[ju >> 2][4 * (ju & 3) + q] = dequant_pair<BITS>(w + q * BITS, U * SL + ju, s2, scl, nz);
        };
        if constexpr (NSL == 2) {
          if (jh == 0) units(std::integral_constant<int, 0>{});
          else units(std::integral_constant<int, 1>{});
        } else {
          switch (jh) {
            case 0: units(std::integral_constant<int, 0>{}); break;
            case 1: units(std::integral_constant<int, 1>{}); break;
            case 2: units(std::integral_constant<int, 2>{}); break;
            default: units(std::integral_constant<int, 3>{}); break;
          }
        }
      } else {
        // weak step: the fp16 weak block, columns c0 .. c0 + 8U - 1 of this row (0 past k_ld)
        const int c0 = (i - nD) * kStepCodes + 8 * U * jh;
        const uint4* src = reinterpret_cast<const uint4*>(p.w_weak + (size_t)row * p.k_ld + c0);
        #pragma unroll
        for (int v = 0; v < U; ++v) {
          const uint4 q = (n0 + r < p.N && c0 + 8 * v < p.k_ld) ? src[v] : make_uint4(0, 0, 0, 0);
          d[v >> 2][4 * (v & 3)] = q.x; d[v >> 2][4 * (v & 3) + 1] = q.y;
          d[v >> 2][4 * (v & 3) + 2] = q.z; d[v >> 2][4 * (v & 3) + 3] = q.w;
        }
      }
      #pragma unroll
      for (int h = 0; h < U / 4; ++h) tmem_st16(at + 16 * h, d[h]);
      tmem_st_wait();
      tc_fence_before();
      if (!(p.skip_arrive && i == 0 && threadIdx.x == 64)) mbar_arrive(&afull[s]);
    }

    // ---------------- epilogue ----------------
    const bool acc_ok = mbar_wait(accf, 0, p.status, p.wait_limit);
    tc_fence_after();
    const int orow = n0 + r;
    #pragma unroll 1
    for (int c0 = jh * (BN / NSL); c0 < (jh + 1) * (BN / NSL); c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base + (uint32_t)c0, v);
      tmem_ld_wait();
      if (acc_ok && orow < p.N) {
        if (TAIL ? nsp > 1 : p.ws != nullptr) {   // split-K: fp32 partial of this split
          // without a tail the partials are [split][M][N] (ws_stride = M N, ws_t0 = 0)
          float* w = TAIL ? p.ws + (size_t)sp * p.ws_stride : p.ws + (size_t)blockIdx.z * p.M * p.N;
          #pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = m0 + c0 + j;
            if (t < p.M) w[(size_t)(TAIL ? t - p.ws_t0 : t) * p.N + orow] = __uint_as_float(v[j]);
          }
        } else {
          #pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = m0 + c0 + j;
            if (t < p.M) p.y[(size_t)t * p.N + orow] = __float2half_rn(__uint_as_float(v[j]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols<BN, S>());
    tmem_relinquish();
  }
}

// ---------------------------------------------------------------- input gradient, many tokens
// dX = dY W_hat on the same pipeline, transposed: one CTA computes a 128-column x BN-token tile
// of dX^T (MMA M = the 128 columns of one packed block, MMA N = tokens), looping over the rows
// (the contraction) in 128-row steps.
//   warp 0      TMA producer: the step's packed block of 8 16-row tiles (the prefill's box, at
//               block b and the step's tiles), their (scale, zero) pairs for block b's group, and
//               two 128B-swizzled BN x 64 fp16 boxes of dY (tokens x rows).
//   warp 1      TMEM allocation and the MMA-issuing thread (unchanged).
//   warps 2..   the A operand W_hat^T: thread (lane quarter, lane) owns column j = TMEM lane and a
//               slab of the step's rows; tensor memory packs two K values (rows 2c, 2c + 1) per
//               32-bit column.  Column j's code sits in the same word of every row (chunk
//               (j / 2) % 4, pair (j / 2) / 4, half j % 2), so one byte permute of two rows'
//               words gives the row pair (moved down a byte where the code sits at bit 8 or
//               above), AND/OR 0x6400 gives 1024 + q 2^o, and fp16x2 fma, subtract and multiply
//               with the row pair's (s, z) give fp16_rn(s (q - z)) bit-exactly.  The weak
//               columns hold q = z, so they come out exactly 0 here; a separate pass writes
//               them.  The same warps run the epilogue.
//   last warp   prep: per step, each row pair's scales and zero points side by side, and (3-bit)
//               the pair whose bits are spread over a chunk's three words rebuilt as an ordinary
//               word, so every A thread runs the same six instructions per row pair.
// Every mbarrier wait is bounded, as in the prefill kernel.
// Stage layout: the prefill's (dY boxes, packed block, (s, z) pairs), then what the prep warp
// derives from them.  The prep warp rewrites the packed block in place with the two rows of
// each row pair interleaved word by word ([64 pairs][4 bits words] of {row 2P, row 2P + 1}),
// rebuilds the 3-bit pair whose bits are spread over a chunk's three words as an ordinary word
// pair ([64 pairs][4 chunks], even code at bits 6-8, odd at 22-24) and writes per row pair and
// offset class {s2, -(1024 2^-o + z2)}.
template <int BITS, int BN>
struct IgSmem {
  static constexpr int kX = Smem<BITS, BN>::kX, kP = Smem<BITS, BN>::kP, kSZ = Smem<BITS, BN>::kSZ;
  static constexpr int kTma = kX + kP + kSZ;
  static constexpr int kCls = BITS == 3 ? 5 : 2;              // code offsets 0, 3, 6, 1, 4 / 0, 4
  static constexpr int kAuxD = BITS == 3 ? 64 * 4 * 8 : 0;    // [64 pairs][4 chunks] uint2
  static constexpr int kAuxS = 64 * kCls * 8;                 // [64 pairs][classes] {s2, nz2}
  static constexpr int kStage = ((kTma + kAuxD + kAuxS) + 1023) & ~1023;
};
// class of a code offset (after the byte shift): 3-bit 0, 3, 6, 1, 4 -> 0..4; 4-bit 0, 4 -> 0, 1
template <int BITS>
__host__ __device__ constexpr int ig_off_cls(int o) {
  return BITS == 3 ? (o == 0 ? 0 : o == 3 ? 1 : o == 6 ? 2 : o == 1 ? 3 : 4) : o / 4;
}
template <int BITS>
__host__ __device__ constexpr int ig_cls_off(int c) {
  return BITS == 3 ? (c == 0 ? 0 : c == 1 ? 3 : c == 2 ? 6 : c == 3 ? 1 : 4) : 4 * c;
}
template <int BITS, int BN, int S>
constexpr int ig_smem_bytes() { return S * IgSmem<BITS, BN>::kStage + 1024 /*barriers*/ + 1024 /*align slack*/; }

struct IgGemmParams {
  __half* dx;
  float* ws;        // split-K partial sums [split][M][K] (NULL: one split, fp16 dx directly)
  int* status;
  int N, K, M, group;
  int rsteps;       // 128-row steps per split (blockIdx.z)
  long long wait_limit;
};

template <int BITS, int BN, int S, int DW>
__global__ void __launch_bounds__(32 * (3 + DW), 1)
k_igemm_sm100(const __grid_constant__ CUtensorMap map_dy, const __grid_constant__ CUtensorMap map_p,
              const __grid_constant__ CUtensorMap map_sz, const __grid_constant__ CUtensorMap map_dx,
              const __grid_constant__ IgGemmParams p) {
  using L = IgSmem<BITS, BN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * L::kStage);
  uint64_t* full = bars;            // [S] TMA landed
  uint64_t* empty = bars + S;       // [S] MMAs of the stage done
  uint64_t* afull = bars + 2 * S;   // [S] A tile written to tensor memory
  uint64_t* accf = bars + 3 * S;    // accumulator complete
  uint64_t* pfull = bars + 3 * S + 1;   // [S] prep warp's words written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * S + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;             // column block (128 columns)
  const int m0 = blockIdx.y * BN;       // first token
  const int nR = (p.N + 127) / 128;
  const int rb0 = blockIdx.z * p.rsteps;                 // first row step of this split
  const int nK = max(0, min(p.rsteps, nR - rb0));
  const int grp = (b * kStepCodes) / p.group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], 32 * DW);
      mbar_init(&pfull[s], 32);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
    prefetch_tmap(&map_dy);
    prefetch_tmap(&map_p);
    prefetch_tmap(&map_sz);
  }
  if (warp == 1) tmem_alloc(tmem_slot, tmem_cols<BN, S>());
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint32_t kBytes = L::kTma;
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nK && ok; ++i) {
        const int s = i % S, u = i / S;
        if (u > 0) ok = mbar_wait(&empty[s], (u - 1) & 1, p.status, p.wait_limit);
        if (!ok) break;
        unsigned char* st = smem + s * L::kStage;
        const int rb = rb0 + i;
        mbar_arrive_expect_tx(&full[s], kBytes);
        tma_load_3d(st + L::kX, &map_p, &full[s], 0, b, rb * 8);
        tma_load_3d(st + L::kX + L::kP, &map_sz, &full[s], 0, grp, rb * 8);
        tma_load_2d(st, &map_dy, &full[s], rb * 128, m0);
        tma_load_2d(st + BN * 128, &map_dy, &full[s], rb * 128 + 64, m0);
        issued = i + 1;
      }
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait(&full[i % S], (i / S) & 1, p.status, p.wait_limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
      const uint64_t dbase = desc_sw128_kmajor(smem_u32(smem));
      bool ok = true;
      for (int i = 0; i < nK && ok; ++i) {
        const int s = i % S, u = i / S;
        ok = mbar_wait(&afull[s], u & 1, p.status, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ds = dbase + (uint64_t)((s * L::kStage) >> 4);
        const uint32_t at = tmem + BN + 64 * s;
        mma_f16_ts(tmem, at, ds, idesc, i != 0);
        #pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          mma_f16_ts(tmem, at + 8 * kk, ds + (uint64_t)((((kk >> 2) * BN * 128) + (kk & 3) * 32) >> 4), idesc, 1u);
        mma_commit(&empty[s]);
      }
      mma_commit(accf);
    }
  } else if (warp == 2 + DW) {
    // ---------------- prep warp ----------------
    bool ok = true;
    for (int i = 0; i < nK && ok; ++i) {
      const int s = i % S, u = i / S;
      ok = mbar_wait(&full[s], u & 1, p.status, p.wait_limit);
      if (!ok) break;
      const uint32_t st = smem_u32(smem) + s * L::kStage;   // shared address of the stage
      constexpr int W = 4 * BITS;   // words of a row's block
      #pragma unroll 1
      for (int P = lane; P < 64; P += 32) {   // one row pair per lane and pass
        uint32_t a[W], c[W];
        const uint32_t ra = st + L::kX + (2 * P) * 16 * BITS;
        #pragma unroll
        for (int v = 0; v < BITS; ++v) {
          const uint4 x = lds_u4(ra + 16 * v), y = lds_u4(ra + 16 * (BITS + v));
          a[4 * v] = x.x; a[4 * v + 1] = x.y; a[4 * v + 2] = x.z; a[4 * v + 3] = x.w;
          c[4 * v] = y.x; c[4 * v + 1] = y.y; c[4 * v + 2] = y.z; c[4 * v + 3] = y.w;
        }
        if constexpr (BITS == 3) {   // bit e of the spread pair: bit 15 / 31 of word e -> 6 + e / 22 + e
          const uint32_t aux_d = st + L::kTma + 32 * P;
          #pragma unroll
          for (int qc = 0; qc < 4; ++qc) {
            const uint32_t* x = a + 3 * qc;
            const uint32_t* y = c + 3 * qc;
            sts_u2(aux_d + 8 * qc,
                   make_uint2(((x[0] >> 9) & 0x00400040u) | ((x[1] >> 8) & 0x00800080u) | ((x[2] >> 7) & 0x01000100u),
                              ((y[0] >> 9) & 0x00400040u) | ((y[1] >> 8) & 0x00800080u) | ((y[2] >> 7) & 0x01000100u)));
          }
        }
        #pragma unroll
        for (int v = 0; v < W / 2; ++v)   // the pair's own bytes, rows interleaved word by word
          sts_u4(ra + 16 * v, make_uint4(a[2 * v], c[2 * v], a[2 * v + 1], c[2 * v + 1]));
        const uint2 z = lds_u2(st + L::kX + L::kP + 8 * P);   // (s, z) of rows 2P, 2P + 1
        const uint32_t s2 = __byte_perm(z.x, z.y, 0x5410), z2 = __byte_perm(z.x, z.y, 0x7632);
        const uint32_t aux_s = st + L::kTma + L::kAuxD + 8 * L::kCls * P;
        #pragma unroll
        for (int cl = 0; cl < L::kCls; ++cl) {
          const uint32_t nego = (0x8000u | ((uint32_t)(25 - ig_cls_off<BITS>(cl)) << 10)) * 0x00010001u;   // -2^(10 - o)
          sts_u2(aux_s + 8 * cl, make_uint2(s2, h2_sub(nego, z2)));
        }
      }
      __syncwarp();
      mbar_arrive(&pfull[s]);
    }
  } else {
    // ---------------- A operand: W_hat^T ----------------
    // NSL = DW / 4 warps per lane quarter; warp w takes lane quarter w % 4 and row slab
    // (w - 2) / 4, RP row pairs of each step (tensor-memory columns RP jh .. RP jh + RP - 1).
    constexpr int NSL = DW / 4, RP = 64 / NSL;
    const int quarter = warp & 3, jh = (warp - 2) >> 2;
    const int j = 32 * quarter + lane;             // column of the block
    const int pj = j >> 1, q = pj & 3, jj = pj >> 2, h = j & 1;
    const bool spread = BITS == 3 && jj == 11;
    // the slot of pair jj (the 3-bit table of owq_format.cuh as packed fields: word, offset / 3)
    const Slot sl = spread ? Slot{0, 6}
                  : BITS == 3 ? Slot{(int)((0xaa244444u >> (2 * jj)) & 3u), 3 * (int)((0x3041024433221100ull >> (4 * jj)) & 15u)}
                              : Slot{2 * (jj / 8) + (jj % 2), 4 * ((jj % 8) / 2)};
    const bool hi8 = !spread && sl.off >= 8;
    const int o2 = hi8 ? sl.off - 8 : sl.off;
    const uint32_t sel = h ? (hi8 ? 0x7733u : 0x7632u) : (hi8 ? 0x5511u : 0x5410u);
    const uint32_t m1 = ((1u << BITS) - 1u) << o2, mask = m1 | (m1 << 16);
    const uint32_t sc = ((uint32_t)(15 - o2) << 10) * 0x00010001u;                // 2^-o
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    // column j's word pair (rows 2P, 2P + 1) in each row pair: the interleaved packed block, or
    // for the spread pair the prep warp's rebuilt pair (then at offset 6, the unshifted half)
    const int woff = spread ? L::kTma + 8 * q : L::kX + 8 * (q * BITS + sl.word);
    const int pstride = spread ? 32 : 32 * BITS;
    const int cls = ig_off_cls<BITS>(o2);
    bool ok = true;
    for (int i = 0; i < nK && ok; ++i) {
      const int s = i % S, u = i / S;
      ok = mbar_wait(&pfull[s], u & 1, p.status, p.wait_limit);   // (implies the TMA landed)
      if (!ok) break;
      tc_fence_after();
      const uint32_t st = smem_u32(smem) + s * L::kStage;   // shared address of the stage
      const uint32_t pk = st + woff + (RP * jh) * pstride;
      const uint32_t snp = st + L::kTma + L::kAuxD + 8 * (L::kCls * RP * jh + cls);
      uint32_t d[RP];
      #pragma unroll
      for (int pr = 0; pr < RP; ++pr) {
        const uint2 w = lds_u2(pk + pr * pstride);
        const uint32_t v = (__byte_perm(w.x, w.y, sel) & mask) | 0x64006400u;
        const uint2 sn = lds_u2(snp + 8 * L::kCls * pr);   // {s2, -(1024 2^-o + z2)} of the pair
        d[pr] = h2_mul(h2_fma(v, sc, sn.y), sn.x);   // fp16_rn(s (q - z))
      }
      const uint32_t at = tmem + lane_base + BN + 64 * s + RP * jh;
      #pragma unroll
      for (int c = 0; c < RP / 16; ++c)
        tmem_st16(at + 16 * c, *reinterpret_cast<const uint32_t(*)[16]>(d + 16 * c));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&afull[s]);
    }

    // ---------------- epilogue ----------------
    // One split: the fp16 tile goes to shared memory as [BN tokens][128 columns] (the stages are
    // idle once the accumulator is complete: every load was consumed by an MMA) and out with one
    // TMA store, which drops the rows past M.  Several splits: fp32 partials straight to the
    // workspace.
    const bool acc_ok = mbar_wait(accf, 0, p.status, p.wait_limit);
    tc_fence_after();
    const int col = b * kStepCodes + j;
    __half* s_out = reinterpret_cast<__half*>(smem);
    #pragma unroll 1
    for (int c0 = jh * (BN / NSL); c0 < (jh + 1) * (BN / NSL); c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base + (uint32_t)c0, v);
      tmem_ld_wait();
      if (p.ws) {
        if (acc_ok) {
          float* w = p.ws + (size_t)blockIdx.z * p.M * p.K;
          #pragma unroll
          for (int t = 0; t < 16; ++t)
            if (m0 + c0 + t < p.M) w[(size_t)(m0 + c0 + t) * p.K + col] = __uint_as_float(v[t]);
        }
      } else {
        #pragma unroll
        for (int t = 0; t < 16; ++t)
          sts_u16(smem_u32(s_out) + 2 * ((c0 + t) * kStepCodes + j), __half_as_ushort(__float2half_rn(__uint_as_float(v[t]))));
      }
    }
    if (!p.ws) {
      fence_proxy_async_smem();          // the tile, written by the generic proxy, to the TMA
      named_bar_sync(1, 32 * DW);        // every A thread's part of the tile is written
      if (warp == 2 && lane == 0 && acc_ok) {
        tma_store_2d(&map_dx, s_out, b * kStepCodes, m0);
        bulk_commit();
        bulk_wait_read0();               // shared memory read out before the CTA may exit
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols<BN, S>());
    tmem_relinquish();
  }
}

// Weak activations of every token, in the weak block's column order: xw[m][t] = x[m][idx[t]]
// (t < k), 0 for t in [k, k_ld).
__global__ void k_gather_weak_x(const __half* __restrict__ x, int M, int K, const int32_t* __restrict__ idx,
                                int k, int k_ld, __half* __restrict__ xw, int* status) {
  const size_t n = (size_t)M * k_ld;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(e / k_ld), t = (int)(e % k_ld);
    xw[e] = t < k && in_range(idx[t], K, status) ? x[(size_t)m * K + idx[t]] : __float2half_rn(0.f);
  }
}

// Split-K: y = fp16_rn(sum of the splits' fp32 partials, in split order); MN outputs, the
// splits' partials MN floats apart.
__global__ void k_splitk_reduce(const float* __restrict__ ws, int splits, size_t MN, __half* __restrict__ y) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < MN; e += (size_t)gridDim.x * blockDim.x) {
    float v = ws[e];
    for (int z = 1; z < splits; ++z) v += ws[(size_t)z * MN + e];
    y[e] = __float2half_rn(v);
  }
}

// ---- host side ----
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
  }
  return fn;
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiled enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_packed_3d(CUtensorMap* m, const void* base, int K, int N, int bits) {
  EncodeTiled enc = get_encoder();
  if (!enc) return false;
  const int Kb = K / kStepCodes;
  const uint64_t tile_blk = 16ull * 16 * bits;          // bytes of one block of a 16-row tile
  const cuuint64_t dims[3] = {tile_blk / 4, (cuuint64_t)Kb, (cuuint64_t)((N + 15) / 16)};
  const cuuint64_t strides[2] = {tile_blk, tile_blk * Kb};
  const cuuint32_t box[3] = {(cuuint32_t)(tile_blk / 4), 1, kBM / 16};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (scale, zero) pairs of the 16-row tiles, tile-major [RT][G][16] 32-bit words: one box is
// the pairs of one group for the 8 tiles of a CTA
bool encode_sz_3d(CUtensorMap* m, const void* base, int G, int N) {
  EncodeTiled enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {16, (cuuint64_t)G, (cuuint64_t)((N + 15) / 16)};
  const cuuint64_t strides[2] = {64, 64ull * G};
  const cuuint32_t box[3] = {16, 1, kBM / 16};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// grow a per-layer device scratch outside stream capture (false: too small and not growable)
bool ensure_scratch(void** buf, size_t* have, size_t need, cudaStream_t s) {
  if (need <= *have) return true;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return false;
  }
  cudaFree(*buf);
  *buf = nullptr;
  *have = 0;
  if (cudaMalloc(buf, need) != cudaSuccess) {
    cudaGetLastError();
    *buf = nullptr;
    return false;
  }
  *have = need;
  return true;
}

}  // namespace

// Token tile width: wider tiles dequantise each weight tile once for more tokens (the
// dequantisation, not the MMA, bounds the narrower tiles); the widest one fits three stages.
int gemm_tile_tokens(int M) { return M <= 64 ? 64 : M <= 256 ? 128 : 256; }

// The launch shape of one product (see GemmPlan).  Two cases leave SMs idle:
//  * fewer tiles than SMs: every tile is split over K (at least 4 steps per split);
//  * a short last wave: the CTAs are dispatched in order, so the last ceil(T / P) - T / P of a
//    wave of whole tiles holds few of them.  The row tiles of the last tt token tiles are then
//    split S ways over K instead; these short CTAs go to the SMs the whole tiles leave free.
//    The choice is a model in units of one whole tile's time: whole tiles end at w (or w + 1
//    with a partial wave of r); a short CTA takes its share of the steps plus a fixed cost
//    (start-up, pipeline fill, fp32 epilogue); the reduction's traffic (partials written and
//    read, the fp16 result) and its launch are charged at the end.  The tail is taken only
//    when the model saves at least kMinGain of a tile's time.
GemmPlan gemm_plan(int N, int K, int M, int sms) {
  constexpr double kSmFlops = 11e12;   // measured per-SM rate of whole 256-token tiles
  constexpr double kHbm = 6e12;        // bytes/s the reduction streams at
  constexpr double kCtaFixed = 3e-6;   // seconds of fixed cost per short CTA
  constexpr double kLaunch = 3e-6;     // seconds for the reduction's launch
  constexpr double kMinGain = 0.15;
  GemmPlan g;
  g.tile_tokens = gemm_tile_tokens(M);
  const int nK = K / kStepCodes;
  g.splits = 1; g.ksteps = nK;
  g.tail_tt = 0; g.tail_sp = 1; g.tail_ksteps = nK;
  if (sms < 1 || nK < 1 || N < 1 || M < 1) return g;
  const long long RT = (N + kBM - 1) / kBM, TT = (M + g.tile_tokens - 1) / g.tile_tokens, T = RT * TT;
  if (T < sms) {
    const int sp = (int)std::max<long long>(1, std::min<long long>(sms / T, nK / 4));
    if (sp > 1) {
      g.ksteps = (nK + sp - 1) / sp;
      g.splits = (nK + g.ksteps - 1) / g.ksteps;
    }
    return g;
  }
  const double tile_s = 2.0 * kBM * g.tile_tokens * (double)K / kSmFlops;
  const double fixed = kCtaFixed / tile_s;
  double best = (double)((T + sms - 1) / sms) - kMinGain;
  for (int tt = 1; tt <= 2 && tt < TT; ++tt) {
    const long long Tm = RT * (TT - tt), w = Tm / sms, r = Tm % sms, f = sms - r;
    for (int S = 2; S <= 8 && nK / S >= 4; ++S) {
      const int ks = (nK + S - 1) / S, se = (nK + ks - 1) / ks;   // the splits actually formed
      const double d = (double)ks / nK + fixed;
      const long long n = RT * tt * se, per = (long long)(1.0 / d);
      double end;
      if (r == 0) end = w + (double)((n + sms - 1) / sms) * d;
      else if (n <= f * per) end = w + 1.0;
      else end = w + 1.0 + (double)((n - f * per + sms - 1) / sms) * d;
      end += ((8.0 * se + 2.0) * tt * g.tile_tokens * (double)N / kHbm + kLaunch) / tile_s;
      if (end < best) {
        best = end;
        g.tail_tt = tt; g.tail_sp = se; g.tail_ksteps = ks;
      }
    }
  }
  return g;
}

namespace {

template <int BITS, int BN, int S, int DW>
owq_status_t run(Layer& L, const __half* x, __half* y, int M, long long wait_limit, bool skip_arrive,
                 cudaStream_t s) {
  if (!L.maps_ready) {
    if (!encode_packed_3d(&L.map_packed, L.packed, L.K, L.N, BITS)) return OWQ_ERR_CUDA;
    if (!encode_sz_3d(&L.map_sz, L.sz_t, L.G, L.N)) return OWQ_ERR_CUDA;   // (used by per-group prefill and the input gradient)
    L.maps_ready = true;
  }
  CUtensorMap mx;
  if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K * 2, 64, BN,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return OWQ_ERR_CUDA;
  GemmParams prm;
  prm.scales = L.scales; prm.zeros = L.zeros; prm.w_weak = L.w_weak; prm.k_ld = L.k_ld;
  prm.y = y; prm.status = device_status_ptr();
  prm.N = L.N; prm.K = L.K; prm.M = M; prm.G = L.G;
  prm.nw = L.k > 0 ? (L.k_ld + kStepCodes - 1) / kStepCodes : 0;
  prm.wait_limit = wait_limit; prm.skip_arrive = skip_arrive ? 1 : 0;
  if (!prm.status) return OWQ_ERR_CUDA;
  int sms = 0;   // SM count of the layer's device
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, L.device) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  GemmPlan g = gemm_plan(L.N, L.K, M, sms);
  const int RT = (L.N + kBM - 1) / kBM, TT = (M + BN - 1) / BN;
  // the split partials live in the layer's workspace, never grown during stream capture (the
  // call then runs unsplit)
  const int t0 = g.tail_sp > 1 ? (TT - g.tail_tt) * BN : 0;   // first token with split partials
  const int nsp = g.tail_sp > 1 ? g.tail_sp : g.splits;
  if (nsp > 1 && !ensure_scratch(reinterpret_cast<void**>(&L.gemm_ws), &L.gemm_ws_bytes,
                                 (size_t)nsp * (M - t0) * L.N * sizeof(float), s)) {
    g.splits = 1; g.ksteps = L.K / kStepCodes;
    g.tail_tt = 0; g.tail_sp = 1;
  }
  prm.ksteps = g.ksteps;
  prm.tail_y0 = TT - g.tail_tt;
  prm.tail_sp = g.tail_sp;
  prm.tail_ksteps = g.tail_ksteps;
  const bool split = g.splits > 1 || g.tail_sp > 1;
  prm.ws = split ? L.gemm_ws : nullptr;
  prm.ws_t0 = g.tail_sp > 1 ? t0 : 0;
  prm.ws_stride = (size_t)(M - prm.ws_t0) * L.N;
  // the tail variant only where a tail can occur (64-token tiles: one token tile per call)
  auto kern = k_gemm_sm100<BITS, BN, S, DW, false>;
  if (g.tail_sp > 1) {
    if constexpr (BN > 64) kern = k_gemm_sm100<BITS, BN, S, DW, true>;
    else return OWQ_ERR_CUDA;   // never planned: a tail needs two token tiles
  }
  constexpr int smem = smem_bytes<BITS, BN, S>();
  static_assert(smem <= 232448, "shared memory budget");
  // the CTAs an SM can hold (by shared memory) never need more than its 512 tensor-memory
  // columns, so an allocation never waits
  static_assert(BN + 64 * S <= (int)tmem_cols<BN, S>(), "tensor memory: accumulator + A stages");
  static_assert((232448 / smem) * tmem_cols<BN, S>() <= 512, "tensor memory per SM");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return OWQ_ERR_CUDA;
  }
  dim3 grid(RT, prm.tail_y0 + g.tail_tt * g.tail_sp, g.splits);
  // the weak activations, gathered once per call into the layer's scratch (grown outside capture)
  CUtensorMap mxw = mx;
  if (L.k > 0) {
    if (!ensure_scratch(reinterpret_cast<void**>(&L.gemm_xw), &L.gemm_xw_bytes, (size_t)M * L.k_ld * sizeof(__half), s))
      return OWQ_ERR_NOMEM;
    const size_t n = (size_t)M * L.k_ld;
    k_gather_weak_x<<<(unsigned)std::min<size_t>((n + 255) / 256, 2048), 256, 0, s>>>(x, M, L.K, L.idx, L.k, L.k_ld, L.gemm_xw,
                                                                                         prm.status);
    if (cudaGetLastError() != cudaSuccess) return OWQ_ERR_CUDA;
    if (!encode_2d(&mxw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, L.gemm_xw, (uint64_t)L.k_ld, (uint64_t)M, (uint64_t)L.k_ld * 2,
                   64, BN, CU_TENSOR_MAP_SWIZZLE_128B))
      return OWQ_ERR_CUDA;
  }
  kern<<<grid, 32 * (2 + DW), smem, s>>>(mx, L.map_packed, mxw, L.G > 1 ? L.map_sz : mx, prm);
  if (cudaGetLastError() != cudaSuccess) return OWQ_ERR_CUDA;
  if (split) {   // the split outputs: every token (K split over all tiles) or the tail's tokens
    const size_t MN = prm.ws_stride;
    k_splitk_reduce<<<(unsigned)std::min<size_t>((MN + 255) / 256, 4096), 256, 0, s>>>(prm.ws, nsp, MN,
                                                                                        y + (size_t)prm.ws_t0 * L.N);
    if (cudaGetLastError() != cudaSuccess) return OWQ_ERR_CUDA;
  }
  return OWQ_OK;
}

template <int BITS>
owq_status_t dispatch(Layer& L, const __half* x, __half* y, int M, long long wl, bool skip, cudaStream_t s) {
  switch (gemm_tile_tokens(M)) {
    case 64: return run<BITS, 64, 6, 8>(L, x, y, M, wl, skip, s);
    case 128: return run<BITS, 128, 4, 8>(L, x, y, M, wl, skip, s);
    default: return run<BITS, 256, 3, 16>(L, x, y, M, wl, skip, s);
  }
}

template <int BITS, int BN, int S, int DW>
owq_status_t ig_run(Layer& L, const __half* dy, __half* dx, int M, long long wait_limit, cudaStream_t s) {
  if (!L.maps_ready) {
    if (!encode_packed_3d(&L.map_packed, L.packed, L.K, L.N, BITS)) return OWQ_ERR_CUDA;
    if (!encode_sz_3d(&L.map_sz, L.sz_t, L.G, L.N)) return OWQ_ERR_CUDA;
    L.maps_ready = true;
  }
  CUtensorMap mdy, mdx;
  if (!encode_2d(&mdy, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dy, (uint64_t)L.N, (uint64_t)M, (uint64_t)L.N * 2, 64, BN,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mdx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dx, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K * 2, kStepCodes, BN,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return OWQ_ERR_CUDA;
  IgGemmParams prm;
  prm.dx = dx;
  prm.status = device_status_ptr();
  prm.N = L.N; prm.K = L.K; prm.M = M; prm.group = L.group;
  prm.wait_limit = wait_limit;
  if (!prm.status) return OWQ_ERR_CUDA;
  // fewer tiles than SMs: split the rows over CTAs (at least 4 steps each), fp32 partials in the
  // layer's prefill workspace, then the split-order reduction; never grown during stream capture
  const int nR = (L.N + 127) / 128, Kb = L.K / kStepCodes;
  const long long tiles = (long long)Kb * ((M + BN - 1) / BN);
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, L.device) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  int splits = tiles < sms ? (int)std::max<long long>(1, std::min<long long>(sms / tiles, nR / 4)) : 1;
  if (splits > 1) {
    prm.rsteps = (nR + splits - 1) / splits;
    splits = (nR + prm.rsteps - 1) / prm.rsteps;
    if (!ensure_scratch(reinterpret_cast<void**>(&L.gemm_ws), &L.gemm_ws_bytes, (size_t)splits * M * L.K * sizeof(float), s))
      splits = 1;
  }
  if (splits == 1) {
    prm.rsteps = nR;
    prm.ws = nullptr;
  } else {
    prm.ws = L.gemm_ws;
  }
  auto kern = k_igemm_sm100<BITS, BN, S, DW>;
  constexpr int smem = ig_smem_bytes<BITS, BN, S>();
  static_assert(smem <= 232448, "shared memory budget");
  static_assert((232448 / smem) * tmem_cols<BN, S>() <= 512, "tensor memory per SM");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return OWQ_ERR_CUDA;
  }
  dim3 grid(Kb, (M + BN - 1) / BN, splits);
  static_assert(BN * kStepCodes * 2 <= IgSmem<BITS, BN>::kStage, "output tile in the first stage");
  kern<<<grid, 32 * (3 + DW), smem, s>>>(mdy, L.map_packed, L.map_sz, mdx, prm);
  if (cudaGetLastError() != cudaSuccess) return OWQ_ERR_CUDA;
  if (splits > 1) {
    const size_t MK = (size_t)M * L.K;
    k_splitk_reduce<<<(unsigned)std::min<size_t>((MK + 255) / 256, 4096), 256, 0, s>>>(prm.ws, splits, MK, dx);
    if (cudaGetLastError() != cudaSuccess) return OWQ_ERR_CUDA;
  }
  return OWQ_OK;
}

template <int BITS>
owq_status_t ig_dispatch(Layer& L, const __half* dy, __half* dx, int M, long long wl, cudaStream_t s) {
  if (M <= 64) return ig_run<BITS, 64, 6, 8>(L, dy, dx, M, wl, s);
  if (M <= 256) return ig_run<BITS, 128, 4, 8>(L, dy, dx, M, wl, s);
  return ig_run<BITS, 256, 3, 16>(L, dy, dx, M, wl, s);
}

}  // namespace

owq_status_t gemm_sm100(Layer& L, const __half* x, __half* y, int M, long long wait_limit,
                        bool skip_arrive, cudaStream_t s) {
  return L.bits == 3 ? dispatch<3>(L, x, y, M, wait_limit, skip_arrive, s)
                     : dispatch<4>(L, x, y, M, wait_limit, skip_arrive, s);
}

owq_status_t igemm_sm100(Layer& L, const __half* dy, __half* dx, int M, long long wait_limit, cudaStream_t s) {
  return L.bits == 3 ? ig_dispatch<3>(L, dy, dx, M, wait_limit, s) : ig_dispatch<4>(L, dy, dx, M, wait_limit, s);
}

}  // namespace owq
