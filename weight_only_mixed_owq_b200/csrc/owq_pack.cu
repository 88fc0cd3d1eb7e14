// Packing (codes -> latency-favoured packed words) and the dequantisation test hook.
#include "owq_internal.cuh"
#include "owq_format.cuh"

namespace owq {
namespace {

// Storage order of the blocks in a layer: rows are grouped in tiles of 16 (the last tile
// padded with zero rows); a tile stores its blocks block-major, so block b of rows
// 16t .. 16t+15 is one contiguous run of 16 blocks at block index (t * Kb + b) * 16 + row % 16.
__host__ __device__ __forceinline__ size_t tiled_block(int row, int b, int Kb) {
  return ((size_t)(row >> 4) * Kb + b) * 16 + (row & 15);
}

// One thread per 128-code block.  Codes of weak columns are replaced by the zero point of
// their (row, group), so the packed dense matrix dequantises to exactly 0 there.
template <int BITS>
__global__ void k_pack(const uint8_t* __restrict__ codes, const __half* __restrict__ zeros,
                       const uint32_t* __restrict__ weak_mask, int N, int K, int group,
                       uint32_t* __restrict__ packed) {
  const int Kb = K / kBlockCodes;
  size_t item = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (size_t)N * Kb) return;
  const int i = (int)(item / Kb), b = (int)(item % Kb);
  const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)i * K + (size_t)b * kBlockCodes);
  uint32_t c[kBlockCodes];
  #pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint4 a = src[v];
    const uint32_t raw[4] = {a.x, a.y, a.z, a.w};
    #pragma unroll
    for (int u = 0; u < 16; ++u) c[16 * v + u] = (raw[u / 4] >> (8 * (u % 4))) & ((1u << BITS) - 1u);
  }
  if (weak_mask) {
    const int G = K / group;
    #pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t wm = weak_mask[b * 4 + m];
      if (!wm) continue;
      #pragma unroll
      for (int q = 0; q < 32; ++q)
        if ((wm >> q) & 1u) {
          const int col = b * kBlockCodes + 32 * m + q;
          c[32 * m + q] = (uint32_t)__half2float(zeros[(size_t)i * G + col / group]);
        }
    }
  }
  uint32_t w[4 * BITS];
  encode_block<BITS>(c, w);
  uint4* dst = reinterpret_cast<uint4*>(packed + tiled_block(i, b, Kb) * 4 * BITS);
  #pragma unroll
  for (int v = 0; v < BITS; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
}

// One thread per block: W_hat = fp16_rn(s * (q - z)) (the product is exact in fp32).
template <int BITS>
__global__ void k_dequant(const uint32_t* __restrict__ packed, const __half* __restrict__ scales,
                          const __half* __restrict__ zeros, int N, int K, int group,
                          __half* __restrict__ w_hat, uint8_t* __restrict__ codes_out) {
  const int Kb = K / kBlockCodes, G = K / group;
  size_t item = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (size_t)N * Kb) return;
  const int i = (int)(item / Kb), b = (int)(item % Kb);
  uint32_t w[4 * BITS];
  const uint4* src = reinterpret_cast<const uint4*>(packed + tiled_block(i, b, Kb) * 4 * BITS);
  #pragma unroll
  for (int v = 0; v < BITS; ++v) {
    const uint4 a = src[v];
    w[4 * v] = a.x; w[4 * v + 1] = a.y; w[4 * v + 2] = a.z; w[4 * v + 3] = a.w;
  }
  uint32_t c[kBlockCodes];
  decode_block<BITS>(w, c);
  const int col0 = b * kBlockCodes;
  const float s = __half2float(scales[(size_t)i * G + col0 / group]);
  const float z = __half2float(zeros[(size_t)i * G + col0 / group]);
  uint4* dst = reinterpret_cast<uint4*>(w_hat + (size_t)i * K + col0);
  #pragma unroll
  for (int v = 0; v < 16; ++v) {
    uint32_t hv[4];
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = 8 * v + 2 * u;
      const __half lo = __float2half_rn(__fmul_rn(s, __fsub_rn((float)c[k], z)));
      const __half hi = __float2half_rn(__fmul_rn(s, __fsub_rn((float)c[k + 1], z)));
      hv[u] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
    }
    dst[v] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
  if (codes_out) {
    uint4* cd = reinterpret_cast<uint4*>(codes_out + (size_t)i * K + col0);
    #pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint32_t cb[4];
      #pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = 16 * v + 4 * u;
        cb[u] = c[k] | (c[k + 1] << 8) | (c[k + 2] << 16) | (c[k + 3] << 24);
      }
      cd[v] = make_uint4(cb[0], cb[1], cb[2], cb[3]);
    }
  }
}

// Tile-major copy of the weak block for the decode kernel: element (row, t) of the row-major
// [N][k_ld] block goes to [row / 16][t / 16][row % 16][t % 16] (rows past N are zero).
__global__ void k_weak_tiles(const __half* __restrict__ w, int N, int k_ld, __half* __restrict__ wt) {
  const size_t RT = (size_t)(N + 15) / 16;
  size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= RT * 16 * k_ld) return;
  const int col = (int)(e % 16), r = (int)((e / 16) % 16);
  const size_t sl = (e / 256) % (size_t)(k_ld / 16), tile = e / ((size_t)256 * (k_ld / 16));
  const size_t row = tile * 16 + r;
  wt[e] = row < (size_t)N ? w[row * k_ld + sl * 16 + col] : __float2half_rn(0.f);
}

// Tile-major (scale, zero) pairs for the decode kernel: entry (row, grp) goes to
// [row / 16][grp][row % 16] (rows past N are (0, 0)).
__global__ void k_sz_tiles(const __half* __restrict__ scales, const __half* __restrict__ zeros, int N, int G,
                           __half2* __restrict__ szt) {
  const size_t RT = (size_t)(N + 15) / 16;
  size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= RT * G * 16) return;
  const int r = (int)(e % 16);
  const size_t grp = (e / 16) % (size_t)G, tile = e / ((size_t)16 * G);
  const size_t row = tile * 16 + r;
  szt[e] = row < (size_t)N ? __halves2half2(scales[row * G + grp], zeros[row * G + grp])
                           : __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
}

}  // namespace

cudaError_t launch_sz_tiles(const __half* scales, const __half* zeros, int N, int G, __half2* sz_t, cudaStream_t s) {
  const size_t n = (size_t)((N + 15) / 16) * G * 16;
  k_sz_tiles<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(scales, zeros, N, G, sz_t);
  return cudaGetLastError();
}

cudaError_t launch_weak_tiles(const __half* w_weak, int N, int k_ld, __half* w_weak_t, cudaStream_t s) {
  const size_t n = (size_t)((N + 15) / 16) * 16 * k_ld;
  k_weak_tiles<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w_weak, N, k_ld, w_weak_t);
  return cudaGetLastError();
}

cudaError_t launch_pack(const uint8_t* codes, const __half* zeros, const uint32_t* weak_mask,
                        int N, int K, int bits, int group, uint32_t* packed, cudaStream_t s) {
  const size_t items = (size_t)N * (K / kBlockCodes);
  const unsigned grid = (unsigned)((items + 127) / 128);
  if (bits == 3) k_pack<3><<<grid, 128, 0, s>>>(codes, zeros, weak_mask, N, K, group, packed);
  else k_pack<4><<<grid, 128, 0, s>>>(codes, zeros, weak_mask, N, K, group, packed);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const Layer& L, __half* w_hat, uint8_t* codes, cudaStream_t s) {
  const size_t items = (size_t)L.N * (L.K / kBlockCodes);
  const unsigned grid = (unsigned)((items + 127) / 128);
  if (L.bits == 3) k_dequant<3><<<grid, 128, 0, s>>>(L.packed, L.scales, L.zeros, L.N, L.K, L.group, w_hat, codes);
  else k_dequant<4><<<grid, 128, 0, s>>>(L.packed, L.scales, L.zeros, L.N, L.K, L.group, w_hat, codes);
  return cudaGetLastError();
}

}  // namespace owq
