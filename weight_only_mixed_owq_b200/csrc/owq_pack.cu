// Packing (codes -> latency-favoured packed words) and the dequantisation test hook.
#include "owq_internal.cuh"
#include "owq_format.cuh"

namespace owq {
namespace {

// One thread per 32-code chunk.  Codes of weak columns are replaced by the zero point of
// their (row, group), so the packed dense matrix dequantises to exactly 0 there.
template <int BITS>
__global__ void k_pack(const uint8_t* __restrict__ codes, const __half* __restrict__ zeros,
                       const uint32_t* __restrict__ weak_mask, int N, int K, int group,
                       uint32_t* __restrict__ packed) {
  const int C = K / kChunkCodes;
  size_t item = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (size_t)N * C) return;
  const int i = (int)(item / C), ch = (int)(item % C);
  const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)i * K + (size_t)ch * kChunkCodes);
  uint4 a = src[0], b = src[1];
  const uint32_t raw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t c[32];
  #pragma unroll
  for (int q = 0; q < 32; ++q) c[q] = (raw[q / 4] >> (8 * (q % 4))) & ((1u << BITS) - 1u);
  uint32_t wm = weak_mask ? weak_mask[ch] : 0u;
  if (wm) {
    const int G = K / group;
    #pragma unroll
    for (int q = 0; q < 32; ++q)
      if ((wm >> q) & 1u) {
        int col = ch * kChunkCodes + q;
        c[q] = (uint32_t)__half2float(zeros[(size_t)i * G + col / group]);
      }
  }
  uint32_t w[BITS];
  encode_chunk<BITS>(c, w);
  uint32_t* dst = packed + item * BITS;
  #pragma unroll
  for (int j = 0; j < BITS; ++j) dst[j] = w[j];
}

// One thread per chunk: W_hat = fp16_rn(s * (q - z)) (the product is exact in fp32).
template <int BITS>
__global__ void k_dequant(const uint32_t* __restrict__ packed, const __half* __restrict__ scales,
                          const __half* __restrict__ zeros, int N, int K, int group,
                          __half* __restrict__ w_hat, uint8_t* __restrict__ codes_out) {
  const int C = K / kChunkCodes, G = K / group;
  size_t item = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (size_t)N * C) return;
  const int i = (int)(item / C), ch = (int)(item % C);
  uint32_t w[BITS];
  #pragma unroll
  for (int j = 0; j < BITS; ++j) w[j] = packed[item * BITS + j];
  uint32_t c[32];
  decode_chunk<BITS>(w, c);
  const int col0 = ch * kChunkCodes;
  const float s = __half2float(scales[(size_t)i * G + col0 / group]);
  const float z = __half2float(zeros[(size_t)i * G + col0 / group]);
  uint32_t hv[16];
  #pragma unroll
  for (int p = 0; p < 16; ++p) {
    __half lo = __float2half_rn(__fmul_rn(s, __fsub_rn((float)c[2 * p], z)));
    __half hi = __float2half_rn(__fmul_rn(s, __fsub_rn((float)c[2 * p + 1], z)));
    hv[p] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(w_hat + (size_t)i * K + col0);
  #pragma unroll
  for (int v = 0; v < 4; ++v) dst[v] = make_uint4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2], hv[4 * v + 3]);
  if (codes_out) {
    uint32_t cb[8];
    #pragma unroll
    for (int v = 0; v < 8; ++v)
      cb[v] = c[4 * v] | (c[4 * v + 1] << 8) | (c[4 * v + 2] << 16) | (c[4 * v + 3] << 24);
    uint4* cd = reinterpret_cast<uint4*>(codes_out + (size_t)i * K + col0);
    cd[0] = make_uint4(cb[0], cb[1], cb[2], cb[3]);
    cd[1] = make_uint4(cb[4], cb[5], cb[6], cb[7]);
  }
}

}  // namespace

cudaError_t launch_pack(const uint8_t* codes, const __half* zeros, const uint32_t* weak_mask,
                        int N, int K, int bits, int group, uint32_t* packed, cudaStream_t s) {
  const size_t items = (size_t)N * (K / kChunkCodes);
  const unsigned grid = (unsigned)((items + 255) / 256);
  if (bits == 3) k_pack<3><<<grid, 256, 0, s>>>(codes, zeros, weak_mask, N, K, group, packed);
  else k_pack<4><<<grid, 256, 0, s>>>(codes, zeros, weak_mask, N, K, group, packed);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const Layer& L, __half* w_hat, uint8_t* codes, cudaStream_t s) {
  const size_t items = (size_t)L.N * (L.K / kChunkCodes);
  const unsigned grid = (unsigned)((items + 255) / 256);
  if (L.bits == 3) k_dequant<3><<<grid, 256, 0, s>>>(L.packed, L.scales, L.zeros, L.N, L.K, L.group, w_hat, codes);
  else k_dequant<4><<<grid, 256, 0, s>>>(L.packed, L.scales, L.zeros, L.N, L.K, L.group, w_hat, codes);
  return cudaGetLastError();
}

}  // namespace owq
