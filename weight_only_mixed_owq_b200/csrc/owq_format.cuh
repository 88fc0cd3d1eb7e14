// Packed-code format of the latency-favoured OWQ layout ("Storage Methods", appendix §2 of
// the OWQ paper as summarised on paperlayer.ai: a full low-precision matrix, zero-filled at
// the weak columns, plus an fp16 block of the weak columns).
//
// A row of K codes is a sequence of 128-code blocks; block b of row i is 4*bits little-endian
// uint32 words at word offset (i*K/128 + b)*4*bits.  Codes 2p and 2p+1 of a block form pair p.
// The block is four chunks of `bits` words; chunk q holds the pairs p = 4j + q (j = 0..15).
// Pair j of a chunk sits at a slot (word, offset): even code at the offset, odd code 16 bits
// higher in the same word.
//   4-bit: word 2(j/8) + j%2, offset 4((j%8)/2).
//   3-bit: (0,0) (1,0) (0,3) (1,3) (0,6) (1,6) (0,9) (1,9) (0,12) (1,12) (2,6) D (2,3) (2,12)
//          (2,0) (2,9); slot D (j = 11): bit e of the even / odd code is bit 15 / 31 of word e.
//
// Why this layout.  The m16n8k16 tensor-core fragment gives lane (g, t) of a warp the k-pairs
// t and t+4 of every 16-wide k slice, i.e. the block pairs p = 4j + t: one chunk per lane.
// Within a chunk, the two pairs one k slice needs (j = 2s, 2s+1) sit at the same bit offset
// (after at most one shift), so one AND per pair lifts them into an fp16x2 register whose
// halves equal code * 2^(o - 24) exactly (the code bits lie in the low 11 bits of each half,
// where fp16 is linear in its bit pattern), and both registers of the slice share the scale
// 2^(o - 24).  With the 3-bit slots above, one right shift by 9 per word serves every pair
// that is not at offset 0, 3 or 6 (offsets 9 and 12 become 0 and 3), and the spread pair D is
// rebuilt at offset 6 from the same shifted words (bit 15 lands on bit 6).  The prefill kernel
// reads the same pairs and forms fp16_rn(s (q - z)) from them.
#pragma once
#include <cstdint>

namespace owq {

// ---- scalar encode / decode of a whole block (pack and dequantise kernels) ----
struct Slot { int word, off; };

__host__ __device__ constexpr Slot slot3(int j) {
  constexpr int w[16] = {0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 2, -1, 2, 2, 2, 2};
  constexpr int o[16] = {0, 0, 3, 3, 6, 6, 9, 9, 12, 12, 6, -1, 3, 12, 0, 9};
  return Slot{w[j], o[j]};
}
__host__ __device__ constexpr Slot slot4(int j) { return Slot{2 * (j / 8) + (j % 2), 4 * ((j % 8) / 2)}; }

// c[0..127] (each < 2^BITS) -> w[0 .. 4*BITS)
template <int BITS>
__host__ __device__ __forceinline__ void encode_block(const uint32_t* c, uint32_t* w) {
  #pragma unroll
  for (int i = 0; i < 4 * BITS; ++i) w[i] = 0u;
  #pragma unroll
  for (int q = 0; q < 4; ++q)
    #pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t ev = c[2 * (4 * j + q)], od = c[2 * (4 * j + q) + 1];
      const Slot sl = BITS == 3 ? slot3(j) : slot4(j);
      if (sl.word < 0) {
        #pragma unroll
        for (int e = 0; e < 3; ++e) w[q * BITS + e] |= (((ev >> e) & 1u) << 15) | (((od >> e) & 1u) << 31);
      } else {
        w[q * BITS + sl.word] |= (ev << sl.off) | (od << (16 + sl.off));
      }
    }
}

template <int BITS>
__host__ __device__ __forceinline__ void decode_block(const uint32_t* w, uint32_t* c) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  #pragma unroll
  for (int q = 0; q < 4; ++q)
    #pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int p = 4 * j + q;
      const Slot sl = BITS == 3 ? slot3(j) : slot4(j);
      if (sl.word < 0) {
        uint32_t ev = 0, od = 0;
        #pragma unroll
        for (int e = 0; e < 3; ++e) {
          ev |= ((w[q * BITS + e] >> 15) & 1u) << e;
          od |= ((w[q * BITS + e] >> 31) & 1u) << e;
        }
        c[2 * p] = ev;
        c[2 * p + 1] = od;
      } else {
        c[2 * p] = (w[q * BITS + sl.word] >> sl.off) & mask;
        c[2 * p + 1] = (w[q * BITS + sl.word] >> (16 + sl.off)) & mask;
      }
    }
}

// ---- register extraction of pair j of a chunk (tensor-core and prefill kernels) ----
// Returns the pair with both codes at bit offset class_off(pair_class(j)) of each 16-bit half
// and every other bit clear.  j is compile-time after unrolling.  The two pairs of one k slice
// (j = 2s, 2s + 1) share a class.  k2 and k4 are 2 and 4: passed in at run time, they keep the
// rebuild of pair D on the multiply-add pipe (as integer multiply-adds) instead of the integer
// logic pipe that the other extractions load.
template <int BITS>
__host__ __device__ constexpr int pair_class(int j) {
  if (BITS == 3) {
    constexpr int c[16] = {0, 0, 1, 1, 2, 2, 0, 0, 1, 1, 2, 2, 1, 1, 0, 0};
    return c[j];
  } else {
    return (j / 2) % 2;   // offsets 0, 4, 0 (after >> 8), 4 (after >> 8)
  }
}
template <int BITS>
__host__ __device__ constexpr int class_off(int cls) { return BITS == 3 ? 3 * cls : 4 * cls; }

template <int BITS>
__device__ __forceinline__ uint32_t pair_bits(const uint32_t* w, int j, uint32_t k2 = 2u, uint32_t k4 = 4u) {
  if constexpr (BITS == 3) {
    constexpr uint32_t m0 = 0x00070007u, m1 = 0x00380038u, m2 = 0x01C001C0u, mD = 0x00400040u;
    switch (j) {
      case 0: return w[0] & m0;
      case 1: return w[1] & m0;
      case 2: return w[0] & m1;
      case 3: return w[1] & m1;
      case 4: return w[0] & m2;
      case 5: return w[1] & m2;
      case 6: return (w[0] >> 9) & m0;
      case 7: return (w[1] >> 9) & m0;
      case 8: return (w[0] >> 9) & m1;
      case 9: return (w[1] >> 9) & m1;
      case 10: return w[2] & m2;
      case 11: return ((w[0] >> 9) & mD) + ((w[1] >> 9) & mD) * k2 + ((w[2] >> 9) & mD) * k4;
      case 12: return w[2] & m1;
      case 13: return (w[2] >> 9) & m1;
      case 14: return w[2] & m0;
      default: return (w[2] >> 9) & m0;
    }
  } else {
    (void)k2;
    (void)k4;
    const uint32_t v = w[2 * (j / 8) + (j % 2)];
    switch ((j % 8) / 2) {
      case 0: return v & 0x000F000Fu;
      case 1: return v & 0x00F000F0u;
      case 2: return (v >> 8) & 0x000F000Fu;
      default: return (v >> 8) & 0x00F000F0u;
    }
  }
}

}  // namespace owq
