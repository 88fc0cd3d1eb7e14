// Packed-code format of the latency-favoured OWQ layout ("Storage Methods", appendix §2 of
// the OWQ paper as summarised on paperlayer.ai: a full low-precision matrix, zero-filled at
// the weak columns, plus an fp16 block of the weak columns).
//
// A row of K codes is a sequence of 32-code chunks; chunk c of row i is `bits` little-endian
// uint32 words at word offset (i*K/32 + c)*bits, so a 128-code block is bits x 16 bytes.
// Codes 2t and 2t+1 of a chunk form pair t: the even code sits at bit offset o of a word
// and the odd code at 16 + o of the same word.
//   4-bit: pair t -> word t/4, o = 4 (t%4).
//   3-bit: pair t < 15 -> word t/5, o = 3 (t%5); pair 15: bit e of code 30 is bit 15 of
//          word e and bit e of code 31 is bit 31 of word e.
// Why: every pair then lies in the two 16-bit halves of one register at the same offset,
// so one AND with a mask such as 0x00070007 lifts a pair into an fp16x2 whose halves are
// the codes times a power of two (the unused high bits stay 0, so each half reads as a
// subnormal or small normal fp16 whose value is exactly code * 2^(o-24) for o + bits <= 11).
#pragma once
#include <cstdint>

namespace owq {

// Encode 32 codes (c[0..31], each < 2^bits) into `bits` words.
template <int BITS>
__host__ __device__ __forceinline__ void encode_chunk(const uint32_t* c, uint32_t* w) {
  if constexpr (BITS == 4) {
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t v = 0;
      #pragma unroll
      for (int r = 0; r < 4; ++r) {
        int t = 4 * j + r;
        v |= (c[2 * t] << (4 * r)) | (c[2 * t + 1] << (16 + 4 * r));
      }
      w[j] = v;
    }
  } else {
    #pragma unroll
    for (int j = 0; j < 3; ++j) {
      uint32_t v = 0;
      #pragma unroll
      for (int r = 0; r < 5; ++r) {
        int t = 5 * j + r;
        v |= (c[2 * t] << (3 * r)) | (c[2 * t + 1] << (16 + 3 * r));
      }
      v |= ((c[30] >> j) & 1u) << 15;
      v |= ((c[31] >> j) & 1u) << 31;
      w[j] = v;
    }
  }
}

// Decode `bits` words into 32 codes.
template <int BITS>
__host__ __device__ __forceinline__ void decode_chunk(const uint32_t* w, uint32_t* c) {
  if constexpr (BITS == 4) {
    #pragma unroll
    for (int t = 0; t < 16; ++t) {
      uint32_t v = w[t / 4] >> (4 * (t % 4));
      c[2 * t] = v & 0xFu;
      c[2 * t + 1] = (v >> 16) & 0xFu;
    }
  } else {
    #pragma unroll
    for (int t = 0; t < 15; ++t) {
      uint32_t v = w[t / 5] >> (3 * (t % 5));
      c[2 * t] = v & 0x7u;
      c[2 * t + 1] = (v >> 16) & 0x7u;
    }
    c[30] = ((w[0] >> 15) & 1u) | (((w[1] >> 15) & 1u) << 1) | (((w[2] >> 15) & 1u) << 2);
    c[31] = ((w[0] >> 31) & 1u) | (((w[1] >> 31) & 1u) << 1) | (((w[2] >> 31) & 1u) << 2);
  }
}

}  // namespace owq
