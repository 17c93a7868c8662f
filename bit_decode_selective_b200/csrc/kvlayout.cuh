// kvlayout.cuh -- the pair-slot layout of KV codes (include/sf.h, sf_kv).
//
// A 32-bit word holds 16/w pairs of w-bit codes; pair slot j keeps its first
// code at bits [w*j, w*j+w) and its second at [16+w*j, 16+w*j+w).  The order
// is the register order of the m16n8k16 tensor-core fragments that read them,
// so a thread turns one word into half2 operands with a mask, an OR of the
// fp16 exponent of 1024 and one fused multiply-add (exact small integers).
//   keys   -- per token, 4 chunks c of w words; pair p = 2s+e of chunk c:
//             dims 16s+2c+8e (first), 16s+2c+8e+1 (second);
//   values -- per 16-token tile, 32 chunks l = 4g+c of 2w words; pair
//             p = 16h+2m+e of chunk l: dim 16m+g+8e of tile tokens 2c+8h
//             (first) and 2c+8h+1 (second).
#pragma once

#include "common.cuh"

namespace sf {

constexpr int kHeadDim = 128;

// Word (within the token) and bit of key element d, w-bit codes.
__host__ __device__ __forceinline__ void key_pos(int d, int w, int& word, int& bit) {
  int s = d >> 4, within = d & 15;
  int e = within >> 3, c = (within & 7) >> 1, second = within & 1;
  int p = 2 * s + e, per = 16 / w;
  word = c * w + p / per;
  bit = 16 * second + w * (p % per);
}

// Word (within the 16-token tile) and bit of value element (tile token tt, dim d).
__host__ __device__ __forceinline__ void value_pos(int tt, int d, int w, int& word, int& bit) {
  int m = d >> 4, within = d & 15;
  int e = within >> 3, g = within & 7;
  int h = tt >> 3, c = (tt & 7) >> 1, second = tt & 1;
  int l = 4 * g + c, p = 16 * h + 2 * m + e, per = 16 / w;
  word = l * (2 * w) + p / per;
  bit = 16 * second + w * (p % per);
}

// Pair slot `slot` of word w as an exact half2 (first code in the low half).
// Codes sitting at bit offsets that fit the fp16 mantissa are masked in
// place; higher slots use the word shifted right by 8.
template <int W, int SLOT>
__device__ __forceinline__ uint32_t pair_h2(uint32_t w, uint32_t w_hi8) {
  constexpr int BIT = W * SLOT;
  constexpr bool SHIFT = BIT + W > 10;
  constexpr int B2 = SHIFT ? BIT - 8 : BIT;
  constexpr uint32_t MASK = (((1u << W) - 1u) << B2) * 0x00010001u;
  uint32_t v = ((SHIFT ? w_hi8 : w) & MASK) | 0x64006400u;  // halves = 1024 + c * 2^B2
  // c = v * 2^-B2 - 1024 * 2^-B2, exact in fp16
  const __half2 sc = __float2half2_rn(1.0f / (float)(1 << B2));
  const __half2 off = __float2half2_rn(-1024.0f / (float)(1 << B2));
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&v), sc, off);
  return *reinterpret_cast<uint32_t*>(&r);
}

}  // namespace sf
