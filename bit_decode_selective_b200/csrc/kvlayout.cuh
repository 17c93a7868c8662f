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
// 3-bit codes are two planes of this layout: the low two bits (w = 2), then the
// high bit (w = 1) -- key words 0..7 and 8..11 of a token, value words 0..127
// and 128..191 of a tile.
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

// b-bit code of key element d of the token whose code words start at kp.
__host__ __device__ __forceinline__ uint32_t key_code(const uint32_t* kp, int d, int b) {
  int word, bit;
  if (b != 3) {
    key_pos(d, b, word, bit);
    return (kp[word] >> bit) & ((1u << b) - 1u);
  }
  key_pos(d, 2, word, bit);
  const uint32_t lo = (kp[word] >> bit) & 3u;
  key_pos(d, 1, word, bit);
  return lo | (((kp[8 + word] >> bit) & 1u) << 2);
}

// b-bit code of value element (tile token tt, dim d) of the tile whose code
// words start at vp.
__host__ __device__ __forceinline__ uint32_t value_code(const uint32_t* vp, int tt, int d, int b) {
  int word, bit;
  if (b != 3) {
    value_pos(tt, d, b, word, bit);
    return (vp[word] >> bit) & ((1u << b) - 1u);
  }
  value_pos(tt, d, 2, word, bit);
  const uint32_t lo = (vp[word] >> bit) & 3u;
  value_pos(tt, d, 1, word, bit);
  return lo | (((vp[128 + word] >> bit) & 1u) << 2);
}

}  // namespace sf
