// wqlayout.cuh -- placement of the packed weight words (the sf_wq layout of
// sf.h), shared by the packer and the GEMV kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace sf {

// Word wi of a row of codes (plane L, or plane H of 3-bit codes) is stored at
// word wq_word(row, wi) of the row: the row's 16-byte units are permuted by an
// XOR with row mod 8 inside every 128-byte block.  Eight consecutive rows then
// hold any given unit in eight different 16-byte bank groups, so a warp that
// reads the same unit of eight rows from shared memory meets no bank conflict.
__host__ __device__ __forceinline__ int wq_word(int row, int wi) {
  return (((wi >> 2) ^ (row & 7)) << 2) | (wi & 3);
}

// Bit position of channel c (0..31) in the high-bit word of a 3-bit base block.
__host__ __device__ __forceinline__ int hi_plane_bit(int c) {
  return c < 16 ? 8 * (c >> 2) + (c & 3) : 8 * ((c - 16) >> 2) + 4 + ((c - 16) & 3);
}

// Base code of weight (n, c) of an N x K matrix of b-bit codes packed at base.
__host__ __device__ __forceinline__ int packed_base_code(const uint32_t* base, int N, int K, int b, long n,
                                                         long c) {
  if (b == 4) return (int)((base[(size_t)n * (K / 8) + wq_word((int)n, (int)(c / 8))] >> (4 * (c & 7))) & 15);
  int q = (int)((base[(size_t)n * (K / 16) + wq_word((int)n, (int)(c / 16))] >> (2 * (c & 15))) & 3);
  if (b == 3) {
    const uint32_t* hp = base + (size_t)N * K / 16;
    q |= (int)((hp[(size_t)n * (K / 32) + wq_word((int)n, (int)(c / 32))] >> hi_plane_bit((int)(c & 31))) & 1) << 2;
  }
  return q;
}

}  // namespace sf
