// wqlayout.cuh -- placement of the packed weight words (the sf_wq layout of
// sf.h), shared by the packer and the GEMV kernels.
#pragma once

namespace sf {

// Word wi of a row of codes (plane L, or plane H of 3-bit codes) is stored at
// word wq_word(row, wi) of the row: the row's 16-byte units are permuted by an
// XOR with row mod 8 inside every 128-byte block.  Eight consecutive rows then
// hold any given unit in eight different 16-byte bank groups, so a warp that
// reads the same unit of eight rows from shared memory meets no bank conflict.
__host__ __device__ __forceinline__ int wq_word(int row, int wi) {
  return (((wi >> 2) ^ (row & 7)) << 2) | (wi & 3);
}

}  // namespace sf
