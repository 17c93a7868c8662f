// radix.cuh -- block-wide exact top-k on unique integer keys.
//
// The k-th largest of n unique keys is found 8 bits at a time from the top:
// each pass histograms the next digit of the keys that share the prefix found
// so far (one private histogram per warp, so atomics only meet within a warp),
// sums the warps' histograms, then one warp scans the 256 bins from the top.  The
// search stops early once the keys sharing the prefix are exactly the ones
// still needed.  The selected keys (key >= threshold) are then written in
// index order with a block prefix sum.
#pragma once

#include "common.cuh"

namespace sf {

constexpr int kRadixMaxWarps = 32;

struct RadixShared {
  int hist[kRadixMaxWarps][256];  // one private histogram per warp
  int tot[256];
  int digit, kleft, done;
  int warp_tot[32];
};

// KeyAt: (int i) -> uint64_t, i < n.  KEY_BITS: significant low bits of the keys.
template <int KEY_BITS, class KeyAt>
__device__ uint64_t block_kth_largest(KeyAt key_at, int n, int k, RadixShared& sh) {
  uint64_t prefix = 0, mask = 0;
  const int lane = threadIdx.x & 31;
  const int n_pad = (n + blockDim.x - 1) / blockDim.x * blockDim.x;
  constexpr int TOP = ((KEY_BITS + 7) / 8 - 1) * 8;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int shift = TOP; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < nwarps * 256; i += blockDim.x) (&sh.hist[0][0])[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n_pad; i += blockDim.x) {
      if (i < n) {
        const uint64_t key = key_at(i);
        if ((key & mask) == prefix) atomicAdd(&sh.hist[warp][(key >> shift) & 255], 1);
      }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      int t = 0;
      for (int w = 0; w < nwarps; w++) t += sh.hist[w][b];
      sh.tot[b] = t;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; j++) tot += (c[j] = sh.tot[255 - 8 * lane - j]);
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int above = incl - tot;
      if (above < k && incl >= k) {
        int run = above;
        for (int j = 0; j < 8; j++) {
          if (run + c[j] >= k) {
            sh.digit = 255 - 8 * lane - j;
            sh.kleft = k - run;
            sh.done = (c[j] == k - run);  // every key of this bucket is needed
            break;
          }
          run += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint64_t)sh.digit << shift;
    mask |= (uint64_t)255 << shift;
    k = sh.kleft;
    const bool done = sh.done;
    __syncthreads();
    if (done) break;  // keys >= prefix (low bits zero) are exactly the top k
  }
  return prefix;
}

// Emit the keys >= tau in index order; emit(pos, i, key).  Each thread owns a
// contiguous range of indices so the order is kept.
template <class KeyAt, class Emit>
__device__ void block_compact(KeyAt key_at, int n, uint64_t tau, RadixShared& sh, Emit emit) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  int mine = 0;
  for (int i = i0; i < i1; i++) mine += key_at(i) >= tau;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sh.warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const int v = lane < nw ? sh.warp_tot[lane] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    if (lane < nw) sh.warp_tot[lane] = x - v;
  }
  __syncthreads();
  int pos = sh.warp_tot[warp] + incl - mine;
  for (int i = i0; i < i1; i++) {
    const uint64_t key = key_at(i);
    if (key >= tau) emit(pos++, i, key);
  }
  __syncthreads();
}

}  // namespace sf
