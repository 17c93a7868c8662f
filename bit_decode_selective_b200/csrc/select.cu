// select.cu -- chunked top-k channel selection.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// which-tiles-count paragraph: a projection's input channels are split into
// chunks of 1,024 and the k channels with the largest activation magnitude in
// each chunk are refined at this step (the error of a projection is the sum of
// activation times weight error, so a large |x| magnifies its channel's error).
//
// One CTA per (batch row, chunk).  Every channel gets the unique key
// (|x| as the 15-bit fp16 magnitude) << 11 | (2047 - index in chunk), so equal
// magnitudes rank the lower index first.  The k-th largest key is found bit by
// bit from the top with block-wide counts; the selected channels are then
// written in ascending index order with a block prefix sum.
#include "common.cuh"
#include "internal.cuh"

namespace sf {
namespace {

template <int E>
__global__ void __launch_bounds__(1024) select_chunks_kernel(const uint16_t* __restrict__ x, int K,
                                                             int chunk, int kch,
                                                             int32_t* __restrict__ sel) {
  pdl_trigger();  // a dependent GEMV may start streaming its base codes now
  __shared__ int warp_sums[32];
  const int b = blockIdx.y, c = blockIdx.x;
  const uint16_t* xc = x + (size_t)b * K + (size_t)c * chunk;
  uint32_t key[E];
#pragma unroll
  for (int e = 0; e < E; e++) {
    int i = threadIdx.x * E + e;
    key[e] = ((uint32_t)(xc[i] & 0x7fff) << 11) | (uint32_t)(2047 - i);
  }
  uint32_t tau = 0;  // largest value with count(key >= tau) >= kch
  for (int bit = 25; bit >= 0; --bit) {
    uint32_t cand = tau | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int e = 0; e < E; e++) cnt += __syncthreads_count(key[e] >= cand);
    if (cnt >= kch) tau = cand;
  }
  // exclusive prefix sum of the per-thread selected counts, in index order
  int mine = 0;
#pragma unroll
  for (int e = 0; e < E; e++) mine += key[e] >= tau;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int nw = blockDim.x >> 5;
    int v = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane < nw) warp_sums[lane] = v - (lane < nw ? warp_sums[lane] : 0);  // exclusive
  }
  __syncthreads();
  int pos = warp_sums[warp] + incl - mine;
  int32_t* out = sel + ((size_t)b * (K / chunk) + c) * kch;
#pragma unroll
  for (int e = 0; e < E; e++) {
    if (key[e] >= tau) out[pos++] = c * chunk + threadIdx.x * E + e;
  }
}

}  // namespace

sf_status check_select_args(const uint16_t* x, int batch, int k, int chunk, int kch) {
  SF_REQUIRE(x && aligned16(x), "x must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(batch >= 1 && batch <= 64, "batch=%d outside [1, 64]", batch);
  SF_UNSUPPORTED(chunk == 256 || chunk == 512 || chunk == 1024 || chunk == 2048,
                 "chunk=%d not in {256,512,1024,2048}", chunk);
  SF_REQUIRE(k > 0 && k % chunk == 0, "k=%d must be a positive multiple of chunk=%d", k, chunk);
  SF_REQUIRE(kch >= 1 && kch <= chunk, "kch=%d outside [1, chunk]", kch);
  return SF_OK;
}

sf_status launch_select(const uint16_t* x, int batch, int k, int chunk, int kch, int32_t* sel,
                        cudaStream_t s) {
  dim3 grid(k / chunk, batch);
  if (chunk <= 1024)
    select_chunks_kernel<1><<<grid, chunk, 0, s>>>(x, k, chunk, kch, sel);
  else
    select_chunks_kernel<2><<<grid, chunk / 2, 0, s>>>(x, k, chunk, kch, sel);
  SF_LAUNCHED();
  return SF_OK;
}

}  // namespace sf

extern "C" sf_status sf_select_channels(const uint16_t* x, int batch, int k, int chunk, int kch,
                                        int32_t* sel, sf_stream_t stream) {
  sf_status st = sf::check_select_args(x, batch, k, chunk, kch);
  if (st != SF_OK) return st;
  SF_REQUIRE(sel && sf::aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  return sf::launch_select(x, batch, k, chunk, kch, sel, sf::as_stream(stream));
}
