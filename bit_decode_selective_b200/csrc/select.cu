// select.cu -- chunked top-k channel selection.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// which-tiles-count paragraph: a projection's input channels are split into
// chunks of 1,024 and the k channels with the largest activation magnitude in
// each chunk are refined at this step (the error of a projection is the sum of
// activation times weight error, so a large |x| magnifies its channel's error).
//
// Every channel gets the unique key (|x| as the 15-bit fp16 magnitude) << 11 |
// (2047 - index in chunk), so equal magnitudes rank the lower index first.
// The k-th largest key is found by a block-wide radix select (radix.cuh); the
// selected channels are then written in ascending index order.
#include "common.cuh"
#include "internal.cuh"
#include "radix.cuh"

namespace sf {
namespace {

constexpr int kSelThreads = 256;

// One CTA per (batch row, chunk of up to 2,048 channels).
__global__ void __launch_bounds__(kSelThreads) select_chunks_kernel(const uint16_t* __restrict__ x,
                                                                   int K, int chunk, int kch,
                                                                   int32_t* __restrict__ sel) {
  pdl_trigger();  // a dependent GEMV may start streaming its base codes now
  pdl_wait();
  __shared__ uint32_t keys[2048];
  __shared__ RadixShared sh;
  const int b = blockIdx.y, c = blockIdx.x;
  const uint16_t* xc = x + (size_t)b * K + (size_t)c * chunk;
  for (int i = threadIdx.x; i < chunk; i += blockDim.x)
    keys[i] = ((uint32_t)(xc[i] & 0x7fff) << 11) | (uint32_t)(2047 - i);
  __syncthreads();
  auto key_at = [&](int i) { return (uint64_t)keys[i]; };
  const uint64_t tau = block_kth_largest<26>(key_at, chunk, kch, sh);
  int32_t* out = sel + ((size_t)b * (K / chunk) + c) * kch;
  block_compact(key_at, chunk, tau, sh, [&](int pos, int i, uint64_t) { out[pos] = c * chunk + i; });
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
  SF_CUDA(launch_pdl(select_chunks_kernel, grid, dim3(kSelThreads), 0, s, x, k, chunk, kch, sel));
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
