// select.cu -- chunked top-k channel selection.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// which-tiles-count paragraph: a projection's input channels are split into
// chunks of 1,024 and the k channels with the largest activation magnitude in
// each chunk are refined at this step (the error of a projection is the sum of
// activation times weight error, so a large |x| magnifies its channel's error).
//
// One warp per (batch row, chunk): lane L holds channels [L per, (L+1) per)
// of the chunk (per = chunk / 32) as 15-bit fp16 magnitudes (bits & 0x7fff,
// so +0 == -0).  The k-th largest magnitude thr is found bit by bit from the
// top (the largest value with at least k magnitudes >= it; one warp-wide
// count per bit), then every channel above thr is taken, and of the channels
// equal to thr the lowest-indexed ones fill the rest (a warp prefix count in
// channel order).  Selected channels are written in ascending order from the
// lanes' exclusive prefix counts.  A CTA is that one warp, with no shared
// memory: it fits in the room every whole-SM kernel leaves free (kSideRegs),
// so a selection on a staging stream never waits for, or delays, them.
#include "common.cuh"
#include "internal.cuh"

namespace sf {
namespace {


__device__ __forceinline__ int warp_exclusive_sum(int v, int lane) {
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  return incl - v;
}

static_assert(32 * 128 <= kSideRegs, "a selection CTA must fit in the room left for staging");
template <int PER>
__global__ void __maxnreg__(128) select_chunks_kernel(const uint16_t* __restrict__ x, int K, int kch,
                                                           int jobs, int32_t* __restrict__ sel) {
  pdl_trigger();  // a dependent GEMV may start streaming its base codes now
  pdl_wait();
  constexpr int chunk = 32 * PER;
  const int lane = threadIdx.x & 31;
  const int job = blockIdx.x;
  const int nch = K / chunk, b = job / nch, c = job - b * nch;
  const uint16_t* xc = x + (size_t)b * K + (size_t)c * chunk + lane * PER;
  uint32_t m[PER];
#pragma unroll
  for (int v = 0; v < PER / 8; v++) {
    const uint4 q = reinterpret_cast<const uint4*>(xc)[v];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; h++) {
      m[8 * v + 2 * h] = w[h] & 0x7fffu;
      m[8 * v + 2 * h + 1] = (w[h] >> 16) & 0x7fffu;
    }
  }
  // thr: the largest value with count(m >= thr) >= kch, i.e. the kch-th largest
  uint32_t thr = 0;
#pragma unroll 1
  for (int bit = 14; bit >= 0; bit--) {
    const uint32_t cand = thr | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < PER; i++) cnt += m[i] >= cand;
    if (__reduce_add_sync(0xffffffffu, cnt) >= kch) thr = cand;
  }
  int gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < PER; i++) gt += m[i] > thr, eq += m[i] == thr;
  const int need_eq = kch - __reduce_add_sync(0xffffffffu, gt);  // >= 1
  const int eq_before = warp_exclusive_sum(eq, lane);
  const int take = max(0, min(eq, need_eq - eq_before));
  int pos = warp_exclusive_sum(gt + take, lane);
  int32_t* out = sel + (size_t)job * kch;
  const int ch0 = c * chunk + lane * PER;
  int taken = 0;
#pragma unroll
  for (int i = 0; i < PER; i++) {
    bool pick = m[i] > thr;
    if (m[i] == thr) pick = taken++ < take;
    if (pick) out[pos++] = ch0 + i;
  }
}

template <int PER>
sf_status launch_select_t(const uint16_t* x, int batch, int k, int kch, int32_t* sel, cudaStream_t s, bool pdl) {
  const int jobs = batch * (k / (32 * PER));
  if (pdl) {
    SF_CUDA(launch_pdl(select_chunks_kernel<PER>, dim3(jobs), dim3(32), 0, s, x, k, kch, jobs, sel));
  } else {
    select_chunks_kernel<PER><<<jobs, 32, 0, s>>>(x, k, kch, jobs, sel);
    SF_LAUNCHED();
  }
  return SF_OK;
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
                        cudaStream_t s, bool pdl) {
  switch (chunk) {
    case 256: return launch_select_t<8>(x, batch, k, kch, sel, s, pdl);
    case 512: return launch_select_t<16>(x, batch, k, kch, sel, s, pdl);
    case 1024: return launch_select_t<32>(x, batch, k, kch, sel, s, pdl);
    default: return launch_select_t<64>(x, batch, k, kch, sel, s, pdl);
  }
}

}  // namespace sf

extern "C" sf_status sf_select_channels(const uint16_t* x, int batch, int k, int chunk, int kch,
                                        int32_t* sel, sf_stream_t stream) {
  sf_status st = sf::check_select_args(x, batch, k, chunk, kch);
  if (st != SF_OK) return st;
  SF_REQUIRE(sel && sf::aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  // a plain launch: on a staging stream the next kernel needs the whole result
  return sf::launch_select(x, batch, k, chunk, kch, sel, sf::as_stream(stream), false);
}
