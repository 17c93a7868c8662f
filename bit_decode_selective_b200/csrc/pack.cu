// pack.cu -- nested quantisation of weights and KV tokens into the packed
// formats of sf.h, and the inverse export used for checking.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// nested-quantization paragraph: the fetched refinement bits subdivide the bin
// the resident base code names.  Each group gets an fp16 step s and offset m;
// the base code is the b-bit round-to-nearest code and the r refinement bits
// index the 2^r equal parts of its bin.  The decisions are taken in fp64 with
// explicitly rounded operations (no contraction) so that they are bit-exact
// with the definition in sf.h.
#include "common.cuh"
#include "quant.cuh"
#include "wqlayout.cuh"

namespace sf {

namespace {

// One thread per (row, group).  Refinement rows are channel-major, so several
// threads share a 32-bit word of R: they OR their bits in atomically into a
// zeroed buffer.
__global__ void pack_weights_kernel(const float* __restrict__ w, int N, int K, int b, int r,
                                    int G, uint32_t* __restrict__ base, uint32_t* __restrict__ R,
                                    uint16_t* __restrict__ sz) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  int gpr = K / G;
  if (idx >= (long)N * gpr) return;
  int n = (int)(idx / gpr), j = (int)(idx % gpr);
  const float* wr = w + (size_t)n * K + (size_t)j * G;
  double lo = (double)wr[0], hi = lo;
  for (int c = 1; c < G; c++) {
    double v = (double)wr[c];  // same comparison order as the definition (keeps
    if (v < lo) lo = v;        // the first of equal extremes, e.g. +0 before -0)
    if (v > hi) hi = v;
  }
  Grid16 g = group_grid(lo, hi, b);
  sz[idx * 2 + 0] = g.s16;
  sz[idx * 2 + 1] = g.m16;
  const int qmax = (1 << (b + r)) - 1;
  uint32_t* hiplane = base + (size_t)N * K / 16;  // b == 3: plane H after plane L
  for (int blk = 0; blk < G / 32; blk++) {
    uint32_t lw[4] = {0, 0, 0, 0};  // up to 128 bits of codes for 32 channels
    uint32_t hw = 0;
    for (int c = 0; c < 32; c++) {
      int ch = j * G + blk * 32 + c;
      int Q = nested_code((double)wr[blk * 32 + c], g, r, qmax);
      int q = Q >> r, rho = Q & ((1 << r) - 1);
      if (b == 4) {
        lw[c >> 3] |= (uint32_t)q << (4 * (c & 7));
      } else {
        lw[c >> 4] |= (uint32_t)(q & 3) << (2 * (c & 15));
        if (b == 3) hw |= (uint32_t)(q >> 2) << hi_plane_bit(c);
      }
      long rbit = ((long)ch * N + n) * r;
      atomicOr(&R[rbit >> 5], (uint32_t)rho << (rbit & 31));
    }
    const int cb = j * G + blk * 32;  // the block's first channel
    if (b == 4) {
      uint32_t* row = base + (size_t)n * (K / 8);
      for (int i = 0; i < 4; i++) row[wq_word(n, cb / 8 + i)] = lw[i];
    } else {
      uint32_t* row = base + (size_t)n * (K / 16);
      row[wq_word(n, cb / 16)] = lw[0];
      row[wq_word(n, cb / 16 + 1)] = lw[1];
      if (b == 3) hiplane[(size_t)n * (K / 32) + wq_word(n, cb / 32)] = hw;
    }
  }
}

__global__ void unpack_weights_kernel(const uint32_t* __restrict__ base,
                                      const uint32_t* __restrict__ R, int N, int K, int b, int r,
                                      uint8_t* __restrict__ qb, uint8_t* __restrict__ rho) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;  // one element
  if (idx >= (long)N * K) return;
  long n = idx / K, c = idx % K;
  qb[idx] = (uint8_t)packed_base_code(base, N, K, b, n, c);
  if (rho && R) {
    long rbit = (c * N + n) * r;
    rho[idx] = (uint8_t)((R[rbit >> 5] >> (rbit & 31)) & ((1u << r) - 1));
  }
}

sf_status check_wq(const sf_wq* w, bool need_refine) {
  SF_REQUIRE(w != nullptr, "null sf_wq");
  SF_REQUIRE(w->n > 0 && w->k > 0, "bad shape n=%d k=%d", w->n, w->k);
  SF_UNSUPPORTED(w->b >= 2 && w->b <= 4, "base bits b=%d not in {2,3,4}", w->b);
  SF_UNSUPPORTED(w->r == 1 || w->r == 2, "refinement bits r=%d not in {1,2}", w->r);
  SF_UNSUPPORTED(w->group == 32 || w->group == 64 || w->group == 128 || w->group == 256,
                 "group %d not in {32,64,128,256}", w->group);
  SF_UNSUPPORTED(w->k % 1024 == 0 && w->k % w->group == 0, "k=%d must be a multiple of 1024", w->k);
  SF_UNSUPPORTED(w->n % 128 == 0, "n=%d must be a multiple of 128", w->n);
  SF_REQUIRE(w->base && aligned16(w->base), "base must be a non-null 16-byte aligned pointer");
  SF_REQUIRE(w->sz && aligned16(w->sz), "sz must be a non-null 16-byte aligned pointer");
  if (need_refine)
    SF_REQUIRE(w->refine && aligned16(w->refine), "refine must be non-null and 16-byte aligned");
  else
    SF_REQUIRE(!w->refine || aligned16(w->refine), "refine must be 16-byte aligned");
  return SF_OK;
}

}  // namespace

sf_status check_kv(const sf_kv* kv) {
  SF_REQUIRE(kv != nullptr, "null sf_kv");
  SF_REQUIRE(kv->batch > 0 && kv->h_kv > 0 && kv->t_max > 0, "bad KV shape");
  SF_UNSUPPORTED(kv->d == 128 && kv->group == 32, "KV needs d=128, group=32 (got %d, %d)", kv->d,
                 kv->group);
  SF_UNSUPPORTED(kv->b >= 2 && kv->b <= 4, "KV base bits %d not in {2,3,4}", kv->b);
  SF_UNSUPPORTED(kv->r == 1 || kv->r == 2, "KV refinement bits %d not in {1,2}", kv->r);
  SF_UNSUPPORTED(kv->t_max % 16 == 0, "t_max=%d must be a multiple of 16", kv->t_max);
  const void* ptrs[6] = {kv->kb, kv->kr, kv->vb, kv->vr, kv->ksz, kv->vsz};
  for (const void* p : ptrs) SF_REQUIRE(p && aligned16(p), "KV buffers must be non-null, 16-byte aligned");
  return SF_OK;
}

sf_status check_wq_public(const sf_wq* w, bool need_refine) { return check_wq(w, need_refine); }

}  // namespace sf

using namespace sf;

extern "C" {

sf_status sf_pack_nested(const float* w, const sf_wq* out, sf_stream_t stream) {
  sf_status st = check_wq(out, true);
  if (st != SF_OK) return st;
  SF_REQUIRE(w && aligned16(w), "w must be a non-null 16-byte aligned device pointer");
  cudaStream_t s = as_stream(stream);
  size_t rbytes = (size_t)out->k * out->n * out->r / 8;
  SF_CUDA(cudaMemsetAsync(out->refine, 0, rbytes, s));
  long total = (long)out->n * (out->k / out->group);
  int threads = 128;
  pack_weights_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, s>>>(
      w, out->n, out->k, out->b, out->r, out->group, (uint32_t*)out->base, (uint32_t*)out->refine,
      out->sz);
  SF_LAUNCHED();
  return SF_OK;
}

sf_status sf_unpack_codes(const sf_wq* w, uint8_t* qb, uint8_t* rho, sf_stream_t stream) {
  sf_status st = check_wq(w, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(qb != nullptr, "qb must be non-null");
  long total = (long)w->n * w->k;
  int threads = 256;
  unpack_weights_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0,
                          as_stream(stream)>>>((const uint32_t*)w->base,
                                               (const uint32_t*)w->refine, w->n, w->k, w->b, w->r,
                                               qb, w->refine ? rho : nullptr);
  SF_LAUNCHED();
  return SF_OK;
}

}  // extern "C"
