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

namespace sf {
namespace {

struct Grid16 {
  uint16_t s16, m16;
  double S, M;
};

__device__ __forceinline__ Grid16 group_grid(double lo, double hi, int b) {
  Grid16 g;
  double step = __ddiv_rn(__dsub_rn(hi, lo), (double)((1 << b) - 1));
  g.s16 = __half_as_ushort(__double2half(step));  // one rounding, nearest-even
  g.m16 = __half_as_ushort(__double2half(lo));
  g.S = h2d(g.s16);
  g.M = h2d(g.m16);
  return g;
}

// (b+r)-bit nested code Q of one value: floor((u + 1/2) * 2^r), clamped.
__device__ __forceinline__ int nested_code(double w, const Grid16& g, int r, int qmax) {
  if (g.S == 0.0) return 0;
  double u = __ddiv_rn(__dsub_rn(w, g.M), g.S);
  double t = __dadd_rn(u, 0.5);
  double f = floor(__dmul_rn(t, (double)(1 << r)));
  f = fmin(fmax(f, 0.0), (double)qmax);
  return (int)f;
}

// Bit position of channel c (0..31) in the high-bit word of a 3-bit base block.
__device__ __forceinline__ int hi_plane_bit(int c) {
  return c < 16 ? 8 * (c >> 2) + (c & 3) : 8 * ((c - 16) >> 2) + 4 + ((c - 16) & 3);
}

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
  const long c0 = (long)n * K + (long)j * G;  // first element of the group
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
    long e0 = c0 + blk * 32;  // element index of the block's first code
    if (b == 4) {
      uint32_t* dst = base + e0 / 8;
      for (int i = 0; i < 4; i++) dst[i] = lw[i];
    } else {
      uint32_t* dst = base + e0 / 16;
      dst[0] = lw[0];
      dst[1] = lw[1];
      if (b == 3) hiplane[e0 / 32] = hw;
    }
  }
}

__global__ void unpack_weights_kernel(const uint32_t* __restrict__ base,
                                      const uint32_t* __restrict__ R, int N, int K, int b, int r,
                                      uint8_t* __restrict__ qb, uint8_t* __restrict__ rho) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;  // one element
  if (idx >= (long)N * K) return;
  long n = idx / K, c = idx % K;
  int q;
  if (b == 4) {
    q = (base[idx / 8] >> (4 * (idx & 7))) & 15;
  } else {
    q = (base[idx / 16] >> (2 * (idx & 15))) & 3;
    if (b == 3) {
      const uint32_t* hp = base + (size_t)N * K / 16;
      q |= ((hp[idx / 32] >> hi_plane_bit((int)(c & 31))) & 1) << 2;
    }
  }
  qb[idx] = (uint8_t)q;
  if (rho && R) {
    long rbit = (c * N + n) * r;
    rho[idx] = (uint8_t)((R[rbit >> 5] >> (rbit & 31)) & ((1u << r) - 1));
  }
}

// One thread per (batch, head, token, group of 32 elements).  A group's codes
// fill whole 32-bit words in both streams, so no two threads share a word.
__global__ void pack_kv_kernel(const uint16_t* __restrict__ x, int BH, int nt, int t_max, int t0,
                               int D, int b, int r, uint32_t* __restrict__ codes,
                               uint32_t* __restrict__ refine, uint16_t* __restrict__ sz) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  int gpt = D / 32;
  if (idx >= (long)BH * nt * gpt) return;
  int j = (int)(idx % gpt);
  long tok = idx / gpt;
  int t = (int)(tok % nt);
  long bh = tok / nt;
  const uint16_t* src = x + (bh * nt + t) * D + j * 32;
  double lo = h2d(src[0]), hi = lo;
  for (int c = 1; c < 32; c++) {
    double v = h2d(src[c]);
    if (v < lo) lo = v;
    if (v > hi) hi = v;
  }
  Grid16 g = group_grid(lo, hi, b);
  long slot = bh * t_max + t0 + t;  // cache token index
  sz[(slot * gpt + j) * 2 + 0] = g.s16;
  sz[(slot * gpt + j) * 2 + 1] = g.m16;
  const int qmax = (1 << (b + r)) - 1;
  uint32_t cw[4] = {0, 0, 0, 0}, rw[2] = {0, 0};
  for (int c = 0; c < 32; c++) {
    int Q = nested_code(h2d(src[c]), g, r, qmax);
    int q = Q >> r, rho = Q & ((1 << r) - 1);
    int cb = c * b, rb = c * r;
    cw[cb >> 5] |= (uint32_t)q << (cb & 31);
    rw[rb >> 5] |= (uint32_t)rho << (rb & 31);
  }
  uint32_t* cdst = codes + (slot * D + j * 32) * b / 32;
  for (int i = 0; i < b; i++) cdst[i] = cw[i];
  uint32_t* rdst = refine + (slot * D + j * 32) * r / 32;
  for (int i = 0; i < r; i++) rdst[i] = rw[i];
}

__global__ void unpack_kv_kernel(const uint32_t* __restrict__ codes,
                                 const uint32_t* __restrict__ refine, int BH, int t, int t_max,
                                 int D, int b, int r, uint8_t* __restrict__ qb,
                                 uint8_t* __restrict__ rho) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)BH * t * D) return;
  int d = (int)(idx % D);
  long tok = idx / D;
  long slot = (tok / t) * t_max + tok % t;
  long e = slot * D + d;
  qb[idx] = (uint8_t)((codes[e * b / 32] >> ((e * b) & 31)) & ((1u << b) - 1));
  if (rho) rho[idx] = (uint8_t)((refine[e * r / 32] >> ((e * r) & 31)) & ((1u << r) - 1));
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
  SF_UNSUPPORTED(kv->b == 2 || kv->b == 4, "KV base bits %d not in {2,4}", kv->b);
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

sf_status sf_kv_pack_tokens(const sf_kv* kv, const uint16_t* k, const uint16_t* v, int t0,
                            int nt, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  SF_REQUIRE(nt >= 0 && t0 >= 0 && t0 + nt <= kv->t_max, "tokens [%d, %d) outside t_max=%d", t0,
             t0 + nt, kv->t_max);
  if (nt == 0) return SF_OK;
  int BH = kv->batch * kv->h_kv;
  long total = (long)BH * nt * (kv->d / 32);
  int threads = 128;
  unsigned blocks = (unsigned)((total + threads - 1) / threads);
  cudaStream_t s = as_stream(stream);
  if (k) {
    pack_kv_kernel<<<blocks, threads, 0, s>>>(k, BH, nt, kv->t_max, t0, kv->d, kv->b, kv->r,
                                              (uint32_t*)kv->kb, (uint32_t*)kv->kr, kv->ksz);
    SF_LAUNCHED();
  }
  if (v) {
    pack_kv_kernel<<<blocks, threads, 0, s>>>(v, BH, nt, kv->t_max, t0, kv->d, kv->b, kv->r,
                                              (uint32_t*)kv->vb, (uint32_t*)kv->vr, kv->vsz);
    SF_LAUNCHED();
  }
  return SF_OK;
}

sf_status sf_kv_unpack_codes(const sf_kv* kv, int which, int t, uint8_t* qb, uint8_t* rho,
                             sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  SF_REQUIRE(which == 0 || which == 1, "which must be 0 (keys) or 1 (values)");
  SF_REQUIRE(t > 0 && t <= kv->t_max, "t=%d outside (0, t_max]", t);
  SF_REQUIRE(qb != nullptr, "qb must be non-null");
  int BH = kv->batch * kv->h_kv;
  long total = (long)BH * t * kv->d;
  int threads = 256;
  unpack_kv_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, as_stream(stream)>>>(
      (const uint32_t*)(which ? kv->vb : kv->kb), (const uint32_t*)(which ? kv->vr : kv->kr), BH, t,
      kv->t_max, kv->d, kv->b, kv->r, qb, rho);
  SF_LAUNCHED();
  return SF_OK;
}

}  // extern "C"
