// kvcache.cu -- nested quantisation of KV tokens into the pair-slot cache
// layout, and the inverse export used for checking.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// nested-quantization paragraph: the same nesting as for weights is applied
// to the KV cache, per token in groups of 32 head-dim elements.
//
// One thread per (batch, head, token).  A key token's words belong to that
// token alone; in a value tile each token owns whole 16-bit halves of the
// words it touches, so tokens packed by different threads never share a store.
#include "common.cuh"
#include "kvlayout.cuh"
#include "quant.cuh"

namespace sf {
namespace {

// Value halves of one token: chunk lane l = 4g + c (c from the token) owns, per
// w-bit stream, w halves: word l*2w + h*w + k, half `second` (h, c, second from
// the token; k = (2m+e) / (16/w)).
template <int W>
struct ValueHalves {
  uint16_t v[8][W];
  __device__ void clear() {
    for (int g = 0; g < 8; g++)
      for (int k = 0; k < W; k++) v[g][k] = 0;
  }
  __device__ void put(int d, uint32_t code) {
    int m = d >> 4, within = d & 15, e = within >> 3, g = within & 7;
    constexpr int per = 16 / W;
    int k = (2 * m + e) / per, slot = (2 * m + e) % per;
    v[g][k] |= (uint16_t)(code << (W * slot));
  }
  __device__ void store(uint16_t* tile_halves, int tt) {
    int h = tt >> 3, c = (tt & 7) >> 1, second = tt & 1;
    for (int g = 0; g < 8; g++)
      for (int k = 0; k < W; k++) {
        int word = (4 * g + c) * 2 * W + h * W + k;
        tile_halves[word * 2 + second] = v[g][k];
      }
  }
};

template <int B, int R>
__global__ void pack_kv_kernel(const uint16_t* __restrict__ x, int BH, int nt, int t_max, int t0,
                               int is_value, uint32_t* __restrict__ codes,
                               uint32_t* __restrict__ refine, uint16_t* __restrict__ sz) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)BH * nt) return;
  const int t = (int)(idx % nt);
  const long bh = idx / nt;
  const uint16_t* src = x + (bh * nt + t) * kHeadDim;
  const long slot = bh * t_max + t0 + t;
  const int qmax = (1 << (B + R)) - 1;
  uint32_t kw[4 * B] = {}, kr[4 * R] = {};
  ValueHalves<B> vb;
  ValueHalves<R> vr;
  vb.clear();
  vr.clear();
  for (int j = 0; j < kHeadDim / 32; j++) {
    double lo = h2d(src[j * 32]), hi = lo;
    for (int c = 1; c < 32; c++) {
      double v = h2d(src[j * 32 + c]);
      if (v < lo) lo = v;
      if (v > hi) hi = v;
    }
    Grid16 g = group_grid(lo, hi, B);
    sz[(slot * 4 + j) * 2 + 0] = g.s16;
    sz[(slot * 4 + j) * 2 + 1] = g.m16;
    for (int c = 0; c < 32; c++) {
      int d = j * 32 + c;
      int Q = nested_code(h2d(src[d]), g, R, qmax);
      uint32_t q = (uint32_t)(Q >> R), rho = (uint32_t)(Q & ((1 << R) - 1));
      if (!is_value) {
        int word, bit;
        key_pos(d, B, word, bit);
        kw[word] |= q << bit;
        key_pos(d, R, word, bit);
        kr[word] |= rho << bit;
      } else {
        vb.put(d, q);
        vr.put(d, rho);
      }
    }
  }
  if (!is_value) {
    uint32_t* kd = codes + slot * 4 * B;
#pragma unroll
    for (int i = 0; i < 4 * B; i++) kd[i] = kw[i];
    uint32_t* rd = refine + slot * 4 * R;
#pragma unroll
    for (int i = 0; i < 4 * R; i++) rd[i] = kr[i];
  } else {
    const long tile = bh * (t_max / 16) + (t0 + t) / 16;
    const int tt = (t0 + t) & 15;
    vb.store(reinterpret_cast<uint16_t*>(codes + tile * 64 * B), tt);
    vr.store(reinterpret_cast<uint16_t*>(refine + tile * 64 * R), tt);
  }
}

__global__ void unpack_kv_kernel(const uint32_t* __restrict__ codes,
                                 const uint32_t* __restrict__ refine, int BH, int t, int t_max,
                                 int b, int r, int is_value, uint8_t* __restrict__ qb,
                                 uint8_t* __restrict__ rho) {
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)BH * t * kHeadDim) return;
  const int d = (int)(idx % kHeadDim);
  const long tok = idx / kHeadDim;
  const long bh = tok / t;
  const int tk = (int)(tok % t);
  int word, bit;
  if (!is_value) {
    const long slot = bh * t_max + tk;
    key_pos(d, b, word, bit);
    qb[idx] = (uint8_t)((codes[slot * 4 * b + word] >> bit) & ((1u << b) - 1));
    if (rho) {
      key_pos(d, r, word, bit);
      rho[idx] = (uint8_t)((refine[slot * 4 * r + word] >> bit) & ((1u << r) - 1));
    }
  } else {
    const long tile = bh * (t_max / 16) + tk / 16;
    value_pos(tk & 15, d, b, word, bit);
    qb[idx] = (uint8_t)((codes[tile * 64 * b + word] >> bit) & ((1u << b) - 1));
    if (rho) {
      value_pos(tk & 15, d, r, word, bit);
      rho[idx] = (uint8_t)((refine[tile * 64 * r + word] >> bit) & ((1u << r) - 1));
    }
  }
}

template <int B, int R>
sf_status launch_pack(const uint16_t* x, int BH, int nt, int t_max, int t0, int is_value,
                      void* codes, void* refine, uint16_t* sz, cudaStream_t s) {
  long total = (long)BH * nt;
  int threads = 128;
  pack_kv_kernel<B, R><<<(unsigned)((total + threads - 1) / threads), threads, 0, s>>>(
      x, BH, nt, t_max, t0, is_value, (uint32_t*)codes, (uint32_t*)refine, sz);
  SF_LAUNCHED();
  return SF_OK;
}

sf_status pack_one(const sf_kv* kv, const uint16_t* x, int t0, int nt, int is_value,
                   cudaStream_t s) {
  int BH = kv->batch * kv->h_kv;
  void* codes = is_value ? kv->vb : kv->kb;
  void* refine = is_value ? kv->vr : kv->kr;
  uint16_t* sz = is_value ? kv->vsz : kv->ksz;
  if (kv->b == 2 && kv->r == 2) return launch_pack<2, 2>(x, BH, nt, kv->t_max, t0, is_value, codes, refine, sz, s);
  if (kv->b == 2 && kv->r == 1) return launch_pack<2, 1>(x, BH, nt, kv->t_max, t0, is_value, codes, refine, sz, s);
  if (kv->b == 4 && kv->r == 2) return launch_pack<4, 2>(x, BH, nt, kv->t_max, t0, is_value, codes, refine, sz, s);
  return launch_pack<4, 1>(x, BH, nt, kv->t_max, t0, is_value, codes, refine, sz, s);
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" sf_status sf_kv_pack_tokens(const sf_kv* kv, const uint16_t* k, const uint16_t* v,
                                       int t0, int nt, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  SF_REQUIRE(nt >= 0 && t0 >= 0 && t0 + nt <= kv->t_max, "tokens [%d, %d) outside t_max=%d", t0,
             t0 + nt, kv->t_max);
  SF_REQUIRE(!k || aligned16(k), "k must be 16-byte aligned");
  SF_REQUIRE(!v || aligned16(v), "v must be 16-byte aligned");
  if (nt == 0) return SF_OK;
  cudaStream_t s = as_stream(stream);
  if (k) {
    st = pack_one(kv, k, t0, nt, 0, s);
    if (st != SF_OK) return st;
  }
  if (v) {
    st = pack_one(kv, v, t0, nt, 1, s);
    if (st != SF_OK) return st;
  }
  return SF_OK;
}

extern "C" sf_status sf_kv_unpack_codes(const sf_kv* kv, int which, int t, uint8_t* qb,
                                        uint8_t* rho, sf_stream_t stream) {
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
      kv->t_max, kv->b, kv->r, which, qb, rho);
  SF_LAUNCHED();
  return SF_OK;
}
