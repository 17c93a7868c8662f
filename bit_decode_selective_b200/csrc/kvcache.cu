// kvcache.cu -- nested quantisation of KV tokens into the pair-slot cache
// layout, and the inverse export used for checking.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// nested-quantization paragraph: the same nesting as for weights is applied
// to the KV cache, per token in groups of 32 head-dim elements.
//
// One warp per (batch, head, token).  A key token's words belong to that
// token alone; in a value tile each token owns whole 16-bit halves of the
// words it touches, so tokens packed by different warps never share a store.
#include "common.cuh"
#include "kvlayout.cuh"
#include "quant.cuh"

namespace sf {
namespace {

constexpr int kPackWarps = 4;  // tokens per CTA of the pack kernel

// Min and max of the 32 elements of a group held by 8 lanes (4 each), with
// the first occurrence winning among equal values (so -0 and +0 keep the
// order-dependent choice of a sequential scan).
__device__ __forceinline__ void group_minmax(const double (&v)[4], int d0, double& lo, double& hi) {
  lo = v[0], hi = v[0];
  int ilo = d0, ihi = d0;
#pragma unroll
  for (int i = 1; i < 4; i++) {
    if (v[i] < lo) lo = v[i], ilo = d0 + i;
    if (v[i] > hi) hi = v[i], ihi = d0 + i;
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const double olo = __shfl_xor_sync(0xffffffffu, lo, o), ohi = __shfl_xor_sync(0xffffffffu, hi, o);
    const int oilo = __shfl_xor_sync(0xffffffffu, ilo, o), oihi = __shfl_xor_sync(0xffffffffu, ihi, o);
    if (olo < lo || (olo == lo && oilo < ilo)) lo = olo, ilo = oilo;
    if (ohi > hi || (ohi == hi && oihi < ihi)) hi = ohi, ihi = oihi;
  }
}

// One warp per (batch, head, token); lane l quantises head-dim elements
// 4l .. 4l+3 (group l / 8).  The token's code words (keys) or 16-bit word
// halves (values) are assembled in shared memory and stored by the first
// lanes; a token owns all of them, so tokens never share a store.
// Keys and values of the same tokens in one launch: blockIdx.y picks the kind.
// With qkv set, the one token comes straight from a qkv projection row: its
// key is turned by the rotary embedding and rounded to fp16 first, its value
// rounded to fp16, and a third kind turns the queries into q_out.
struct PackArgs {
  const uint16_t* x[2];  // [BH][nt][128] fp16 keys, values (either may be null)
  uint32_t* codes[2];
  uint32_t* refine[2];
  uint16_t* sz[2];
  int BH, nt, t_max, t0, first_kind;
  const float* qkv;      // nullable: [batch][(h_q + 2 h_kv) 128] fp32 (nt = 1)
  uint16_t* q_out;       // with qkv: [batch][h_q][128] fp16
  int h_q, h_kv, pos;
  double theta;
};

// The lane's 4 consecutive elements (4 lane .. 4 lane + 3) of a 128-element
// head row, turned by the rotary embedding: element e < 64 pairs with e + 64,
// held by lane ^ 16; cs[i] = (cos, sin) of pair i (rope_cos_sin).
__device__ __forceinline__ void rope_lane4(float (&x)[4], int lane, const float2* cs) {
  float xp[4];
#pragma unroll
  for (int i = 0; i < 4; i++) xp[i] = __shfl_xor_sync(0xffffffffu, x[i], 16);
  const bool first = lane < 16;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int e = 4 * lane + i, k = first ? e : e - kHeadDim / 2;
    const float2 t = cs[k];
    x[i] = first ? rope_first(x[i], xp[i], t.x, t.y) : rope_second(xp[i], x[i], t.x, t.y);
  }
}

__device__ __forceinline__ float f16_round(float x) { return __half2float(__float2half_rn(x)); }

template <int B, int R>
__global__ void __launch_bounds__(kPackWarps * 32) pack_kv_kernel(PackArgs pa) {
  // keys: 4B code words + 4R refinement words; values: 8B + 8R halves
  __shared__ uint32_t acc[kPackWarps][8 * (B + R)];
  pdl_trigger();
  pdl_wait();
  const int kind = pa.first_kind + blockIdx.y;  // 0 keys, 1 values, 2 queries (with qkv)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the rotation of every pair, once per CTA (the same for all heads)
  __shared__ float2 rope_cs[kHeadDim / 2];
  if (pa.qkv && kind != 1) {
    for (int i = threadIdx.x; i < kHeadDim / 2; i += blockDim.x) {
      float c, sn;
      rope_cos_sin(pa.pos, pa.theta, i, kHeadDim, c, sn);
      rope_cs[i] = make_float2(c, sn);
    }
    __syncthreads();
  }
  if (kind == 2) {  // queries: the rotary embedding only
    const long idx = (long)blockIdx.x * kPackWarps + warp;
    if (idx >= (long)(pa.BH / pa.h_kv) * pa.h_q) return;  // whole warps only
    const long b = idx / pa.h_q, h = idx % pa.h_q;
    const float4 r4 = *reinterpret_cast<const float4*>(pa.qkv + (b * (pa.h_q + 2 * pa.h_kv) + h) * kHeadDim +
                                                       4 * lane);
    float y[4] = {r4.x, r4.y, r4.z, r4.w};
    rope_lane4(y, lane, rope_cs);
    const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(y[0])) |
                        ((uint32_t)__half_as_ushort(__float2half_rn(y[1])) << 16);
    const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(y[2])) |
                        ((uint32_t)__half_as_ushort(__float2half_rn(y[3])) << 16);
    *reinterpret_cast<uint2*>(pa.q_out + idx * kHeadDim + 4 * lane) = make_uint2(lo, hi);
    return;
  }
  const int is_value = kind;
  const uint16_t* __restrict__ x = pa.x[is_value];
  uint32_t* __restrict__ codes = pa.codes[is_value];
  uint32_t* __restrict__ refine = pa.refine[is_value];
  uint16_t* __restrict__ sz = pa.sz[is_value];
  const int BH = pa.BH, nt = pa.nt, t_max = pa.t_max, t0 = pa.t0;
  const long idx = (long)blockIdx.x * kPackWarps + warp;
  if (idx >= (long)BH * nt) return;  // whole warps only
  const int t = (int)(idx % nt);
  const long bh = idx / nt;
  const long slot = bh * t_max + t0 + t;
  uint32_t* a = acc[warp];
  for (int i = lane; i < 8 * (B + R); i += 32) a[i] = 0;
  const int d0 = 4 * lane;
  double v[4];
  if (pa.qkv) {  // the one token from its projection row: key turned, both rounded to fp16
    const long b = bh / pa.h_kv, g = bh % pa.h_kv;
    const float4 r4 = *reinterpret_cast<const float4*>(
        pa.qkv + (b * (pa.h_q + 2 * pa.h_kv) + pa.h_q + (long)is_value * pa.h_kv + g) * kHeadDim + d0);
    float y[4] = {r4.x, r4.y, r4.z, r4.w};
    if (!is_value) rope_lane4(y, lane, rope_cs);
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] = (double)f16_round(y[i]);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2*>(x + (bh * nt + t) * kHeadDim + d0);
    v[0] = h2d((uint16_t)(raw.x & 0xffff)), v[1] = h2d((uint16_t)(raw.x >> 16));
    v[2] = h2d((uint16_t)(raw.y & 0xffff)), v[3] = h2d((uint16_t)(raw.y >> 16));
  }
  double lo, hi;
  group_minmax(v, d0, lo, hi);
  const Grid16 g = group_grid(lo, hi, B);
  const int j = lane >> 3;
  if ((lane & 7) == 0) {
    sz[(slot * 4 + j) * 2 + 0] = g.s16;
    sz[(slot * 4 + j) * 2 + 1] = g.m16;
  }
  __syncwarp();
  const int qmax = (1 << (B + R)) - 1;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int d = d0 + i;
    const int Q = nested_code(v[i], g, R, qmax);
    const uint32_t q = (uint32_t)(Q >> R), rho = (uint32_t)(Q & ((1 << R) - 1));
    if (!is_value) {
      int word, bit;
      if constexpr (B == 3) {  // low two bits: words 0..7; high bit: words 8..11
        key_pos(d, 2, word, bit);
        atomicOr(&a[word], (q & 3u) << bit);
        key_pos(d, 1, word, bit);
        atomicOr(&a[8 + word], (q >> 2) << bit);
      } else {
        key_pos(d, B, word, bit);
        atomicOr(&a[word], q << bit);
      }
      key_pos(d, R, word, bit);
      atomicOr(&a[4 * B + word], rho << bit);
    } else {
      // half (gg, k) of the token's value words, slot `sl` of 16/w codes; with
      // 3-bit codes halves (gg, 0..1) of the low-bit plane and (gg, 2) of the
      // high-bit plane
      const int m = d >> 4, within = d & 15, e = within >> 3, gg = within & 7;
      const int pp = 2 * m + e;
      if constexpr (B == 3) {
        atomicOr(&a[gg * 3 + pp / 8], (q & 3u) << (2 * (pp % 8)));
        atomicOr(&a[gg * 3 + 2], (q >> 2) << pp);
      } else {
        atomicOr(&a[gg * B + pp / (16 / B)], q << (B * (pp % (16 / B))));
      }
      atomicOr(&a[8 * B + gg * R + pp / (16 / R)], rho << (R * (pp % (16 / R))));
    }
  }
  __syncwarp();
  if (!is_value) {
    if (lane < 4 * B) codes[slot * 4 * B + lane] = a[lane];
    else if (lane < 4 * (B + R)) refine[slot * 4 * R + lane - 4 * B] = a[lane];
  } else {
    const long tile = bh * (t_max / 16) + (t0 + t) / 16;
    const int tt = (t0 + t) & 15;
    const int h = tt >> 3, c = (tt & 7) >> 1, second = tt & 1;
    for (int i = lane; i < 8 * (B + R); i += 32) {
      const bool base = i < 8 * B;
      const int W = base ? B : R, ii = base ? i : i - 8 * B;
      const int gg = ii / W, k = ii % W;
      int word = (4 * gg + c) * 2 * W + h * W + k;
      if (B == 3 && base) word = k < 2 ? (4 * gg + c) * 4 + h * 2 + k : 128 + (4 * gg + c) * 2 + h;
      uint16_t* halves = reinterpret_cast<uint16_t*>((base ? codes + tile * 64 * B : refine + tile * 64 * R));
      halves[word * 2 + second] = (uint16_t)a[i];
    }
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
  if (!is_value) {
    const long slot = bh * t_max + tk;
    qb[idx] = (uint8_t)key_code(codes + slot * 4 * b, d, b);
    if (rho) rho[idx] = (uint8_t)key_code(refine + slot * 4 * r, d, r);
  } else {
    const long tile = bh * (t_max / 16) + tk / 16;
    qb[idx] = (uint8_t)value_code(codes + tile * 64 * b, tk & 15, d, b);
    if (rho) rho[idx] = (uint8_t)value_code(refine + tile * 64 * r, tk & 15, d, r);
  }
}

template <int B, int R>
sf_status launch_pack(const PackArgs& pa, int kinds, cudaStream_t s) {
  long total = (long)pa.BH * pa.nt;
  if (pa.qkv && (long)(pa.BH / pa.h_kv) * pa.h_q > total) total = (long)(pa.BH / pa.h_kv) * pa.h_q;
  SF_CUDA(launch_pdl(pack_kv_kernel<B, R>, dim3((unsigned)((total + kPackWarps - 1) / kPackWarps), kinds),
                     dim3(kPackWarps * 32), 0, s, pa));
  return SF_OK;
}

sf_status launch_pack_any(const sf_kv* kv, const PackArgs& pa, int kinds, cudaStream_t s) {
  if (kv->b == 2 && kv->r == 2) return launch_pack<2, 2>(pa, kinds, s);
  if (kv->b == 2 && kv->r == 1) return launch_pack<2, 1>(pa, kinds, s);
  if (kv->b == 3 && kv->r == 2) return launch_pack<3, 2>(pa, kinds, s);
  if (kv->b == 3 && kv->r == 1) return launch_pack<3, 1>(pa, kinds, s);
  if (kv->b == 4 && kv->r == 2) return launch_pack<4, 2>(pa, kinds, s);
  return launch_pack<4, 1>(pa, kinds, s);
}

PackArgs pack_args(const sf_kv* kv, int t0, int nt) {
  PackArgs pa = {};
  pa.codes[0] = (uint32_t*)kv->kb, pa.codes[1] = (uint32_t*)kv->vb;
  pa.refine[0] = (uint32_t*)kv->kr, pa.refine[1] = (uint32_t*)kv->vr;
  pa.sz[0] = kv->ksz, pa.sz[1] = kv->vsz;
  pa.BH = kv->batch * kv->h_kv, pa.nt = nt, pa.t_max = kv->t_max, pa.t0 = t0;
  pa.h_kv = kv->h_kv;
  return pa;
}

sf_status pack_both(const sf_kv* kv, const uint16_t* k, const uint16_t* v, int t0, int nt, cudaStream_t s) {
  PackArgs pa = pack_args(kv, t0, nt);
  pa.x[0] = k, pa.x[1] = v;
  pa.first_kind = k ? 0 : 1;
  const int kinds = (k ? 1 : 0) + (v ? 1 : 0);
  if (kinds == 0) return SF_OK;
  return launch_pack_any(kv, pa, kinds, s);
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
  return pack_both(kv, k, v, t0, nt, as_stream(stream));
}

extern "C" sf_status sf_kv_append_rope(const sf_kv* kv, const float* qkv, int h_q, int pos, float theta,
                                       int t, uint16_t* q, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  SF_REQUIRE(t >= 0 && t < kv->t_max, "t=%d outside [0, t_max=%d)", t, kv->t_max);
  SF_REQUIRE(pos >= 0, "pos=%d < 0", pos);
  SF_REQUIRE(h_q > 0 && h_q % kv->h_kv == 0, "h_q=%d must be a positive multiple of h_kv=%d", h_q, kv->h_kv);
  SF_REQUIRE(qkv && aligned16(qkv), "qkv must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(q && aligned16(q), "q must be a non-null 16-byte aligned device pointer");
  PackArgs pa = pack_args(kv, t, 1);
  pa.qkv = qkv, pa.q_out = q, pa.h_q = h_q, pa.pos = pos, pa.theta = (double)theta;
  pa.first_kind = 0;
  return launch_pack_any(kv, pa, 3, as_stream(stream));
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
