// kv.cu -- KV token scoring, per-KV-head top-k selection and refined split-K
// attention over a nested-quantised KV cache.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?":
//   which-tiles-count paragraph -- every cached token is scored by the
//     attention it receives, computed from the resident low-bit keys, and the
//     highest-scoring tokens are refined for each KV head (the keys and values
//     a group of query heads shares); unselected tokens still take part at
//     low precision;
//   nested-quantization paragraph -- refinement bits subdivide the base bin;
//   where-it-earns-its-keep paragraph -- KV refinement is a step that cannot
//     overlap the attention around it, since the selection depends on the
//     attention scores.
//
// Schedule (one pass over the resident cache, then work on the selected
// tokens only):
//   kv_base_kernel     per 16-token tile, logits of the group's query heads
//                      from the base keys and the base attention (online
//                      softmax, split-K partials) from the base values; the
//                      logits are stored for scoring.  Codes are turned into
//                      exact fp16 integers in registers and contracted on the
//                      tensor cores (mma.sync m16n8k16, fp32 accumulation);
//                      the per-token fp16 steps/offsets are applied in fp32.
//   kv_stats_kernel    softmax max/sum of every query head from the partials;
//   kv_local_kernel    per context span, score every token and keep the
//                      span's k_tok best (a token in the global top-k is in
//                      the top-k of its own span), in token order;
//   kv_final_kernel    per KV head, the k_tok best of the candidates;
//   kv_correct_kernel  for the selected tokens only: swap each token's base
//                      contribution for its refined one (refined logit, refined
//                      value), relative to the head's softmax max;
//   kv_merge_kernel    log-sum-exp merge of the partials plus the correction.
// The result equals softmax(q.k~) v~ with refined k~, v~ on the selected
// tokens, up to fp32 rounding.
#include <cfloat>
#include <mutex>

#include "common.cuh"
#include "kvlayout.cuh"
#include "radix.cuh"

namespace sf {
namespace {

constexpr int kD = kHeadDim;
constexpr int kRec = kD + 2;     // partial record: acc[kD], m, l
constexpr int kWarps = 4;        // warps per base-pass CTA (independent splits)
constexpr int kStages = 4;       // cp.async ring depth per warp
constexpr int kMaxCand = 16384;  // candidates per KV head in the final select
constexpr int kMaxSpan = 8192;   // tokens per local-select CTA
constexpr int kCorrTok = 16;     // selected tokens per correction CTA

// ---- small PTX helpers -------------------------------------------------------

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Pair slot `slot` (compile-time after unrolling) of a w-bit pair-slot word as
// an exact half2 of CENTRED codes c - (2^W - 1)/2 (for 2-bit codes
// -1.5, -0.5, 0.5, 1.5).  The code is masked in place, OR-ed into the
// mantissa of 1024.0 and rescaled with one fused multiply-add; the word is
// shifted first so that the code sits at a bit offset b2 in [2, 10 - W], which
// keeps the fma constant exactly representable.  w_l2 = w << 2, w_r = w >> 8
// (W = 2) or w >> 6 (W = 4).
template <int W>
__device__ __forceinline__ uint32_t pair_at(uint32_t w, uint32_t w_l2, uint32_t w_r, int slot) {
  const int bit = W * slot;
  const int rsh = W == 2 ? 8 : 6;
  const bool left = bit < 2;
  const bool right = !left && bit + W > 10;
  const int b2 = left ? bit + 2 : right ? bit - rsh : bit;
  const uint32_t src = left ? w_l2 : right ? w_r : w;
  const uint32_t mask = (((1u << W) - 1u) << b2) * 0x00010001u;
  uint32_t v = (src & mask) | 0x64006400u;  // 1024 + c * 2^b2 per half
  // fp16 bit patterns: 2^-b2, and -(2^(10-b2) + centre) whose mantissa is
  // centre * 2^b2 = (2^W - 1) * 2^(b2-1)
  const uint32_t sc = (uint32_t)((15 - b2) << 10) * 0x00010001u;
  const uint32_t off = (0x8000u | ((uint32_t)(25 - b2) << 10) | (((1u << W) - 1u) << (b2 - 1))) * 0x00010001u;
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&v), *reinterpret_cast<const __half2*>(&sc),
                      *reinterpret_cast<const __half2*>(&off));
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int W>
struct Words {
  uint32_t w, l2, r;
  __device__ __forceinline__ void set(uint32_t x) {
    w = x;
    l2 = x << 2;
    r = x >> (W == 2 ? 8 : 6);
  }
};

template <int W, int N>
__device__ __forceinline__ uint32_t pair_of(const Words<W> (&ws)[N], int p) {
  constexpr int per = 16 / W;
  const Words<W>& x = ws[p / per];
  return pair_at<W>(x.w, x.l2, x.r, p % per);
}

// ---------------------------------------------------------------------------
// base pass

struct BaseArgs {
  const uint8_t* kb;
  const uint8_t* vb;
  const uint16_t* ksz;
  const uint16_t* vsz;
  int h_kv, t_max, T;
  const uint16_t* q;
  int h_q, gq;
  float* logits;  // [batch][h_q][T]
  float* part;    // [batch][h_q][nrec][rec]  (rec = kRec with values, 2 without)
  int span, nsplit, nrec;
  float scale;
};

template <int B, bool PV>
struct Stage {
  static constexpr int kBytes = 256 * B;           // key codes of 16 tokens
  static constexpr int vBytes = PV ? 256 * B : 0;  // value tile
  static constexpr int szBytes = PV ? 512 : 256;   // key (+ value) step/offset (fp16)
  static constexpr int bytes = kBytes + vBytes + szBytes;
};

template <int B, bool PV>
struct WarpSmem {
  static constexpr int ring = kStages * Stage<B, PV>::bytes;
  static constexpr int zf = 16 * 4 * 2 * 4 * (PV ? 2 : 1);  // fp32 (s, m') of 16 tokens x 4 groups
  static constexpr int ps = 16 * 9 * 4;                      // transposed probabilities
  static constexpr int bytes = ring + zf + ps;
};

// GQP: query heads per KV head padded to 4 or 8.  B: base bits (2 or 4).
template <int GQP, int B, bool PV>
__global__ void __launch_bounds__(kWarps * 32, GQP == 4 ? 4 : 2) kv_base_kernel(BaseArgs a) {
  using St = Stage<B, PV>;
  using WS = WarpSmem<B, PV>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int g = blockIdx.y, bat = blockIdx.z;
  const int split = blockIdx.x * kWarps + warp;
  uint8_t* wsm = smem + warp * WS::bytes;
  float* Zs = reinterpret_cast<float*>(wsm + WS::ring);        // [PV+1][16][4][2]
  float* Ps = reinterpret_cast<float*>(wsm + WS::ring + WS::zf);  // [16][9]
  const float centre = 0.5f * (float)((1 << B) - 1);

  const int tw0 = split * a.span;
  const int tw1 = min(a.T, tw0 + a.span);
  const int ntile = (split < a.nsplit && tw1 > tw0) ? (tw1 - tw0 + 15) / 16 : 0;
  const long slot0 = ((long)bat * a.h_kv + g) * a.t_max;  // first token slot of this head
  const int gq = a.gq;
  const int h0 = 2 * tig, h1 = 2 * tig + 1;  // the lane's logit / output head columns

  // ---- query fragments (B operand of the key contraction): head gid
  const uint16_t* qg = a.q + ((long)bat * a.h_q + (long)g * gq) * kD;
  uint32_t qf[8][2];
  float qsum[4] = {0.f, 0.f, 0.f, 0.f};  // per group j: the lane's 8 dims of head gid
#pragma unroll
  for (int s = 0; s < 8; s++) {
    uint32_t lo = 0, hi = 0;
    if (gid < gq) {
      lo = *reinterpret_cast<const uint32_t*>(qg + gid * kD + 16 * s + 2 * tig);
      hi = *reinterpret_cast<const uint32_t*>(qg + gid * kD + 16 * s + 2 * tig + 8);
    }
    qf[s][0] = lo, qf[s][1] = hi;
    float2 f0 = __half22float2(*reinterpret_cast<__half2*>(&lo));
    float2 f1 = __half22float2(*reinterpret_cast<__half2*>(&hi));
    qsum[s >> 1] += (f0.x + f0.y) + (f1.x + f1.y);
  }
  float Q0[4], Q1[4];  // per-group sums of q for heads 2tig, 2tig+1
#pragma unroll
  for (int j = 0; j < 4; j++) {
    float v = qsum[j];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    Q0[j] = __shfl_sync(0xffffffffu, v, 8 * tig);
    Q1[j] = __shfl_sync(0xffffffffu, v, 8 * tig + 4);
  }

  // softmax state of heads 2tig, 2tig+1 (the lane's logit and output columns)
  float mrun0 = -INFINITY, mrun1 = -INFINITY, lsum0 = 0.f, lsum1 = 0.f;
  constexpr int NT = GQP == 4 ? 1 : 2;  // value-side n-tiles (hi/lo of 8 heads: two)
  float accv[NT][8][4];
  float mt[4] = {0.f, 0.f, 0.f, 0.f};  // sum_t p m'_t,j of the B-operand head
#pragma unroll
  for (int nt = 0; nt < NT; nt++)
#pragma unroll
    for (int m = 0; m < 8; m++)
#pragma unroll
      for (int i = 0; i < 4; i++) accv[nt][m][i] = 0.f;

  auto issue = [&](int it) {
    if (it < ntile) {
      uint8_t* st = wsm + (it % kStages) * St::bytes;
      const long slot = slot0 + tw0 + 16 * it;
#pragma unroll
      for (int c = 0; c < B / 2; c++) {
        const int ci = lane + 32 * c;
        cp_async16(st + 16 * ci, a.kb + slot * 16 * B + 16 * ci);
        if (PV) cp_async16(st + St::kBytes + 16 * ci, a.vb + (slot / 16) * 256 * B + 16 * ci);
      }
      if (lane < 16)
        cp_async16(st + St::kBytes + St::vBytes + 16 * lane,
                   reinterpret_cast<const uint8_t*>(a.ksz) + slot * 16 + 16 * lane);
      else if (PV)
        cp_async16(st + St::kBytes + St::vBytes + 16 * lane,
                   reinterpret_cast<const uint8_t*>(a.vsz) + slot * 16 + 16 * (lane - 16));
    }
    cp_async_commit();
  };

#pragma unroll
  for (int i = 0; i < kStages - 1; i++) issue(i);

  for (int it = 0; it < ntile; it++) {
    issue(it + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint8_t* st = wsm + (it % kStages) * St::bytes;
    const int t0 = tw0 + 16 * it;
    // (s, m') = (s, m + centre * s) in fp32 for the tile's tokens; tokens past
    // the end of the span get (0, 0) so they contribute nothing
    {
      const uint32_t* zh = reinterpret_cast<const uint32_t*>(st + St::kBytes + St::vBytes);
#pragma unroll
      for (int i = 0; i < (PV ? 4 : 2); i++) {
        const int e = lane + 32 * i;  // (which, token, group) = (e / 64, (e / 4) % 16, e % 4)
        uint32_t z = zh[e];
        float2 sm = __half22float2(*reinterpret_cast<__half2*>(&z));
        const bool valid = t0 + ((e >> 2) & 15) < tw1;
        reinterpret_cast<float2*>(Zs)[e] = valid ? make_float2(sm.x, fmaf(centre, sm.x, sm.y)) : make_float2(0.f, 0.f);
      }
    }
    __syncwarp();

    // ---- logits: tokens on M (gid, gid+8), heads on N, k-steps of 16 dims
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
      for (int i = 0; i < 4; i++) acc[j][i] = 0.f;
    {
      const uint32_t* kc = reinterpret_cast<const uint32_t*>(st);
      Words<B> w0[B], w8[B];
#pragma unroll
      for (int i = 0; i < B; i++) {
        w0[i].set(kc[gid * 4 * B + tig * B + i]);
        w8[i].set(kc[(gid + 8) * 4 * B + tig * B + i]);
      }
#pragma unroll
      for (int s = 0; s < 8; s++) {
        uint32_t a0 = pair_of<B>(w0, 2 * s), a1 = pair_of<B>(w8, 2 * s);
        uint32_t a2 = pair_of<B>(w0, 2 * s + 1), a3 = pair_of<B>(w8, 2 * s + 1);
        mma16816(acc[s >> 1], a0, a1, a2, a3, qf[s][0], qf[s][1]);
      }
    }
    float l[4];  // (tok gid, head 2tig), (gid, 2tig+1), (gid+8, 2tig), (gid+8, 2tig+1)
#pragma unroll
    for (int r = 0; r < 2; r++) {
      const int tok = gid + 8 * r;
      const float4* zk = reinterpret_cast<const float4*>(Zs + tok * 8);
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int jj = 0; jj < 2; jj++) {
        const float4 z = zk[jj];  // groups 2jj, 2jj+1: (s, m')
        x0 = fmaf(z.x, acc[2 * jj][2 * r], fmaf(z.y, Q0[2 * jj], x0));
        x1 = fmaf(z.x, acc[2 * jj][2 * r + 1], fmaf(z.y, Q1[2 * jj], x1));
        x0 = fmaf(z.z, acc[2 * jj + 1][2 * r], fmaf(z.w, Q0[2 * jj + 1], x0));
        x1 = fmaf(z.z, acc[2 * jj + 1][2 * r + 1], fmaf(z.w, Q1[2 * jj + 1], x1));
      }
      const bool valid = t0 + tok < tw1;
      l[2 * r + 0] = valid ? x0 * a.scale : -INFINITY;
      l[2 * r + 1] = valid ? x1 * a.scale : -INFINITY;
    }
    {
      float* lg = a.logits + ((long)bat * a.h_q + (long)g * gq) * a.T;
#pragma unroll
      for (int r = 0; r < 2; r++) {
        const int t = t0 + gid + 8 * r;
        if (t < tw1) {
          if (h0 < gq) lg[(long)h0 * a.T + t] = l[2 * r];
          if (h1 < gq) lg[(long)h1 * a.T + t] = l[2 * r + 1];
        }
      }
    }
    // ---- online softmax over this warp's tokens (heads 2tig, 2tig+1)
    float mx0 = fmaxf(l[0], l[2]), mx1 = fmaxf(l[1], l[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(mrun0, mx0), mn1 = fmaxf(mrun1, mx1);  // finite: the tile has a token
    const float al0 = __expf(mrun0 - mn0), al1 = __expf(mrun1 - mn1);
    float p[4];
    p[0] = h0 < gq ? __expf(l[0] - mn0) : 0.f;
    p[1] = h1 < gq ? __expf(l[1] - mn1) : 0.f;
    p[2] = h0 < gq ? __expf(l[2] - mn0) : 0.f;
    p[3] = h1 < gq ? __expf(l[3] - mn1) : 0.f;
    lsum0 = fmaf(lsum0, al0, p[0] + p[2]);
    lsum1 = fmaf(lsum1, al1, p[1] + p[3]);
    mrun0 = mn0, mrun1 = mn1;

    if constexpr (PV) {
      Ps[gid * 9 + h0] = p[0];
      Ps[gid * 9 + h1] = p[1];
      Ps[(gid + 8) * 9 + h0] = p[2];
      Ps[(gid + 8) * 9 + h1] = p[3];
      // rescale factors of the heads of the lane's output columns; with four
      // heads the columns are (head, hi/lo part): tig < 2 hi, tig >= 2 lo of
      // heads 2(tig&1), 2(tig&1)+1, held by lane tig ^ 2 in the logit layout
      float ac0 = al0, ac1 = al1;
      if constexpr (GQP == 4) {
        const float x0 = __shfl_xor_sync(0xffffffffu, al0, 2), x1 = __shfl_xor_sync(0xffffffffu, al1, 2);
        if (tig >= 2) ac0 = x0, ac1 = x1;
      }
      // rescale factor of the B-operand head (held by the lanes with tig = hb / 2)
      const int hb = GQP == 4 ? (gid & 3) : gid;
      const float ala = __shfl_sync(0xffffffffu, al0, hb >> 1);
      const float alb = __shfl_sync(0xffffffffu, al1, hb >> 1);
      const float alg = (hb & 1) ? alb : ala;
      __syncwarp();
      // B operand: p * s of head hb for the lane's tokens 2tig, 2tig+1,
      // 2tig+8, 2tig+9, split into an fp16 high part and an fp16 low part
      // (v - hi) so the product keeps ~22 bits; the offsets m' go to the fp32
      // m-term.  Four heads: lanes gid < 4 carry hi, gid >= 4 lo (one n-tile).
      // Eight heads: n-tile 0 hi, n-tile 1 lo.
      const float* zv = Zs + 16 * 8;
      float pv[4];
#pragma unroll
      for (int i = 0; i < 4; i++) pv[i] = Ps[(2 * tig + (i & 1) + 8 * (i >> 1)) * 9 + hb];
      uint32_t bf[NT][4][2];
#pragma unroll
      for (int jj = 0; jj < 2; jj++) {
        float4 z[4];
#pragma unroll
        for (int i = 0; i < 4; i++)
          z[i] = reinterpret_cast<const float4*>(zv + (2 * tig + (i & 1) + 8 * (i >> 1)) * 8)[jj];
#pragma unroll
        for (int e = 0; e < 2; e++) {  // group 2jj + e
          float v[4];
#pragma unroll
          for (int i = 0; i < 4; i++) v[i] = pv[i] * (e ? z[i].z : z[i].x);
          const __half2 h01 = __floats2half2_rn(v[0], v[1]), h23 = __floats2half2_rn(v[2], v[3]);
          const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
          const __half2 l01 = __floats2half2_rn(v[0] - f01.x, v[1] - f01.y);
          const __half2 l23 = __floats2half2_rn(v[2] - f23.x, v[3] - f23.y);
          if constexpr (GQP == 4) {
            const bool lo = gid >= 4;
            bf[0][2 * jj + e][0] = *reinterpret_cast<const uint32_t*>(lo ? &l01 : &h01);
            bf[0][2 * jj + e][1] = *reinterpret_cast<const uint32_t*>(lo ? &l23 : &h23);
          } else {
            bf[0][2 * jj + e][0] = *reinterpret_cast<const uint32_t*>(&h01);
            bf[0][2 * jj + e][1] = *reinterpret_cast<const uint32_t*>(&h23);
            bf[NT - 1][2 * jj + e][0] = *reinterpret_cast<const uint32_t*>(&l01);
            bf[NT - 1][2 * jj + e][1] = *reinterpret_cast<const uint32_t*>(&l23);
          }
        }
        float s0 = mt[2 * jj] * alg, s1 = mt[2 * jj + 1] * alg;
#pragma unroll
        for (int i = 0; i < 4; i++) {
          s0 = fmaf(pv[i], z[i].y, s0);
          s1 = fmaf(pv[i], z[i].w, s1);
        }
        mt[2 * jj] = s0, mt[2 * jj + 1] = s1;
      }
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + St::kBytes);
      Words<B> vw[2 * B];
#pragma unroll
      for (int i = 0; i < 2 * B; i++) vw[i].set(vc[lane * 2 * B + i]);
      // Each tile's product starts from zero and is folded into the running
      // sum with one fp32 FMA that also applies the softmax rescale: long
      // accumulation chains inside the tensor-core accumulator would drift.
#pragma unroll
      for (int m = 0; m < 8; m++) {
        uint32_t a0 = pair_of<B>(vw, 2 * m), a1 = pair_of<B>(vw, 2 * m + 1);
        uint32_t a2 = pair_of<B>(vw, 16 + 2 * m), a3 = pair_of<B>(vw, 17 + 2 * m);
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
          float t4[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(t4, a0, a1, a2, a3, bf[nt][m >> 1][0], bf[nt][m >> 1][1]);
          accv[nt][m][0] = fmaf(accv[nt][m][0], ac0, t4[0]);
          accv[nt][m][1] = fmaf(accv[nt][m][1], ac1, t4[1]);
          accv[nt][m][2] = fmaf(accv[nt][m][2], ac0, t4[2]);
          accv[nt][m][3] = fmaf(accv[nt][m][3], ac1, t4[3]);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // ---- per-warp state of heads 2tig, 2tig+1, then merge the CTA's warps
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lsum0 += __shfl_xor_sync(0xffffffffu, lsum0, o);
    lsum1 += __shfl_xor_sync(0xffffffffu, lsum1, o);
  }
  __syncwarp();
  // warp record in its own smem: [GQP][kRec] (the stage ring is free now)
  float* wrec = reinterpret_cast<float*>(wsm);
  const int rec = PV ? kRec : 2;
  if constexpr (PV) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
      float v = mt[j];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      mt[j] = v;  // head gid
    }
    float m0[4], m1[4];  // m-terms of heads 2tig, 2tig+1 (held by the hi lanes gid = head)
#pragma unroll
    for (int j = 0; j < 4; j++) {
      m0[j] = __shfl_sync(0xffffffffu, mt[j], 8 * tig);
      m1[j] = __shfl_sync(0xffffffffu, mt[j], 8 * tig + 4);
    }
#pragma unroll
    for (int m = 0; m < 8; m++) {
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        if constexpr (GQP == 4) {
          o[i] = accv[0][m][i] + __shfl_xor_sync(0xffffffffu, accv[0][m][i], 2);  // hi + lo
        } else {
          o[i] = accv[0][m][i] + accv[NT - 1][m][i];
        }
      }
      if (GQP == 8 || tig < 2) {
        wrec[h0 * kRec + 16 * m + gid] = o[0] + m0[m >> 1];
        wrec[h1 * kRec + 16 * m + gid] = o[1] + m1[m >> 1];
        wrec[h0 * kRec + 16 * m + gid + 8] = o[2] + m0[m >> 1];
        wrec[h1 * kRec + 16 * m + gid + 8] = o[3] + m1[m >> 1];
      }
    }
  }
  if (gid == 0) {
    wrec[h0 * rec + rec - 2] = mrun0, wrec[h0 * rec + rec - 1] = lsum0;
    wrec[h1 * rec + rec - 2] = mrun1, wrec[h1 * rec + rec - 1] = lsum1;
  }
  __syncthreads();
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  for (int e = threadIdx.x; e < gq * rec; e += blockDim.x) {
    const int h = e / rec, d = e % rec;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++)
      M = fmaxf(M, reinterpret_cast<const float*>(smem + w * WS::bytes)[h * rec + rec - 2]);
    float v = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float* r = reinterpret_cast<const float*>(smem + w * WS::bytes) + h * rec;
        const float mw = r[rec - 2];
        if (mw > -INFINITY) v = fmaf(__expf(mw - M), d == rec - 2 ? 0.f : r[d], v);
      }
    }
    if (d == rec - 2) v = M;
    a.part[((hq0 + h) * a.nrec + blockIdx.x) * rec + d] = v;
  }
}

// Softmax max and sum of every query head: M = max_s m_s, Z = sum_s l_s e^(m_s - M).
__global__ void kv_stats_kernel(const float* __restrict__ part, int nsplit, int rec,
                                float2* __restrict__ stats) {
  const long bh = blockIdx.x;
  const float* p = part + bh * nsplit * rec;
  const int mo = rec - 2;
  __shared__ float sm[256];
  float m = -INFINITY;
  for (int i = threadIdx.x; i < nsplit; i += blockDim.x) m = fmaxf(m, p[(long)i * rec + mo]);
  sm[threadIdx.x] = m;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) sm[threadIdx.x] = fmaxf(sm[threadIdx.x], sm[threadIdx.x + o]);
    __syncthreads();
  }
  const float M = sm[0];
  __syncthreads();
  float s = 0.f;
  for (int i = threadIdx.x; i < nsplit; i += blockDim.x) {
    float mi = p[(long)i * rec + mo];
    if (mi > -INFINITY) s += p[(long)i * rec + mo + 1] * expf(mi - M);
  }
  sm[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) sm[threadIdx.x] += sm[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) stats[bh] = make_float2(M, sm[0]);
}

// ---------------------------------------------------------------------------
// selection

// Unique ranking key: score bits (positive floats order like their bits) above
// the complement of the token index, so equal scores rank the lower token first.
__device__ __forceinline__ uint64_t score_key(float score, int t) {
  return ((uint64_t)__float_as_uint(score) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
}
__device__ __forceinline__ int key_token(uint64_t key) {
  return (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu));
}

__global__ void __launch_bounds__(1024) kv_local_kernel(const float* __restrict__ logits,
                                                        const float2* __restrict__ stats, int T,
                                                        int span, int h_q, int h_kv, int k_tok,
                                                        float* __restrict__ scores,
                                                        uint64_t* __restrict__ cand) {
  extern __shared__ uint64_t keys[];  // span entries
  __shared__ RadixShared sh;
  __shared__ float Ms[8], invZ[8];
  const int gq = h_q / h_kv;
  const int sp = blockIdx.x, g = blockIdx.y, bat = blockIdx.z;
  const int t0 = sp * span, n = min(T, t0 + span) - t0;
  if (threadIdx.x < gq) {
    const float2 st = stats[(long)bat * h_q + g * gq + threadIdx.x];
    Ms[threadIdx.x] = st.x, invZ[threadIdx.x] = 1.0f / st.y;
  }
  __syncthreads();
  const float* lg = logits + ((long)bat * h_q + g * gq) * T + t0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float s = 0.f;
    for (int h = 0; h < gq; h++) s += expf(lg[(long)h * T + i] - Ms[h]) * invZ[h];
    if (scores) scores[((long)bat * h_kv + g) * T + t0 + i] = s;
    keys[i] = score_key(s, t0 + i);
  }
  __syncthreads();
  const int kl = min(k_tok, n);
  auto key_at = [&](int i) { return keys[i]; };
  const uint64_t tau = block_kth_largest<64>(key_at, n, kl, sh);
  uint64_t* out = cand + (((long)bat * h_kv + g) * gridDim.x + sp) * (long)min(k_tok, span);
  block_compact(key_at, n, tau, sh, [&](int pos, int, uint64_t key) { out[pos] = key; });
}

__global__ void __launch_bounds__(1024) kv_final_kernel(const uint64_t* __restrict__ cand, int nspan,
                                                        int span, int T, int h_kv, int k_tok,
                                                        int32_t* __restrict__ sel) {
  extern __shared__ uint64_t keys[];  // all candidates of this KV head
  __shared__ RadixShared sh;
  const int g = blockIdx.x, bat = blockIdx.y;
  const int per = min(k_tok, span);
  const uint64_t* src = cand + ((long)bat * h_kv + g) * nspan * (long)per;
  // every span but the last holds `per` keys, so the candidates are one run
  const int last = min(k_tok, T - (nspan - 1) * span);
  const int n = (nspan - 1) * per + last;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = src[i];
  __syncthreads();
  auto key_at = [&](int i) { return keys[i]; };
  const uint64_t tau = block_kth_largest<64>(key_at, n, k_tok, sh);
  int32_t* out = sel + ((long)bat * h_kv + g) * k_tok;
  block_compact(key_at, n, tau, sh, [&](int pos, int, uint64_t key) { out[pos] = key_token(key); });
}

// ---------------------------------------------------------------------------
// correction on the selected tokens

struct CorrArgs {
  const uint8_t *kb, *kr, *vb, *vr;
  const uint16_t *ksz, *vsz;
  int h_kv, t_max, b, r, T;
  const uint16_t* q;
  int h_q, gq;
  const int32_t* sel;
  int k_tok;
  const float* logits;  // base logits [batch][h_q][T]
  const float2* stats;  // [batch][h_q] (max, sum)
  float* corr;          // [batch][h_q][ncorr][kRec]: d-acc[kD], d-sum, unused
  int ncorr;
  float scale;
};


// block = kD threads (thread = head-dim element); every token of the chunk is
// loaded with independent loads before anything is computed
__global__ void __launch_bounds__(kD) kv_correct_kernel(CorrArgs a) {
  __shared__ float kf[kCorrTok][kD + 4];
  __shared__ float vbs[kCorrTok][kD];
  __shared__ float vfs[kCorrTok][kD];
  __shared__ float qs[8][kD + 4];
  __shared__ float wf[kCorrTok][8], wb[kCorrTok][8];
  __shared__ int ts[kCorrTok];
  const int d = threadIdx.x;
  const int chunk = blockIdx.x, g = blockIdx.y, bat = blockIdx.z;
  const int gq = a.gq;
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  for (int h = 0; h < gq; h++) qs[h][d] = h2f(a.q[(hq0 + h) * kD + d]);
  const int j0 = chunk * kCorrTok;
  const int nsel = min(kCorrTok, a.k_tok - j0);
  const int32_t* sg = a.sel + ((long)bat * a.h_kv + g) * a.k_tok + j0;
  if (d < nsel) ts[d] = sg[d];
  __syncthreads();
  const long slot0 = ((long)bat * a.h_kv + g) * a.t_max;
  const float half = 0.5f * (float)(1 << a.r), inv = 1.0f / (float)(1 << a.r);
  int kw, kbit, krw, krbit;
  key_pos(d, a.b, kw, kbit);
  key_pos(d, a.r, krw, krbit);
  // all loads first (independent), then the arithmetic
  uint32_t rqk[kCorrTok], rrk[kCorrTok], rzk[kCorrTok], rqv[kCorrTok], rrv[kCorrTok], rzv[kCorrTok];
  int rvb[kCorrTok], rvr[kCorrTok];
#pragma unroll
  for (int i = 0; i < kCorrTok; i++) {
    if (i < nsel) {
      const int t = ts[i];
      const long slot = slot0 + t;
      const long tile = slot / 16;
      int vw, vbit, vrw, vrbit;
      value_pos(t & 15, d, a.b, vw, vbit);
      value_pos(t & 15, d, a.r, vrw, vrbit);
      rqk[i] = reinterpret_cast<const uint32_t*>(a.kb + slot * 16 * a.b)[kw];
      rrk[i] = reinterpret_cast<const uint32_t*>(a.kr + slot * 16 * a.r)[krw];
      rzk[i] = *reinterpret_cast<const uint32_t*>(a.ksz + (slot * 4 + d / 32) * 2);
      rqv[i] = reinterpret_cast<const uint32_t*>(a.vb + tile * 256 * a.b)[vw];
      rrv[i] = reinterpret_cast<const uint32_t*>(a.vr + tile * 256 * a.r)[vrw];
      rzv[i] = *reinterpret_cast<const uint32_t*>(a.vsz + (slot * 4 + d / 32) * 2);
      rvb[i] = vbit, rvr[i] = vrbit;
    }
  }
#pragma unroll
  for (int i = 0; i < kCorrTok; i++) {
    if (i < nsel) {
      const uint32_t qk = (rqk[i] >> kbit) & ((1u << a.b) - 1);
      const uint32_t rk = (rrk[i] >> krbit) & ((1u << a.r) - 1);
      const uint32_t qv = (rqv[i] >> rvb[i]) & ((1u << a.b) - 1);
      const uint32_t rv = (rrv[i] >> rvr[i]) & ((1u << a.r) - 1);
      const float2 k2 = __half22float2(*reinterpret_cast<const __half2*>(&rzk[i]));
      const float2 v2 = __half22float2(*reinterpret_cast<const __half2*>(&rzv[i]));
      kf[i][d] = fmaf(k2.x, (float)qk + ((float)rk + 0.5f - half) * inv, k2.y);
      vbs[i][d] = fmaf(v2.x, (float)qv, v2.y);
      vfs[i][d] = fmaf(v2.x, (float)qv + ((float)rv + 0.5f - half) * inv, v2.y);
    }
  }
  __syncthreads();
  // refined logits of (token, head) pairs; base logits as the base pass stored them
  for (int pr = d; pr < nsel * gq; pr += kD) {
    const int i = pr / gq, h = pr % gq;
    float acc = 0.f;
#pragma unroll 8
    for (int e = 0; e < kD; e++) acc = fmaf(qs[h][e], kf[i][e], acc);
    const float M = a.stats[hq0 + h].x;
    const float lb = a.logits[(hq0 + h) * a.T + ts[i]];
    wf[i][h] = __expf(acc * a.scale - M);
    wb[i][h] = __expf(lb - M);
  }
  __syncthreads();
  for (int h = 0; h < gq; h++) {
    float da = 0.f, dz = 0.f;
    for (int i = 0; i < nsel; i++) {
      da = fmaf(wf[i][h], vfs[i][d], fmaf(-wb[i][h], vbs[i][d], da));
      dz += wf[i][h] - wb[i][h];
    }
    float* rec = a.corr + ((hq0 + h) * a.ncorr + chunk) * kRec;
    rec[d] = da;
    if (d == 0) rec[kD] = dz;
  }
}

// out = (sum_s e^(m_s - M) acc_s + sum_c dA_c) / (Z + sum_c dZ_c).
// 4 x kD threads: thread group r sums every 4th record.
constexpr int kMergeGroups = 4;
constexpr int kMaxRec = 4096;

__global__ void __launch_bounds__(kMergeGroups * kD) kv_merge_kernel(
    const float* __restrict__ part, int nrec, const float* __restrict__ corr, int ncorr,
    const float2* __restrict__ stats, float* __restrict__ out) {
  __shared__ float wts[kMaxRec];
  __shared__ float red[kMergeGroups][kD + 1];
  const long bh = blockIdx.x;
  const float2 st = stats[bh];
  const float* p = part + bh * nrec * kRec;
  for (int s = threadIdx.x; s < nrec; s += blockDim.x) {
    const float ms = p[(long)s * kRec + kD];
    wts[s] = ms > -INFINITY ? expf(ms - st.x) : 0.f;
  }
  __syncthreads();
  const int d = threadIdx.x % kD, grp = threadIdx.x / kD;
  float num = 0.f, dz = 0.f;
  int s = grp;
  for (; s + 3 * kMergeGroups < nrec; s += 4 * kMergeGroups) {
    const float v0 = p[(long)s * kRec + d], v1 = p[(long)(s + kMergeGroups) * kRec + d];
    const float v2 = p[(long)(s + 2 * kMergeGroups) * kRec + d], v3 = p[(long)(s + 3 * kMergeGroups) * kRec + d];
    num = fmaf(wts[s], v0, num);
    num = fmaf(wts[s + kMergeGroups], v1, num);
    num = fmaf(wts[s + 2 * kMergeGroups], v2, num);
    num = fmaf(wts[s + 3 * kMergeGroups], v3, num);
  }
  for (; s < nrec; s += kMergeGroups) num = fmaf(wts[s], p[(long)s * kRec + d], num);
  if (corr) {
    const float* c = corr + bh * ncorr * kRec;
    for (int i = grp; i < ncorr; i += kMergeGroups) {
      num += c[(long)i * kRec + d];
      dz += c[(long)i * kRec + kD];
    }
  }
  red[grp][d] = num;
  if (d == 0) red[grp][kD] = dz;
  __syncthreads();
  if (grp == 0) {
    float n = 0.f, z = st.y;
#pragma unroll
    for (int r = 0; r < kMergeGroups; r++) {
      n += red[r][d];
      z += red[r][kD];
    }
    out[bh * kD + d] = n / z;
  }
}

// ---------------------------------------------------------------------------
// host side

struct Plan {
  int nsplit, span, nrec; // base pass (warp splits; one record per CTA of kWarps splits)
  int sspan, ns;          // selection spans
  int ncorr;              // correction chunks per KV head
  size_t off_logits, off_part, off_stats, off_cand, off_corr, total;
};

Plan make_plan(const sf_kv* kv, int t, int h_q, int k_tok, bool need_logits, bool with_pv,
               bool select, int n_splits) {
  Plan P;
  const int sms = num_sms();
  const int heads = kv->batch * kv->h_kv;
  int ns = n_splits > 0 ? n_splits : (16 * sms + heads - 1) / heads;
  int maxs = (t + 15) / 16;
  if (ns > maxs) ns = maxs;
  if (ns < 1) ns = 1;
  P.span = ((t + ns - 1) / ns + 15) / 16 * 16;
  P.nsplit = (t + P.span - 1) / P.span;
  P.nrec = (P.nsplit + kWarps - 1) / kWarps;  // <= kMaxRec is checked by the callers
  // selection spans
  int ss = (sms + heads - 1) / heads;
  if (ss < 1) ss = 1;
  int span = (t + ss - 1) / ss;
  if (span > kMaxSpan) span = kMaxSpan;
  if (span < 32) span = 32;
  ss = (t + span - 1) / span;
  while (ss > 1 && (long)ss * (k_tok < span ? k_tok : span) > kMaxCand && span < kMaxSpan) {
    span = span * 2 > kMaxSpan ? kMaxSpan : span * 2;
    ss = (t + span - 1) / span;
  }
  P.sspan = span, P.ns = ss;
  P.ncorr = k_tok > 0 ? (k_tok + kCorrTok - 1) / kCorrTok : 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const int rec = with_pv ? kRec : 2;
  P.off_logits = need_logits ? take((size_t)kv->batch * h_q * t * 4) : 0;
  P.off_part = take((size_t)kv->batch * h_q * P.nrec * rec * 4);
  P.off_stats = take((size_t)kv->batch * h_q * 8);
  P.off_cand = select ? take((size_t)heads * P.ns * (k_tok < span ? k_tok : span) * 8) : 0;
  P.off_corr = (with_pv && P.ncorr) ? take((size_t)kv->batch * h_q * P.ncorr * kRec * 4) : 0;
  P.total = off;
  return P;
}

sf_status check_q(const sf_kv* kv, int t, const uint16_t* q, int h_q) {
  SF_REQUIRE(t >= 1 && t <= kv->t_max, "t=%d outside [1, t_max=%d]", t, kv->t_max);
  SF_REQUIRE(q && aligned16(q), "q must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(h_q > 0 && h_q % kv->h_kv == 0 && h_q / kv->h_kv <= 8,
                 "h_q=%d must be a multiple of h_kv=%d with at most 8 query heads per KV head", h_q,
                 kv->h_kv);
  return SF_OK;
}

template <int GQP, int B, bool PV>
sf_status launch_base_t(const BaseArgs& a, int batch, cudaStream_t s) {
  const size_t smem = kWarps * WarpSmem<B, PV>::bytes;
  auto kern = kv_base_kernel<GQP, B, PV>;
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid((a.nsplit + kWarps - 1) / kWarps, a.h_kv, batch);
  kern<<<grid, kWarps * 32, smem, s>>>(a);
  SF_LAUNCHED();
  return SF_OK;
}

sf_status launch_base(const sf_kv* kv, const BaseArgs& a, bool pv, cudaStream_t s) {
  const int gqp = a.gq <= 4 ? 4 : 8;
  if (kv->b == 2) {
    if (gqp == 4) return pv ? launch_base_t<4, 2, true>(a, kv->batch, s) : launch_base_t<4, 2, false>(a, kv->batch, s);
    return pv ? launch_base_t<8, 2, true>(a, kv->batch, s) : launch_base_t<8, 2, false>(a, kv->batch, s);
  }
  if (gqp == 4) return pv ? launch_base_t<4, 4, true>(a, kv->batch, s) : launch_base_t<4, 4, false>(a, kv->batch, s);
  return pv ? launch_base_t<8, 4, true>(a, kv->batch, s) : launch_base_t<8, 4, false>(a, kv->batch, s);
}

BaseArgs base_args(const sf_kv* kv, int t, const uint16_t* q, int h_q, float* logits, float* part,
                   const Plan& P) {
  BaseArgs a;
  a.kb = (const uint8_t*)kv->kb, a.vb = (const uint8_t*)kv->vb;
  a.ksz = kv->ksz, a.vsz = kv->vsz;
  a.h_kv = kv->h_kv, a.t_max = kv->t_max, a.T = t;
  a.q = q, a.h_q = h_q, a.gq = h_q / kv->h_kv;
  a.logits = logits, a.part = part;
  a.span = P.span, a.nsplit = P.nsplit, a.nrec = P.nrec;
  a.scale = 1.0f / sqrtf((float)kD);
  return a;
}

sf_status launch_select(const sf_kv* kv, int t, int h_q, int k_tok, const Plan& P,
                        const float* logits, const float2* stats, float* scores, uint64_t* cand,
                        int32_t* sel, cudaStream_t s) {
  long ncand = (long)P.ns * (k_tok < P.sspan ? k_tok : P.sspan);
  SF_UNSUPPORTED(ncand <= kMaxCand, "t=%d with k_tok=%d needs %ld candidates (max %d)", t, k_tok,
                 ncand, kMaxCand);
  SF_CUDA(cudaFuncSetAttribute(kv_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSpan * 8));
  kv_local_kernel<<<dim3(P.ns, kv->h_kv, kv->batch), 1024, (size_t)P.sspan * 8, s>>>(
      logits, stats, t, P.sspan, h_q, kv->h_kv, k_tok, scores, cand);
  SF_LAUNCHED();
  SF_CUDA(cudaFuncSetAttribute(kv_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxCand * 8));
  kv_final_kernel<<<dim3(kv->h_kv, kv->batch), 1024, (size_t)ncand * 8, s>>>(cand, P.ns, P.sspan, t,
                                                                           kv->h_kv, k_tok, sel);
  SF_LAUNCHED();
  return SF_OK;
}

sf_status launch_correct_merge(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                               const int32_t* sel, int k_tok, const Plan& P, const float* logits,
                               const float* part, const float2* stats, float* corr, float* out,
                               cudaStream_t s) {
  if (k_tok > 0) {
    CorrArgs c;
    c.kb = (const uint8_t*)kv->kb, c.kr = (const uint8_t*)kv->kr;
    c.vb = (const uint8_t*)kv->vb, c.vr = (const uint8_t*)kv->vr;
    c.ksz = kv->ksz, c.vsz = kv->vsz;
    c.h_kv = kv->h_kv, c.t_max = kv->t_max, c.b = kv->b, c.r = kv->r, c.T = t;
    c.q = q, c.h_q = h_q, c.gq = h_q / kv->h_kv;
    c.sel = sel, c.k_tok = k_tok, c.logits = logits, c.stats = stats;
    c.corr = corr, c.ncorr = P.ncorr;
    c.scale = 1.0f / sqrtf((float)kD);
    kv_correct_kernel<<<dim3(P.ncorr, kv->h_kv, kv->batch), kD, 0, s>>>(c);
    SF_LAUNCHED();
  }
  kv_merge_kernel<<<kv->batch * h_q, kMergeGroups * kD, 0, s>>>(part, P.nrec, k_tok > 0 ? corr : nullptr,
                                                                P.ncorr, stats, out);
  SF_LAUNCHED();
  return SF_OK;
}

sf_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws_bytes < need || (need > 0 && !ws)) {
    set_error("workspace: need %zu bytes, got %zu", need, ws_bytes);
    return SF_ERR_WORKSPACE;
  }
  SF_REQUIRE(!ws || aligned16(ws), "ws must be 16-byte aligned");
  return SF_OK;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_kv_score_select_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                                     int logits_given) {
  if (!kv || t <= 0 || h_q <= 0 || k_tok <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, !logits_given, false, true, 0).total;
}

extern "C" sf_status sf_kv_score_select(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                        int k_tok, int32_t* sel, float* logits, float* scores,
                                        void* ws, size_t ws_bytes, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok >= 1 && k_tok <= t, "k_tok=%d outside [1, t=%d]", k_tok, t);
  SF_UNSUPPORTED(k_tok <= 4096, "k_tok=%d above 4096", k_tok);
  SF_REQUIRE(sel && aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(!logits || aligned16(logits), "logits must be 16-byte aligned");
  SF_REQUIRE(!scores || aligned16(scores), "scores must be 16-byte aligned");
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, false, true, 0);
  SF_UNSUPPORTED(P.nrec <= kMaxRec, "t=%d needs %d partial records (max %d)", t, P.nrec, kMaxRec);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  cudaStream_t s = as_stream(stream);
  BaseArgs a = base_args(kv, t, q, h_q, lg, (float*)(w + P.off_part), P);
  st = launch_base(kv, a, false, s);
  if (st != SF_OK) return st;
  float2* stats = (float2*)(w + P.off_stats);
  kv_stats_kernel<<<kv->batch * h_q, 256, 0, s>>>((const float*)(w + P.off_part), P.nrec, 2, stats);
  SF_LAUNCHED();
  return launch_select(kv, t, h_q, k_tok, P, lg, stats, scores, (uint64_t*)(w + P.off_cand), sel, s);
}

extern "C" size_t sf_kv_attn_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                             int n_splits) {
  if (!kv || t <= 0 || h_q <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, true, true, false, n_splits).total;
}

extern "C" sf_status sf_kv_attn_refined(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                        const int32_t* sel, int k_tok, int n_splits, float* out,
                                        void* ws, size_t ws_bytes, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok >= 0 && k_tok <= t, "k_tok=%d outside [0, t=%d]", k_tok, t);
  SF_REQUIRE(k_tok == 0 || (sel && aligned16(sel)), "sel must be non-null and 16-byte aligned");
  SF_REQUIRE(n_splits >= 0, "n_splits=%d < 0", n_splits);
  SF_REQUIRE(out && aligned16(out), "out must be a non-null 16-byte aligned device pointer");
  Plan P = make_plan(kv, t, h_q, k_tok, true, true, false, n_splits);
  SF_UNSUPPORTED(P.nrec <= kMaxRec, "t=%d needs %d partial records (max %d)", t, P.nrec, kMaxRec);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  cudaStream_t s = as_stream(stream);
  float* lg = (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  float2* stats = (float2*)(w + P.off_stats);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  kv_stats_kernel<<<kv->batch * h_q, 256, 0, s>>>(part, P.nrec, kRec, stats);
  SF_LAUNCHED();
  return launch_correct_merge(kv, t, q, h_q, sel, k_tok, P, lg, part, stats,
                              (float*)(w + P.off_corr), out, s);
}

extern "C" size_t sf_kv_attend_selective_workspace_bytes(const sf_kv* kv, int t, int h_q,
                                                         int k_tok, int logits_given) {
  if (!kv || t <= 0 || h_q <= 0 || k_tok <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, !logits_given, true, true, 0).total;
}

extern "C" sf_status sf_kv_attend_selective(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                            int k_tok, int32_t* sel, float* logits, float* out,
                                            void* ws, size_t ws_bytes, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok >= 1 && k_tok <= t, "k_tok=%d outside [1, t=%d]", k_tok, t);
  SF_UNSUPPORTED(k_tok <= 4096, "k_tok=%d above 4096", k_tok);
  SF_REQUIRE(sel && aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(!logits || aligned16(logits), "logits must be 16-byte aligned");
  SF_REQUIRE(out && aligned16(out), "out must be a non-null 16-byte aligned device pointer");
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, true, true, 0);
  SF_UNSUPPORTED(P.nrec <= kMaxRec, "t=%d needs %d partial records (max %d)", t, P.nrec, kMaxRec);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  cudaStream_t s = as_stream(stream);
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  float2* stats = (float2*)(w + P.off_stats);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  kv_stats_kernel<<<kv->batch * h_q, 256, 0, s>>>(part, P.nrec, kRec, stats);
  SF_LAUNCHED();
  st = launch_select(kv, t, h_q, k_tok, P, lg, stats, nullptr, (uint64_t*)(w + P.off_cand), sel, s);
  if (st != SF_OK) return st;
  return launch_correct_merge(kv, t, q, h_q, sel, k_tok, P, lg, part, stats,
                              (float*)(w + P.off_corr), out, s);
}

// ---------------------------------------------------------------------------
// sf_kv_attend_selective with library-owned scratch.
//
// Some callers cannot allocate device memory for the workspace.  A plain C
// host program or an embedding runtime has no caching allocator to draw from,
// so every call would need cudaMalloc + cudaFree, and cudaFree synchronises the
// whole device.  A latency-critical decode loop must not stall on that
// synchronisation.  For those callers the workspace is this file-scope device
// array: it is part of the library's module image, so using it allocates
// nothing at call time.  All calls on one device share it, so two such calls
// that overlap on the GPU (different streams or threads with no ordering
// between them) race on it.  None of the scratch needs to start at zero:
// every kernel of the pass writes each scratch word it later reads.

namespace sf {
namespace {

constexpr size_t kStaticWsBytes = (size_t)SF_KV_STATIC_WS_BYTES;
constexpr int kStaticWsDevices = 64;

__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_static_ws_mu;
void* g_static_ws_ptr[kStaticWsDevices] = {};

// Device address of g_static_ws on the current device, looked up once per
// device (the first lookup loads the module on that device).
sf_status static_ws(void** ptr) {
  int dev = -1;
  SF_CUDA(cudaGetDevice(&dev));
  SF_UNSUPPORTED(dev >= 0 && dev < kStaticWsDevices, "device %d outside [0, %d)", dev,
                 kStaticWsDevices);
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess || !p) {
      set_error("cudaGetSymbolAddress(static KV workspace) on device %d failed: %s", dev,
                cudaGetErrorString(e));
      return SF_ERR_CUDA;
    }
    g_static_ws_ptr[dev] = p;
  }
  *ptr = g_static_ws_ptr[dev];
  return SF_OK;
}

}  // namespace
}  // namespace sf

extern "C" sf_status sf_kv_attend_selective_static(const sf_kv* kv, int t, const uint16_t* q,
                                                   int h_q, int k_tok, int32_t* sel, float* logits,
                                                   float* out, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok >= 1 && k_tok <= t, "k_tok=%d outside [1, t=%d]", k_tok, t);
  const size_t need = make_plan(kv, t, h_q, k_tok, logits == nullptr, true, true, 0).total;
  if (need > kStaticWsBytes) {
    set_error("workspace of %zu bytes needed (batch=%d, h_q=%d, t=%d, k_tok=%d, logits %s) is above "
              "the static scratch of %zu bytes; use sf_kv_attend_selective with a caller workspace",
              need, kv->batch, h_q, t, k_tok, logits ? "given" : "in scratch", kStaticWsBytes);
    return SF_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  st = static_ws(&ws);
  if (st != SF_OK) return st;
  return sf_kv_attend_selective(kv, t, q, h_q, k_tok, sel, logits, out, ws, kStaticWsBytes, stream);
}
