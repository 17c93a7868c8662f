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
//   kv_base_kernel  per 16-token tile, logits of the group's query heads from
//                   the base keys and the base attention (online softmax,
//                   split-K partials) from the base values; the logits are
//                   stored for scoring.  Codes are turned into exact fp16
//                   integers in registers and contracted on the tensor cores
//                   (mma.sync m16n8k16, fp32 accumulation); the per-token fp16
//                   steps/offsets are applied in fp32.
//   kv_post_kernel  one thread-block cluster per KV head: softmax statistics
//                   from the partials, token scores, a cluster-wide radix
//                   select of the top k_tok (histograms exchanged through
//                   distributed shared memory), then the correction of the
//                   selected tokens (each token's base contribution swapped
//                   for its refined one, relative to the head's softmax
//                   maximum) and the log-sum-exp merge of the partials.
// The result equals softmax(q.k~) v~ with refined k~, v~ on the selected
// tokens, up to fp32 rounding.
#include <cooperative_groups.h>

#include <algorithm>
#include <cfloat>
#include <mutex>

#include "common.cuh"
#include "kvlayout.cuh"

namespace sf {
namespace {

constexpr int kD = kHeadDim;
constexpr int kRec = kD + 2;     // partial record: acc[kD], m, l
constexpr int kWarps = 4;        // warps per base-pass CTA (independent splits)
constexpr int kStages = 4;       // cp.async ring depth per warp

// ---- small PTX helpers -------------------------------------------------------

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(gmem) : "memory");
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
// four CTAs of 128 threads per SM at 120 registers (GQP = 4) leave kSideRegs
// of the SM's registers free; GQP = 8 takes two CTAs of up to 255
static_assert(65536 - 4 * 120 * kWarps * 32 >= kSideRegs, "base pass registers leave no room for a staging CTA");
template <int GQP, int B, bool PV>
__global__ void __maxnreg__(GQP == 4 ? 120 : 255) kv_base_kernel(BaseArgs a) {
  using St = Stage<B, PV>;
  using WS = WarpSmem<B, PV>;
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_trigger();  // the kernel after the base pass may be scheduled now; it waits for this grid
  pdl_wait();     // q and the cache (including a token appended just before) are complete
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

// ---------------------------------------------------------------------------
// after the base pass: one thread-block cluster per (batch, KV head)
//
// The cluster's CTAs split the context: each scores its tokens (sum over the
// group's query heads of the softmax probability, from the stored base
// logits) into shared memory.  The k_tok-th largest score is found by a radix
// select over the score bits (non-negative floats order like their bits),
// 9 bits per pass from bit 30: every CTA histograms its keys, stores the
// histogram into every peer's shared memory (distributed shared memory) and,
// after the cluster barrier, all CTAs take the same decision from their local
// copies.  Equal scores rank the lower token first; the selected tokens are
// written in ascending order and also handed, by position, to the CTA that
// refines them.  Each CTA then copies its share of the selected tokens' codes
// and scales into shared memory with cp.async in one go and refines them, each
// warp four tokens together (swapping each token's base contribution for its
// refined one, relative to the head's softmax maximum; the refined logits of
// the warp's (token, head) slots summed by one transposed butterfly, each
// warp's sums kept in its own slot rather than added with shared-memory
// atomics), sums an interleaved share of the base partial records, and CTA h
// merges query head h.

constexpr int kPostThreads = 512;
constexpr int kPostMaxTok = 16640;  // tokens per CTA scored in shared memory (cluster of 8)
constexpr int kPostCl = 8;
constexpr int kPostStage = 64;      // selected tokens staged in shared memory at a time
constexpr int kPostMaxSel = 512;    // selected tokens per CTA (k_tok <= 4096)
constexpr int kMaxKTok = 4096;      // the largest k_tok every attention entry point accepts
static_assert(kPostCl * kPostMaxSel == kMaxKTok, "the cluster's selection buffers must hold k_tok tokens");
constexpr int kHistBins = 512;
// a warp's share of one staging batch, times 8 query heads, fits its 32 lanes
static_assert(kPostStage / (kPostThreads / 32) * 8 <= 32, "staging batch too large for the lane layout");
// the per-warp partial numerators reuse the score keys' space
static_assert((kPostThreads / 32) * 8 * kD <= kPostMaxTok, "key space too small for the partial numerators");

struct PostArgs {
  const uint8_t *kb, *kr, *vb, *vr;
  const uint16_t *ksz, *vsz;
  int h_kv, t_max, b, r, T;
  const uint16_t* q;
  int h_q, gq;
  const float* logits;  // base logits [batch][h_q][T]
  const float* part;    // base partial records [batch][h_q][nrec][rec]
  int nrec, rec;        // rec = kRec (with values) or 2 (scores only)
  int k_tok;
  int32_t* sel;         // [batch][h_kv][k_tok]: written when select, else read
  int select;
  float* scores;        // nullable [batch][h_kv][T]
  float* out;           // nullable [batch][h_q][kD]
  uint16_t* out16;      // nullable [batch][h_q][kD], the same rounded to fp16
  int chunk;            // tokens per CTA
  float scale;
};

struct PostShared {
  int hist[kHistBins];  // this CTA's histogram of the current pass
  int tot[kHistBins];
  int warp_tot[32];
  int cnt;
  int digit, kleft, done;
  float M[8], Z[8];
  float wden[kPostThreads / 32][8];      // per warp: its tokens' change of each head's denominator
  float wtab[kPostThreads / 32][2 * 32];  // per warp: (w_refined, w_base) of its (token, head) slots
};

// Filled by the peers (distributed shared memory stores, which do not stall the
// writer); read locally after a cluster barrier.
struct PostMail {
  int hist[2][kPostCl][kHistBins];  // per pass (alternating): every CTA's histogram
  int cnt[kPostCl];                 // every CTA's packed (above, equal) counts
  int tok[kPostMaxSel];             // the selected tokens this CTA refines, by position
  float num[kPostCl][kD];           // this CTA's query head: every CTA's partial numerator
  float den[kPostCl];
};

// Words of one staged token: K codes (4b), K refinement (4r), K and V (s, m)
// (4 + 4), the token's 8 value chunks of codes (8 x 2b) and refinement (8 x 2r).
__host__ __device__ constexpr int tok_words(int b, int r) { return 20 * (b + r) + 8; }

// Sums each of the N (16 or 32) per-lane values v over the warp; returns the
// sum of value lane % N.  Each round keeps the half of the values that the
// lane's bit selects and adds the partner's copy of it.
template <int N>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[N], int lane) {
  static_assert(N == 16 || N == 32, "16 or 32 values");
#pragma unroll
  for (int n = N, o = N / 2; n > 1; n >>= 1, o >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int j = 0; j < n / 2; j++) {
      const float keep = up ? v[j + n / 2] : v[j], send = up ? v[j] : v[j + n / 2];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float r = v[0];
  if constexpr (N == 16) r += __shfl_xor_sync(0xffffffffu, r, 16);
  return r;
}

// GQP: query heads per KV head, padded to 4 or 8 (register arrays); B, R:
// the cache's base and refinement bits.
template <int GQP, int B, int R>
__global__ void __launch_bounds__(kPostThreads, 1) kv_post_kernel(PostArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int cr = (int)cluster.block_rank(), CL = (int)cluster.num_blocks();
  extern __shared__ __align__(16) uint8_t dyn[];
  PostMail& mail = *reinterpret_cast<PostMail*>(dyn);
  uint32_t* stage = reinterpret_cast<uint32_t*>(dyn + sizeof(PostMail));  // staged selected tokens
  uint32_t* keys = stage + kPostStage * tok_words(B, R);               // this CTA's score keys
  __shared__ PostShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kPostThreads / 32;
  const int g = blockIdx.y, bat = blockIdx.z;
  const int gq = a.gq;
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  pdl_trigger();
  // every CTA of the cluster must have started before peers touch its shared
  // memory: arrive now, wait right before the first distributed access
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  pdl_wait();  // the base pass is complete

  // softmax statistics of the group's query heads: every record's (m, l)
  // loaded in one batch per lane
  if (warp < gq) {
    const float* pr = a.part + (hq0 + warp) * a.nrec * a.rec;
    constexpr int PER = 8;
    float ms[PER], ls[PER];
    float m = -INFINITY, z = 0.f;
    for (int s0 = 0; s0 < a.nrec; s0 += 32 * PER) {
#pragma unroll
      for (int k = 0; k < PER; k++) {
        const int s = s0 + lane + 32 * k;
        ms[k] = s < a.nrec ? pr[(long)s * a.rec + a.rec - 2] : -INFINITY;
        ls[k] = s < a.nrec ? pr[(long)s * a.rec + a.rec - 1] : 0.f;
      }
      float mb = -INFINITY;
#pragma unroll
      for (int k = 0; k < PER; k++) mb = fmaxf(mb, ms[k]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      const float mn = fmaxf(m, mb);
      float zb = 0.f;
#pragma unroll
      for (int k = 0; k < PER; k++)
        if (ms[k] > -INFINITY) zb += ls[k] * expf(ms[k] - mn);
      z = (m > -INFINITY ? z * expf(m - mn) : 0.f) + zb;
      m = mn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) sh.M[warp] = m, sh.Z[warp] = z;
  }
  __syncthreads();

  const int ja = (int)((long)cr * a.k_tok / CL), jb = (int)((long)(cr + 1) * a.k_tok / CL);
  if (a.select) {
    const int t0 = cr * a.chunk, n = max(0, min(a.T, t0 + a.chunk) - t0);
    const float* lg = a.logits + hq0 * a.T + t0;
    float Mh[GQP], invZ[GQP];
#pragma unroll
    for (int h = 0; h < GQP; h++) Mh[h] = h < gq ? sh.M[h] : 0.f, invZ[h] = h < gq ? 1.0f / sh.Z[h] : 0.f;
    // eight tokens per thread per step (token tid + 512 e: coalesced), every load
    // of the step issued first
    constexpr int TPT = 8;
    for (int i0 = tid; i0 < n; i0 += TPT * kPostThreads) {
      float l[GQP][TPT];
#pragma unroll
      for (int h = 0; h < GQP; h++)
#pragma unroll
        for (int e = 0; e < TPT; e++) {
          const int i = i0 + e * kPostThreads;
          l[h][e] = (h < gq && i < n) ? lg[(long)h * a.T + i] : -INFINITY;
        }
#pragma unroll
      for (int e = 0; e < TPT; e++) {
        const int i = i0 + e * kPostThreads;
        if (i < n) {
          float sc = 0.f;
#pragma unroll
          for (int h = 0; h < GQP; h++)
            if (h < gq) sc += expf(l[h][e] - Mh[h]) * invZ[h];  // full-accuracy exp: the score decides the selection
          if (a.scores) a.scores[((long)bat * a.h_kv + g) * a.T + t0 + i] = sc;
          keys[i] = __float_as_uint(sc);
        }
      }
    }
    // ---- radix select of the k_tok-th largest key over the cluster: digits of
    // bits 30..22, 21..13, 12..4, 3..0 (bit 31 is 0 for non-negative scores)
    uint32_t prefix = 0, mask = 0x80000000u;
    int kleft = a.k_tok, buf = 0;
    bool done = false;
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    for (int pass = 0; pass < 4 && !done; pass++) {
      const int shift = pass < 3 ? 22 - 9 * pass : 0;
      const int bits = pass < 3 ? 9 : 4, bins = 1 << bits;
      for (int i = tid; i < bins; i += kPostThreads) sh.hist[i] = 0;
      __syncthreads();
      for (int i0 = warp * 32; i0 < n; i0 += kPostThreads) {  // whole warps: lanes with equal bins add once
        const int i = i0 + lane;
        const uint32_t key = i < n ? keys[i] : 0u;
        const bool in = i < n && (key & mask) == prefix;
        const int bn = in ? (int)((key >> shift) & (bins - 1)) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, bn);
        if (in && (__ffs(same) - 1) == lane) atomicAdd(&sh.hist[bn], __popc(same));
      }
      __syncthreads();
      for (int i = tid; i < bins * CL; i += kPostThreads)  // my histogram into every peer's mailbox
        cluster.map_shared_rank(&mail.hist[buf][cr][0], i / bins)[i % bins] = sh.hist[i % bins];
      cluster.sync();  // every CTA's histogram is in every mailbox
      for (int bn = tid; bn < bins; bn += kPostThreads) {
        int t = 0;
        for (int rk = 0; rk < CL; rk++) t += mail.hist[buf][rk][bn];
        sh.tot[bn] = t;
      }
      __syncthreads();
      if (warp == 0) {
        // lane covers the bins below bins - 1 - PL lane, from the top
        const int PL = bins >= 32 ? bins / 32 : 1;
        int c[16], tot = 0;
#pragma unroll
        for (int j = 0; j < 16; j++) {
          const int bn = bins - 1 - PL * lane - j;
          c[j] = (j < PL && bn >= 0) ? sh.tot[bn] : 0;
          tot += c[j];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int above = incl - tot;
        if (above < kleft && incl >= kleft) {
          int run = above;
          for (int j = 0; j < PL; j++) {
            if (run + c[j] >= kleft) {
              sh.digit = bins - 1 - PL * lane - j;
              sh.kleft = kleft - run;
              sh.done = c[j] == kleft - run;  // the whole bucket is needed
              break;
            }
            run += c[j];
          }
        }
      }
      __syncthreads();
      prefix |= (uint32_t)sh.digit << shift;
      mask |= (uint32_t)(bins - 1) << shift;
      kleft = sh.kleft;
      done = sh.done;
      buf ^= 1;  // the next pass fills the other mailbox while this one may still be read
    }
    // keys above `prefix` (or, when the last bucket was taken whole, at or above
    // it) are selected; of the keys equal to it, the first `kleft` in token order
    const int per = (n + kPostThreads - 1) / kPostThreads;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int ngt = 0, neq = 0;
    for (int i = i0; i < i1; i++) {
      const uint32_t key = keys[i];
      if (done ? key >= prefix : key > prefix) ngt++;
      else if (!done && key == prefix) neq++;
    }
    // one block scan of the packed counts (above + equal << 16), in token order
    const int v = ngt + (neq << 16);
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) sh.warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = lane < NW ? sh.warp_tot[lane] : 0;
      int x = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += u;
      }
      if (lane < NW) sh.warp_tot[lane] = x - wv;
      if (lane == 31) sh.cnt = x;
    }
    __syncthreads();
    const int ex = sh.warp_tot[warp] + incl - v;
    const int gt_ex = ex & 0xFFFF, eq_ex = ex >> 16;
    if (tid < CL) cluster.map_shared_rank(&mail.cnt[cr], tid)[0] = sh.cnt;
    cluster.sync();  // every CTA's counts are in every mailbox
    int sel_before = 0, eq_before = 0;
    for (int rk = 0; rk < cr; rk++) {
      const int c = mail.cnt[rk];
      sel_before += (c & 0xFFFF) + max(0, min(c >> 16, kleft - eq_before));
      eq_before += c >> 16;
    }
    // my selected tokens: above-threshold ones, and equal ones while the budget lasts
    const int eq_mine = done ? 0 : max(0, min(neq, kleft - (eq_before + eq_ex)));
    int pos = sel_before + gt_ex + max(0, min(eq_ex, kleft - eq_before));
    int eq_seen = 0;
    int32_t* selw = a.sel + ((long)bat * a.h_kv + g) * a.k_tok;
    for (int i = i0; i < i1; i++) {
      const uint32_t key = keys[i];
      bool take = done ? key >= prefix : key > prefix;
      if (!done && key == prefix) take = eq_seen++ < eq_mine;
      if (take && pos < a.k_tok) {
        selw[pos] = t0 + i;
        if (a.out || a.out16) {  // hand the token to the CTA that refines position pos
          const int dst = (int)(((long)(pos + 1) * CL + a.k_tok - 1) / a.k_tok) - 1;
          const int dja = (int)((long)dst * a.k_tok / CL);
          cluster.map_shared_rank(&mail.tok[0], dst)[pos - dja] = t0 + i;
        }
      }
      if (take) pos++;
    }
    cluster.sync();  // every selected token is in its refining CTA's mailbox
  } else {
    const int32_t* selg = a.sel + ((long)bat * a.h_kv + g) * a.k_tok;
    for (int j = ja + tid; j < jb; j += kPostThreads) mail.tok[j - ja] = selg[j];
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    __syncthreads();
  }
  if (!a.out && !a.out16) return;  // no peer reads or writes this CTA's shared memory any more

  // ---- refined attention on this CTA's share of the selected tokens
  {
    const int W = tok_words(B, R);
    const int oK = 0, oKr = 4 * B, oZk = 4 * (B + R), oZv = oZk + 4, oV = oZv + 4, oVr = oV + 16 * B;
    const long slot0 = ((long)bat * a.h_kv + g) * a.t_max;
    const float half = 0.5f * (float)(1 << R), inv = 1.0f / (float)(1 << R);
    const uint32_t bmask = (1u << B) - 1u, rmask = (1u << R) - 1u;
    // lane owns head dims d_e = lane + 32 e (scale group e)
    int kw[4], kbit[4], krw[4], krbit[4];
    float qv[GQP][4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
      key_pos(lane + 32 * e, B, kw[e], kbit[e]);
      key_pos(lane + 32 * e, R, krw[e], krbit[e]);
#pragma unroll
      for (int h = 0; h < GQP; h++) qv[h][e] = h < gq ? h2f(a.q[(hq0 + h) * kD + lane + 32 * e]) : 0.f;
    }
    constexpr int TPW = kPostStage / NW;  // tokens of a staging batch per warp
    float an[GQP][4], ad_own = 0.f;
#pragma unroll
    for (int h = 0; h < GQP; h++)
#pragma unroll
      for (int e = 0; e < 4; e++) an[h][e] = 0.f;
    // pieces of one staged token: 16-byte copies (8-byte for 1-bit value refinement chunks)
    const int pk = B, pkr = R, pv = 8 * (B >= 2 ? B / 2 : 1), pvr = 8 * (R >= 2 ? R / 2 : 1);
    const int npiece = pk + pkr + 2 + pv + pvr;
    for (int j0 = ja; j0 < jb; j0 += kPostStage) {
      const int nt = min(kPostStage, jb - j0);
      __syncthreads();  // the previous batch is consumed
      for (int it = tid; it < nt * npiece; it += kPostThreads) {
        const int i = it / npiece, pc = it % npiece;
        int t = mail.tok[j0 - ja + i];
        if (t < 0 || t >= a.T) t = 0;  // out-of-range indices are never produced by the selection
        const long slot = slot0 + t, tile = slot / 16;
        const int c = (t & 7) >> 1;  // the token's value chunk column
        uint32_t* dst = stage + i * W;
        if (pc < pk) {
          cp_async16(dst + oK + 4 * pc, a.kb + slot * 16 * B + 16 * pc);
        } else if (pc < pk + pkr) {
          const int q4 = pc - pk;
          cp_async16(dst + oKr + 4 * q4, a.kr + slot * 16 * R + 16 * q4);
        } else if (pc == pk + pkr) {
          cp_async16(dst + oZk, reinterpret_cast<const uint8_t*>(a.ksz) + slot * 16);
        } else if (pc == pk + pkr + 1) {
          cp_async16(dst + oZv, reinterpret_cast<const uint8_t*>(a.vsz) + slot * 16);
        } else if (pc < pk + pkr + 2 + pv) {
          // value codes: chunk l = 4 gg + c holds 2b words; b = 4 takes two 16-byte copies
          const int q4 = pc - (pk + pkr + 2), gg = B >= 2 ? q4 / (B / 2) : q4, part = B >= 2 ? q4 % (B / 2) : 0;
          cp_async16(dst + oV + gg * 2 * B + 4 * part,
                     a.vb + tile * 256 * B + (size_t)(4 * gg + c) * 8 * B + 16 * part);
        } else {
          const int q4 = pc - (pk + pkr + 2 + pv);
          if constexpr (R >= 2) {
            const int gg = q4 / (R / 2), part = q4 % (R / 2);
            cp_async16(dst + oVr + gg * 2 * R + 4 * part,
                       a.vr + tile * 256 * R + (size_t)(4 * gg + c) * 8 * R + 16 * part);
          } else {
            cp_async8(dst + oVr + q4 * 2, a.vr + tile * 256 * R + (size_t)(4 * q4 + c) * 8 * R);
          }
        }
      }
      cp_async_commit();
      // while the copies fly: the base weights exp(l_base - M) of the warp's
      // tokens; lane L holds slot u = L % (TPW GQP), i.e. token i = warp + NW
      // (u / GQP), head u % GQP (the slot the transposed reduction below
      // leaves in lane L)
      float wbl = 0.f;
      const int u_own = lane % (TPW * GQP), m_own = u_own / GQP, h_own = u_own % GQP;
      const bool own_ok = h_own < gq && warp + NW * m_own < nt;
      if (own_ok)
        wbl = __expf(a.logits[(hq0 + h_own) * a.T + mail.tok[j0 - ja + warp + NW * m_own]] - sh.M[h_own]);
      cp_async_wait<0>();
      __syncthreads();
      // the warp's TPW tokens together: refined keys, base and refined values
      float kf[TPW][4], vbs[TPW][4], vfs[TPW][4];
#pragma unroll
      for (int m = 0; m < TPW; m++) {
        const int i = warp + NW * m;
        const bool ok = i < nt;
        const uint32_t* st = stage + (ok ? i : 0) * W;
        const int tt = ok ? (mail.tok[j0 - ja + i] & 15) : 0;
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int d = lane + 32 * e;
          int vw, vbit, vrw, vrbit;
          value_pos(tt, d, B, vw, vbit);
          value_pos(tt, d, R, vrw, vrbit);
          // staged chunk gg = d & 7 holds words [l 2w, l 2w + 2w) of the tile
          const int vwl = vw - (4 * (d & 7) + ((tt & 7) >> 1)) * 2 * B + (d & 7) * 2 * B;
          const int vrwl = vrw - (4 * (d & 7) + ((tt & 7) >> 1)) * 2 * R + (d & 7) * 2 * R;
          const uint32_t zk = st[oZk + e], zv = st[oZv + e];
          const float2 k2 = __half22float2(*reinterpret_cast<const __half2*>(&zk));
          const float2 v2 = __half22float2(*reinterpret_cast<const __half2*>(&zv));
          const uint32_t qk = (st[oK + kw[e]] >> kbit[e]) & bmask, rk = (st[oKr + krw[e]] >> krbit[e]) & rmask;
          const uint32_t qq = (st[oV + vwl] >> vbit) & bmask, rv = (st[oVr + vrwl] >> vrbit) & rmask;
          kf[m][e] = fmaf(k2.x, (float)qk + ((float)rk + 0.5f - half) * inv, k2.y);
          vbs[m][e] = ok ? fmaf(v2.x, (float)qq, v2.y) : 0.f;
          vfs[m][e] = ok ? fmaf(v2.x, (float)qq + ((float)rv + 0.5f - half) * inv, v2.y) : 0.f;
        }
      }
      // refined logits of the TPW x GQP (token, head) slots: per-lane partial
      // dot products, summed over the warp by a transposed butterfly that
      // leaves slot lane % (TPW GQP) in each lane
      float lg[TPW * GQP];
#pragma unroll
      for (int m = 0; m < TPW; m++)
#pragma unroll
        for (int h = 0; h < GQP; h++) {
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 4; e++) acc = fmaf(qv[h][e], kf[m][e], acc);
          lg[m * GQP + h] = acc;
        }
      const float lg_own = warp_transpose_sum<TPW * GQP>(lg, lane);
      float wfl = 0.f;
      if (own_ok) wfl = __expf(lg_own * a.scale - sh.M[h_own]);
      // every lane needs every slot's (w_refined, w_base): through the warp's table
      float2* wtab = reinterpret_cast<float2*>(&sh.wtab[warp][0]);
      if (lane < TPW * GQP) wtab[lane] = make_float2(wfl, wbl);
      ad_own += wfl - wbl;
      __syncwarp();
#pragma unroll
      for (int m = 0; m < TPW; m++)
#pragma unroll
        for (int h = 0; h < GQP; h++) {
          const float2 w = wtab[m * GQP + h];
#pragma unroll
          for (int e = 0; e < 4; e++) an[h][e] = fmaf(w.x, vfs[m][e], fmaf(-w.y, vbs[m][e], an[h][e]));
        }
      __syncwarp();
    }
    // per-warp partial numerators and denominators (the score keys are no
    // longer needed: their space holds them), summed in the merge below
    float* wnum = reinterpret_cast<float*>(keys);
#pragma unroll
    for (int h = 0; h < GQP; h++)
      if (h < gq) {
#pragma unroll
        for (int e = 0; e < 4; e++) wnum[(warp * GQP + h) * kD + lane + 32 * e] = an[h][e];
      }
    // slot u's denominator change sits in lanes u, u + TPW GQP, ...; sum over
    // the TPW tokens of each head
    float dsum = lane < TPW * GQP ? ad_own : 0.f;
#pragma unroll
    for (int o = GQP; o < 32; o <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
    if (lane < gq) sh.wden[warp][lane] = dsum;
  }
  __syncthreads();
  // this CTA's share of the base records: records s = cr, cr + CL, ... (loads batched)
  for (int e = tid; e < gq * kD; e += kPostThreads) {
    const int hh = e / kD, d = e % kD;
    const float* pr = a.part + (hq0 + hh) * a.nrec * a.rec;
    float num = 0.f;  // the correction: every warp's partial
    for (int w = 0; w < NW; w++) num += reinterpret_cast<const float*>(keys)[(w * GQP + hh) * kD + d];
    constexpr int PER = 8;
    for (int s0 = cr; s0 < a.nrec; s0 += CL * PER) {
      float mv[PER], av[PER];
#pragma unroll
      for (int k = 0; k < PER; k++) {
        const int s = s0 + CL * k;
        mv[k] = s < a.nrec ? pr[(long)s * a.rec + kD] : -INFINITY;
        av[k] = s < a.nrec ? pr[(long)s * a.rec + d] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < PER; k++)
        if (mv[k] > -INFINITY) num = fmaf(__expf(mv[k] - sh.M[hh]), av[k], num);
    }
    cluster.map_shared_rank(&mail.num[cr][0], hh)[d] = num;  // to the CTA that merges head hh
  }
  if (tid < gq) {
    float den = 0.f;
    for (int w = 0; w < NW; w++) den += sh.wden[w][tid];
    cluster.map_shared_rank(&mail.den[cr], tid)[0] = den;
  }
  cluster.sync();  // every partial numerator is in its head's mailbox
  if (cr < gq) {
    for (int d = tid; d < kD; d += kPostThreads) {
      float num = 0.f, den = sh.Z[cr];
      for (int rk = 0; rk < CL; rk++) num += mail.num[rk][d], den += mail.den[rk];
      const float o = num / den;
      if (a.out) a.out[(hq0 + cr) * kD + d] = o;
      if (a.out16) a.out16[(hq0 + cr) * kD + d] = __half_as_ushort(__float2half_rn(o));
    }
  }
}

// ---------------------------------------------------------------------------
// host side

struct Plan {
  int nsplit, span, nrec;  // base pass (warp splits; one record per CTA of kWarps splits)
  int cl, chunk;           // cluster size and tokens per CTA after the base pass
  size_t off_logits, off_part, total;
};

Plan make_plan(const sf_kv* kv, int t, int h_q, int k_tok, bool need_logits, bool with_pv,
               bool select, int n_splits) {
  (void)k_tok, (void)select;
  Plan P;
  const int sms = num_sms();
  const int heads = kv->batch * kv->h_kv;
  int ns = n_splits > 0 ? n_splits : (16 * sms + heads - 1) / heads;
  int maxs = (t + 15) / 16;
  if (ns > maxs) ns = maxs;
  if (ns < 1) ns = 1;
  P.span = ((t + ns - 1) / ns + 15) / 16 * 16;
  P.nsplit = (t + P.span - 1) / P.span;
  P.nrec = (P.nsplit + kWarps - 1) / kWarps;
  P.cl = kPostCl;
  P.chunk = (t + P.cl - 1) / P.cl;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const int rec = with_pv ? kRec : 2;
  P.off_logits = need_logits ? take((size_t)kv->batch * h_q * t * 4) : 0;
  P.off_part = take((size_t)kv->batch * h_q * P.nrec * rec * 4);
  P.total = off;
  return P;
}

// k_tok of every entry point: at most t, at most kMaxKTok (each of the kPostCl
// CTAs of a head's cluster holds up to kPostMaxSel of the selected tokens), and
// at least 1 unless a base-only call (allow_zero) is meant.
sf_status check_ktok(int k_tok, int t, bool allow_zero) {
  SF_REQUIRE(k_tok >= (allow_zero ? 0 : 1) && k_tok <= t, "k_tok=%d outside [%d, t=%d]", k_tok,
             allow_zero ? 0 : 1, t);
  SF_UNSUPPORTED(k_tok <= kMaxKTok, "k_tok=%d above %d", k_tok, kMaxKTok);
  return SF_OK;
}

sf_status check_q(const sf_kv* kv, int t, const uint16_t* q, int h_q) {
  SF_REQUIRE(t >= 1 && t <= kv->t_max, "t=%d outside [1, t_max=%d]", t, kv->t_max);
  SF_REQUIRE(q && aligned16(q), "q must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(h_q > 0 && h_q % kv->h_kv == 0 && h_q / kv->h_kv <= 8,
                 "h_q=%d must be a multiple of h_kv=%d with at most 8 query heads per KV head", h_q,
                 kv->h_kv);
  SF_UNSUPPORTED(t <= kPostCl * kPostMaxTok, "t=%d above %d", t, kPostCl * kPostMaxTok);
  return SF_OK;
}

template <int GQP, int B, bool PV>
sf_status launch_base_t(const BaseArgs& a, int batch, cudaStream_t s) {
  const size_t smem = kWarps * WarpSmem<B, PV>::bytes;
  auto kern = kv_base_kernel<GQP, B, PV>;
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.nsplit + kWarps - 1) / kWarps, a.h_kv, batch);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;  // launch overlaps the previous kernel's tail
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SF_CUDA(cudaLaunchKernelEx(&cfg, kern, a));
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

// The cluster kernel after the base pass (launched with programmatic
// serialization: its CTAs start while the base pass drains).
sf_status launch_post(const sf_kv* kv, int t, const uint16_t* q, int h_q, int k_tok, const Plan& P,
                      const float* logits, const float* part, int rec, int32_t* sel, int select,
                      float* scores, float* out, cudaStream_t s, uint16_t* out16 = nullptr) {
  PostArgs a;
  a.kb = (const uint8_t*)kv->kb, a.kr = (const uint8_t*)kv->kr;
  a.vb = (const uint8_t*)kv->vb, a.vr = (const uint8_t*)kv->vr;
  a.ksz = kv->ksz, a.vsz = kv->vsz;
  a.h_kv = kv->h_kv, a.t_max = kv->t_max, a.b = kv->b, a.r = kv->r, a.T = t;
  a.q = q, a.h_q = h_q, a.gq = h_q / kv->h_kv;
  a.logits = logits, a.part = part, a.nrec = P.nrec, a.rec = rec;
  a.k_tok = k_tok, a.sel = sel, a.select = select, a.scores = scores, a.out = out, a.out16 = out16;
  a.chunk = P.chunk;
  a.scale = 1.0f / sqrtf((float)kD);
  // the score keys' space, which later holds the per-warp partial numerators
  // of the refined attention [warps][GQP][kD]
  const size_t gqp = a.gq <= 4 ? 4 : 8;
  const size_t key_words = (out || out16) ? std::max((size_t)P.chunk, (size_t)(kPostThreads / 32) * gqp * kD) : (size_t)P.chunk;
  const size_t smem = sizeof(PostMail) + ((size_t)kPostStage * tok_words(kv->b, kv->r) + key_words) * 4;
  void (*kern)(PostArgs);
  if (a.gq <= 4)
    kern = kv->b == 2 ? (kv->r == 2 ? kv_post_kernel<4, 2, 2> : kv_post_kernel<4, 2, 1>)
                      : (kv->r == 2 ? kv_post_kernel<4, 4, 2> : kv_post_kernel<4, 4, 1>);
  else
    kern = kv->b == 2 ? (kv->r == 2 ? kv_post_kernel<8, 2, 2> : kv_post_kernel<8, 2, 1>)
                      : (kv->r == 2 ? kv_post_kernel<8, 4, 2> : kv_post_kernel<8, 4, 1>);
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(PostMail) + ((size_t)kPostStage * tok_words(4, 2) + kPostMaxTok) * 4)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.cl, kv->h_kv, kv->batch);
  cfg.blockDim = dim3(kPostThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P.cl, attr[0].val.clusterDim.y = 1, attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  SF_CUDA(cudaLaunchKernelEx(&cfg, kern, a));
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
  st = check_ktok(k_tok, t, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(sel && aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(!logits || aligned16(logits), "logits must be 16-byte aligned");
  SF_REQUIRE(!scores || aligned16(scores), "scores must be 16-byte aligned");
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, false, true, 0);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  cudaStream_t s = as_stream(stream);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, P);
  st = launch_base(kv, a, false, s);
  if (st != SF_OK) return st;
  return launch_post(kv, t, q, h_q, k_tok, P, lg, part, 2, sel, 1, scores, nullptr, s);
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
  st = check_ktok(k_tok, t, true);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok == 0 || (sel && aligned16(sel)), "sel must be non-null and 16-byte aligned");
  SF_REQUIRE(n_splits >= 0, "n_splits=%d < 0", n_splits);
  SF_REQUIRE(out && aligned16(out), "out must be a non-null 16-byte aligned device pointer");
  Plan P = make_plan(kv, t, h_q, k_tok, true, true, false, n_splits);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  cudaStream_t s = as_stream(stream);
  float* lg = (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  return launch_post(kv, t, q, h_q, k_tok, P, lg, part, kRec, const_cast<int32_t*>(sel), 0, nullptr,
                     out, s);
}

extern "C" size_t sf_kv_attend_selective_workspace_bytes(const sf_kv* kv, int t, int h_q,
                                                         int k_tok, int logits_given) {
  if (!kv || t <= 0 || h_q <= 0 || k_tok <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, !logits_given, true, true, 0).total;
}

namespace sf {
namespace {

// Score, select and attend; the output in fp32 (out) and/or fp16 (out16).
sf_status attend_selective(const sf_kv* kv, int t, const uint16_t* q, int h_q, int k_tok, int32_t* sel,
                           float* logits, float* out, uint16_t* out16, void* ws, size_t ws_bytes,
                           cudaStream_t s) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  st = check_ktok(k_tok, t, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(sel && aligned16(sel), "sel must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(!logits || aligned16(logits), "logits must be 16-byte aligned");
  SF_REQUIRE((out || out16) && (!out || aligned16(out)) && (!out16 || aligned16(out16)),
             "out must be a non-null 16-byte aligned device pointer");
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, true, true, 0);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  return launch_post(kv, t, q, h_q, k_tok, P, lg, part, kRec, sel, 1, nullptr, out, s, out16);
}

}  // namespace
}  // namespace sf

extern "C" sf_status sf_kv_attend_selective(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                            int k_tok, int32_t* sel, float* logits, float* out,
                                            void* ws, size_t ws_bytes, sf_stream_t stream) {
  SF_REQUIRE(out, "out must be a non-null 16-byte aligned device pointer");
  return attend_selective(kv, t, q, h_q, k_tok, sel, logits, out, nullptr, ws, ws_bytes, as_stream(stream));
}

extern "C" sf_status sf_kv_attend_selective_f16(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                                int k_tok, int32_t* sel, float* logits, uint16_t* out,
                                                void* ws, size_t ws_bytes, sf_stream_t stream) {
  SF_REQUIRE(out, "out must be a non-null 16-byte aligned device pointer");
  return attend_selective(kv, t, q, h_q, k_tok, sel, logits, nullptr, out, ws, ws_bytes, as_stream(stream));
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
  st = check_ktok(k_tok, t, false);
  if (st != SF_OK) return st;
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
