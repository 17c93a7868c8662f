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
//   kv_score_kernel, kv_pick_kernel  score every token (sum over the group's
//                   query heads of the softmax probability, from the stored
//                   logits and the statistics of the partials) and select the
//                   top k_tok per KV head: a histogram of the score bits, the
//                   boundary bucket, and in the head's last CTA the exact
//                   k_tok-th score and the selected tokens in ascending order;
//   kv_refine_kernel  swaps the selected tokens' base contributions for
//                   their refined ones (relative to the head's softmax
//                   maximum) and merges the partials by log-sum-exp.
// The result equals softmax(q.k~) v~ with refined k~, v~ on the selected
// tokens, up to fp32 rounding.

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
constexpr int kCtlWords = 2048 + 32;  // per head: selection histogram, two counters, statistics (kCtl below)

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

// 3-bit codes are two planes: the low two bits in a 2-bit pair-slot word, the
// high bit in a 1-bit pair-slot word (16 slots; slot j at bits j and 16 + j).
// The high-bit word is kept as given, shifted left by 3 and right by 6, so that
// every slot's bit sits at an offset bh in [3, 9].
struct HiWord {
  uint32_t w, l3, r6;
  __device__ __forceinline__ void set(uint32_t x) {
    w = x;
    l3 = x << 3;
    r6 = x >> 6;
  }
};

// Pair p of 3-bit codes as an exact half2 of centred codes c - 3.5: low bits
// from slot p % 8 of lo[p / 8], high bit from slot p % 16 of hi[p / 16].
// The low pair is placed at b2 as in pair_at<2> and rescaled with an offset
// that also removes 4096 * 2^-bh; the second fused multiply-add adds the high
// pair, 1024 + hi 2^bh, times 4 * 2^-bh.  Every intermediate is a multiple of
// 0.5 below 1024 in magnitude, so both steps are exact in fp16.
template <int NL, int NH>
__device__ __forceinline__ uint32_t pair3_of(const Words<2> (&lo)[NL], const HiWord (&hi)[NH], int p) {
  const Words<2>& x = lo[p / 8];
  const int bit = 2 * (p % 8);
  const bool left = bit < 2, right = !left && bit + 2 > 10;
  const int b2 = left ? bit + 2 : right ? bit - 8 : bit;
  const uint32_t src = left ? x.l2 : right ? x.r : x.w;
  const uint32_t vl = (src & ((3u << b2) * 0x00010001u)) | 0x64006400u;  // 1024 + lo 2^b2 per half
  const HiWord& y = hi[p / 16];
  const int hb = p % 16;
  const int bh = hb < 3 ? hb + 3 : hb < 10 ? hb : hb - 6;
  const uint32_t hsrc = hb < 3 ? y.l3 : hb < 10 ? y.w : y.r6;
  const uint32_t vh = (hsrc & ((1u << bh) * 0x00010001u)) | 0x64006400u;  // 1024 + hi 2^bh per half
  // offset -(1024 2^-b2 + 4096 2^-bh + 3.5) = -n / 2 with n < 2048 an integer:
  // fp16 exponent field e + 14 and mantissa (n - 2^e) 2^(10-e), e = floor(log2 n)
  const uint32_t n = (2048u >> b2) + (8192u >> bh) + 7u;
  const int e = 31 - __clz(n);
  const uint32_t off = (0x8000u | ((uint32_t)(e + 14) << 10) | ((n - (1u << e)) << (10 - e))) * 0x00010001u;
  const uint32_t sc = (uint32_t)((15 - b2) << 10) * 0x00010001u;  // 2^-b2
  const uint32_t sh = (uint32_t)((17 - bh) << 10) * 0x00010001u;  // 4 * 2^-bh
  __half2 c = __hfma2(*reinterpret_cast<const __half2*>(&vl), *reinterpret_cast<const __half2*>(&sc),
                      *reinterpret_cast<const __half2*>(&off));
  c = __hfma2(*reinterpret_cast<const __half2*>(&vh), *reinterpret_cast<const __half2*>(&sh), c);
  return *reinterpret_cast<uint32_t*>(&c);
}

// The code words of one chunk of PAIRS pairs (a key token's chunk: 16; a value
// tile's chunk: 32) in registers, B-bit codes.  load() takes the chunk's words
// in the w = B layout (B = 3: its 2-bit plane words, and its 1-bit plane words
// in hi).
template <int B, int PAIRS>
struct ChunkCodes {
  static constexpr int NW = PAIRS * B / 16;
  Words<B> w[NW];
  __device__ __forceinline__ void load(const uint32_t* lo, const uint32_t*) {
#pragma unroll
    for (int i = 0; i < NW; i++) w[i].set(lo[i]);
  }
  __device__ __forceinline__ uint32_t pair(int p) const { return pair_of<B>(w, p); }
};

template <int PAIRS>
struct ChunkCodes<3, PAIRS> {
  static constexpr int NL = PAIRS / 8, NH = PAIRS / 16;
  Words<2> lo[NL];
  HiWord hi[NH];
  __device__ __forceinline__ void load(const uint32_t* l, const uint32_t* h) {
#pragma unroll
    for (int i = 0; i < NL; i++) lo[i].set(l[i]);
#pragma unroll
    for (int i = 0; i < NH; i++) hi[i].set(h[i]);
  }
  __device__ __forceinline__ uint32_t pair(int p) const { return pair3_of(lo, hi, p); }
};

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
  int* ctl;       // [batch][h_kv][kCtl]: zeroed here for the kernels after the base pass
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

// GQP: query heads per KV head padded to 4 or 8.  B: base bits (2, 3 or 4).
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
  if (blockIdx.x == 0 && a.ctl) {  // the histogram and counters of the kernels after this one
    int* c = a.ctl + ((long)bat * a.h_kv + g) * kCtlWords;
    for (int i = threadIdx.x; i < kCtlWords; i += blockDim.x) c[i] = 0;
  }
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
      for (int c = 0; c < (B + 1) / 2; c++) {  // 16 B chunks of 16 tokens' keys (and the value tile)
        const int ci = lane + 32 * c;
        if (ci < 16 * B) {
          cp_async16(st + 16 * ci, a.kb + slot * 16 * B + 16 * ci);
          if (PV) cp_async16(st + St::kBytes + 16 * ci, a.vb + (slot / 16) * 256 * B + 16 * ci);
        }
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
      // chunk tig of tokens gid and gid + 8 (3-bit codes: 2-bit plane words
      // 2 tig, 2 tig + 1 and 1-bit plane word 8 + tig of the token)
      const uint32_t* kc = reinterpret_cast<const uint32_t*>(st);
      constexpr int LW = B == 3 ? 2 : B;
      ChunkCodes<B, 16> w0, w8;
      w0.load(kc + gid * 4 * B + tig * LW, kc + gid * 4 * B + 8 + tig);
      w8.load(kc + (gid + 8) * 4 * B + tig * LW, kc + (gid + 8) * 4 * B + 8 + tig);
#pragma unroll
      for (int s = 0; s < 8; s++) {
        uint32_t a0 = w0.pair(2 * s), a1 = w8.pair(2 * s);
        uint32_t a2 = w0.pair(2 * s + 1), a3 = w8.pair(2 * s + 1);
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
      // chunk `lane` of the value tile (3-bit codes: 2-bit plane words 4 lane ..
      // 4 lane + 3, 1-bit plane words 128 + 2 lane, 128 + 2 lane + 1)
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + St::kBytes);
      ChunkCodes<B, 32> vw;
      vw.load(vc + lane * 2 * (B == 3 ? 2 : B), vc + 128 + 2 * lane);
      // Each tile's product starts from zero and is folded into the running
      // sum with one fp32 FMA that also applies the softmax rescale: long
      // accumulation chains inside the tensor-core accumulator would drift.
#pragma unroll
      for (int m = 0; m < 8; m++) {
        uint32_t a0 = vw.pair(2 * m), a1 = vw.pair(2 * m + 1);
        uint32_t a2 = vw.pair(16 + 2 * m), a3 = vw.pair(17 + 2 * m);
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
// after the base pass: scoring and selection, then refinement and merge
//
// kv_score_kernel -- CTAs of kSelThreads threads over slices of kSelTok
// tokens of one (batch, KV head).  Each computes the softmax statistics of the
// group's query heads from the base pass's split records, the scores of its
// tokens from the stored logits (written out: the sum over the group's query
// heads of each head's softmax probability), and the histogram of the score
// keys' bits 30..20, added into the head's histogram in the workspace.  Scores
// are non-negative, so their bit patterns order like their values; bits 30..20
// are the exponent and the top three mantissa bits.
//
// kv_pick_kernel -- the same CTAs again: each finds, from the complete
// histogram, the bucket that holds the k_tok-th largest key, writes the bitmap
// words of its tokens in higher buckets and appends its boundary-bucket
// (key, token) pairs to the head's list.  The last CTA of the head to finish
// (an atomic counter: no CTA ever waits for another) loads the bitmap and the
// list, pins the k_tok-th largest key K* with two 10-bit digits over the list,
// marks the tokens above K* and the lowest-indexed ones equal to it, and
// writes the marked tokens in ascending order.
//
// kv_refine_kernel -- kRefParts CTAs per (batch, KV head), each with a share
// of the selected tokens and of the base pass's split records.  Per selected
// token a warp reads its base and refinement codes and scales, swaps the
// token's base contribution for its refined one (weights relative to the
// head's softmax maximum: numerator v~ exp(l~ - M) - v^ exp(l^ - M), the
// denominator likewise), and adds the CTA's records rescaled to M; the last
// CTA of the head to finish divides the summed numerators by the summed
// denominators.

constexpr int kSelThreads = 512;
constexpr size_t kSpreadSmem = 120 * 1024;  // more than half an SM's shared memory
constexpr int kSelTok = 2048;        // tokens scored per CTA
constexpr int kBins1 = 2048;         // first digit: key bits 30..20
constexpr int kBins2 = 1024;         // then bits 19..10 and 9..0
constexpr int kCandCap = 4096;       // boundary-bucket keys held in shared memory
constexpr int kTieCap = 2048;        // tokens equal to the k-th key ranked in shared memory
constexpr int kMaxT = 1 << 18;       // tokens a head's bitmap holds in shared memory
// per head: histogram, selection counter, refinement counter, a flag, then
// (M, Z) of each of the group's query heads (up to 8), written by the selection
constexpr int kCtl = kBins1 + 32;
constexpr int kCtlStats = kBins1 + 4;
static_assert(kCtl == kCtlWords, "the base pass zeroes exactly the control words");
constexpr int kRefThreads = 256;
constexpr int kRefWarps = kRefThreads / 32;
constexpr int kRefTPW = 4;           // tokens a warp refines together
constexpr int kRefPartsMax = 16;     // CTAs per head that refine
constexpr int kMaxKTok = 4096;       // the largest k_tok every attention entry point accepts
static_assert(kRefTPW * 8 <= 32, "a warp's (token, head) slots must fit its lanes");

// Softmax statistics of query head h from the split records: M = max m,
// Z = sum l exp(m - M), in one pass (online rescaling).  One warp.
__device__ __forceinline__ void head_stats(const float* __restrict__ pr, int nrec, int rec, int lane, float& M,
                                           float& Z) {
  float m = -INFINITY, z = 0.f;
  for (int s = lane; s < nrec; s += 32) {
    const float ms = pr[(long)s * rec + rec - 2], ls = pr[(long)s * rec + rec - 1];
    if (ms > -INFINITY) {
      const float mn = fmaxf(m, ms);
      z = z * expf(m - mn) + ls * expf(ms - mn);
      m = mn;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o), zo = __shfl_xor_sync(0xffffffffu, z, o);
    const float mn = fmaxf(m, mo);
    z = (m > -INFINITY ? z * expf(m - mn) : 0.f) + (mo > -INFINITY ? zo * expf(mo - mn) : 0.f);
    m = mn;
  }
  M = m, Z = z;
}

// Exclusive prefix sum of v over the block's threads (in thread order), and the
// total.  ws: 32 ints of shared memory.
template <int NT>
__device__ __forceinline__ int block_exclusive_sum(int v, int* ws, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  __syncthreads();  // ws may still be read by a previous call
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < NT / 32 ? ws[lane] : 0;
    int x = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    if (lane < NT / 32) ws[lane] = x - wv;
    if (lane == 31) ws[NT / 32] = x;
  }
  __syncthreads();
  total = ws[NT / 32];
  return ws[warp] + incl - v;
}

// The bucket of the kneed-th largest key: hist[0, nb) counts keys per digit;
// bucket b is taken when the keys of higher buckets number fewer than kneed
// and those at or above it kneed or more.  Returns b; *kleft = kneed minus the
// keys above b.  Every thread gets the result.
template <int NT>
__device__ int find_bucket(const int* __restrict__ hist, int nb, int kneed, int* ws, int* res, int* kleft) {
  const int per = nb / NT;  // 2 or 4 bins per thread, from the top
  int c[4], tot = 0;
#pragma unroll
  for (int j = 0; j < 4; j++) {
    c[j] = j < per ? hist[nb - 1 - per * (int)threadIdx.x - j] : 0;
    tot += c[j];
  }
  int all;
  const int above = block_exclusive_sum<NT>(tot, ws, all);
  if (above < kneed && above + tot >= kneed) {
    int run = above;
    for (int j = 0; j < per; j++) {
      if (run + c[j] >= kneed) {
        res[0] = nb - 1 - per * (int)threadIdx.x - j;
        res[1] = kneed - run;
        break;
      }
      run += c[j];
    }
  }
  __syncthreads();
  *kleft = res[1];
  return res[0];
}

// Add 1 to hist[bin] for every lane with bin >= 0; lanes with equal bins add
// once, by their count (scores often share a bucket: one same-address atomic
// per lane would serialise).  Whole warps only.
__device__ __forceinline__ void hist_add(int* hist, int bin) {
  const unsigned same = __match_any_sync(0xffffffffu, bin);
  if (bin >= 0 && (__ffs(same) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], __popc(same));
}

struct SelArgs {
  const float* logits;  // [batch][h_q][T] base logits (scaled)
  const float* part;    // [batch][h_q][nrec][rec]
  int nrec, rec;
  int h_kv, h_q, gq, T, Tp, k_tok, nblk;
  float* scores;        // [batch][h_kv][Tp] (Tp = T rounded up to 32: whole 16-byte rows)
  float* scores_out;    // nullable [batch][h_kv][T]: the scores for the caller
  int* ctl;             // [batch][h_kv][kCtl]
  uint32_t* bitmap;     // [batch][h_kv][Tp / 32]: tokens of the buckets above the boundary
  uint2* cand;          // [batch][h_kv][kCandCap]: (key, token) of the boundary bucket
  int32_t* sel;         // [batch][h_kv][k_tok]
};

struct SelShared {
  int hist[kBins1];
  int ws[40];
  int res[2];
  int ncand, last;
  float M[8], iZ[8];
  uint32_t words[kSelTok / 32];
};

// kv_score_kernel: the statistics, the scores of the CTA's tokens and their
// histogram, added into the head's histogram.
template <int GQP>
__global__ void __launch_bounds__(kSelThreads) kv_score_kernel(SelArgs a) {
  __shared__ SelShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.y, bat = blockIdx.z, gq = a.gq;
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  const long head = (long)bat * a.h_kv + g;
  pdl_trigger();
  pdl_wait();  // the base pass (logits, records, zeroed histogram) is complete
  // the CTA's logits are loaded first: their latency overlaps the statistics
  const int t0 = blockIdx.x * kSelTok, t1 = min(a.T, t0 + kSelTok);
  constexpr int U = kSelTok / kSelThreads;
  float l[GQP][U];
  {
    const float* lg = a.logits + hq0 * a.T;
#pragma unroll
    for (int h = 0; h < GQP; h++)
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int t = t0 + tid + kSelThreads * u;
        l[h][u] = (h < gq && t < t1) ? lg[(long)h * a.T + t] : -INFINITY;
      }
  }
  if (warp < gq) {
    float M, Z;
    head_stats(a.part + (hq0 + warp) * a.nrec * a.rec, a.nrec, a.rec, lane, M, Z);
    if (lane == 0) {
      sh.M[warp] = M, sh.iZ[warp] = 1.0f / Z;
      if (blockIdx.x == 0) {  // for the refinement after it
        float* st = reinterpret_cast<float*>(a.ctl + head * kCtl + kCtlStats);
        st[2 * warp] = M, st[2 * warp + 1] = Z;
      }
    }
  }
  for (int i = tid; i < kBins1; i += kSelThreads) sh.hist[i] = 0;
  __syncthreads();
  float* sc = a.scores + head * a.Tp;
  float* sco = a.scores_out ? a.scores_out + head * a.T : nullptr;
  {
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int t = t0 + tid + kSelThreads * u;
      int bin = -1;
      if (t < t1) {
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < GQP; h++)
          if (h < gq) s += expf(l[h][u] - sh.M[h]) * sh.iZ[h];  // full-accuracy exp: the score decides
        sc[t] = s;
        if (sco) sco[t] = s;
        bin = (int)(__float_as_uint(s) >> 20);
      }
      // one shared atomic per token: cheaper here than aggregating equal bins
      // over the warp first (measured)
      if (bin >= 0) atomicAdd(&sh.hist[bin], 1);
    }
  }
  __syncthreads();
  int* gh = a.ctl + head * kCtl;
  for (int i = tid; i < kBins1; i += kSelThreads)
    if (sh.hist[i]) atomicAdd(&gh[i], sh.hist[i]);
}

// Dynamic shared memory of a pick CTA: the bitmap of selected tokens, the
// boundary bucket's keys and tokens, the tied tokens.
constexpr size_t kSelDyn = (size_t)(kMaxT / 32) * 4 + (size_t)kCandCap * 8 + (size_t)kTieCap * 4;

// kv_pick_kernel: every CTA finds the bucket of the k_tok-th largest key from
// the head's complete histogram, writes its tokens' bitmap words (tokens of
// higher buckets) and appends its boundary-bucket tokens to the head's
// candidate list; the head's last CTA pins the k_tok-th key among the
// candidates, marks them and the lowest tied tokens, and writes the selection
// in ascending order.
__global__ void __launch_bounds__(kSelThreads) kv_pick_kernel(SelArgs a) {
  __shared__ SelShared sh;
  extern __shared__ __align__(16) uint32_t dyn_sel[];
  uint32_t* bits = dyn_sel;                                    // [kMaxT / 32]
  uint32_t* ck = bits + kMaxT / 32;                            // [kCandCap] keys
  int* ct = reinterpret_cast<int*>(ck + kCandCap);             // [kCandCap] tokens
  int* tie_t = ct + kCandCap;                                  // [kTieCap]
  const int tid = threadIdx.x, lane = tid & 31;
  const int g = blockIdx.y, bat = blockIdx.z;
  const long head = (long)bat * a.h_kv + g;
  pdl_trigger();
  pdl_wait();  // every score and the complete histogram
  const int T = a.T;
  const float* sc = a.scores + head * a.Tp;
  // the CTA's scores (four consecutive tokens per thread) are loaded first:
  // their latency overlaps the histogram's load and the bucket search
  const int t0 = blockIdx.x * kSelTok + 4 * tid;
  uint32_t key[4] = {0u, 0u, 0u, 0u};
  if (t0 + 4 <= a.Tp) {
    const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + t0));
    key[0] = __float_as_uint(f.x), key[1] = __float_as_uint(f.y);
    key[2] = __float_as_uint(f.z), key[3] = __float_as_uint(f.w);
  }
  int* gh = a.ctl + head * kCtl;
  for (int i = tid; i < kBins1; i += kSelThreads) sh.hist[i] = __ldcg(gh + i);
  if (tid < kSelTok / 32) sh.words[tid] = 0u;
  __syncthreads();
  int kneed;
  const uint32_t b1 = (uint32_t)find_bucket<kSelThreads>(sh.hist, kBins1, a.k_tok, sh.ws, sh.res, &kneed);
  uint2* cl = a.cand + head * kCandCap;
  int* ncand_g = gh + kBins1 + 3;
  {
    uint32_t m = 0;
    int nc = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const bool in = t0 + i < T;
      const uint32_t d = key[i] >> 20;
      if (in && d > b1) m |= 1u << i;
      nc += in && d == b1;
    }
    if (m) atomicOr(&sh.words[(4 * tid) >> 5], m << ((4 * tid) & 31));
    // boundary-bucket tokens into the head's list: one atomic per warp
    int incl = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    int base = 0;
    if (lane == 31 && incl) base = atomicAdd(ncand_g, incl);
    base = __shfl_sync(0xffffffffu, base, 31) + incl - nc;
#pragma unroll
    for (int i = 0; i < 4; i++)
      if (t0 + i < T && (key[i] >> 20) == b1) {
        if (base < kCandCap) cl[base] = make_uint2(key[i], (uint32_t)(t0 + i));
        base++;
      }
  }
  __syncthreads();
  {
    const int w0 = blockIdx.x * (kSelTok / 32), nw = (T + 31) / 32;
    if (tid < kSelTok / 32 && w0 + tid < nw) a.bitmap[head * (a.Tp / 32) + w0 + tid] = sh.words[tid];
  }
  __threadfence();  // this CTA's words and candidates before its count
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(gh + kBins1 + 2, 1) == a.nblk - 1;
  __syncthreads();
  if (!sh.last) return;
  __threadfence();  // every other CTA's words and candidates are visible

  // ---- the head's last CTA
  const int nw = (T + 31) / 32;
  const int wper = (nw + kSelThreads - 1) / kSelThreads;
  const int w0 = min(nw, tid * wper), w1 = min(nw, w0 + wper);
  for (int w = tid; w < nw; w += kSelThreads) bits[w] = __ldcg(a.bitmap + head * (a.Tp / 32) + w);
  const int ncand = __ldcg(ncand_g);
  const bool in_smem = ncand <= kCandCap;
  if (in_smem)
    for (int j = tid; j < ncand; j += kSelThreads) {
      const uint2 e = __ldcg(cl + j);
      ck[j] = e.x, ct[j] = (int)e.y;
    }
  __syncthreads();
  // f(valid, key, token) on whole warps (lanes past the end pass valid = false)
  auto for_cands = [&](auto&& f) {
    if (in_smem) {
      for (int j0 = tid - lane; j0 < ncand; j0 += kSelThreads) {
        const int j = j0 + lane;
        const bool v = j < ncand;
        f(v, v ? ck[j] : 0u, v ? ct[j] : 0);
      }
    } else {
      for (int t0 = tid - lane; t0 < T; t0 += kSelThreads) {
        const int t = t0 + lane;
        const uint32_t key = t < T ? __float_as_uint(__ldcg(sc + t)) : 0u;
        f(t < T && (key >> 20) == b1, key, t);
      }
    }
  };
  uint32_t prefix = b1 << 20, mask = 0xFFF00000u;
#pragma unroll 1
  for (int shift = 10; shift >= 0; shift -= 10) {
    for (int i = tid; i < kBins2; i += kSelThreads) sh.hist[i] = 0;
    __syncthreads();
    for_cands([&](bool v, uint32_t key, int t) {
      (void)t;
      hist_add(sh.hist, v && (key & mask) == prefix ? (int)((key >> shift) & (kBins2 - 1)) : -1);
    });
    __syncthreads();
    int kl;
    const uint32_t d = (uint32_t)find_bucket<kSelThreads>(sh.hist, kBins2, kneed, sh.ws, sh.res, &kl);
    kneed = kl;
    prefix |= d << shift;
    mask |= (uint32_t)(kBins2 - 1) << shift;
  }
  // prefix is the k_tok-th largest key K*; kneed of the keys equal to it are
  // taken, the lowest tokens first
  if (tid == 0) sh.res[0] = 0;
  __syncthreads();
  for_cands([&](bool v, uint32_t key, int t) {
    if (v && key > prefix) atomicOr(&bits[t >> 5], 1u << (t & 31));
    const bool eq = v && key == prefix;
    const unsigned m = __ballot_sync(0xffffffffu, eq);
    if (m) {  // one atomic per warp
      int base = 0;
      if (lane == __ffs(m) - 1) base = atomicAdd(&sh.res[0], __popc(m));
      base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
      const int slot = base + __popc(m & ((1u << lane) - 1u));
      if (eq && slot < kTieCap) tie_t[slot] = t;
    }
  });
  __syncthreads();
  const int nties = sh.res[0];
  if (nties <= kTieCap) {
    // a tie is taken when fewer than kneed tied tokens lie below it
    for (int i = tid; i < nties; i += kSelThreads) {
      const int t = tie_t[i];
      int below = 0;
      for (int k2 = 0; k2 < nties; k2++) below += tie_t[k2] < t;
      if (below < kneed) atomicOr(&bits[t >> 5], 1u << (t & 31));
    }
  } else {
    // many equal keys: per-thread counts of its own tied tokens, then each
    // thread marks the first ones of its range that the budget still allows
    int mine = 0;
    for (int w = w0; w < w1; w++)
      for (int i = 32 * w; i < min(T, 32 * w + 32); i++) mine += __float_as_uint(__ldcg(sc + i)) == prefix;
    int ties_all;
    const int ties_before = block_exclusive_sum<kSelThreads>(mine, sh.ws, ties_all);
    int take = max(0, min(mine, kneed - ties_before));
    for (int w = w0; w < w1 && take > 0; w++) {
      uint32_t m = bits[w];
      for (int i = 0; i < 32 && take > 0; i++) {
        const int t = 32 * w + i;
        if (t < T && __float_as_uint(__ldcg(sc + t)) == prefix) m |= 1u << i, take--;
      }
      bits[w] = m;
    }
  }
  __syncthreads();
  int cnt = 0;
  for (int w = w0; w < w1; w++) cnt += __popc(bits[w]);
  int total;
  int pos = block_exclusive_sum<kSelThreads>(cnt, sh.ws, total);
  int32_t* out = a.sel + head * a.k_tok;
  for (int w = w0; w < w1; w++) {
    uint32_t m = bits[w];
    while (m) {
      const int i = __ffs(m) - 1;
      m &= m - 1;
      if (pos < a.k_tok) out[pos] = 32 * w + i;
      pos++;
    }
  }
}

struct RefArgs {
  const uint8_t *kb, *kr, *vb, *vr;
  const uint16_t *ksz, *vsz;
  int h_kv, t_max, T;
  const uint16_t* q;
  int h_q, gq;
  const float* logits;  // base logits (scaled), [batch][h_q][T]
  const float* part;    // [batch][h_q][nrec][kRec]
  int nrec;
  int k_tok, parts;
  int stats_given;      // the selection left (M, Z) in the control words
  const int32_t* sel;   // [batch][h_kv][k_tok]
  int* ctl;             // [batch][h_kv][kCtl]
  float* rpart;         // [batch][h_kv][parts][gq][kD + 1]
  float* out;           // nullable [batch][h_q][kD]
  uint16_t* out16;      // nullable [batch][h_q][kD]
  float scale;
};

template <int GQP>
struct RefShared {
  float M[8], Z[8];
  float num[kRefWarps][GQP][kD];
  float den[kRefWarps][GQP];
  float2 wtab[kRefWarps][kRefTPW * GQP];
  int last;
};

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

// Per-lane constants of the refinement: the lane owns head dims lane + 32 e
// (scale group e): their word and bit in a token's key codes and refinements,
// and the query values of the group's heads there.
template <int GQP, int B, int R>
struct RefLane {
  // 3-bit codes: (kw, kbit) in the 2-bit plane, (khw, khbit) in the 1-bit plane
  int kw[4], kbit[4], khw[4], khbit[4], krw[4], krbit[4];
  float qv[GQP][4];
  __device__ __forceinline__ void init(const RefArgs& a, long hq0, int lane) {
#pragma unroll
    for (int e = 0; e < 4; e++) {
      key_pos(lane + 32 * e, B == 3 ? 2 : B, kw[e], kbit[e]);
      key_pos(lane + 32 * e, 1, khw[e], khbit[e]);
      khw[e] += 8;
      key_pos(lane + 32 * e, R, krw[e], krbit[e]);
#pragma unroll
      for (int h = 0; h < GQP; h++) qv[h][e] = h < a.gq ? h2f(a.q[(hq0 + h) * kD + lane + 32 * e]) : 0.f;
    }
  }
};

// One warp swaps the base contributions of up to kRefTPW tokens (tok[m] < 0:
// none) for their refined ones: adds v~ exp(l~ - M) - v^ exp(l^ - M) into
// an[h][e] (head h, dim lane + 32 e) and exp(l~ - M) - exp(l^ - M) of the
// lane's (token, head) slot into ad_own.  wtab: the warp's kRefTPW * GQP
// float2 of shared memory.
template <int GQP, int B, int R>
__device__ __forceinline__ void refine_batch(const RefArgs& a, const RefLane<GQP, B, R>& rl, const float* M,
                                             long slot0, long hq0, const int (&tok)[kRefTPW], int lane,
                                             float (&an)[GQP][4], float& ad_own, float2* wtab) {
  const float half = 0.5f * (float)(1 << R), inv = 1.0f / (float)(1 << R);
  const uint32_t bmask = (1u << B) - 1u, rmask = (1u << R) - 1u;
  const int u_own = lane % (kRefTPW * GQP), m_own = u_own / GQP, h_own = u_own % GQP;
  // every load of the warp's tokens first
  uint32_t wk[kRefTPW][4], wkr[kRefTPW][4], wv[kRefTPW][4], wvr[kRefTPW][4], zk[kRefTPW][4], zv[kRefTPW][4];
#pragma unroll
  for (int m = 0; m < kRefTPW; m++) {
    const int t = tok[m] < 0 ? 0 : tok[m];
    const long slot = slot0 + t, tile = slot / 16;
    const uint32_t* kp = reinterpret_cast<const uint32_t*>(a.kb + slot * 16 * B);
    const uint32_t* krp = reinterpret_cast<const uint32_t*>(a.kr + slot * 16 * R);
    const uint32_t* vp = reinterpret_cast<const uint32_t*>(a.vb + tile * 256 * B);
    const uint32_t* vrp = reinterpret_cast<const uint32_t*>(a.vr + tile * 256 * R);
    const uint32_t* zkp = reinterpret_cast<const uint32_t*>(a.ksz) + slot * 4;
    const uint32_t* zvp = reinterpret_cast<const uint32_t*>(a.vsz) + slot * 4;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int d = lane + 32 * e;
      int vrw, vrbit;
      value_pos(t & 15, d, R, vrw, vrbit);
      if constexpr (B == 3)
        wk[m][e] = ((kp[rl.kw[e]] >> rl.kbit[e]) & 3u) | (((kp[rl.khw[e]] >> rl.khbit[e]) & 1u) << 2);
      else
        wk[m][e] = (kp[rl.kw[e]] >> rl.kbit[e]) & bmask;
      wkr[m][e] = (krp[rl.krw[e]] >> rl.krbit[e]) & rmask;
      wv[m][e] = value_code(vp, t & 15, d, B);
      wvr[m][e] = (vrp[vrw] >> vrbit) & rmask;
      zk[m][e] = zkp[e];
      zv[m][e] = zvp[e];
    }
  }
  int tok_own = tok[0];
#pragma unroll
  for (int m = 1; m < kRefTPW; m++)
    if (m == m_own) tok_own = tok[m];
  float wbl = 0.f;
  const bool own_ok = h_own < a.gq && tok_own >= 0;
  if (own_ok) wbl = expf(a.logits[(hq0 + h_own) * a.T + tok_own] - M[h_own]);
  float kf[kRefTPW][4], vbs[kRefTPW][4], vfs[kRefTPW][4];
#pragma unroll
  for (int m = 0; m < kRefTPW; m++) {
    const bool ok = tok[m] >= 0;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float2 k2 = __half22float2(*reinterpret_cast<const __half2*>(&zk[m][e]));
      const float2 v2 = __half22float2(*reinterpret_cast<const __half2*>(&zv[m][e]));
      kf[m][e] = fmaf(k2.x, (float)wk[m][e] + ((float)wkr[m][e] + 0.5f - half) * inv, k2.y);
      vbs[m][e] = ok ? fmaf(v2.x, (float)wv[m][e], v2.y) : 0.f;
      vfs[m][e] = ok ? fmaf(v2.x, (float)wv[m][e] + ((float)wvr[m][e] + 0.5f - half) * inv, v2.y) : 0.f;
    }
  }
  // refined logits of the TPW x GQP (token, head) slots
  float lg[kRefTPW * GQP];
#pragma unroll
  for (int m = 0; m < kRefTPW; m++)
#pragma unroll
    for (int h = 0; h < GQP; h++) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; e++) acc = fmaf(rl.qv[h][e], kf[m][e], acc);
      lg[m * GQP + h] = acc;
    }
  const float lg_own = warp_transpose_sum<kRefTPW * GQP>(lg, lane);
  float wfl = 0.f;
  if (own_ok) wfl = expf(lg_own * a.scale - M[h_own]);
  if (lane < kRefTPW * GQP) wtab[lane] = make_float2(wfl, wbl);
  ad_own += wfl - wbl;
  __syncwarp();
#pragma unroll
  for (int m = 0; m < kRefTPW; m++)
#pragma unroll
    for (int h = 0; h < GQP; h++) {
      const float2 w = wtab[m * GQP + h];
#pragma unroll
      for (int e = 0; e < 4; e++) an[h][e] = fmaf(w.x, vfs[m][e], fmaf(-w.y, vbs[m][e], an[h][e]));
    }
  __syncwarp();
}

// The share s = part, part + parts, ... of the base pass's split records of
// the group's heads, rescaled to M: num[(h, d)] for the (h, d) pairs e =
// tid, tid + nthreads, ... (at most 4 per thread), every load issued first.
template <int GQP>
__device__ __forceinline__ void record_share(const RefArgs& a, long hq0, const float* M, int part, int parts,
                                             int tid, int nthreads, float (&num)[4]) {
  constexpr int PER = 8;
#pragma unroll
  for (int i = 0; i < 4; i++) num[i] = 0.f;
  for (int s0 = part; s0 < a.nrec; s0 += parts * PER) {
    float mv[4][PER], av[4][PER];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int e = tid + i * nthreads, h = e / kD, d = e % kD;
      const float* pr = a.part + (hq0 + (h < a.gq ? h : 0)) * a.nrec * kRec;
#pragma unroll
      for (int k = 0; k < PER; k++) {
        const int sidx = s0 + parts * k;
        const bool ok = e < a.gq * kD && sidx < a.nrec;
        mv[i][k] = ok ? pr[(long)sidx * kRec + kD] : -INFINITY;
        av[i][k] = ok ? pr[(long)sidx * kRec + d] : 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int e = tid + i * nthreads, h = (e / kD) < a.gq ? e / kD : 0;
#pragma unroll
      for (int k = 0; k < PER; k++)
        if (mv[i][k] > -INFINITY) num[i] = fmaf(expf(mv[i][k] - M[h]), av[i][k], num[i]);
    }
  }
}

// The head's output from every CTA's partial: out[h] = sum of the parts'
// numerators (+ extra) / (Z + sum of their denominators (+ extra_den)).
template <int NT>
__device__ __forceinline__ void merge_parts(const RefArgs& a, long hq0, long head, const float* Z, int parts,
                                            const float* extra_num, const float* extra_den) {
  const int gq = a.gq;
  const float* rh = a.rpart + head * a.parts * gq * (kD + 1);
  for (int e = threadIdx.x; e < gq * kD; e += NT) {
    const int h = e / kD, d = e % kD;
    float nv[kRefPartsMax], dv[kRefPartsMax];  // every part's load in flight together
    float num = extra_num ? extra_num[e] : 0.f, den = Z[h] + (extra_den ? extra_den[h] : 0.f);
    for (int p0 = 0; p0 < parts; p0 += kRefPartsMax) {
#pragma unroll
      for (int k = 0; k < kRefPartsMax; k++) {
        const int p = p0 + k;
        nv[k] = p < parts ? __ldcg(rh + (p * gq + h) * (kD + 1) + d) : 0.f;
        dv[k] = p < parts ? __ldcg(rh + (p * gq + h) * (kD + 1) + kD) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kRefPartsMax; k++) num += nv[k], den += dv[k];
    }
    const float o = num / den;
    if (a.out) a.out[(hq0 + h) * kD + d] = o;
    if (a.out16) a.out16[(hq0 + h) * kD + d] = __half_as_ushort(__float2half_rn(o));
  }
}

// The CTA's partial (its warps' numerators in num_w [warps][GQP][kD], their
// denominators in den_w [warps][GQP], plus its record share rec[i] for pairs
// tid + i NT) into the head's slot `part` of the workspace.
template <int GQP, int NT>
__device__ __forceinline__ void write_part(const RefArgs& a, long head, int part, const float* num_w,
                                           const float* den_w, const float (&rec)[4]) {
  constexpr int NW = NT / 32;
  float* rp = a.rpart + (head * a.parts + part) * a.gq * (kD + 1);
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int e = threadIdx.x + i * NT;
    if (e < a.gq * kD) {
      const int h = e / kD, d = e % kD;
      float num = rec[i];
      for (int w = 0; w < NW; w++) num += num_w[(w * GQP + h) * kD + d];
      rp[h * (kD + 1) + d] = num;
    }
  }
  if ((int)threadIdx.x < a.gq) {
    float den = 0.f;
    for (int w = 0; w < NW; w++) den += den_w[w * GQP + threadIdx.x];
    rp[threadIdx.x * (kD + 1) + kD] = den;
  }
}

// A warp's numerators and denominator changes into shared memory.
template <int GQP>
__device__ __forceinline__ void stash_warp(float (&an)[GQP][4], float ad_own, int warp, int lane, float* num_w,
                                           float* den_w) {
#pragma unroll
  for (int h = 0; h < GQP; h++)
#pragma unroll
    for (int e = 0; e < 4; e++) num_w[(warp * GQP + h) * kD + lane + 32 * e] = an[h][e];
  // slot u's denominator change sits in lanes u, u + TPW GQP, ...: sum each head's
  float dsum = lane < kRefTPW * GQP ? ad_own : 0.f;
#pragma unroll
  for (int o = GQP; o < 32; o <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane < GQP) den_w[warp * GQP + lane] = dsum;
}

// kv_refine_kernel (a selection given): kRefParts CTAs per head, each a share
// of the selected tokens and of the split records; the head's last CTA merges.
// MINB = 2 holds the registers to two CTAs per SM (for grids of more than one
// wave, e.g. 8 caches at once; a few spills), MINB = 1 lets one CTA take what it
// needs (no spills).
template <int GQP, int B, int R, int MINB>
__global__ void __launch_bounds__(kRefThreads, MINB) kv_refine_kernel(RefArgs a) {
  __shared__ RefShared<GQP> sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int part = blockIdx.x, g = blockIdx.y, bat = blockIdx.z, gq = a.gq;
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  const long head = (long)bat * a.h_kv + g;
  pdl_trigger();
  pdl_wait();  // the base pass (and the selection, when it ran before) is complete
  if (a.stats_given) {
    // the statistics the scoring left in the control words (the same
    // computation over the same records)
    if (tid < gq) {
      const float* st = reinterpret_cast<const float*>(a.ctl + head * kCtl + kCtlStats);
      sh.M[tid] = __ldcg(st + 2 * tid), sh.Z[tid] = __ldcg(st + 2 * tid + 1);
    }
  } else if (warp < gq) {
    float M, Z;
    head_stats(a.part + (hq0 + warp) * a.nrec * kRec, a.nrec, kRec, lane, M, Z);
    if (lane == 0) sh.M[warp] = M, sh.Z[warp] = Z;
  }
  __syncthreads();
  const int ja = (int)((long)part * a.k_tok / a.parts), jb = (int)((long)(part + 1) * a.k_tok / a.parts);
  const long slot0 = head * a.t_max;
  RefLane<GQP, B, R> rl;
  rl.init(a, hq0, lane);
  float rec[4];
  record_share<GQP>(a, hq0, sh.M, part, a.parts, tid, kRefThreads, rec);
  float an[GQP][4], ad_own = 0.f;
#pragma unroll
  for (int h = 0; h < GQP; h++)
#pragma unroll
    for (int e = 0; e < 4; e++) an[h][e] = 0.f;
  const int32_t* selg = a.sel + head * a.k_tok;
  for (int j0 = ja + warp * kRefTPW; j0 < jb; j0 += kRefWarps * kRefTPW) {
    int tok[kRefTPW];
#pragma unroll
    for (int m = 0; m < kRefTPW; m++) {
      const int j = j0 + m;
      const int t = j < jb ? selg[j] : -1;
      tok[m] = (t >= 0 && t < a.T) ? t : -1;  // a foreign index is skipped, never dereferenced
    }
    refine_batch<GQP, B, R>(a, rl, sh.M, slot0, hq0, tok, lane, an, ad_own, &sh.wtab[warp][0]);
  }
  stash_warp<GQP>(an, ad_own, warp, lane, &sh.num[0][0][0], &sh.den[0][0]);
  __syncthreads();
  write_part<GQP, kRefThreads>(a, head, part, &sh.num[0][0][0], &sh.den[0][0], rec);
  __threadfence();  // this CTA's partial before its count
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(a.ctl + head * kCtl + kBins1 + 1, 1) == a.parts - 1;
  __syncthreads();
  if (!sh.last) return;
  __threadfence();  // every other CTA's partial is visible
  merge_parts<kRefThreads>(a, hq0, head, sh.Z, a.parts, nullptr, nullptr);
}

// ---------------------------------------------------------------------------
// host side

struct Plan {
  int nsplit, span, nrec;  // base pass (warp splits; one record per CTA of kWarps splits)
  int Tp, sel_blocks, parts;
  size_t off_logits, off_part, off_scores, off_bitmap, off_cand, off_ctl, off_rpart, total;
};

// The workspace: [logits] [records] [scores, Tp-pitched] [control words] [refinement partials].
Plan make_plan(const sf_kv* kv, int t, int h_q, int k_tok, bool need_logits, bool with_pv, bool select,
               bool refine, int n_splits) {
  Plan P;
  const int sms = num_sms();
  const int heads = kv->batch * kv->h_kv;
  // splits per head: whole CTAs of kWarps splits, all (batch, head) CTAs in one
  // wave of 4 CTAs per SM (e.g. 296 for 8 heads, 36 for 64)
  int ns = n_splits > 0 ? n_splits : kWarps * std::max(1, 4 * sms / heads);
  int maxs = (t + 15) / 16;
  if (ns > maxs) ns = maxs;
  if (ns < 1) ns = 1;
  P.span = ((t + ns - 1) / ns + 15) / 16 * 16;
  P.nsplit = (t + P.span - 1) / P.span;
  P.nrec = (P.nsplit + kWarps - 1) / kWarps;
  P.Tp = (t + 31) / 32 * 32;
  P.sel_blocks = (t + kSelTok - 1) / kSelTok;
  // refinement CTAs per head: enough for the selected tokens and for the
  // split records (a few per CTA: each CTA's record loads are in flight together)
  P.parts = std::max(1, std::min(kRefPartsMax, std::max((k_tok + kRefWarps * kRefTPW - 1) / (kRefWarps * kRefTPW),
                                                        (P.nrec + 7) / 8)));
  const int gq = h_q / kv->h_kv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const int rec = with_pv ? kRec : 2;
  P.off_logits = need_logits ? take((size_t)kv->batch * h_q * t * 4) : 0;
  P.off_part = take((size_t)kv->batch * h_q * P.nrec * rec * 4);
  P.off_scores = select ? take((size_t)heads * P.Tp * 4) : 0;
  P.off_bitmap = select ? take((size_t)heads * (P.Tp / 32) * 4) : 0;
  P.off_cand = select ? take((size_t)heads * kCandCap * 8) : 0;
  P.off_ctl = take((size_t)heads * kCtl * 4);
  P.off_rpart = refine ? take((size_t)heads * P.parts * gq * (kD + 1) * 4) : 0;
  P.total = off;
  return P;
}

sf_status check_q(const sf_kv* kv, int t, const uint16_t* q, int h_q) {
  SF_REQUIRE(t >= 1 && t <= kv->t_max, "t=%d outside [1, t_max=%d]", t, kv->t_max);
  SF_REQUIRE(q && aligned16(q), "q must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(h_q > 0 && h_q % kv->h_kv == 0 && h_q / kv->h_kv <= 8,
                 "h_q=%d must be a multiple of h_kv=%d with at most 8 query heads per KV head", h_q,
                 kv->h_kv);
  SF_UNSUPPORTED(t <= kMaxT, "t=%d above %d", t, kMaxT);
  return SF_OK;
}

// k_tok of every entry point: at most t and kMaxKTok, at least 1 unless a
// base-only call (allow_zero) is meant.
sf_status check_ktok(int k_tok, int t, bool allow_zero) {
  SF_REQUIRE(k_tok >= (allow_zero ? 0 : 1) && k_tok <= t, "k_tok=%d outside [%d, t=%d]", k_tok,
             allow_zero ? 0 : 1, t);
  SF_UNSUPPORTED(k_tok <= kMaxKTok, "k_tok=%d above %d", k_tok, kMaxKTok);
  return SF_OK;
}

// kv_logits_fma_kernel -- the base pass without values on the CUDA cores: the
// same logits and per-CTA (max, sum) records as kv_base_kernel<4, 2, false>,
// with the key contraction done by fp32 FMAs (a lane per token, up to 4 query
// heads) instead of mma.sync.  Kept to measure the two against each other
// (2-bit keys).  The query heads sit in shared memory in the order of the code
// stream (qs[code][head]: one 16-byte load gives a code's 4 heads); code k of
// a token's key word w (bit 2k) is dim 16 s + 2 c + 8 e + (k >= 8) with
// c = w / 2, pair p = 8 (w % 2) + k % 8 = 2 s + e, in scale group s / 2.
__global__ void __launch_bounds__(kWarps * 32) kv_logits_fma_kernel(BaseArgs a) {
  __shared__ __align__(16) float qs[kD][4];
  __shared__ float Qg[4][4];              // [head][group]: sum of q over the group
  __shared__ float wr[kWarps][4][2];      // warp records: (max, sum) per head
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y, bat = blockIdx.z, gq = a.gq;
  const uint16_t* qg = a.q + ((long)bat * a.h_q + (long)g * gq) * kD;
  for (int e = threadIdx.x; e < 4 * kD; e += blockDim.x) {
    const int h = e / kD, d = e % kD;
    int word, bit;
    key_pos(d, 2, word, bit);
    qs[word * 16 + bit / 2][h] = h < gq ? h2f(qg[h * kD + d]) : 0.f;
  }
  if (threadIdx.x < 16) {
    const int h = threadIdx.x >> 2, j = threadIdx.x & 3;
    float v = 0.f;
    for (int d = 32 * j; d < 32 * j + 32; d++) v += h < gq ? h2f(qg[h * kD + d]) : 0.f;
    Qg[h][j] = v;
  }
  __syncthreads();
  const int split = blockIdx.x * kWarps + warp;
  const int tw0 = split * a.span, tw1 = split < a.nsplit ? min(a.T, tw0 + a.span) : tw0;
  const long slot0 = ((long)bat * a.h_kv + g) * a.t_max;
  float mrun[4], lsum[4];
#pragma unroll
  for (int h = 0; h < 4; h++) mrun[h] = -INFINITY, lsum[h] = 0.f;
  float* lg = a.logits + ((long)bat * a.h_q + (long)g * gq) * a.T;
  for (int tb = tw0; tb < tw1; tb += 32) {
    const int t = tb + lane;
    const bool ok = t < tw1;
    uint4 c0 = make_uint4(0u, 0u, 0u, 0u), c1 = c0, zz = c0;
    if (ok) {
      const uint4* kp = reinterpret_cast<const uint4*>(a.kb + (slot0 + t) * 32);
      c0 = __ldg(kp), c1 = __ldg(kp + 1);
      zz = __ldg(reinterpret_cast<const uint4*>(a.ksz) + (slot0 + t));
    }
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    float acc[4][4];  // [head][group]
#pragma unroll
    for (int h = 0; h < 4; h++)
#pragma unroll
      for (int j = 0; j < 4; j++) acc[h][j] = 0.f;
#pragma unroll
    for (int wi = 0; wi < 8; wi++)
#pragma unroll
      for (int k = 0; k < 16; k++) {
        const int grp = (wi & 1) * 2 + (k & 7) / 4;
        const float c = (float)((w[wi] >> (2 * k)) & 3u);
        const float4 qv = *reinterpret_cast<const float4*>(&qs[wi * 16 + k][0]);
        acc[0][grp] = fmaf(qv.x, c, acc[0][grp]);
        acc[1][grp] = fmaf(qv.y, c, acc[1][grp]);
        acc[2][grp] = fmaf(qv.z, c, acc[2][grp]);
        acc[3][grp] = fmaf(qv.w, c, acc[3][grp]);
      }
    // (s, m') per group, m' = m + 1.5 s: the codes enter uncentred, so the
    // offset term is m, not m'
    const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
    float l[4];
#pragma unroll
    for (int h = 0; h < 4; h++) {
      float x = 0.f;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float2 sm = __half22float2(*reinterpret_cast<const __half2*>(&zw[j]));
        x = fmaf(sm.x, acc[h][j], fmaf(sm.y, Qg[h][j], x));
      }
      l[h] = ok && h < gq ? x * a.scale : -INFINITY;
      if (ok && h < gq) lg[(long)h * a.T + t] = l[h];
    }
    // online softmax over the warp's tokens, one warp-wide max per chunk
#pragma unroll
    for (int h = 0; h < 4; h++) {
      float mx = l[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (mx > -INFINITY) {
        const float mn = fmaxf(mrun[h], mx);
        lsum[h] = lsum[h] * __expf(mrun[h] - mn) + (l[h] > -INFINITY ? __expf(l[h] - mn) : 0.f);
        mrun[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 4; h++) {
    float v = lsum[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) wr[warp][h][0] = mrun[h], wr[warp][h][1] = v;
  }
  __syncthreads();
  const long hq0 = (long)bat * a.h_q + (long)g * gq;
  if (threadIdx.x < gq) {
    const int h = threadIdx.x;
    float M = -INFINITY, L = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kWarps; w2++) M = fmaxf(M, wr[w2][h][0]);
    if (M > -INFINITY)
#pragma unroll
      for (int w2 = 0; w2 < kWarps; w2++)
        if (wr[w2][h][0] > -INFINITY) L = fmaf(__expf(wr[w2][h][0] - M), wr[w2][h][1], L);
    a.part[((hq0 + h) * a.nrec + blockIdx.x) * 2 + 0] = M;
    a.part[((hq0 + h) * a.nrec + blockIdx.x) * 2 + 1] = L;
  }
}

template <int GQP, int B, bool PV>
sf_status launch_base_t(const BaseArgs& a, int batch, cudaStream_t s) {
  const size_t smem = kWarps * WarpSmem<B, PV>::bytes;
  auto kern = kv_base_kernel<GQP, B, PV>;
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  SF_CUDA(launch_pdl(kern, dim3((a.nsplit + kWarps - 1) / kWarps, a.h_kv, batch), dim3(kWarps * 32), smem, s, a));
  return SF_OK;
}

sf_status launch_base(const sf_kv* kv, const BaseArgs& a, bool pv, cudaStream_t s) {
  const int gqp = a.gq <= 4 ? 4 : 8;
  if (kv->b == 2) {
    if (gqp == 4) return pv ? launch_base_t<4, 2, true>(a, kv->batch, s) : launch_base_t<4, 2, false>(a, kv->batch, s);
    return pv ? launch_base_t<8, 2, true>(a, kv->batch, s) : launch_base_t<8, 2, false>(a, kv->batch, s);
  }
  if (kv->b == 3) {
    if (gqp == 4) return pv ? launch_base_t<4, 3, true>(a, kv->batch, s) : launch_base_t<4, 3, false>(a, kv->batch, s);
    return pv ? launch_base_t<8, 3, true>(a, kv->batch, s) : launch_base_t<8, 3, false>(a, kv->batch, s);
  }
  if (gqp == 4) return pv ? launch_base_t<4, 4, true>(a, kv->batch, s) : launch_base_t<4, 4, false>(a, kv->batch, s);
  return pv ? launch_base_t<8, 4, true>(a, kv->batch, s) : launch_base_t<8, 4, false>(a, kv->batch, s);
}

BaseArgs base_args(const sf_kv* kv, int t, const uint16_t* q, int h_q, float* logits, float* part, int* ctl,
                   const Plan& P) {
  BaseArgs a;
  a.kb = (const uint8_t*)kv->kb, a.vb = (const uint8_t*)kv->vb;
  a.ksz = kv->ksz, a.vsz = kv->vsz;
  a.h_kv = kv->h_kv, a.t_max = kv->t_max, a.T = t;
  a.q = q, a.h_q = h_q, a.gq = h_q / kv->h_kv;
  a.logits = logits, a.part = part, a.ctl = ctl;
  a.span = P.span, a.nsplit = P.nsplit, a.nrec = P.nrec;
  a.scale = 1.0f / sqrtf((float)kD);
  return a;
}

// Scoring, then selection, after the base pass (programmatic serialization:
// the CTAs of each start while the kernel before it drains).
sf_status launch_select(const sf_kv* kv, int t, int h_q, int k_tok, const Plan& P, const float* logits,
                        const float* part, int rec, char* ws, float* scores_out, int* ctl, int32_t* sel,
                        cudaStream_t s) {
  SelArgs a;
  a.logits = logits, a.part = part, a.nrec = P.nrec, a.rec = rec;
  a.h_kv = kv->h_kv, a.h_q = h_q, a.gq = h_q / kv->h_kv, a.T = t, a.Tp = P.Tp, a.k_tok = k_tok;
  a.nblk = P.sel_blocks;
  a.scores = (float*)(ws + P.off_scores), a.scores_out = scores_out, a.ctl = ctl, a.sel = sel;
  a.bitmap = (uint32_t*)(ws + P.off_bitmap), a.cand = (uint2*)(ws + P.off_cand);
  const dim3 grid(P.sel_blocks, kv->h_kv, kv->batch);
  // a grid of at most one CTA per SM is spread over the SMs: the CTA reserves
  // shared memory enough that no second one fits beside it (the scoring of a
  // head's tokens is latency-bound; two CTAs on one SM would share its load path)
  auto score = a.gq <= 4 ? kv_score_kernel<4> : kv_score_kernel<8>;
  const size_t spread = (long)grid.x * grid.y * grid.z <= num_sms() ? kSpreadSmem : 0;
  if (spread) SF_CUDA(cudaFuncSetAttribute(score, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)spread));
  SF_CUDA(launch_pdl(score, grid, dim3(kSelThreads), spread, s, a));
  SF_CUDA(cudaFuncSetAttribute(kv_pick_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelDyn));
  SF_CUDA(launch_pdl(kv_pick_kernel, grid, dim3(kSelThreads), kSelDyn, s, a));
  return SF_OK;
}

template <int GQP, int MINB>
void (*refine_kernel_for(int b, int r))(RefArgs) {
  if (b == 2) return r == 2 ? kv_refine_kernel<GQP, 2, 2, MINB> : kv_refine_kernel<GQP, 2, 1, MINB>;
  if (b == 3) return r == 2 ? kv_refine_kernel<GQP, 3, 2, MINB> : kv_refine_kernel<GQP, 3, 1, MINB>;
  return r == 2 ? kv_refine_kernel<GQP, 4, 2, MINB> : kv_refine_kernel<GQP, 4, 1, MINB>;
}

// Refinement of the selected tokens and the merge (programmatic serialization).
sf_status launch_refine(const sf_kv* kv, int t, const uint16_t* q, int h_q, int k_tok, const Plan& P,
                        const float* logits, const float* part, const int32_t* sel, int* ctl, float* rpart,
                        float* out, uint16_t* out16, int stats_given, cudaStream_t s) {
  RefArgs a;
  a.kb = (const uint8_t*)kv->kb, a.kr = (const uint8_t*)kv->kr;
  a.vb = (const uint8_t*)kv->vb, a.vr = (const uint8_t*)kv->vr;
  a.ksz = kv->ksz, a.vsz = kv->vsz;
  a.h_kv = kv->h_kv, a.t_max = kv->t_max, a.T = t;
  a.q = q, a.h_q = h_q, a.gq = h_q / kv->h_kv;
  a.logits = logits, a.part = part, a.nrec = P.nrec;
  a.k_tok = k_tok, a.parts = P.parts, a.sel = sel, a.ctl = ctl, a.rpart = rpart;
  a.stats_given = stats_given;
  a.out = out, a.out16 = out16;
  a.scale = 1.0f / sqrtf((float)kD);
  // two CTAs per SM when the grid is more than one wave of one CTA per SM
  const bool two = (long)P.parts * kv->h_kv * kv->batch > num_sms();
  void (*kern)(RefArgs);
  if (a.gq <= 4) kern = two ? refine_kernel_for<4, 2>(kv->b, kv->r) : refine_kernel_for<4, 1>(kv->b, kv->r);
  else kern = two ? refine_kernel_for<8, 2>(kv->b, kv->r) : refine_kernel_for<8, 1>(kv->b, kv->r);
  SF_CUDA(launch_pdl(kern, dim3(P.parts, kv->h_kv, kv->batch), dim3(kRefThreads), 0, s, a));
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
  return make_plan(kv, t, h_q, k_tok, !logits_given, false, true, false, 0).total;
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
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, false, true, false, 0);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  int* ctl = (int*)(w + P.off_ctl);
  cudaStream_t s = as_stream(stream);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, ctl, P);
  st = launch_base(kv, a, false, s);
  if (st != SF_OK) return st;
  return launch_select(kv, t, h_q, k_tok, P, lg, part, 2, w, scores, ctl, sel, s);
}

extern "C" size_t sf_kv_logits_fma_workspace_bytes(const sf_kv* kv, int t, int h_q) {
  if (!kv || t <= 0 || h_q <= 0) return 0;
  return make_plan(kv, t, h_q, 0, false, false, false, false, 0).total;
}

extern "C" sf_status sf_kv_logits_fma(const sf_kv* kv, int t, const uint16_t* q, int h_q, float* logits,
                                      void* ws, size_t ws_bytes, sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_UNSUPPORTED(kv->b == 2 && h_q / kv->h_kv <= 4, "the CUDA-core form takes 2-bit keys and <= 4 query heads per KV head");
  SF_REQUIRE(logits && aligned16(logits), "logits must be a non-null 16-byte aligned device pointer");
  Plan P = make_plan(kv, t, h_q, 0, false, false, false, false, 0);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  BaseArgs a = base_args(kv, t, q, h_q, logits, (float*)(w + P.off_part), nullptr, P);
  SF_CUDA(launch_pdl(kv_logits_fma_kernel, dim3((a.nsplit + kWarps - 1) / kWarps, a.h_kv, kv->batch),
                     dim3(kWarps * 32), 0, as_stream(stream), a));
  return SF_OK;
}

extern "C" size_t sf_kv_attn_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                             int n_splits) {
  if (!kv || t <= 0 || h_q <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, true, true, false, true, n_splits).total;
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
  Plan P = make_plan(kv, t, h_q, k_tok, true, true, false, true, n_splits);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  cudaStream_t s = as_stream(stream);
  float* lg = (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  int* ctl = (int*)(w + P.off_ctl);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, ctl, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  return launch_refine(kv, t, q, h_q, k_tok, P, lg, part, sel, ctl, (float*)(w + P.off_rpart), out, nullptr, 0, s);
}

extern "C" size_t sf_kv_attend_selective_workspace_bytes(const sf_kv* kv, int t, int h_q,
                                                         int k_tok, int logits_given) {
  if (!kv || t <= 0 || h_q <= 0 || k_tok <= 0) return 0;
  return make_plan(kv, t, h_q, k_tok, !logits_given, true, true, true, 0).total;
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
  Plan P = make_plan(kv, t, h_q, k_tok, logits == nullptr, true, true, true, 0);
  st = check_ws(ws, ws_bytes, P.total);
  if (st != SF_OK) return st;
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float* part = (float*)(w + P.off_part);
  int* ctl = (int*)(w + P.off_ctl);
  BaseArgs a = base_args(kv, t, q, h_q, lg, part, ctl, P);
  st = launch_base(kv, a, true, s);
  if (st != SF_OK) return st;
  st = launch_select(kv, t, h_q, k_tok, P, lg, part, kRec, w, nullptr, ctl, sel, s);
  if (st != SF_OK) return st;
  return launch_refine(kv, t, q, h_q, k_tok, P, lg, part, sel, ctl, (float*)(w + P.off_rpart), out, out16, 1, s);
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
  const size_t need = make_plan(kv, t, h_q, k_tok, logits == nullptr, true, true, true, 0).total;
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
