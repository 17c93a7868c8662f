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
//     attention scores.  Hence the order: logits -> softmax stats -> scores ->
//     selection -> refined attention.
//
// Kernels:
//   kv_logits_kernel   base logits of a span of tokens for the query heads of
//                      one KV head, plus the span's (max, sum exp) per head;
//   kv_stats_kernel    merge the spans' (max, sum) into the softmax stats;
//   kv_local_kernel    per span, score every token and keep the span's
//                      k_tok best (a token in the global top-k is in the top-k
//                      of its own span), in token order;
//   kv_final_kernel    per KV head, the k_tok best of the candidates;
//   kv_attn_kernel     per context split, online-softmax attention with the
//                      selected tokens dequantised at b+r bits;
//   kv_merge_kernel    log-sum-exp merge of the splits.
#include <cfloat>

#include "common.cuh"

namespace sf {
namespace {

constexpr int kD = 128;          // head dim (validated)
constexpr int kGroups = kD / 32; // quantisation groups per token
constexpr int kTile = 64;        // tokens per shared-memory tile (logits)
constexpr int kATile = 32;       // tokens per shared-memory tile (attention)
constexpr int kMaxCand = 16384;  // candidates per KV head in the final select
constexpr int kMaxSpan = 8192;   // tokens per local-select CTA

struct KvView {
  const uint32_t *kb, *kr, *vb, *vr;
  const uint16_t *ksz, *vsz;
  int h_kv, t_max, b, r;
};

__device__ __forceinline__ long slot_of(const KvView& kv, int bat, int g, int t) {
  return ((long)bat * kv.h_kv + g) * kv.t_max + t;
}

// Dequantise element d of token `slot` (base, or refined when `refined`).
__device__ __forceinline__ float kv_value(const uint32_t* codes, const uint32_t* refine,
                                          const uint16_t* sz, long slot, int d, int b, int r,
                                          bool refined) {
  long e = slot * kD + d;
  uint32_t q = (codes[(e * b) >> 5] >> ((e * b) & 31)) & ((1u << b) - 1);
  const uint16_t* z = sz + (slot * kGroups + d / 32) * 2;
  float s = h2f(z[0]), m = h2f(z[1]);
  float v = (float)q;
  if (refined) {
    uint32_t rho = (refine[(e * r) >> 5] >> ((e * r) & 31)) & ((1u << r) - 1);
    v += ((float)rho + 0.5f - 0.5f * (float)(1 << r)) / (float)(1 << r);
  }
  return fmaf(s, v, m);
}

// ---------------------------------------------------------------------------
// logits

__global__ void __launch_bounds__(256) kv_logits_kernel(KvView kv, int T, int span,
                                                        const uint16_t* __restrict__ q, int h_q,
                                                        float* __restrict__ logits,
                                                        float2* __restrict__ part) {
  const int gq = h_q / kv.h_kv;
  const int sp = blockIdx.x, g = blockIdx.y, bat = blockIdx.z;
  const int t0 = sp * span, t1 = min(T, t0 + span);
  __shared__ float qs[8][kD + 1];
  __shared__ float kd[kTile][kD + 1];
  __shared__ float red[8][kTile];
  const float scale = rsqrtf((float)kD);
  for (int i = threadIdx.x; i < gq * kD; i += blockDim.x)
    qs[i / kD][i % kD] = h2f(q[((long)bat * h_q + g * gq + i / kD) * kD + i % kD]) * scale;
  float run_m[8], run_s[8];  // used by threads 0..gq-1
  for (int h = 0; h < 8; h++) run_m[h] = -FLT_MAX, run_s[h] = 0.f;
  __syncthreads();
  for (int tt = t0; tt < t1; tt += kTile) {
    const int nt = min(kTile, t1 - tt);
    for (int i = threadIdx.x; i < nt * kD; i += blockDim.x) {
      int t = i / kD, d = i % kD;
      kd[t][d] = kv_value(kv.kb, kv.kr, kv.ksz, slot_of(kv, bat, g, tt + t), d, kv.b, kv.r, false);
    }
    __syncthreads();
    for (int pr = threadIdx.x; pr < nt * gq; pr += blockDim.x) {
      int t = pr / gq, h = pr % gq;
      float acc = 0.f;
      for (int d = 0; d < kD; d++) acc = fmaf(qs[h][d], kd[t][d], acc);
      logits[((long)bat * h_q + g * gq + h) * T + tt + t] = acc;
      red[h][t] = acc;
    }
    __syncthreads();
    if (threadIdx.x < gq) {
      int h = threadIdx.x;
      float m = run_m[h];
      for (int t = 0; t < nt; t++) m = fmaxf(m, red[h][t]);
      float s = run_s[h] * expf(run_m[h] - m);
      for (int t = 0; t < nt; t++) s += expf(red[h][t] - m);
      run_m[h] = m, run_s[h] = s;
    }
    __syncthreads();
  }
  if (threadIdx.x < gq) {
    int h = g * gq + threadIdx.x;
    part[((long)bat * h_q + h) * gridDim.x + sp] = make_float2(run_m[threadIdx.x], run_s[threadIdx.x]);
  }
}

// (max, sum exp) of every query head from the spans' partials.
__global__ void kv_stats_kernel(const float2* __restrict__ part, int nspan, float2* __restrict__ stats) {
  const long bh = blockIdx.x;  // bat * h_q + h
  const float2* p = part + bh * nspan;
  __shared__ float sm[256];
  float m = -FLT_MAX;
  for (int i = threadIdx.x; i < nspan; i += blockDim.x) m = fmaxf(m, p[i].x);
  sm[threadIdx.x] = m;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) sm[threadIdx.x] = fmaxf(sm[threadIdx.x], sm[threadIdx.x + o]);
    __syncthreads();
  }
  const float M = sm[0];
  __syncthreads();
  float s = 0.f;
  for (int i = threadIdx.x; i < nspan; i += blockDim.x) s += p[i].y * expf(p[i].x - M);
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

// k-th largest of n unique keys (1 <= k <= n), 8 bits per pass from the top.
// keys in shared memory; hist: 256 ints of shared scratch.
__device__ uint64_t block_kth_largest(const uint64_t* keys, int n, int k, int* hist) {
  __shared__ int s_digit, s_k;
  uint64_t prefix = 0, mask = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      uint64_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      const int lane = threadIdx.x;
      int c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; j++) tot += (c[j] = hist[255 - 8 * lane - j]);
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int above = incl - tot;  // keys with a larger digit
      if (above < k && incl >= k) {
        int run = above;
        for (int j = 0; j < 8; j++) {
          if (run + c[j] >= k) {
            s_digit = 255 - 8 * lane - j;
            s_k = k - run;
            break;
          }
          run += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint64_t)s_digit << shift;
    mask |= (uint64_t)255 << shift;
    k = s_k;
    __syncthreads();
  }
  return prefix;
}

// Write the keys >= tau in index order: out[pos] for pos = rank among them.
// Thread i handles a contiguous range of indices, so order is preserved.
template <class Emit>
__device__ void block_compact(const uint64_t* keys, int n, uint64_t tau, Emit emit) {
  __shared__ int warp_tot[32];
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  int mine = 0;
  for (int i = i0; i < i1; i++) mine += keys[i] >= tau;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int nw = blockDim.x >> 5;
    int v = lane < nw ? warp_tot[lane] : 0;
    int x = v;
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += u;
    }
    if (lane < nw) warp_tot[lane] = x - v;
  }
  __syncthreads();
  int pos = warp_tot[warp] + incl - mine;
  for (int i = i0; i < i1; i++)
    if (keys[i] >= tau) emit(pos++, keys[i]);
  __syncthreads();
}

__global__ void __launch_bounds__(1024) kv_local_kernel(const float* __restrict__ logits,
                                                        const float2* __restrict__ stats, int T,
                                                        int span, int h_q, int h_kv, int k_tok,
                                                        float* __restrict__ scores,
                                                        uint64_t* __restrict__ cand) {
  extern __shared__ uint64_t keys[];  // span entries
  __shared__ int hist[256];
  const int gq = h_q / h_kv;
  const int sp = blockIdx.x, g = blockIdx.y, bat = blockIdx.z;
  const int t0 = sp * span, n = min(T, t0 + span) - t0;
  float M[8], invZ[8];
  for (int h = 0; h < gq; h++) {
    float2 st = stats[(long)bat * h_q + g * gq + h];
    M[h] = st.x, invZ[h] = 1.0f / st.y;
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float s = 0.f;
    for (int h = 0; h < gq; h++)
      s += expf(logits[((long)bat * h_q + g * gq + h) * T + t0 + i] - M[h]) * invZ[h];
    if (scores) scores[((long)bat * h_kv + g) * T + t0 + i] = s;
    keys[i] = score_key(s, t0 + i);
  }
  __syncthreads();
  const int kl = min(k_tok, n);
  uint64_t tau = block_kth_largest(keys, n, kl, hist);
  uint64_t* out = cand + (((long)bat * h_kv + g) * gridDim.x + sp) * (long)min(k_tok, span);
  block_compact(keys, n, tau, [&](int pos, uint64_t key) { out[pos] = key; });
}

__global__ void __launch_bounds__(1024) kv_final_kernel(const uint64_t* __restrict__ cand, int nspan,
                                                        int span, int T, int h_kv, int k_tok,
                                                        int32_t* __restrict__ sel) {
  extern __shared__ uint64_t keys[];  // all candidates of this KV head
  __shared__ int hist[256];
  const int g = blockIdx.x, bat = blockIdx.y;
  const int per = min(k_tok, span);
  const uint64_t* src = cand + ((long)bat * h_kv + g) * nspan * (long)per;
  int n = 0;
  for (int sp = 0; sp < nspan; sp++) {  // spans hold min(k_tok, their length) keys
    int len = min(T, (sp + 1) * span) - sp * span;
    int cnt = min(k_tok, len);
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) keys[n + i] = src[(long)sp * per + i];
    n += cnt;
  }
  __syncthreads();
  uint64_t tau = block_kth_largest(keys, n, k_tok, hist);
  int32_t* out = sel + ((long)bat * h_kv + g) * k_tok;
  block_compact(keys, n, tau, [&](int pos, uint64_t key) { out[pos] = key_token(key); });
}

// ---------------------------------------------------------------------------
// refined attention (split over the context, partials merged by log-sum-exp)

__global__ void __launch_bounds__(256) kv_attn_kernel(KvView kv, int T, int span,
                                                      const uint16_t* __restrict__ q, int h_q,
                                                      const int32_t* __restrict__ sel, int k_tok,
                                                      const float* __restrict__ base_logits,
                                                      float* __restrict__ part) {
  const int gq = h_q / kv.h_kv;
  const int sp = blockIdx.x, g = blockIdx.y, bat = blockIdx.z;
  const int t0 = sp * span, t1 = min(T, t0 + span);
  __shared__ float qs[8][kD + 1];
  __shared__ float kd[kATile][kD + 1];
  __shared__ float vd[kATile][kD + 1];
  __shared__ float pl[8][kATile];
  __shared__ float s_m[8], s_l[8], s_alpha[8];
  extern __shared__ uint32_t selmask[];  // one bit per token of the span
  const float scale = rsqrtf((float)kD);
  for (int i = threadIdx.x; i < gq * kD; i += blockDim.x)
    qs[i / kD][i % kD] = h2f(q[((long)bat * h_q + g * gq + i / kD) * kD + i % kD]) * scale;
  for (int i = threadIdx.x; i < (span + 31) / 32; i += blockDim.x) selmask[i] = 0;
  if (threadIdx.x < 8) s_m[threadIdx.x] = -FLT_MAX, s_l[threadIdx.x] = 0.f;
  __syncthreads();
  const int32_t* sg = sel + ((long)bat * kv.h_kv + g) * k_tok;
  for (int j = threadIdx.x; j < k_tok; j += blockDim.x) {
    int t = sg[j];
    if (t >= t0 && t < t1) atomicOr(&selmask[(t - t0) >> 5], 1u << ((t - t0) & 31));
  }
  // accumulators: thread owns (head, dim) pairs idx, idx + 256, ...
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  __syncthreads();
  for (int tt = t0; tt < t1; tt += kATile) {
    const int nt = min(kATile, t1 - tt);
    for (int i = threadIdx.x; i < nt * kD; i += blockDim.x) {
      int t = i / kD, d = i % kD;
      int lt = tt + t - t0;
      bool rf = (selmask[lt >> 5] >> (lt & 31)) & 1;
      long slot = slot_of(kv, bat, g, tt + t);
      if (rf || !base_logits) kd[t][d] = kv_value(kv.kb, kv.kr, kv.ksz, slot, d, kv.b, kv.r, rf);
      vd[t][d] = kv_value(kv.vb, kv.vr, kv.vsz, slot, d, kv.b, kv.r, rf);
    }
    __syncthreads();
    for (int pr = threadIdx.x; pr < nt * gq; pr += blockDim.x) {
      int t = pr / gq, h = pr % gq;
      int lt = tt + t - t0;
      bool rf = (selmask[lt >> 5] >> (lt & 31)) & 1;
      float l;
      if (rf || !base_logits) {
        l = 0.f;
        for (int d = 0; d < kD; d++) l = fmaf(qs[h][d], kd[t][d], l);
      } else {
        l = base_logits[((long)bat * h_q + g * gq + h) * T + tt + t];
      }
      pl[h][t] = l;
    }
    __syncthreads();
    if (threadIdx.x < gq) {  // online softmax update of head h
      int h = threadIdx.x;
      float m = s_m[h];
      for (int t = 0; t < nt; t++) m = fmaxf(m, pl[h][t]);
      float alpha = expf(s_m[h] - m);
      float l = s_l[h] * alpha;
      for (int t = 0; t < nt; t++) {
        float p = expf(pl[h][t] - m);
        pl[h][t] = p;
        l += p;
      }
      s_m[h] = m, s_l[h] = l, s_alpha[h] = alpha;
    }
    __syncthreads();
    for (int k = 0; k < 4; k++) {
      int idx = threadIdx.x + 256 * k;
      if (idx < gq * kD) {
        int h = idx / kD, d = idx % kD;
        float a = acc[k] * s_alpha[h];
        for (int t = 0; t < nt; t++) a = fmaf(pl[h][t], vd[t][d], a);
        acc[k] = a;
      }
    }
    __syncthreads();
  }
  // partial layout: [bat][h_q][nsplit][kD + 2] = (acc[kD], m, l)
  for (int k = 0; k < 4; k++) {
    int idx = threadIdx.x + 256 * k;
    if (idx < gq * kD) {
      int h = idx / kD, d = idx % kD;
      part[(((long)bat * h_q + g * gq + h) * gridDim.x + sp) * (kD + 2) + d] = acc[k];
    }
  }
  if (threadIdx.x < gq) {
    float* p = part + (((long)bat * h_q + g * gq + threadIdx.x) * gridDim.x + sp) * (kD + 2);
    p[kD] = s_m[threadIdx.x];
    p[kD + 1] = s_l[threadIdx.x];
  }
}

__global__ void kv_merge_kernel(const float* __restrict__ part, int nsplit, float* __restrict__ out) {
  const long bh = blockIdx.x;
  const float* p = part + bh * nsplit * (kD + 2);
  float M = -FLT_MAX;
  for (int s = 0; s < nsplit; s++) M = fmaxf(M, p[s * (kD + 2) + kD]);
  float L = 0.f, a = 0.f;
  const int d = threadIdx.x;
  for (int s = 0; s < nsplit; s++) {
    float w = expf(p[s * (kD + 2) + kD] - M);
    L += w * p[s * (kD + 2) + kD + 1];
    a += w * p[s * (kD + 2) + d];
  }
  out[bh * kD + d] = a / L;
}

KvView view_of(const sf_kv* kv) {
  KvView v;
  v.kb = (const uint32_t*)kv->kb, v.kr = (const uint32_t*)kv->kr;
  v.vb = (const uint32_t*)kv->vb, v.vr = (const uint32_t*)kv->vr;
  v.ksz = kv->ksz, v.vsz = kv->vsz;
  v.h_kv = kv->h_kv, v.t_max = kv->t_max, v.b = kv->b, v.r = kv->r;
  return v;
}

// ---- launch geometry --------------------------------------------------------

struct ScorePlan {
  int lspan, nl;       // logits spans
  int sspan, ns;       // selection spans
  size_t off_logits, off_part, off_stats, off_cand, total;
};

ScorePlan score_plan(const sf_kv* kv, int t, int h_q, int k_tok, bool logits_given) {
  ScorePlan P;
  const int sms = num_sms();
  const int heads = kv->batch * kv->h_kv;
  P.lspan = 256;
  P.nl = (t + P.lspan - 1) / P.lspan;
  int ns = (sms + heads - 1) / heads;
  if (ns < 1) ns = 1;
  int span = (t + ns - 1) / ns;
  if (span > kMaxSpan) span = kMaxSpan;
  if (span < 32) span = 32;
  ns = (t + span - 1) / span;
  while (ns > 1 && (long)ns * (k_tok < span ? k_tok : span) > kMaxCand) {
    span = (span * 2 > kMaxSpan) ? kMaxSpan : span * 2;
    int ns2 = (t + span - 1) / span;
    if (ns2 == ns) break;
    ns = ns2;
  }
  P.sspan = span, P.ns = ns;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  P.off_logits = logits_given ? 0 : take((size_t)kv->batch * h_q * t * 4);
  P.off_part = take((size_t)kv->batch * h_q * P.nl * 8);
  P.off_stats = take((size_t)kv->batch * h_q * 8);
  P.off_cand = take((size_t)heads * ns * (k_tok < span ? k_tok : span) * 8);
  P.total = off;
  return P;
}

int attn_splits(const sf_kv* kv, int t, int n_splits) {
  if (n_splits > 0) return n_splits < t ? n_splits : t;
  const int heads = kv->batch * kv->h_kv;
  int s = (2 * num_sms() + heads - 1) / heads;
  int maxs = (t + kATile - 1) / kATile;
  if (s > maxs) s = maxs;
  return s < 1 ? 1 : s;
}

sf_status check_q(const sf_kv* kv, int t, const uint16_t* q, int h_q) {
  SF_REQUIRE(t >= 1 && t <= kv->t_max, "t=%d outside [1, t_max=%d]", t, kv->t_max);
  SF_REQUIRE(q && aligned16(q), "q must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(h_q > 0 && h_q % kv->h_kv == 0 && h_q / kv->h_kv <= 8,
                 "h_q=%d must be a multiple of h_kv=%d with at most 8 query heads per KV head", h_q,
                 kv->h_kv);
  return SF_OK;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_kv_score_select_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                                     int logits_given) {
  if (!kv || t <= 0 || h_q <= 0 || k_tok <= 0) return 0;
  return score_plan(kv, t, h_q, k_tok, logits_given != 0).total;
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
  ScorePlan P = score_plan(kv, t, h_q, k_tok, logits != nullptr);
  long ncand = (long)P.ns * (k_tok < P.sspan ? k_tok : P.sspan);
  SF_UNSUPPORTED(ncand <= kMaxCand, "t=%d with k_tok=%d needs %ld candidates (max %d)", t, k_tok,
                 ncand, kMaxCand);
  if (ws_bytes < P.total || (P.total > 0 && !ws)) {
    set_error("workspace: need %zu bytes, got %zu", P.total, ws_bytes);
    return SF_ERR_WORKSPACE;
  }
  SF_REQUIRE(!ws || aligned16(ws), "ws must be 16-byte aligned");
  char* w = (char*)ws;
  float* lg = logits ? logits : (float*)(w + P.off_logits);
  float2* part = (float2*)(w + P.off_part);
  float2* stats = (float2*)(w + P.off_stats);
  uint64_t* cand = (uint64_t*)(w + P.off_cand);
  cudaStream_t s = as_stream(stream);
  KvView v = view_of(kv);
  kv_logits_kernel<<<dim3(P.nl, kv->h_kv, kv->batch), 256, 0, s>>>(v, t, P.lspan, q, h_q, lg, part);
  SF_LAUNCHED();
  kv_stats_kernel<<<kv->batch * h_q, 256, 0, s>>>(part, P.nl, stats);
  SF_LAUNCHED();
  size_t smem_l = (size_t)P.sspan * 8;
  SF_CUDA(cudaFuncSetAttribute(kv_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kMaxSpan * 8));
  kv_local_kernel<<<dim3(P.ns, kv->h_kv, kv->batch), 1024, smem_l, s>>>(
      lg, stats, t, P.sspan, h_q, kv->h_kv, k_tok, scores, cand);
  SF_LAUNCHED();
  SF_CUDA(cudaFuncSetAttribute(kv_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kMaxCand * 8));
  kv_final_kernel<<<dim3(kv->h_kv, kv->batch), 1024, (size_t)ncand * 8, s>>>(
      cand, P.ns, P.sspan, t, kv->h_kv, k_tok, sel);
  SF_LAUNCHED();
  return SF_OK;
}

extern "C" size_t sf_kv_attn_workspace_bytes(const sf_kv* kv, int t, int h_q, int n_splits) {
  if (!kv || t <= 0 || h_q <= 0) return 0;
  int ns = attn_splits(kv, t, n_splits);
  return (size_t)kv->batch * h_q * ns * (kD + 2) * 4;
}

extern "C" sf_status sf_kv_attn_refined(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                        const int32_t* sel, int k_tok, const float* base_logits,
                                        int n_splits, float* out, void* ws, size_t ws_bytes,
                                        sf_stream_t stream) {
  sf_status st = check_kv(kv);
  if (st != SF_OK) return st;
  st = check_q(kv, t, q, h_q);
  if (st != SF_OK) return st;
  SF_REQUIRE(k_tok >= 0 && k_tok <= t, "k_tok=%d outside [0, t=%d]", k_tok, t);
  SF_REQUIRE(k_tok == 0 || (sel && aligned16(sel)), "sel must be non-null and 16-byte aligned");
  SF_REQUIRE(n_splits >= 0, "n_splits=%d < 0", n_splits);
  SF_REQUIRE(out && aligned16(out), "out must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(!base_logits || aligned16(base_logits), "base_logits must be 16-byte aligned");
  int ns = attn_splits(kv, t, n_splits);
  size_t need = (size_t)kv->batch * h_q * ns * (kD + 2) * 4;
  if (ws_bytes < need || !ws) {
    set_error("workspace: need %zu bytes, got %zu", need, ws_bytes);
    return SF_ERR_WORKSPACE;
  }
  SF_REQUIRE(aligned16(ws), "ws must be 16-byte aligned");
  int span = (t + ns - 1) / ns;
  ns = (t + span - 1) / span;
  cudaStream_t s = as_stream(stream);
  size_t smem = (size_t)((span + 31) / 32) * 4;
  SF_UNSUPPORTED(smem <= 64 * 1024, "split of %d tokens too long", span);
  SF_CUDA(cudaFuncSetAttribute(kv_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024));
  kv_attn_kernel<<<dim3(ns, kv->h_kv, kv->batch), 256, smem, s>>>(
      view_of(kv), t, span, q, h_q, k_tok ? sel : nullptr, k_tok, base_logits, (float*)ws);
  SF_LAUNCHED();
  kv_merge_kernel<<<kv->batch * h_q, kD, 0, s>>>((const float*)ws, ns, out);
  SF_LAUNCHED();
  return SF_OK;
}
