// gemv.cu -- refined low-bit GEMV: y = W~ x with base codes for every channel and
// nested refinements for the selected ones.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?":
//   which-tiles-count paragraph -- the k channels with the largest |x| in each
//     chunk of 1,024 input channels are refined; every other channel still
//     contributes at base precision;
//   nested-quantization paragraph -- the refined value is the centre of the
//     refinement's sub-bin inside the base bin:
//       w~ = w^ + s * (2*rho + 1 - 2^r) / 2^(r+1).
//   the-map-app-also-loads-tiles paragraph -- with fetch lag the correction
//     of a projection is applied later than its base product; the
//     correction-only kernel below computes it on its own.
//
// Decomposition, per output row i (fp32 accumulation):
//   y_i = sum_groups [ s_ig * sum_{c in g} x_c q_ic + m_ig * sum_{c in g} x_c ]
//       + sum_{c selected} x_c * s_i,g(c) * (rho_ic + 1/2 - 2^(r-1)) / 2^r
//
// Activation prologue (in every CTA, after griddepcontrol.wait): each
// 64-channel lane group of x becomes exact fixed point x = x_fix * 2^e with
// |x_fix| < 2^21, split into three byte planes laid out in the order of the
// code byte vectors below, plus the group's sums, in shared memory.

// Base pass (HBM-bound: every resident code is read once).  One CTA of 16
// warps per SM owns a contiguous, 4-aligned range of rows.  Its work is a list
// of (2,048-channel segment, 4-row step) tasks split evenly over the warps; a
// warp keeps the byte planes of its current segment in registers (a lane owns
// 64 channels) and streams the codes of its rows through a per-lane cp.async
// ring.  A lane turns 16 B of 2-bit codes into byte vectors with one AND per
// four codes (codes at bit offsets 2 and 6 keep a factor 4 that is removed
// once per row), takes integer dot products with dp4a (four code x byte
// products per instruction) and combines the planes in 32-bit integers, so the
// lane's partial dot product is exact.  Partial sums of four rows are reduced
// across the warp with a transposed butterfly.
//
// Correction pass: a table of the selected channels (x_c, group, refinement
// row) and the refinement words covering the CTA's rows are copied into shared
// memory while the base pass streams (the base pass also keeps the rows'
// (s, m) words), then each lane owns 1, 2 or 4 rows
// and every warp walks a range of the table, summing x_c (rho_ic + 1/2 -
// 2^(r-1)) / 2^r over each run of channels that share a scale group and
// scaling each run once.
#include "common.cuh"
#include "internal.cuh"

namespace sf {
namespace {

constexpr int kLaneCh = 64;                 // input channels per lane
constexpr int kSegChannels = 32 * kLaneCh;  // 2,048 channels per warp segment
constexpr int kWarps = 16;                  // one CTA of 16 warps per SM
constexpr int kThreads = kWarps * 32;
#ifndef SF_GEMV_XPLANES
#define SF_GEMV_XPLANES 3
#endif
constexpr int kXP = SF_GEMV_XPLANES;        // byte planes of the fixed-point activations
constexpr int kXShift = 8 * kXP - 4;        // x_fix = x * 2^-(ilogb(max|x|) - kXShift), |x_fix| < 2^(8 kXP - 3)
constexpr int kXR = 16 * kXP;               // plane words per lane group
constexpr int kXWords = kXR + 4;            // then sum0, sum1, 2^e, sum
constexpr int kRowUnit = 4;                 // CTA row ranges start at multiples of 4
constexpr size_t kSmemLimit = 226 * 1024;  // one block reservation (1 KB) below the SM's 228 KB

struct GemvParams {
  const uint32_t* base;
  const uint32_t* refine;  // channel-major rows, or staged rows [batch][n_sel]
  const uint16_t* sz;
  const uint16_t* x;       // [batch][K] fp16
  const int32_t* sel;      // [batch][n_sel]
  float* y;
  int N, K, G, gshift, r, batch, n_sel, segs;
  int refine_row_words;  // N * r / 32
  int staged;            // refine holds [batch][n_sel] staged rows
  int rows_max;          // most rows a CTA owns
  int plane_words;       // shared words of the activation planes
  int area_words;        // shared words of the copy rings (reused by the slow correction path)
  int fast;              // correction tables in their own shared region, filled before the base pass
  int w_span;            // stride of the refinement-word table (words a CTA's rows can span)
  int corr_rows;         // rows per lane in the correction (1, 2 or 4)
  int corr_split;        // fast path: the warps' correction partials go to the free ring area
  int pstride;           // row stride of the partial sums: segs base columns, then the correction
  float* y_corr;         // non-null: the correction goes here ([batch][N]) and y gets the base only
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Per lane and row: CW words of codes (64 channels), U rows per task.
template <int BITS>
struct Lane {
  static constexpr int CW = BITS == 2 ? 4 : BITS == 3 ? 6 : 8;
  static constexpr int U = BITS == 4 ? 2 : 4;
};

// Ring slot of one task (words): codes [U][C16][32 lanes][4] in 16-byte chunks,
// for b = 3 then the high-bit words [U][32][2], then (s, m) [U][ZW][32].
// Consecutive lanes read consecutive chunks, so reads are conflict-free.
template <int BITS, int ZW>
struct Ring {
  static constexpr int CW = Lane<BITS>::CW, U = Lane<BITS>::U;
  static constexpr int C16 = BITS == 3 ? 1 : CW / 4;
  static constexpr int hi_off() { return U * C16 * 32 * 4; }
  static constexpr int z_off = U * 32 * CW;
  static constexpr int words = U * 32 * (CW + ZW);
};

// Copies of one row into ring slot position u: the lane's codes (lane_base:
// the row-0 address of the lane's 16-byte chunks, row_bytes apart) and its
// (s, m) word(s) (lane_z: row 0's, gpr words apart).
template <int BITS, int ZW>
__device__ __forceinline__ void issue_row(const uint8_t* lane_base, const uint8_t* lane_hi, size_t row_bytes,
                                          const uint32_t* lane_z, int gpr, int row, uint32_t* slot, int u,
                                          int lane) {
  using R = Ring<BITS, ZW>;
  const uint8_t* rb = lane_base + (size_t)row * row_bytes;
#pragma unroll
  for (int c = 0; c < R::C16; c++) cp_async16(slot + ((u * R::C16 + c) * 32 + lane) * 4, rb + 16 * c);
  if constexpr (BITS == 3) cp_async8(slot + R::hi_off() + (u * 32 + lane) * 2, lane_hi + (size_t)row * (row_bytes / 2));
  const uint32_t* zr = lane_z + (size_t)row * gpr;
#pragma unroll
  for (int h = 0; h < ZW; h++) cp_async4(slot + R::z_off + (u * ZW + h) * 32 + lane, zr + h);
}

// Code byte vector v (0..15) of a lane's 64 channels; byte L holds the code of
// channel chan_of(v, L).
template <int BITS>
__host__ __device__ __forceinline__ int chan_of(int v, int L) {
  if (BITS == 4) return 8 * (v >> 1) + (v & 1) + 2 * L;
  return 16 * (v >> 2) + (v & 3) + 4 * L;
}

template <int BITS>
__device__ __forceinline__ uint32_t code_vec(const uint32_t (&w)[Lane<BITS>::CW], int v) {
  if constexpr (BITS == 4) {
    return (w[v >> 1] >> (4 * (v & 1))) & 0x0F0F0F0Fu;
  } else {
    const int wi = v >> 2, j = v & 3;
    uint32_t c = (w[wi] >> (2 * j)) & 0x03030303u;
    if constexpr (BITS == 3) c |= ((w[4 + (wi >> 1)] >> (4 * (wi & 1) + j)) << 2) & 0x04040404u;
    return c;
  }
}

// sum_c code_c * x_fix_c over the lane's 64 channels (ZW = 1) or over each
// 32-channel half (ZW = 2), exact in 32-bit integers: |x_fix| < 2^(8 kXP - 3)
// and codes < 16 keep every partial below 2^31 (intermediate wrap-around
// cancels).  Plane p of vector v is xr[kXP v + p]; the top plane is signed.
template <int BITS, int ZW>
__device__ __forceinline__ void lane_dot(const uint32_t (&w)[Lane<BITS>::CW], const uint32_t (&xr)[kXR],
                                         int32_t (&d)[ZW]) {
  auto mac = [&](uint32_t c, int v, uint32_t (&acc)[kXP]) {
#pragma unroll
    for (int q = 0; q < kXP; q++)
      acc[q] = q == kXP - 1 ? (uint32_t)dp4a_us(c, xr[kXP * v + q], (int32_t)acc[q]) : dp4a_uu(c, xr[kXP * v + q], acc[q]);
  };
  auto combine = [&](const uint32_t (&acc)[kXP]) {
    uint32_t t = acc[0];
#pragma unroll
    for (int q = 1; q < kXP; q++) t += acc[q] << (8 * q);
    return (int32_t)t;
  };
  if constexpr (BITS == 2) {
    // c0 = w & 0x03.. (channels 4L), c1 = w & 0x0C.. = 4 x (channels 4L+1),
    // the same on w >> 4 for 4L+2 and 4L+3: set A has factor 1, set B factor 4
    uint32_t A[ZW][kXP], B[ZW][kXP];
#pragma unroll
    for (int h = 0; h < ZW; h++)
#pragma unroll
      for (int q = 0; q < kXP; q++) A[h][q] = B[h][q] = 0;
#pragma unroll
    for (int wi = 0; wi < 4; wi++) {
      const int h = ZW == 2 ? (wi >> 1) : 0;
      const uint32_t w0 = w[wi], w4 = w0 >> 4;
      mac(w0 & 0x03030303u, 4 * wi + 0, A[h]);
      mac(w0 & 0x0C0C0C0Cu, 4 * wi + 1, B[h]);
      mac(w4 & 0x03030303u, 4 * wi + 2, A[h]);
      mac(w4 & 0x0C0C0C0Cu, 4 * wi + 3, B[h]);
    }
#pragma unroll
    for (int h = 0; h < ZW; h++) d[h] = combine(A[h]) + (combine(B[h]) >> 2);
  } else {
    uint32_t A[ZW][kXP];
#pragma unroll
    for (int h = 0; h < ZW; h++)
#pragma unroll
      for (int q = 0; q < kXP; q++) A[h][q] = 0;
#pragma unroll
    for (int v = 0; v < 16; v++) mac(code_vec<BITS>(w, v), v, A[ZW == 2 ? (chan_of<BITS>(v, 0) >= 32) : 0]);
#pragma unroll
    for (int h = 0; h < ZW; h++) d[h] = combine(A[h]);
  }
}

// Sum each of U per-lane values over the warp.  Returns the full sum of row
// lane >> 3 (U = 4) or lane >> 4 (U = 2) in every lane.
template <int U>
__device__ __forceinline__ float warp_sum_rows(float (&a)[U], int lane) {
  if constexpr (U == 4) {
    const bool up = lane & 16;
    float k0 = up ? a[2] : a[0], k1 = up ? a[3] : a[1];
    float s0 = up ? a[0] : a[2], s1 = up ? a[1] : a[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool up8 = lane & 8;
    float k = up8 ? k1 : k0, s = up8 ? k0 : k1;
    k += __shfl_xor_sync(0xffffffffu, s, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
  } else {
    const bool up = lane & 16;
    float k = up ? a[1] : a[0], s = up ? a[0] : a[1];
    k += __shfl_xor_sync(0xffffffffu, s, 16);
    k += __shfl_xor_sync(0xffffffffu, k, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;
  }
}

// ---------------------------------------------------------------------------
// correction table entries: (x_c, x_c (1 - off/2^r), group of c, word offset of
// the refinement row of c), off = 1/2 - 2^(r-1)

__device__ __forceinline__ uint4 make_jd(const GemvParams& p, int b, int j) {
  const int c = __ldg(p.sel + (size_t)b * p.n_sel + j);
  const float xc = h2f(__ldg(p.x + (size_t)b * p.K + c));
  const float cfac = 1.0f - (0.5f - 0.5f * (float)(1 << p.r)) / (float)(1 << p.r);
  const uint32_t off = p.staged ? (uint32_t)(((size_t)b * p.n_sel + j) * p.refine_row_words)
                                : (uint32_t)((size_t)c * p.refine_row_words);
  return make_uint4(__float_as_uint(xc), __float_as_uint(xc * cfac), (uint32_t)(c >> p.gshift), off);
}

// ---------------------------------------------------------------------------
// activation prologue: every CTA turns batch row b of x into the fixed-point
// byte planes of all K/64 lane groups in shared memory, one warp per group

template <int BITS>
__device__ void prep_planes(const GemvParams& p, int b, uint32_t* __restrict__ xs, int* __restrict__ scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ngrp = p.K / kLaneCh;
  // UNR groups per warp at a time (independent shuffle chains interleave); the
  // warp's scratch holds their 64 fixed-point values each, by (vector, byte)
  constexpr int UNR = 4;
  int* sw = scratch + warp * UNR * kLaneCh;
  auto slot_of = [](int c) {
    const int v = BITS == 4 ? 2 * (c >> 3) + (c & 1) : 4 * (c >> 4) + (c & 3);
    const int L = BITS == 4 ? (c >> 1) & 3 : (c >> 2) & 3;
    return 4 * v + L;
  };
  for (int g0 = warp; g0 < ngrp; g0 += UNR * kWarps) {
    uint32_t xw[UNR];
#pragma unroll
    for (int u = 0; u < UNR; u++) {
      const int grp = g0 + u * kWarps;
      xw[u] = grp < ngrp ? __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)b * p.K + (size_t)grp * kLaneCh) + lane)
                         : 0u;
    }
    float2 xv[UNR];
    float mx[UNR], sm[UNR];
#pragma unroll
    for (int u = 0; u < UNR; u++) {
      xv[u] = __half22float2(*reinterpret_cast<const __half2*>(&xw[u]));
      mx[u] = fmaxf(fabsf(xv[u].x), fabsf(xv[u].y));
      sm[u] = xv[u].x + xv[u].y;  // channels 2 lane, 2 lane + 1: halves are lanes 0-15, 16-31
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < UNR; u++) mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], o));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < UNR; u++) sm[u] += __shfl_xor_sync(0xffffffffu, sm[u], o);
    int eb[UNR];
    float s1[UNR];
#pragma unroll
    for (int u = 0; u < UNR; u++) {
      // x_fix = x 2^-e with e = ilogb(max |x|) - kXShift; every nonzero fp16 value
      // is a normal float, so the exponent and 2^-e come from the float bits (exact)
      eb[u] = (__float_as_int(mx[u]) >> 23) & 0xff;  // biased exponent; 0 only for max 0
      const float scale = eb[u] ? __int_as_float((254 + kXShift - eb[u]) << 23) : 0.f;
      sw[u * kLaneCh + slot_of(2 * lane)] = __float2int_rn(xv[u].x * scale);
      sw[u * kLaneCh + slot_of(2 * lane + 1)] = __float2int_rn(xv[u].y * scale);
      s1[u] = __shfl_sync(0xffffffffu, sm[u], 16);
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < UNR; u++) {
      const int grp = g0 + u * kWarps;
      if (grp < ngrp) {
        uint32_t* dst = xs + grp * kXWords;
        if (lane < 16) {  // lane v: plane q of vector v = byte q of its four values
          const int4 f = reinterpret_cast<const int4*>(sw + u * kLaneCh)[lane];
#pragma unroll
          for (int q = 0; q < kXP; q++) {
            const uint32_t sel = (uint32_t)q | ((uint32_t)(4 + q) << 4);
            const uint32_t t01 = __byte_perm((uint32_t)f.x, (uint32_t)f.y, sel);
            const uint32_t t23 = __byte_perm((uint32_t)f.z, (uint32_t)f.w, sel);
            dst[kXP * lane + q] = __byte_perm(t01, t23, 0x5410);
          }
        }
        if (lane == 0) {  // lane 0 holds the first half's sum, s1 the second's
          reinterpret_cast<float*>(dst)[kXR + 0] = sm[u];
          reinterpret_cast<float*>(dst)[kXR + 1] = s1[u];
          reinterpret_cast<float*>(dst)[kXR + 2] = eb[u] ? __int_as_float((eb[u] - kXShift) << 23) : 1.0f;
          reinterpret_cast<float*>(dst)[kXR + 3] = sm[u] + s1[u];
        }
      }
    }
    __syncwarp();  // the scratch is rewritten by the next groups
  }
}

// ---------------------------------------------------------------------------
// correction

// Table entries [j0, j0 + jn) of batch row b into jd, and the refinement words
// [w_lo, w_lo + nwr) of each entry's row into wt (stride nwr), by cp.async.
__device__ void corr_fill(const GemvParams& p, int b, int j0, int jn, int w_lo, int nwr, uint4* jd,
                          uint32_t* wt) {
  for (int i = threadIdx.x; i < jn; i += kThreads) {
    if (p.staged) {  // the staged row of entry j is known without the selection: copy it first
      const uint32_t off = (uint32_t)(((size_t)b * p.n_sel + j0 + i) * p.refine_row_words);
      for (int k = 0; k < nwr; k++) cp_async4(wt + (size_t)i * nwr + k, p.refine + off + w_lo + k);
      jd[i] = make_jd(p, b, j0 + i);
    } else {
      const uint4 d = make_jd(p, b, j0 + i);
      jd[i] = d;
      for (int k = 0; k < nwr; k++) cp_async4(wt + (size_t)i * nwr + k, p.refine + d.w + w_lo + k);
    }
  }
  cp_async_commit();
}

// Warp tasks of the correction: row blocks of 32 lanes x RL rows, times
// splits of the table entries.
__device__ __forceinline__ void corr_tasks(int rows, int RL, int& nblk, int& js_n) {
  nblk = (rows / RL + 31) / 32;
  js_n = nblk >= kWarps ? 1 : kWarps / nblk;
}

// The correction of table entries [0, jn): into cpart[js][row] (entry split
// js, stride rows_max; every row of every split written), or added into
// the correction column part[row][segs] when cpart is NULL.  Lanes own RL consecutive rows (inside one
// refinement word); warps split the entries.
// Entries come in ascending channel order, so channels of one scale group are
// consecutive: each run is summed unscaled and multiplied by s once.  szt:
// the CTA's (s, m) words group-major, [gpr][rows_max], so that the lanes of a
// warp (consecutive rows) read consecutive words; or NULL (scales read from
// global memory).
template <int RL>
__device__ void corr_process(const GemvParams& p, int n0, int rows, int w_lo, int nwr, int jn,
                             const uint4* __restrict__ jd, const uint32_t* __restrict__ wt,
                             const uint32_t* __restrict__ szt, float* part, float* cpart) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gpr = p.K >> p.gshift;
  const int units = rows / RL;
  int nblk, js_n;
  corr_tasks(rows, RL, nblk, js_n);
  const int ntasks = nblk * js_n;
  const int r = p.r;
  const uint32_t fmask = ((1u << r) - 1u) << (23 - r);
  for (int task = warp; task < ntasks; task += kWarps) {
    const int blk = task % nblk, js = task / nblk;
    const int qu = blk * 32 + lane;
    const bool ok = qu < units;
    const int rl0 = RL * qu;
    const int bit0 = (n0 + rl0) * r;
    const int wr = (bit0 >> 5) - w_lo;
    int rot[RL];
#pragma unroll
    for (int t = 0; t < RL; t++) rot[t] = (23 - r - ((bit0 & 31) + r * t)) & 31;
    const int ia = (int)((long)js * jn / js_n), ib = (int)((long)(js + 1) * jn / js_n);
    float acc[RL], run[RL];
#pragma unroll
    for (int t = 0; t < RL; t++) acc[t] = run[t] = 0.f;
    float C = 0.f;
    int gcur = -1;
    auto flush = [&]() {
      if (gcur >= 0 && ok) {
        // the lane's RL rows of group gcur are consecutive words of szt
        uint32_t zt[RL];
        if (szt) {
          const uint32_t* zp = szt + gcur * p.rows_max + rl0;
          if constexpr (RL == 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(zp);
            zt[0] = v.x, zt[1] = v.y, zt[2] = v.z, zt[3] = v.w;
          } else if constexpr (RL == 2) {
            const uint2 v = *reinterpret_cast<const uint2*>(zp);
            zt[0] = v.x, zt[1] = v.y;
          } else {
            zt[0] = zp[0];
          }
        }
#pragma unroll
        for (int t = 0; t < RL; t++) {
          const uint32_t zw = szt ? zt[t]
                                  : __ldg(reinterpret_cast<const uint32_t*>(p.sz) + (size_t)(n0 + rl0 + t) * gpr + gcur);
          const float sc = __low2float(*reinterpret_cast<const __half2*>(&zw));
          acc[t] = fmaf(sc, run[t] - C, acc[t]);
        }
      }
    };
    for (int i = ia; i < ib; i++) {
      const uint4 d = jd[i];
      if ((int)d.z != gcur) {
        flush();
        gcur = (int)d.z;
        C = 0.f;
#pragma unroll
        for (int t = 0; t < RL; t++) run[t] = 0.f;
      }
      const uint32_t w = ok ? wt[(size_t)i * nwr + wr] : 0u;
      const float xc = __uint_as_float(d.x);
      // f = 1 + rho / 2^r; sum x f - sum x (1 - off/2^r) = sum x (rho + off) / 2^r
#pragma unroll
      for (int t = 0; t < RL; t++)
        run[t] = fmaf(__uint_as_float(0x3F800000u | (__funnelshift_l(w, w, rot[t]) & fmask)), xc, run[t]);
      C += __uint_as_float(d.y);
    }
    flush();
    if (ok && cpart) {
#pragma unroll
      for (int t = 0; t < RL; t++) cpart[js * p.rows_max + rl0 + t] = acc[t];
    } else if (ok && ib > ia) {
#pragma unroll
      for (int t = 0; t < RL; t++) atomicAdd(&part[(rl0 + t) * p.pstride + p.segs], acc[t]);
    }
  }
}

__device__ __forceinline__ void corr_dispatch(const GemvParams& p, int n0, int rows, int w_lo, int nwr, int jn,
                                              const uint4* jd, const uint32_t* wt, const uint32_t* szt,
                                              float* part, float* cpart) {
  if (p.corr_rows == 4)
    corr_process<4>(p, n0, rows, w_lo, nwr, jn, jd, wt, szt, part, cpart);
  else if (p.corr_rows == 2)
    corr_process<2>(p, n0, rows, w_lo, nwr, jn, jd, wt, szt, part, cpart);
  else
    corr_process<1>(p, n0, rows, w_lo, nwr, jn, jd, wt, szt, part, cpart);
}

// ---------------------------------------------------------------------------
// the GEMV

// 120 registers x 512 threads: kSideRegs of the SM's registers stay free
static_assert(65536 - 120 * kThreads >= kSideRegs, "GEMV registers leave no room for a staging CTA");
template <int BITS, int ZW, int PD>
__global__ void __maxnreg__(120) gemv_kernel(GemvParams p) {
  using R = Ring<BITS, ZW>;
  constexpr int U = Lane<BITS>::U, CW = Lane<BITS>::CW;
  extern __shared__ __align__(16) uint32_t smem[];
  pdl_trigger();  // the next kernel of the stream may be scheduled; it waits for this grid
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int units = p.N / kRowUnit;
  const int n0 = (int)((long)blockIdx.x * units / gridDim.x) * kRowUnit;
  const int n1 = (int)((long)(blockIdx.x + 1) * units / gridDim.x) * kRowUnit;
  const int rows = n1 - n0;
  const int ngrp = p.K / kLaneCh, gpr = p.K >> p.gshift;
  // shared memory: partial sums [rows][segs] | rings | (fast) table, words, scales
  float* part = reinterpret_cast<float*>(smem);
  uint32_t* xs = smem + ((p.rows_max * p.pstride + 3) & ~3);  // activation planes [K/64][kXWords], prologue scratch
  uint32_t* area = xs + p.plane_words;
  uint4* jd_fast = reinterpret_cast<uint4*>(area + p.area_words);
  uint32_t* wt_fast = reinterpret_cast<uint32_t*>(jd_fast + p.n_sel);
  uint32_t* szt = wt_fast + (((size_t)p.n_sel * p.w_span + 3) & ~(size_t)3);
  const int w_lo = (n0 * p.r) >> 5;
  const int nwr = (((n1 * p.r) + 31) >> 5) - w_lo;
  const int steps = (rows + U - 1) / U, ntask = p.segs * steps;
  const int ta = (int)((long)warp * ntask / kWarps), tb = (int)((long)(warp + 1) * ntask / kWarps);
  const size_t row_bytes = (size_t)p.K * (BITS == 3 ? 2 : BITS) / 8;
  const bool fill_szt = p.fast && p.n_sel > 0;
  // the fast correction's per-warp partials: in the ring area, free once the base pass is done
  float* cpart = p.corr_split && p.fast && p.n_sel > 0 ? reinterpret_cast<float*>(area) : nullptr;

  for (int b = 0; b < p.batch; b++) {
    {
      // ---- base pass of batch row b: every (row, segment) partial is written once
      uint32_t* ring = area + warp * PD * R::words;
      int iseg = ta / steps, ist = ta - iseg * steps, islot = 0, left = tb - ta;
      auto issue = [&]() {
        if (left > 0) {
          const int lg = iseg * 32 + lane;
          if (lg < ngrp) {
            const uint8_t* lb = reinterpret_cast<const uint8_t*>(p.base) + 16 * R::C16 * lg;
            const uint8_t* lh = reinterpret_cast<const uint8_t*>(p.base) + (size_t)p.N * p.K / 4 + 8 * lg;
            const uint32_t* lz = reinterpret_cast<const uint32_t*>(p.sz) + ((lg * kLaneCh) >> p.gshift);
            uint32_t* slot = ring + islot * R::words;
            const int r0 = n0 + ist * U;
#pragma unroll
            for (int u = 0; u < U; u++) issue_row<BITS, ZW>(lb, lh, row_bytes, lz, gpr, r0 + u, slot, u, lane);
          }
          if (++ist == steps) ist = 0, ++iseg;
          --left;
        }
        islot = islot + 1 == PD ? 0 : islot + 1;
        cp_async_commit();
      };
#pragma unroll
      for (int i = 0; i < PD - 1; i++) issue();
      if (b == 0) pdl_wait();  // x, the selection and the staged rows are complete
      for (int i = threadIdx.x; i < rows; i += kThreads) part[i * p.pstride + p.segs] = 0.f;  // correction column
      prep_planes<BITS>(p, b, xs, reinterpret_cast<int*>(xs + ngrp * kXWords));
      if (p.fast && p.n_sel > 0) corr_fill(p, b, 0, p.n_sel, w_lo, nwr, jd_fast, wt_fast);
      __syncthreads();  // planes complete
      uint32_t xr[kXR];
      float xsum0 = 0.f, xsum1 = 0.f, xscale = 0.f;
      int cseg = ta / steps, cst = ta - cseg * steps, cslot = 0, cur = -1;
      for (int t = ta; t < tb; t++) {
        issue();
        const int lg = cseg * 32 + lane;
        const bool la = lg < ngrp;
        if (cseg != cur) {
          cur = cseg;
          if (la) {
            const uint4* src = reinterpret_cast<const uint4*>(xs + lg * kXWords);
#pragma unroll
            for (int k = 0; k < kXR / 4; k++) {
              const uint4 q = src[k];
              xr[4 * k + 0] = q.x, xr[4 * k + 1] = q.y, xr[4 * k + 2] = q.z, xr[4 * k + 3] = q.w;
            }
            const float4 f = reinterpret_cast<const float4*>(src)[kXR / 4];
            xsum0 = ZW == 2 ? f.x : f.w, xsum1 = f.y, xscale = f.z;
          } else {
#pragma unroll
            for (int k = 0; k < kXR; k++) xr[k] = 0;
            xsum0 = xsum1 = xscale = 0.f;
          }
        }
        cp_async_wait<PD - 1>();
        const uint32_t* slot = ring + cslot * R::words;
        const int r0 = n0 + cst * U;
        const int zg = (lg * kLaneCh) >> p.gshift;
        const bool zown = fill_szt && la && ((lg * kLaneCh) & (p.G - 1)) == 0;
        float acc[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
          acc[u] = 0.f;
          if (la) {
            uint32_t w[CW];
#pragma unroll
            for (int c = 0; c < R::C16; c++) {
              const uint4 q = *reinterpret_cast<const uint4*>(slot + ((u * R::C16 + c) * 32 + lane) * 4);
              w[4 * c + 0] = q.x, w[4 * c + 1] = q.y, w[4 * c + 2] = q.z, w[4 * c + 3] = q.w;
            }
            if constexpr (BITS == 3) {
              const uint2 h = *reinterpret_cast<const uint2*>(slot + R::hi_off() + (u * 32 + lane) * 2);
              w[4] = h.x, w[5] = h.y;
            }
            int32_t d[ZW];
            lane_dot<BITS, ZW>(w, xr, d);
            const uint32_t z0 = slot[R::z_off + (u * ZW) * 32 + lane];
            const float2 sm0 = __half22float2(*reinterpret_cast<const __half2*>(&z0));
            if constexpr (ZW == 1) {
              acc[u] = fmaf(sm0.x * xscale, (float)d[0], sm0.y * xsum0);
              if (zown) szt[zg * p.rows_max + (r0 + u - n0)] = z0;
            } else {
              const uint32_t z1 = slot[R::z_off + (u * ZW + 1) * 32 + lane];
              const float2 sm1 = __half22float2(*reinterpret_cast<const __half2*>(&z1));
              acc[u] = fmaf(sm0.x * xscale, (float)d[0],
                            fmaf(sm1.x * xscale, (float)d[1], fmaf(sm0.y, xsum0, sm1.y * xsum1)));
              if (fill_szt && la) szt[zg * p.rows_max + (r0 + u - n0)] = z0, szt[(zg + 1) * p.rows_max + (r0 + u - n0)] = z1;
            }
          }
        }
        const float tot = warp_sum_rows<U>(acc, lane);
        const int u = U == 4 ? (lane >> 3) : (lane >> 4);
        if ((lane & (32 / U - 1)) == 0) part[(r0 + u - n0) * p.pstride + cseg] = tot;
        if (++cst == steps) cst = 0, ++cseg;
        cslot = cslot + 1 == PD ? 0 : cslot + 1;
      }
      cp_async_wait<0>();
    }
    __syncthreads();

    // ---- correction of the selected channels of batch row b
    if (p.n_sel > 0) {
      if (p.fast) {
        corr_dispatch(p, n0, rows, w_lo, nwr, p.n_sel, jd_fast, wt_fast, szt, part, cpart);
      } else {
        // tables in chunks in the ring area; scales from global memory
        const int jcap = p.area_words / (4 + nwr);
        uint4* jd = reinterpret_cast<uint4*>(area);
        for (int j0 = 0; j0 < p.n_sel; j0 += jcap) {
          const int jn = min(jcap, p.n_sel - j0);
          uint32_t* wt = reinterpret_cast<uint32_t*>(jd + jn);
          corr_fill(p, b, j0, jn, w_lo, nwr, jd, wt);
          cp_async_wait<0>();
          __syncthreads();
          corr_dispatch(p, n0, rows, w_lo, nwr, jn, jd, wt, nullptr, part, nullptr);
          __syncthreads();
        }
      }
    }
    __syncthreads();

    int cjs = 0;  // entry splits of the correction partials in cpart
    if (cpart) {
      int nblk;
      corr_tasks(rows, p.corr_rows, nblk, cjs);
    }
    for (int row = n0 + threadIdx.x; row < n1; row += kThreads) {
      const float* pr = part + (row - n0) * p.pstride;
      float base = 0.f, corr = pr[p.segs];
      for (int s = 0; s < p.segs; s++) base += pr[s];
      for (int js = 0; js < cjs; js++) corr += cpart[js * p.rows_max + row - n0];
      float* dst = p.y + (size_t)b * p.N + row;
      if (p.y_corr) {
        *dst = base;
        p.y_corr[(size_t)b * p.N + row] = corr;
      } else {
        *dst = base + corr;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// the correction on its own (fetch lag), added into y
//
// A thread owns 8 consecutive output rows of one batch row and walks every
// selected channel in order, so the sum is deterministic: per channel it reads
// the refinement word that covers its rows (consecutive threads read
// consecutive words), adds x_c f_t, f_t = 1 + rho_t / 2^r, into a per-row run,
// and scales each run of channels that share a scale group once,
// s (run - sum x_c cfac) = s sum x_c (rho + off) / 2^r.  CTAs of 64 threads,
// at most 64 registers and no shared memory fit in the room every whole-SM
// kernel of the library leaves free, so on a staging stream the correction
// neither waits for them nor delays them.

constexpr int kCorrThreads = 64;
constexpr int kCorrRows = 8;
static_assert(kCorrThreads * 64 <= kSideRegs, "a correction CTA must fit in the room left for staging");

struct CorrArgs {
  const uint32_t* refine;  // channel-major rows [K][row_words], or staged rows [batch][n_sel][row_words]
  const uint16_t* sz;
  const uint16_t* x;
  const int32_t* sel;
  float* y;
  int N, K, gshift, r, n_sel, row_words, staged, units;  // units = batch * N / kCorrRows
};

template <int R>
__global__ void __maxnreg__(64) corr_only_kernel(CorrArgs a) {
  const int u = blockIdx.x * kCorrThreads + threadIdx.x;
  if (u >= a.units) return;
  const int per_b = a.N / kCorrRows;
  const int b = u / per_b, row0 = (u - b * per_b) * kCorrRows;
  const int bit0 = row0 * a.r, wi = bit0 >> 5;
  const int gpr = a.K >> a.gshift;
  // the rows' bits start at bit sh of the word (a multiple of 8); the word is
  // shifted down first, so row t's field sits at bit R t
  const int sh = bit0 & 31;
  constexpr uint32_t fmask = ((1u << R) - 1u) << (23 - R);
  const float cfac = 1.0f - (0.5f - 0.5f * (float)(1 << R)) / (float)(1 << R);
  const uint32_t* zrow = reinterpret_cast<const uint32_t*>(a.sz) + (size_t)row0 * gpr;
  const int32_t* sel = a.sel + (size_t)b * a.n_sel;
  const uint16_t* xb = a.x + (size_t)b * a.K;
  float acc[kCorrRows], run[kCorrRows];
#pragma unroll
  for (int t = 0; t < kCorrRows; t++) acc[t] = run[t] = 0.f;
  float C = 0.f;
  int gcur = -1;
  auto flush = [&]() {
    if (gcur >= 0) {
#pragma unroll
      for (int t = 0; t < kCorrRows; t++) {
        const uint32_t zw = __ldg(zrow + (size_t)t * gpr + gcur);
        acc[t] = fmaf(__low2float(*reinterpret_cast<const __half2*>(&zw)), run[t] - C, acc[t]);
      }
    }
  };
  auto word_of = [&](int j, int c) {
    const size_t row = a.staged ? (size_t)b * a.n_sel + j : (size_t)c;
    return __ldg(a.refine + row * a.row_words + wi) >> sh;
  };
  // channel j + 1's index, activation and word are loaded while j is summed
  int c = a.n_sel > 0 ? __ldg(sel) : 0;
  float xc = a.n_sel > 0 ? h2f(__ldg(xb + c)) : 0.f;
  uint32_t w = a.n_sel > 0 ? word_of(0, c) : 0u;
  for (int j = 0; j < a.n_sel; j++) {
    const int cn = j + 1 < a.n_sel ? __ldg(sel + j + 1) : 0;
    const float xn = j + 1 < a.n_sel ? h2f(__ldg(xb + cn)) : 0.f;
    const uint32_t wn = j + 1 < a.n_sel ? word_of(j + 1, cn) : 0u;
    const int g = c >> a.gshift;
    if (g != gcur) {
      flush();
      gcur = g, C = 0.f;
#pragma unroll
      for (int t = 0; t < kCorrRows; t++) run[t] = 0.f;
    }
#pragma unroll
    for (int t = 0; t < kCorrRows; t++)
      run[t] = fmaf(__uint_as_float(0x3F800000u | (__funnelshift_l(w, w, (23 - R - R * t) & 31) & fmask)), xc,
                    run[t]);
    C = fmaf(xc, cfac, C);
    c = cn, xc = xn, w = wn;
  }
  flush();
  float4* yv = reinterpret_cast<float4*>(a.y + (size_t)b * a.N + row0);
#pragma unroll
  for (int q = 0; q < kCorrRows / 4; q++) {
    float4 v = yv[q];
    v.x += acc[4 * q], v.y += acc[4 * q + 1], v.z += acc[4 * q + 2], v.w += acc[4 * q + 3];
    yv[q] = v;
  }
}

// ---------------------------------------------------------------------------
// host side

size_t slot_words(int bits, int zw) {
  if (bits == 2) return zw == 1 ? Ring<2, 1>::words : Ring<2, 2>::words;
  if (bits == 3) return zw == 1 ? Ring<3, 1>::words : Ring<3, 2>::words;
  return zw == 1 ? Ring<4, 1>::words : Ring<4, 2>::words;
}

template <int BITS, int ZW>
void* kernel_for(int pd) {
  if (pd == 4) return (void*)gemv_kernel<BITS, ZW, 4>;
  if (pd == 3) return (void*)gemv_kernel<BITS, ZW, 3>;
  return (void*)gemv_kernel<BITS, ZW, 2>;
}

// Rows per lane in the correction: the fewest warp steps, counting ~6 + 3 RL
// instructions per step of RL rows.
int pick_corr_rows(int rows) {
  int best = 1;
  long best_cost = -1;
  for (int rl = 1; rl <= 4; rl *= 2) {
    const long blocks = (rows / rl + 31) / 32;
    const long cost = blocks * (6 + 3 * rl);
    if (best_cost < 0 || cost < best_cost) best = rl, best_cost = cost;
  }
  return best;
}

sf_status gemv_launch(const sf_wq* w, const uint16_t* x, int batch, int chunk, int kch,
                      const int32_t* sel_in, int32_t* sel_out, const void* refine_rows, float* y,
                      cudaStream_t s, float* y_corr = nullptr) {
  sf_status st = check_wq_public(w, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(x && aligned16(x), "x must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(y && aligned16(y), "y must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(batch >= 1 && batch <= 8, "batch=%d outside [1, 8]", batch);
  SF_REQUIRE(kch >= 0, "kch=%d < 0", kch);
  int n_sel = 0;
  if (kch > 0) {
    st = check_select_args(x, batch, w->k, chunk, kch);
    if (st != SF_OK) return st;
    n_sel = (w->k / chunk) * kch;
    SF_REQUIRE(refine_rows || w->refine, "kch > 0 needs w->refine or staged refine_rows");
    SF_REQUIRE(!refine_rows || aligned16(refine_rows), "refine_rows must be 16-byte aligned");
    if (sel_in) {
      SF_REQUIRE(aligned16(sel_in), "sel_in must be 16-byte aligned");
    } else {
      SF_REQUIRE(sel_out && aligned16(sel_out), "sel_out is needed when sel_in is NULL");
    }
  }

  GemvParams p = {};
  p.base = (const uint32_t*)w->base;
  p.refine = (const uint32_t*)(refine_rows ? refine_rows : w->refine);
  p.sz = w->sz;
  p.x = x;
  p.y = y;
  p.y_corr = y_corr;
  p.N = w->n, p.K = w->k, p.G = w->group, p.r = w->r, p.batch = batch, p.n_sel = n_sel;
  p.gshift = 0;
  while ((1 << p.gshift) < w->group) p.gshift++;
  p.segs = (w->k + kSegChannels - 1) / kSegChannels;
  p.refine_row_words = w->n * w->r / 32;
  p.staged = refine_rows != nullptr;

  const int zw = w->group == 32 ? 2 : 1;
  int grid = num_sms();
  const int units = w->n / kRowUnit;
  if (grid > units) grid = units;
  p.rows_max = ((units + grid - 1) / grid) * kRowUnit;
  p.w_span = p.rows_max * w->r / 32 + 2;
  p.corr_rows = pick_corr_rows(p.rows_max);
  p.plane_words = (w->k / kLaneCh) * kXWords + kWarps * 4 * kLaneCh;  // planes, then per-warp scratch
  const size_t gpr = (size_t)(w->k / w->group);
  p.pstride = p.segs + 1;
  const size_t part_words = ((size_t)p.rows_max * p.pstride + 3) & ~(size_t)3;
  const size_t table_words = (size_t)n_sel * 4 + (((size_t)n_sel * p.w_span + 3) & ~(size_t)3) +
                             (size_t)p.rows_max * gpr;
  const size_t limit_words = kSmemLimit / 4;
  const size_t fixed = part_words + p.plane_words;
  // ring depth: the deepest that leaves room for the correction tables, else
  // the deepest that fits (the tables then go through the ring area in chunks)
  int pd = 0;
  size_t area = 0;
  for (int d = (w->b == 3 ? 3 : 4); d >= 2 && !pd; d--) {
    const size_t ring = (size_t)kWarps * d * slot_words(w->b, zw);
    if (fixed + ring + (n_sel > 0 ? table_words : 0) <= limit_words) pd = d, area = ring, p.fast = n_sel > 0;
  }
  for (int d = (w->b == 3 ? 3 : 4); d >= 2 && !pd; d--) {
    const size_t ring = (size_t)kWarps * d * slot_words(w->b, zw);
    if (fixed + ring <= limit_words) pd = d, area = ring, p.fast = 0;
  }
  SF_UNSUPPORTED(pd > 0, "n=%d, k=%d does not fit in shared memory", w->n, w->k);
  p.corr_split = p.fast && area >= (size_t)kWarps * p.rows_max;
  if (!p.fast && n_sel > 0)
    SF_UNSUPPORTED(area >= (size_t)(4 + p.w_span) * 16, "n=%d, k=%d: no room for the correction", w->n, w->k);
  const size_t smem = (fixed + area + (p.fast ? table_words : 0)) * 4;
  SF_UNSUPPORTED(smem <= kSmemLimit, "n=%d, k=%d needs %zu bytes of shared memory", w->n, w->k, smem);
  p.area_words = (int)area;

  // the selection (when not given), then the GEMV, which waits for it (and for
  // x) through programmatic dependent launch while its first code copies fly
  if (kch > 0 && !sel_in) {
    st = launch_select(x, batch, w->k, chunk, kch, sel_out, s, true);
    if (st != SF_OK) return st;
    p.sel = sel_out;
  } else {
    p.sel = sel_in;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* kern;
  if (w->b == 2)
    kern = zw == 1 ? kernel_for<2, 1>(pd) : kernel_for<2, 2>(pd);
  else if (w->b == 3)
    kern = zw == 1 ? kernel_for<3, 1>(pd) : kernel_for<3, 2>(pd);
  else
    kern = zw == 1 ? kernel_for<4, 1>(pd) : kernel_for<4, 2>(pd);
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit));
  void* args[] = {&p};
  SF_CUDA(cudaLaunchKernelExC(&cfg, kern, args));
  return SF_OK;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_gemv_workspace_bytes(const sf_wq* w, int batch, int chunk, int kch) {
  (void)w, (void)batch, (void)chunk, (void)kch;
  return 0;
}

extern "C" sf_status sf_gemv_refined(const sf_wq* w, const uint16_t* x, int batch, int chunk,
                                     int kch, const int32_t* sel_in, int32_t* sel_out,
                                     const void* refine_rows, float* y, void* ws, size_t ws_bytes,
                                     sf_stream_t stream) {
  (void)ws, (void)ws_bytes;
  return gemv_launch(w, x, batch, chunk, kch, sel_in, sel_out, refine_rows, y, as_stream(stream));
}

extern "C" sf_status sf_gemv_correction(const sf_wq* w, const uint16_t* x, int batch, int chunk,
                                        int kch, const int32_t* sel, const void* refine_rows,
                                        float* y, sf_stream_t stream) {
  sf_status st = check_wq_public(w, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(kch >= 0, "kch=%d < 0", kch);
  if (kch == 0) return SF_OK;  // nothing to correct
  SF_REQUIRE(sel && aligned16(sel), "sel must be non-null and 16-byte aligned");
  SF_REQUIRE(y && aligned16(y), "y must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(batch >= 1 && batch <= 8, "batch=%d outside [1, 8]", batch);
  st = check_select_args(x, batch, w->k, chunk, kch);
  if (st != SF_OK) return st;
  SF_REQUIRE(refine_rows || w->refine, "the correction needs w->refine or staged refine_rows");
  SF_REQUIRE(!refine_rows || aligned16(refine_rows), "refine_rows must be 16-byte aligned");
  CorrArgs a;
  a.refine = (const uint32_t*)(refine_rows ? refine_rows : w->refine);
  a.sz = w->sz, a.x = x, a.sel = sel, a.y = y;
  a.N = w->n, a.K = w->k, a.r = w->r;
  a.gshift = 0;
  while ((1 << a.gshift) < w->group) a.gshift++;
  a.n_sel = (w->k / chunk) * kch;
  a.row_words = w->n * w->r / 32;
  a.staged = refine_rows != nullptr;
  a.units = batch * (w->n / kCorrRows);
  // a plain launch: on a staging stream it follows an event wait
  const int blocks = (a.units + kCorrThreads - 1) / kCorrThreads;
  if (a.r == 2)
    corr_only_kernel<2><<<blocks, kCorrThreads, 0, as_stream(stream)>>>(a);
  else
    corr_only_kernel<1><<<blocks, kCorrThreads, 0, as_stream(stream)>>>(a);
  SF_LAUNCHED();
  return SF_OK;
}

extern "C" sf_status sf_gemv_refined_split(const sf_wq* w, const uint16_t* x, int batch, int chunk,
                                           int kch, const int32_t* sel_in, const void* refine_rows,
                                           float* y_base, float* y_corr, sf_stream_t stream) {
  SF_REQUIRE(kch >= 1, "kch=%d: the split form needs a correction (kch >= 1)", kch);
  SF_REQUIRE(sel_in && aligned16(sel_in), "sel_in must be non-null and 16-byte aligned");
  SF_REQUIRE(y_corr && aligned16(y_corr), "y_corr must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(w && batch >= 1, "null weights or batch < 1");
  const size_t bytes = (size_t)batch * (size_t)w->n * sizeof(float);
  const char *a0 = (const char*)y_base, *b0 = (const char*)y_corr;
  SF_REQUIRE(!y_base || a0 + bytes <= b0 || b0 + bytes <= a0, "y_base and y_corr overlap");
  return gemv_launch(w, x, batch, chunk, kch, sel_in, nullptr, refine_rows, y_base, as_stream(stream), y_corr);
}
