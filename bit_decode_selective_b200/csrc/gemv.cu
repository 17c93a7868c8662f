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
//     correction-only mode below computes it on its own.
//
// Decomposition, per output row i (fp32 accumulation):
//   y_i = sum_groups [ s_ig * sum_{c in g} x_c q_ic + m_ig * sum_{c in g} x_c ]
//       + sum_{c selected} x_c * s_i,g(c) * (2 rho_ic + 1 - 2^r) / 2^(r+1)
//
// Base pass (HBM-bound: every resident code is read once).  Each CTA owns a
// contiguous range of rows; each warp owns one 2,048-channel segment of K and
// keeps that segment's activations in registers as exact fixed point: per
// 64-channel lane group x = x_fix * 2^e with |x_fix| < 2^23, split into three
// byte planes.  A lane streams 64 channels of a row per step (16 B of 2-bit
// codes), expands them to byte vectors with shifts and masks and takes the
// integer dot products with dp4a (4 code x byte products per instruction).
// Rows are prefetched one step ahead in registers; partial sums of four rows
// are reduced across the warp with a transposed butterfly.
//
// Correction pass: after griddepcontrol.wait (the selection kernel may still
// be running while the base pass streams), the CTA stages the selected
// channels' activations and the refinement words covering its rows in shared
// memory with independent loads, then one warp per row sums the corrections.
#include "common.cuh"
#include "internal.cuh"

namespace sf {
namespace {

constexpr int kSegChannels = 2048;  // 32 lanes x 64 channels
constexpr int kWarps = 8;
constexpr int kCtasPerSm = 2;
constexpr int kXWords = 52;         // per 64-channel group: 16 vectors x 3 planes, sum, 2^e, pad
constexpr int kCorrSmemWords = 12 * 1024;

struct GemvParams {
  const uint32_t* base;
  const uint32_t* refine;  // channel-major rows, or staged rows
  const uint16_t* sz;
  const uint16_t* x;
  const int32_t* sel;
  float* y;
  int N, K, G, r, batch, n_sel, segs, row_warps;
  int refine_row_words;  // N * r / 32
  int staged;            // refine holds [batch][n_sel] staged rows
  int mode;              // 0: base + correction, 1: correction only, added into y
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

// Words of packed codes per lane per row (64 channels).
template <int BITS>
struct Lane {
  static constexpr int W = BITS == 2 ? 4 : BITS == 3 ? 6 : 8;
  static constexpr int U = BITS == 4 ? 2 : 4;  // rows per step
};

// Ring slot layout (per warp, words): codes [U][W/4 chunks][32 lanes][4 words]
// (b = 3: then [U][32 lanes][2 words] of high bits), then sz [U][2][32 lanes].
// Consecutive lanes read consecutive 16-byte chunks, so reads are conflict-free.
template <int BITS>
struct Ring {
  static constexpr int W = Lane<BITS>::W, U = Lane<BITS>::U;
  static constexpr int CW = BITS == 3 ? 4 : W;           // words in 16-byte chunks
  static constexpr int slot_words = U * 32 * (W + 2);   // one item of U rows
};

template <int BITS>
__device__ __forceinline__ void issue_row(const GemvParams& p, int row, int lg, int gpr, int g0,
                                          int g1, uint32_t* slot, int u, int lane) {
  using R = Ring<BITS>;
  const uint8_t* rowbase;
  if constexpr (BITS == 4) {
    rowbase = reinterpret_cast<const uint8_t*>(p.base + (size_t)row * (p.K / 8)) + 32 * lg;
  } else {
    rowbase = reinterpret_cast<const uint8_t*>(p.base + (size_t)row * (p.K / 16)) + 16 * lg;
  }
#pragma unroll
  for (int c = 0; c < R::CW / 4; c++)
    cp_async16(slot + ((u * (R::CW / 4) + c) * 32 + lane) * 4, rowbase + 16 * c);
  if constexpr (BITS == 3) {
    const uint8_t* hb = reinterpret_cast<const uint8_t*>(p.base + (size_t)p.N * p.K / 16 +
                                                         (size_t)row * (p.K / 32)) + 8 * lg;
    cp_async8(slot + R::U * R::CW * 32 + (u * 32 + lane) * 2, hb);
  }
  uint32_t* zs = slot + R::U * 32 * R::W;
  const uint32_t* szrow = reinterpret_cast<const uint32_t*>(p.sz) + (size_t)row * gpr;
  cp_async4(zs + (u * 2 + 0) * 32 + lane, szrow + g0);
  if (g1 != g0) cp_async4(zs + (u * 2 + 1) * 32 + lane, szrow + g1);
}

template <int BITS>
__device__ __forceinline__ void read_row(const uint32_t* slot, int u, int lane,
                                         uint32_t (&w)[Lane<BITS>::W], uint32_t (&z)[2], bool split) {
  using R = Ring<BITS>;
#pragma unroll
  for (int c = 0; c < R::CW / 4; c++) {
    const uint4 v = *reinterpret_cast<const uint4*>(slot + ((u * (R::CW / 4) + c) * 32 + lane) * 4);
    w[4 * c + 0] = v.x, w[4 * c + 1] = v.y, w[4 * c + 2] = v.z, w[4 * c + 3] = v.w;
  }
  if constexpr (BITS == 3) {
    const uint2 h = *reinterpret_cast<const uint2*>(slot + R::U * R::CW * 32 + (u * 32 + lane) * 2);
    w[4] = h.x, w[5] = h.y;
  }
  const uint32_t* zs = slot + R::U * 32 * R::W;
  z[0] = zs[(u * 2 + 0) * 32 + lane];
  z[1] = split ? zs[(u * 2 + 1) * 32 + lane] : z[0];
}

// Code byte-vector v (0..15) of the lane's 64 channels; byte L holds the code
// of channel chan_of(v, L) (0..63).
template <int BITS>
__device__ __forceinline__ uint32_t code_vec(const uint32_t (&w)[Lane<BITS>::W], int v) {
  if constexpr (BITS == 4) {
    return (w[v >> 1] >> (4 * (v & 1))) & 0x0F0F0F0Fu;  // word v/2: 8 channels
  } else {
    const int wi = v >> 2, j = v & 3;  // word wi: 16 channels
    uint32_t c = (w[wi] >> (2 * j)) & 0x03030303u;
    if constexpr (BITS == 3) {
      const int sh = 4 * (wi & 1) + j;  // high bits of the 32-channel block wi/2
      c |= ((w[4 + (wi >> 1)] >> sh) << 2) & 0x04040404u;
    }
    return c;
  }
}

template <int BITS>
__host__ __device__ __forceinline__ int chan_of(int v, int L) {
  if (BITS == 4) return 8 * (v >> 1) + (v & 1) + 2 * L;
  return 16 * (v >> 2) + (v & 3) + 4 * L;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum each of U per-lane values over the warp; lane (u * 32 / U) .. holds row u.
// Returns the full sum of row (lane >> (5 - log2 U)) in every lane.
template <int U>
__device__ __forceinline__ float warp_sum_rows(float (&a)[U], int lane) {
  if constexpr (U == 4) {
    // xor 16: lanes < 16 keep rows 0,1; lanes >= 16 keep rows 2,3
    const bool up = lane & 16;
    float k0 = up ? a[2] : a[0], k1 = up ? a[3] : a[1];
    float s0 = up ? a[0] : a[2], s1 = up ? a[1] : a[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    // xor 8: keep one row
    const bool up8 = lane & 8;
    float k = up8 ? k1 : k0, s = up8 ? k0 : k1;
    k += __shfl_xor_sync(0xffffffffu, s, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;  // row 2*(lane>>4) + ((lane>>3)&1) = lane >> 3
  } else {
    const bool up = lane & 16;
    float k = up ? a[1] : a[0], s = up ? a[0] : a[1];
    k += __shfl_xor_sync(0xffffffffu, s, 16);
    k += __shfl_xor_sync(0xffffffffu, k, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    return k;  // row lane >> 4
  }
}

// x of one batch row -> fixed-point byte planes per 64-channel group.
template <int BITS>
__device__ void prep_x(const uint16_t* __restrict__ x, int K, uint16_t* xraw, uint32_t* xs) {
  // all loads first (16 B per thread per step), then the per-group work
  for (int i = threadIdx.x; i < K / 8; i += blockDim.x)
    reinterpret_cast<uint4*>(xraw)[i] = __ldg(reinterpret_cast<const uint4*>(x) + i);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  uint8_t* xb = reinterpret_cast<uint8_t*>(xs);
  for (int grp = warp; grp < K / 64; grp += nwarps) {
    // lane handles channels 2*lane, 2*lane + 1 of the group
    __half2 hv = reinterpret_cast<const __half2*>(xraw + grp * 64)[lane];
    float2 xv = __half22float2(hv);
    float mx = fmaxf(fabsf(xv.x), fabsf(xv.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const int e = mx > 0.f ? ilogbf(mx) - 22 : 0;  // |x| * 2^-e < 2^23
    uint8_t* base = xb + (size_t)grp * kXWords * 4;
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int c = 2 * lane + h;
      const float xc = h ? xv.y : xv.x;
      const int xf = mx > 0.f ? __float2int_rn(ldexpf(xc, -e)) : 0;
      int v, L;
      if (BITS == 4) {
        v = 2 * (c >> 3) + (c & 1);
        L = (c & 7) >> 1;
      } else {
        v = 4 * (c >> 4) + (c & 3);
        L = (c & 15) >> 2;
      }
      uint8_t* dst = base + v * 12 + L;
      dst[0] = (uint8_t)(xf & 0xff);
      dst[4] = (uint8_t)((xf >> 8) & 0xff);
      dst[8] = (uint8_t)((xf >> 16) & 0xff);
    }
    float s = warp_sum(xv.x + xv.y);
    if (lane == 0) {
      reinterpret_cast<float*>(base)[48] = s;
      reinterpret_cast<float*>(base)[49] = ldexpf(1.0f, e);
    }
  }
}

template <int BITS>
__device__ __forceinline__ float group_dot(const uint32_t (&w)[Lane<BITS>::W], const uint32_t (&xr)[48]) {
  uint32_t lo = 0, mid = 0;
  int32_t hi = 0;
#pragma unroll
  for (int v = 0; v < 16; v++) {
    uint32_t c = code_vec<BITS>(w, v);
    lo = dp4a_uu(c, xr[3 * v + 0], lo);
    mid = dp4a_uu(c, xr[3 * v + 1], mid);
    hi = dp4a_us(c, xr[3 * v + 2], hi);
  }
  return fmaf((float)hi, 65536.0f, (float)mid * 256.0f + (float)lo);
}

// Same, split into the two 32-channel halves (groups of 32 channels).
template <int BITS>
__device__ __forceinline__ float2 group_dot_halves(const uint32_t (&w)[Lane<BITS>::W],
                                                   const uint32_t (&xr)[48]) {
  uint32_t lo[2] = {0, 0}, mid[2] = {0, 0};
  int32_t hi[2] = {0, 0};
#pragma unroll
  for (int v = 0; v < 16; v++) {
    const int h = chan_of<BITS>(v, 0) >= 32;
    uint32_t c = code_vec<BITS>(w, v);
    lo[h] = dp4a_uu(c, xr[3 * v + 0], lo[h]);
    mid[h] = dp4a_uu(c, xr[3 * v + 1], mid[h]);
    hi[h] = dp4a_us(c, xr[3 * v + 2], hi[h]);
  }
  return make_float2(fmaf((float)hi[0], 65536.0f, (float)mid[0] * 256.0f + (float)lo[0]),
                     fmaf((float)hi[1], 65536.0f, (float)mid[1] * 256.0f + (float)lo[1]));
}

template <int BITS, int PD>
__global__ void __launch_bounds__(kWarps * 32, kCtasPerSm) gemv_kernel(GemvParams p) {
  constexpr int W = Lane<BITS>::W, U = Lane<BITS>::U;
  extern __shared__ __align__(16) uint32_t smem[];
  const int ngrp = p.K / 64;
  uint32_t* xs = smem;                                       // ngrp * kXWords
  float* part = reinterpret_cast<float*>(xs + ngrp * kXWords);  // rows x segs
  const int n0 = (int)((long)blockIdx.x * p.N / gridDim.x);
  const int n1 = (int)((long)(blockIdx.x + 1) * p.N / gridDim.x);
  const int rows = n1 - n0;
  // scratch: x staging (prologue), then the per-warp copy rings (base pass),
  // then the correction staging
  uint32_t* scratch = reinterpret_cast<uint32_t*>(part + ((rows * p.segs + 3) & ~3));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = warp % p.segs, rw = warp / p.segs;
  const bool warp_active = p.mode == 0 && rw < p.row_warps;
  const int lg = seg * 32 + lane;  // lane's 64-channel group
  const bool lane_active = warp_active && lg < ngrp;
  const int G = p.G;
  const bool split = G == 32;

  for (int b = 0; b < p.batch; b++) {
    const uint16_t* xrow = p.x + (size_t)b * p.K;
    if (p.mode == 0) {
      // every (row, segment) partial is written by exactly one warp below
      prep_x<BITS>(xrow, p.K, reinterpret_cast<uint16_t*>(scratch), xs);
    } else {
      for (int i = threadIdx.x; i < rows * p.segs; i += blockDim.x) part[i] = 0.f;
    }
    __syncthreads();
    if (warp_active) {
      uint32_t xr[48];
      float xsum = 0.f, xscale = 0.f;
      if (lane_active) {
        const uint4* src = reinterpret_cast<const uint4*>(xs + lg * kXWords);
#pragma unroll
        for (int i = 0; i < 12; i++) {
          uint4 v = src[i];
          xr[4 * i + 0] = v.x, xr[4 * i + 1] = v.y, xr[4 * i + 2] = v.z, xr[4 * i + 3] = v.w;
        }
        xsum = __uint_as_float(xs[lg * kXWords + 48]);
        xscale = __uint_as_float(xs[lg * kXWords + 49]);
      } else {
#pragma unroll
        for (int i = 0; i < 48; i++) xr[i] = 0;
      }
      // sums of x over the two 32-channel halves (groups of 32 only)
      float xs0 = 0.f, xs1 = 0.f;
      if (split && lane_active) {
        const __half2* xh = reinterpret_cast<const __half2*>(xrow + lg * 64);
        for (int i = 0; i < 16; i++) {
          float2 a = __half22float2(xh[i]), c = __half22float2(xh[16 + i]);
          xs0 += a.x + a.y;
          xs1 += c.x + c.y;
        }
      }
      const int gpr = p.K / G;
      const int g0 = (lg * 64) / G, g1 = (lg * 64 + 32) / G;
      const int step = p.row_warps * U;
      const int first = n0 + rw * U;
      const int nitems = first < n1 ? (n1 - first + step - 1) / step : 0;
      uint32_t* ring = scratch + warp * PD * Ring<BITS>::slot_words;
      auto issue = [&](int k) {
        if (k < nitems && lane_active) {
          uint32_t* slot = ring + (k % PD) * Ring<BITS>::slot_words;
#pragma unroll
          for (int u = 0; u < U; u++) {
            const int row = first + k * step + u;
            if (row < n1) issue_row<BITS>(p, row, lg, gpr, g0, g1, slot, u, lane);
          }
        }
        cp_async_commit();
      };
#pragma unroll
      for (int k = 0; k < PD - 1; k++) issue(k);
      for (int k = 0; k < nitems; k++) {
        issue(k + PD - 1);
        cp_async_wait<PD - 1>();
        const uint32_t* slot = ring + (k % PD) * Ring<BITS>::slot_words;
        const int i0 = first + k * step;
        float acc[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
          acc[u] = 0.f;
          if (lane_active && i0 + u < n1) {
            uint32_t w[W], z[2];
            read_row<BITS>(slot, u, lane, w, z, split);
            float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&z[0]));
            if (!split) {
              const float d = group_dot<BITS>(w, xr) * xscale;
              acc[u] = fmaf(s0.x, d, s0.y * xsum);
            } else {
              float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&z[1]));
              const float2 d = group_dot_halves<BITS>(w, xr);
              acc[u] = fmaf(s0.x, d.x * xscale, fmaf(s1.x, d.y * xscale, fmaf(s0.y, xs0, s1.y * xs1)));
            }
          }
        }
        const float tot = warp_sum_rows<U>(acc, lane);
        const int u = U == 4 ? (lane >> 3) : (lane >> 4);
        const int row = i0 + u;
        if ((lane & (32 / U - 1)) == 0 && row < n1) part[(row - n0) * p.segs + seg] = tot;
      }
      cp_async_wait<0>();
    }
    __syncthreads();

    // ---- correction of the selected channels of batch row b
    if (p.n_sel > 0) {
      pdl_wait();  // selection (and staged rows) complete and visible
      const int32_t* sel = p.sel + (size_t)b * p.n_sel;
      const int w0 = (n0 * p.r) >> 5;
      const int nw = (((n1 * p.r) + 31) >> 5) - w0;
      const float half = 0.5f * (float)(1 << p.r), inv = 1.0f / (float)(1 << p.r);
      const int per_sel = 2 + nw;
      const bool staged_smem = (long)p.n_sel * per_sel <= kCorrSmemWords;
      if (staged_smem) {
        // [n_sel] x * 2^-r, [n_sel] group, [n_sel][nw] refinement words
        float* cx = reinterpret_cast<float*>(scratch);
        int* cg = reinterpret_cast<int*>(cx + p.n_sel);
        uint32_t* cw = reinterpret_cast<uint32_t*>(cg + p.n_sel);
        for (int j = threadIdx.x; j < p.n_sel; j += blockDim.x) {
          const int c = __ldg(sel + j);
          cx[j] = h2f(__ldg(xrow + c)) * inv;
          cg[j] = c / G;
        }
        for (int i = threadIdx.x; i < p.n_sel * nw; i += blockDim.x) {
          const int j = i / nw, k = i % nw;
          const uint32_t* rrow = p.staged ? p.refine + ((size_t)b * p.n_sel + j) * p.refine_row_words
                                          : p.refine + (size_t)__ldg(sel + j) * p.refine_row_words;
          cw[j * nw + k] = __ldg(rrow + w0 + k);
        }
        __syncthreads();
        const int nwarps = blockDim.x >> 5;
        for (int row = n0 + warp; row < n1; row += nwarps) {
          const int bit = row * p.r - w0 * 32;
          const uint16_t* zr = p.sz + (size_t)row * (p.K / G) * 2;
          float corr = 0.f;
          for (int j = lane; j < p.n_sel; j += 32) {
            const uint32_t rho = (cw[j * nw + (bit >> 5)] >> (bit & 31)) & ((1u << p.r) - 1);
            const float s = h2f(__ldg(zr + 2 * cg[j]));
            corr = fmaf(cx[j] * s, (float)rho + 0.5f - half, corr);
          }
          corr = warp_sum(corr);
          if (lane == 0) part[(row - n0) * p.segs] += corr;
        }
      } else {
        const int nwarps = blockDim.x >> 5;
        for (int row = n0 + warp; row < n1; row += nwarps) {
          float corr = 0.f;
          const int rbit = row * p.r;
          for (int j = lane; j < p.n_sel; j += 32) {
            const int c = __ldg(sel + j);
            const uint32_t* rrow = p.staged ? p.refine + ((size_t)b * p.n_sel + j) * p.refine_row_words
                                            : p.refine + (size_t)c * p.refine_row_words;
            const uint32_t rho = (__ldg(rrow + (rbit >> 5)) >> (rbit & 31)) & ((1u << p.r) - 1);
            const float s = h2f(__ldg(p.sz + ((size_t)row * (p.K / G) + c / G) * 2));
            corr = fmaf(h2f(__ldg(xrow + c)) * inv * s, (float)rho + 0.5f - half, corr);
          }
          corr = warp_sum(corr);
          if (lane == 0) part[(row - n0) * p.segs] += corr;
        }
      }
      __syncthreads();
    }
    for (int row = n0 + threadIdx.x; row < n1; row += blockDim.x) {
      float acc = 0.f;
      for (int s = 0; s < p.segs; s++) acc += part[(row - n0) * p.segs + s];
      float* dst = p.y + (size_t)b * p.N + row;
      *dst = p.mode == 1 ? *dst + acc : acc;
    }
    __syncthreads();
  }
}

sf_status gemv_launch(const sf_wq* w, const uint16_t* x, int batch, int chunk, int kch,
                      const int32_t* sel_in, int32_t* sel_out, const void* refine_rows, float* y,
                      int mode, cudaStream_t s) {
  sf_status st = check_wq_public(w, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(x && aligned16(x), "x must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(y && aligned16(y), "y must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(batch >= 1 && batch <= 8, "batch=%d outside [1, 8]", batch);
  SF_REQUIRE(kch >= 0, "kch=%d < 0", kch);
  const int32_t* sel = nullptr;
  int n_sel = 0;
  if (kch > 0) {
    st = check_select_args(x, batch, w->k, chunk, kch);
    if (st != SF_OK) return st;
    n_sel = (w->k / chunk) * kch;
    SF_REQUIRE(refine_rows || w->refine, "kch > 0 needs w->refine or staged refine_rows");
    SF_REQUIRE(!refine_rows || aligned16(refine_rows), "refine_rows must be 16-byte aligned");
    if (sel_in) {
      SF_REQUIRE(aligned16(sel_in), "sel_in must be 16-byte aligned");
      sel = sel_in;
    } else {
      SF_REQUIRE(sel_out && aligned16(sel_out), "sel_out is needed when sel_in is NULL");
      st = launch_select(x, batch, w->k, chunk, kch, sel_out, s);
      if (st != SF_OK) return st;
      sel = sel_out;
    }
  } else if (mode == 1) {
    return SF_OK;  // nothing to correct
  }
  GemvParams p;
  p.base = (const uint32_t*)w->base;
  p.refine = (const uint32_t*)(refine_rows ? refine_rows : w->refine);
  p.sz = w->sz;
  p.x = x;
  p.sel = sel;
  p.y = y;
  p.N = w->n, p.K = w->k, p.G = w->group, p.r = w->r, p.batch = batch, p.n_sel = n_sel;
  p.mode = mode;
  p.segs = (w->k + kSegChannels - 1) / kSegChannels;
  SF_UNSUPPORTED(p.segs <= kWarps, "k=%d above %d", w->k, kWarps * kSegChannels);
  p.refine_row_words = w->n * w->r / 32;
  p.staged = refine_rows != nullptr;
  const int U = w->b == 4 ? 2 : 4;
  const int W = w->b == 2 ? 4 : w->b == 3 ? 6 : 8;
  const size_t slot_bytes = (size_t)U * 32 * (W + 2) * 4;
  const size_t xs_bytes = (size_t)(w->k / 64) * kXWords * 4;
  const size_t xraw_bytes = (size_t)w->k * 2;
  const size_t corr_bytes = (size_t)kCorrSmemWords * 4;
  auto smem_for = [&](int ctas_per_sm, int pd) {
    int grid = ctas_per_sm * num_sms();
    if (grid > w->n / 4) grid = w->n / 4;
    const size_t rows = (w->n + grid - 1) / grid;
    const size_t segs = (w->k + kSegChannels - 1) / kSegChannels;
    const size_t part = ((rows * segs + 3) & ~(size_t)3) * 4;
    size_t scratch = (size_t)kWarps * pd * slot_bytes;
    if (scratch < xraw_bytes) scratch = xraw_bytes;
    if (scratch < corr_bytes) scratch = corr_bytes;
    return xs_bytes + part + scratch;
  };
  const size_t per_sm = 227 * 1024;
  int ctas = kCtasPerSm, pd = 3;
  if (smem_for(ctas, 3) * ctas > per_sm - ctas * 1024) pd = 2;
  if (smem_for(ctas, pd) * ctas > per_sm - ctas * 1024) ctas = 1, pd = 3;
  int grid = ctas * num_sms();
  if (grid > w->n / 4) grid = w->n / 4;
  const int rows_per_cta = (w->n + grid - 1) / grid;
  p.row_warps = kWarps / p.segs;
  const int needed = (rows_per_cta + U - 1) / U;
  if (p.row_warps > needed) p.row_warps = needed;
  if (p.row_warps < 1) p.row_warps = 1;
  const size_t smem = smem_for(ctas, pd);
  SF_UNSUPPORTED(smem <= 200 * 1024, "k=%d needs too much shared memory", w->k);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (kch > 0 && !sel_in) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void (*kern)(GemvParams);
  if (pd == 3)
    kern = w->b == 2 ? gemv_kernel<2, 3> : w->b == 3 ? gemv_kernel<3, 3> : gemv_kernel<4, 3>;
  else
    kern = w->b == 2 ? gemv_kernel<2, 2> : w->b == 3 ? gemv_kernel<3, 2> : gemv_kernel<4, 2>;
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
  SF_CUDA(cudaLaunchKernelEx(&cfg, kern, p));
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
  return gemv_launch(w, x, batch, chunk, kch, sel_in, sel_out, refine_rows, y, 0, as_stream(stream));
}

extern "C" sf_status sf_gemv_correction(const sf_wq* w, const uint16_t* x, int batch, int chunk,
                                        int kch, const int32_t* sel, const void* refine_rows,
                                        float* y, sf_stream_t stream) {
  SF_REQUIRE(kch == 0 || (sel && aligned16(sel)), "sel must be non-null and 16-byte aligned");
  return gemv_launch(w, x, batch, chunk, kch, sel, nullptr, refine_rows, y, 1, as_stream(stream));
}
