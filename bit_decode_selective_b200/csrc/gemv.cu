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
//     of a projection is applied later than its base product; the split form
//     writes it to its own output and the correction-only kernel computes it
//     on its own.
//
// Decomposition, per output row i (fp32 accumulation):
//   y_i = sum_groups [ s_ig * sum_{c in g} x_c q_ic + m_ig * sum_{c in g} x_c ]
//       + sum_{c selected} x_c * s_i,g(c) * (rho_ic + 1/2 - 2^(r-1)) / 2^r
//
// One CTA per SM owns a contiguous range of rows (a multiple of 4).
//
// Producer warp: one lane streams the CTA's codes through a ring of shared
// memory stages with 1-D bulk copies (cp.async.bulk, completion counted on an
// mbarrier per stage), and copies the rows' (s, m) words once.  The weights do
// not depend on earlier kernels, so these copies start before the grid
// dependency wait and overlap the previous kernel's tail.
//
// Compute warps: after the grid dependency wait they build the correction
// tables (selected channel, x_c, group; the refinement words of the CTA's rows
// copied with cp.async) and the activation planes (four threads per 64-channel
// block) together.  Warp w owns the 2,048-channel segment w % segs (lane L: 64
// consecutive channels) for every row whose index in its stage is congruent to
// w / segs.  Its activations are turned once into fixed point
// x = x_fix * 2^e per 64-channel lane block (e from the block's largest |x|,
// |x_fix| < 2^20: every value within 2^9 of the block's largest is exact, the
// rest round to 2^-20 of it) held as three byte planes in registers, in the
// order of the code byte vectors: a 32-bit word of
// 2-bit codes gives four byte vectors with one AND each (the codes at bit
// offsets 2 and 6 of a byte carry a factor 4 that is folded into the scale),
// dp4a takes four code x byte products per instruction, and the planes are
// combined in 32-bit integers: the lane's partial dot product over its block is
// exact for its fixed-point x.  Per row: s * 2^e * dot + m * sum(x), summed over
// the warp with a transposed butterfly into a per-(row, segment) slot.
//
// Correction (after the base pass, all threads): a thread owns 4 consecutive
// rows (the r bits of 4 rows never straddle a 32-bit word) and a share of the
// selected channels; per channel it reads one refinement word and adds
// x_c * (1 + rho/2^r) to a per-row run, and every run of channels in one scale
// group is scaled once, s * (run - sum x_c (1 - off/2^r)) with
// off = 1/2 - 2^(r-1).  The base pass leaves the scales group-major for it.
// Every partial has its own slot, so the sums are deterministic.
#include "common.cuh"
#include "internal.cuh"

#include <algorithm>

namespace sf {
namespace {

constexpr int kLaneCh = 64;                 // input channels per lane
constexpr int kSegCh = 32 * kLaneCh;        // channels per warp segment
constexpr int kMaxSegs = 16;                // k <= 32,768
constexpr int kMaxWarps = 15;               // compute warps per CTA (plus the producer: 16 warps)
#ifndef SF_GEMV_PLANES
#define SF_GEMV_PLANES 3
#endif
constexpr int kXP = SF_GEMV_PLANES;         // byte planes of the fixed-point activations (2 or 3)
constexpr int kXW = 16 * kXP + 4;           // shared words per lane block: planes, sum0, sum1, scale, pad
// x_fix = x * 2^(kXE - ilogb(max |x| of the block)): |x_fix| < 2^(kXE + 1), so
// 4 * sum code * x_fix over 64 channels fits an int32 for every base width
constexpr int kXE = kXP == 2 ? 14 : 19;
constexpr int kRowUnit = 4;                 // CTA row ranges start at multiples of 4
constexpr size_t kSmemLimit = 227 * 1024;   // dynamic shared memory of one CTA
constexpr size_t kStageTarget = 36 * 1024;  // bytes of codes per ring stage, at most
constexpr int kMaxStages = 6;
constexpr unsigned long long kWaitNs = 1000000000ull;  // bounded waits give up after 1 s

// Bounded waits that ran out (the host reads it with sf_device_wait_timeouts).
__device__ unsigned int g_wait_timeouts;

struct GemvArgs {
  const uint8_t* base;      // codes; b = 3: plane L then plane H (hi_off bytes in)
  const uint32_t* refine;   // channel-major rows [K][row_words], or staged rows [n_sel][row_words]
  const uint32_t* sz;       // [N][gpr] words: fp16 (s, m)
  const uint16_t* x;        // [K] fp16
  const int32_t* sel;       // [n_sel]
  float* y;                 // [N]
  float* y_corr;            // non-null: the correction goes here, y gets the base product
  size_t hi_off;
  int N, K, gpr, gshift, r, n_sel;
  int segs, R, W;           // segments, warps per segment, compute warps (segs * R)
  int rc, stages;           // rows per stage (R * RPW), ring depth
  int rowL, rowH;           // bytes per row of plane L (all codes for b = 2, 4) and of plane H
  int stage_bytes;
  int row_words, staged, rows_max;
  int off_ring, off_sz, off_x, off_part, off_szt, off_jd, off_wt, off_cpart;  // shared memory offsets
  int szt_pitch, wt_pitch, cparts;
};

// ---- PTX helpers ------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase of `bar` with this parity to complete, for at most
// kWaitNs; false (and the timeout counted) if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitNs) {
      atomicAdd(&g_wait_timeouts, 1u);
      return false;
    }
  }
  return true;
}
// 1-D bulk copy global -> this CTA's shared memory, completion counted on bar.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Named barrier over `count` threads (whole warps).
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t dp4a_us(uint32_t a, uint32_t b, uint32_t c) {
  int32_t d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"((int32_t)c));
  return (uint32_t)d;
}

// ---- activations -------------------------------------------------------------

// Byte L of code vector v of a lane's 64 channels holds the code of channel
// chan_of(v, L) (local to the lane block).
template <int BITS>
__host__ __device__ __forceinline__ int chan_of(int v, int L) {
  if (BITS == 4) return 8 * (v >> 1) + (v & 1) + 2 * L;
  return 16 * (v >> 2) + (v & 3) + 4 * L;
}

// A quarter of lane block b of x (64 channels) as fixed point, by the four
// consecutive lanes of a quad (quarter q = lane & 3: channels 16q .. 16q + 15,
// which are exactly the channels of code vectors 4q .. 4q + 3).  The block's
// exponent comes from the quad's largest |x|; dst = the block's shared words:
// planes[kXP * v + p] = byte p of x_fix for the four channels of vector v,
// then the sum of channels 0-31, of 32-63 and the factor that turns the
// integer dot product back into x units (2^e, divided by 4 where the byte
// vectors carry the factor 4).  Whole warps (valid = false: the lane computes
// nothing but takes part in the shuffles).
template <int BITS>
__device__ __forceinline__ void quarter_planes(bool valid, const uint16_t* __restrict__ xq, int q,
                                               uint32_t* __restrict__ dst) {
  uint32_t h[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (valid) {
    const uint4 a0 = reinterpret_cast<const uint4*>(xq)[0], a1 = reinterpret_cast<const uint4*>(xq)[1];
    h[0] = a0.x, h[1] = a0.y, h[2] = a0.z, h[3] = a0.w, h[4] = a1.x, h[5] = a1.y, h[6] = a1.z, h[7] = a1.w;
  }
  uint32_t mx2 = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) mx2 = __vmaxu2(mx2, h[i] & 0x7fff7fffu);
  uint32_t mx = max(mx2 & 0xffffu, mx2 >> 16);
  mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    sq += f.x, sq += f.y;
  }
  const float sh = sq + __shfl_xor_sync(0xffffffffu, sq, 1);  // quarters 0+1 or 2+3
  const float so = __shfl_xor_sync(0xffffffffu, sh, 2);       // the other half
  // x_fix = x * 2^(kXE - ilogb(max |x|)): the largest values are fp16
  // mantissas times 2^(kXE - 10) (exact), smaller ones round to that step
  const int eb = mx ? ((__float_as_int(h2f((uint16_t)mx)) >> 23) & 0xff) - 127 : 0;  // ilogb(max |x|)
  const float scale = mx ? __int_as_float((127 + kXE - eb) << 23) : 0.f;
  if (!valid) return;
  int qv[16];
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    // round to nearest even through the float mantissa: 1.5 * 2^23 + x_fix
    qv[2 * i] = __float_as_int(fmaf(f.x, scale, 12582912.0f)) - 0x4B400000;
    qv[2 * i + 1] = __float_as_int(fmaf(f.y, scale, 12582912.0f)) - 0x4B400000;
  }
#pragma unroll
  for (int vv = 0; vv < 4; vv++) {
    const int v = 4 * q + vv;
    const int a = qv[chan_of<BITS>(vv, 0) & 15], b = qv[chan_of<BITS>(vv, 1) & 15];
    const int c = qv[chan_of<BITS>(vv, 2) & 15], d = qv[chan_of<BITS>(vv, 3) & 15];
#pragma unroll
    for (int p = 0; p < kXP; p++) {
      const uint32_t sel = (uint32_t)p | ((uint32_t)(4 + p) << 4);
      const uint32_t t01 = __byte_perm((uint32_t)a, (uint32_t)b, sel);
      const uint32_t t23 = __byte_perm((uint32_t)c, (uint32_t)d, sel);
      dst[kXP * v + p] = __byte_perm(t01, t23, 0x5410);
    }
  }
  if (q == 0) {
    float* f = reinterpret_cast<float*>(dst + 16 * kXP);
    f[0] = sh;
    f[1] = so;
    f[2] = mx ? __int_as_float((127 + eb - kXE - (BITS == 4 ? 0 : 2)) << 23) : 1.0f;
    f[3] = 0.f;
  }
}

// ---- the base pass of one row -------------------------------------------------

// The lane's partial sum of one row: the integer dot products of its block
// (per 32-channel half when ZW = 2), then s * 2^e * dot + m * sum(x).
// cw: the row's codes of this lane (plane L), hw: plane H (b = 3),
// zw: the row's (s, m) word(s) for the lane's group(s).
template <int BITS, int ZW>
__device__ __forceinline__ float lane_row(const uint8_t* __restrict__ cw, const uint8_t* __restrict__ hw,
                                          const uint32_t (&xr)[16 * kXP], float xs0, float xs1,
                                          float xsc, uint32_t z0, uint32_t z1) {
  uint32_t A[ZW][kXP], B[ZW][kXP];
#pragma unroll
  for (int h = 0; h < ZW; h++)
#pragma unroll
    for (int p = 0; p < kXP; p++) A[h][p] = B[h][p] = 0u;
  auto mac = [&](uint32_t c, int v, uint32_t(&acc)[kXP]) {
#pragma unroll
    for (int p = 0; p < kXP; p++)
      acc[p] = p == kXP - 1 ? dp4a_us(c, xr[kXP * v + p], acc[p]) : dp4a_uu(c, xr[kXP * v + p], acc[p]);
  };
  if constexpr (BITS == 4) {
    const uint4 q0 = reinterpret_cast<const uint4*>(cw)[0], q1 = reinterpret_cast<const uint4*>(cw)[1];
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int h = ZW == 2 ? (i >> 2) : 0;
      mac(w[i] & 0x0F0F0F0Fu, 2 * i, A[h]);
      mac((w[i] >> 4) & 0x0F0F0F0Fu, 2 * i + 1, A[h]);
    }
  } else {
    const uint4 q0 = *reinterpret_cast<const uint4*>(cw);
    const uint32_t w[4] = {q0.x, q0.y, q0.z, q0.w};
    uint32_t hi[2] = {0u, 0u};
    if constexpr (BITS == 3) {
      const uint2 t = *reinterpret_cast<const uint2*>(hw);
      hi[0] = t.x, hi[1] = t.y;
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int h = ZW == 2 ? (i >> 1) : 0;
      const uint32_t w0 = w[i], w4 = w0 >> 4;
      uint32_t c0 = w0 & 0x03030303u, c1 = w0 & 0x0C0C0C0Cu;
      uint32_t c2 = w4 & 0x03030303u, c3 = w4 & 0x0C0C0C0Cu;
      if constexpr (BITS == 3) {
        // the high bit of the codes of vector 4i + m sits at bit 4 (i & 1) + m of
        // each byte of hi[i / 2]; it joins at bit 2 (factor-1 vectors) or 4
        const uint32_t H = hi[i >> 1];
        if ((i & 1) == 0) {
          c0 |= (H << 2) & 0x04040404u;
          c1 |= (H << 3) & 0x10101010u;
          c2 |= H & 0x04040404u;
          c3 |= (H << 1) & 0x10101010u;
        } else {
          c0 |= (H >> 2) & 0x04040404u;
          c1 |= (H >> 1) & 0x10101010u;
          c2 |= (H >> 4) & 0x04040404u;
          c3 |= (H >> 3) & 0x10101010u;
        }
      }
      mac(c0, 4 * i + 0, A[h]);
      mac(c1, 4 * i + 1, B[h]);
      mac(c2, 4 * i + 2, A[h]);
      mac(c3, 4 * i + 3, B[h]);
    }
  }
  // 4 x sum(code x_fix) (b = 2, 3: set B carries the factor 4) or sum(code x_fix) (b = 4)
  int32_t J[ZW];
#pragma unroll
  for (int h = 0; h < ZW; h++) {
    uint32_t a = A[h][0], bb = B[h][0];
#pragma unroll
    for (int p = 1; p < kXP; p++) a += A[h][p] << (8 * p), bb += B[h][p] << (8 * p);
    J[h] = BITS == 4 ? (int32_t)a : (int32_t)((a << 2) + bb);
  }
  const float2 sm0 = __half22float2(*reinterpret_cast<const __half2*>(&z0));
  if constexpr (ZW == 1) {
    return fmaf(sm0.x * xsc, (float)J[0], sm0.y * (xs0 + xs1));
  } else {
    const float2 sm1 = __half22float2(*reinterpret_cast<const __half2*>(&z1));
    return fmaf(sm0.x * xsc, (float)J[0], fmaf(sm1.x * xsc, (float)J[1], fmaf(sm0.y, xs0, sm1.y * xs1)));
  }
}

// Sum each of U per-lane values over the warp.  Returns the full sum of value
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

// ---- the kernel -----------------------------------------------------------------

// RPW: rows per compute warp per stage (2 or 4).  A CTA's warps are spread
// over the SM's four schedulers, each with a quarter of the register file:
// four warps of 120 registers a thread leave kSideRegs / 4 of every quarter
// free for a staging CTA.
static_assert(((kMaxWarps + 1 + 3) / 4) * 120 * 32 + kSideRegs / 4 <= 65536 / 4,
              "GEMV registers leave no room for a staging CTA");
template <int BITS, int ZW, int RPW>
__global__ void __maxnreg__(120) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  uint64_t* szbar = empty + kMaxStages;
  uint8_t* ring = smem + a.off_ring;
  uint32_t* szs = reinterpret_cast<uint32_t*>(smem + a.off_sz);
  uint32_t* xpl = reinterpret_cast<uint32_t*>(smem + a.off_x);
  float* part = reinterpret_cast<float*>(smem + a.off_part);
  uint32_t* szt = reinterpret_cast<uint32_t*>(smem + a.off_szt);
  uint2* jd = reinterpret_cast<uint2*>(smem + a.off_jd);
  uint32_t* wt = reinterpret_cast<uint32_t*>(smem + a.off_wt);
  float* cpart = reinterpret_cast<float*>(smem + a.off_cpart);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int units = a.N / kRowUnit;
  const int n0 = (int)((long)blockIdx.x * units / gridDim.x) * kRowUnit;
  const int n1 = (int)((long)(blockIdx.x + 1) * units / gridDim.x) * kRowUnit;
  const int rows = n1 - n0;
  const int nst = (rows + a.rc - 1) / a.rc;
  const int w_lo = (n0 * a.r) >> 5;
  const int nwr = (((n1 * a.r) + 31) >> 5) - w_lo;
  const bool corr = a.n_sel > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; s++) mbar_init(&full[s], 1), mbar_init(&empty[s], a.W);
    mbar_init(szbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  pdl_trigger();  // the next kernel of the stream may be scheduled; it waits for this grid

  if (warp == a.W) {
    // ---------------- producer warp
    int issued = 0;
    auto issue = [&](int i) {
      const int slot = i % S;
      const int r0 = i * a.rc, nr = min(a.rc, rows - r0);
      const uint32_t bl = (uint32_t)(nr * a.rowL), bh = (uint32_t)(nr * a.rowH);
      uint8_t* dst = ring + (size_t)slot * a.stage_bytes;
      mbar_expect_tx(&full[slot], bl + bh);
      bulk_g2s(dst, a.base + (size_t)(n0 + r0) * a.rowL, bl, &full[slot]);
      if (BITS == 3) bulk_g2s(dst + (size_t)a.rc * a.rowL, a.base + a.hi_off + (size_t)(n0 + r0) * a.rowH, bh, &full[slot]);
    };
    if (lane == 0) {
      const uint32_t zb = (uint32_t)(rows * a.gpr * 4);
      mbar_expect_tx(szbar, zb);
      bulk_g2s(szs, a.sz + (size_t)n0 * a.gpr, zb, szbar);
      for (; issued < min(S, nst); issued++) issue(issued);
    }
    pdl_wait();  // the previous kernel is complete (no data of it is read here)
    if (lane == 0) {
      for (; issued < nst; issued++) {
        const int slot = issued % S;
        if (!mbar_wait(&empty[slot], ((issued / S) - 1) & 1)) break;
        issue(issued);
      }
      // nothing may still be landing in this CTA's shared memory when it exits
      for (int i = max(0, issued - S); i < issued; i++) mbar_wait(&full[i % S], (i / S) & 1);
      mbar_wait(szbar, 0);
    }
    __syncwarp();
  } else {
    // ---------------- compute warps
    const int seg = warp % a.segs, jw = warp / a.segs;
    const int lg = seg * 32 + lane;  // lane block
    const bool la = lg * kLaneCh < a.K;
    const int tc = threadIdx.x, ntc = a.W * 32;
    pdl_wait();  // x, the selection and the staged rows are complete
    // correction tables, entries tc, tc + ntc, ...: the selection's loads are
    // issued first, their activations after the planes (every load of a round
    // in flight together)
    constexpr int kJ = 2;
    int rawj[kJ];
    if (corr)
#pragma unroll
      for (int u = 0; u < kJ; u++) rawj[u] = tc + u * ntc < a.n_sel ? __ldg(a.sel + tc + u * ntc) : 0;
    // activation planes: four threads per 64-channel lane block
    {
      const int nq = (a.K / kLaneCh) * 4;
      for (int b0 = warp * 32; b0 < nq; b0 += ntc) {
        const int idx = b0 + lane, b = idx >> 2, q = idx & 3;
        quarter_planes<BITS>(idx < nq, a.x + (size_t)b * kLaneCh + 16 * q, q, xpl + (size_t)b * kXW);
      }
    }
    if (corr) {
      // -1 - c: channel c selected but not refined now (no correction); a
      // foreign index is clamped, so it never leaves the buffers
      for (int j0 = 0; j0 < a.n_sel; j0 += kJ * ntc) {
#pragma unroll
        for (int u = 0; u < kJ; u++) {
          const int j = j0 + tc + u * ntc;
          if (j >= a.n_sel) continue;
          const int raw = j0 == 0 ? rawj[u] : __ldg(a.sel + j);
          const int c = min(max(raw < 0 ? -1 - raw : raw, 0), a.K - 1);
          const uint32_t xc = raw < 0 ? 0u : __float_as_uint(h2f(__ldg(a.x + c)));
          jd[j] = make_uint2(xc, (uint32_t)(c >> a.gshift));
          const uint32_t* src = a.refine + (size_t)(a.staged ? j : c) * a.row_words + w_lo;
          for (int k = 0; k < nwr; k++) cp_async4(wt + (size_t)j * a.wt_pitch + k, src + k);
        }
      }
      cp_async_commit();
    }
    bar_sync(1, a.W * 32);
    uint32_t xr[16 * kXP];
    float xs0, xs1, xsc;
    {
      const uint4* src = reinterpret_cast<const uint4*>(xpl + ((size_t)seg * 32 + lane) * kXW);
#pragma unroll
      for (int k = 0; k < 4 * kXP; k++) {
        const uint4 q = src[k];
        xr[4 * k] = q.x, xr[4 * k + 1] = q.y, xr[4 * k + 2] = q.z, xr[4 * k + 3] = q.w;
      }
      const float4 f = reinterpret_cast<const float4*>(src)[4 * kXP];
      xs0 = f.x, xs1 = f.y, xsc = f.z;
    }
    const int g0 = (lg * kLaneCh) >> a.gshift;            // the lane's (first) group
    const bool zown = corr && la && ((lg * kLaneCh) & ((1 << a.gshift) - 1)) == 0;
    bool ok = mbar_wait(szbar, 0);
    const size_t codeL = (size_t)lg * (BITS == 4 ? 32 : 16);
    for (int i = 0; i < nst && ok; i++) {
      const int slot = i % S;
      if (!mbar_wait(&full[slot], (i / S) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* sl = ring + (size_t)slot * a.stage_bytes;
      float pv[RPW];
#pragma unroll
      for (int t = 0; t < RPW; t++) {
        const int rr = jw + a.R * t, lr = i * a.rc + rr;
        pv[t] = 0.f;
        if (la && lr < rows) {
          const uint32_t* zr = szs + (size_t)lr * a.gpr + g0;
          const uint32_t z0 = zr[0], z1 = ZW == 2 ? zr[1] : 0u;
          if (zown) {
            szt[(size_t)g0 * a.szt_pitch + lr] = z0;
            if (ZW == 2) szt[(size_t)(g0 + 1) * a.szt_pitch + lr] = z1;
          }
          pv[t] = lane_row<BITS, ZW>(sl + (size_t)rr * a.rowL + codeL,
                                     sl + (size_t)a.rc * a.rowL + (size_t)rr * a.rowH + (size_t)lg * 8, xr, xs0,
                                     xs1, xsc, z0, z1);
        }
      }
      const float tot = warp_sum_rows<RPW>(pv, lane);
      const int t = RPW == 4 ? (lane >> 3) : (lane >> 4);
      const int lr = i * a.rc + jw + a.R * t;
      if ((lane & (32 / RPW - 1)) == 0 && lr < rows) part[(size_t)lr * a.segs + seg] = tot;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    cp_async_wait_all();  // this thread's refinement words
  }
  bar_sync(2, blockDim.x);  // base pass, tables and refinement words complete

  // ---------------- correction of the selected channels (all threads)
  if (corr) {
    const int nb = rows / 4;
    const int Q = a.cparts;
    const int r = a.r;
    const uint32_t fmask = ((1u << r) - 1u) << (23 - r);
    const float cfac = 1.0f - (0.5f - 0.5f * (float)(1 << r)) / (float)(1 << r);
    for (int task = threadIdx.x; task < nb * Q; task += blockDim.x) {
      const int blk = task % nb, q = task / nb;
      const int j0 = (int)((long)q * a.n_sel / Q), j1 = (int)((long)(q + 1) * a.n_sel / Q);
      const int bit0 = (n0 + 4 * blk) * r;
      const int wi = (bit0 >> 5) - w_lo;
      int rot[4];
#pragma unroll
      for (int t = 0; t < 4; t++) rot[t] = (23 - r - ((bit0 & 31) + r * t)) & 31;
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, run[4] = {0.f, 0.f, 0.f, 0.f};
      float C = 0.f;
      int gcur = -1;
      auto flush = [&]() {
        if (gcur >= 0) {
          const uint4 z = *reinterpret_cast<const uint4*>(szt + (size_t)gcur * a.szt_pitch + 4 * blk);
          const uint32_t zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
          for (int t = 0; t < 4; t++)
            acc[t] = fmaf(__low2float(*reinterpret_cast<const __half2*>(&zz[t])), run[t] - C, acc[t]);
        }
      };
      for (int j = j0; j < j1; j++) {
        const uint2 d = jd[j];
        if ((int)d.y != gcur) {
          flush();
          gcur = (int)d.y, C = 0.f;
#pragma unroll
          for (int t = 0; t < 4; t++) run[t] = 0.f;
        }
        const uint32_t w = wt[(size_t)j * a.wt_pitch + wi];
        const float xc = __uint_as_float(d.x);
        // f = 1 + rho / 2^r; sum x f - sum x (1 - off/2^r) = sum x (rho + off) / 2^r
#pragma unroll
        for (int t = 0; t < 4; t++)
          run[t] = fmaf(__uint_as_float(0x3F800000u | (__funnelshift_l(w, w, rot[t]) & fmask)), xc, run[t]);
        C = fmaf(xc, cfac, C);
      }
      flush();
      *reinterpret_cast<float4*>(cpart + (size_t)q * a.rows_max + 4 * blk) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    bar_sync(2, blockDim.x);
  }

  // ---------------- output
  for (int lr = threadIdx.x; lr < rows; lr += blockDim.x) {
    float base = 0.f, c = 0.f;
    for (int s = 0; s < a.segs; s++) base += part[(size_t)lr * a.segs + s];
    if (corr)
      for (int q = 0; q < a.cparts; q++) c += cpart[(size_t)q * a.rows_max + lr];
    if (a.y_corr) {
      a.y[n0 + lr] = base;
      a.y_corr[n0 + lr] = c;
    } else {
      a.y[n0 + lr] = base + c;
    }
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
  // entry j: channel and activation (-1 - c: selected, not refined now: x = 0)
  auto chan = [&](int j) {
    const int raw = __ldg(sel + j);
    return min(max(raw < 0 ? -1 - raw : raw, 0), a.K - 1);
  };
  auto act = [&](int j, int c) { return __ldg(sel + j) < 0 ? 0.f : h2f(__ldg(xb + c)); };
  // channel j + 1's index, activation and word are loaded while j is summed
  int c = a.n_sel > 0 ? chan(0) : 0;
  float xc = a.n_sel > 0 ? act(0, c) : 0.f;
  uint32_t w = a.n_sel > 0 ? word_of(0, c) : 0u;
  for (int j = 0; j < a.n_sel; j++) {
    const int cn = j + 1 < a.n_sel ? chan(j + 1) : 0;
    const float xn = j + 1 < a.n_sel ? act(j + 1, cn) : 0.f;
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

size_t align128(size_t v) { return (v + 127) & ~(size_t)127; }

struct Plan {
  GemvArgs a;  // shape and shared memory layout (pointers are set per launch)
  int grid, threads, rpw, zw;
  size_t smem;
};

// Work split and shared memory layout of one GEMV shape: segments of 2,048
// channels, warps per segment (at most 16 compute warps), rows per stage (the
// warps of a segment take RPW rows each), the ring depth that fits.
sf_status make_plan(const sf_wq* w, int n_sel, Plan& P) {
  GemvArgs& a = P.a;
  a = GemvArgs{};
  const int N = w->n, K = w->k;
  a.N = N, a.K = K, a.r = w->r, a.n_sel = n_sel;
  a.gpr = K / w->group;
  a.gshift = 0;
  while ((1 << a.gshift) < w->group) a.gshift++;
  a.segs = (K + kSegCh - 1) / kSegCh;
  SF_UNSUPPORTED(a.segs <= kMaxSegs, "k=%d above %d", K, kMaxSegs * kSegCh);
  a.R = std::max(1, kMaxWarps / a.segs);
  a.W = a.segs * a.R;
  a.rowL = K * (w->b == 4 ? 4 : 2) / 8;
  a.rowH = w->b == 3 ? K / 8 : 0;
  a.hi_off = w->b == 3 ? (size_t)N * K / 4 : 0;
  const size_t rowB = (size_t)a.rowL + a.rowH;
  const int units = N / kRowUnit;
  P.grid = std::min(num_sms(), units);
  a.rows_max = ((units + P.grid - 1) / P.grid) * kRowUnit;
  // four rows per warp per stage when a stage stays small and a CTA still gets
  // two or more stages (compute starts as soon as the first one lands)
  P.rpw = (size_t)a.R * 4 * rowB <= kStageTarget && a.rows_max >= 2 * a.R * 4 ? 4 : 2;
  a.rc = a.R * P.rpw;
  a.stage_bytes = (int)(a.rc * rowB);
  a.row_words = N * w->r / 32;
  a.wt_pitch = ((a.rows_max * w->r + 31) >> 5) + 1;
  a.szt_pitch = (a.rows_max + 3) & ~3;
  if (a.szt_pitch % 32 == 0) a.szt_pitch += 4;  // spread the group-major scale stores over banks
  P.threads = (a.W + 1) * 32;
  P.zw = w->group == 32 ? 2 : 1;
  const int nb_max = a.rows_max / 4;
  // channel shares of the correction: enough threads busy, and few partial
  // sums per row for the output's serial add
  a.cparts = n_sel > 0 ? std::max(1, std::min(std::min(n_sel, 16), P.threads / nb_max)) : 0;
  size_t off = align128((2 * kMaxStages + 1) * sizeof(uint64_t));
  a.off_sz = (int)off;
  off += align128((size_t)a.rows_max * a.gpr * 4);
  a.off_part = (int)off;
  off += align128((size_t)a.rows_max * a.segs * 4);
  // the activation planes are read once, before the correction partials are written
  a.off_x = a.off_cpart = (int)off;
  off += align128(std::max((size_t)a.segs * 32 * kXW * 4, (size_t)a.cparts * a.rows_max * 4));
  if (n_sel > 0) {
    a.off_szt = (int)off;
    off += align128((size_t)a.gpr * a.szt_pitch * 4);
    a.off_jd = (int)off;
    off += align128((size_t)n_sel * 8);
    a.off_wt = (int)off;
    off += align128((size_t)n_sel * a.wt_pitch * 4);
  }
  a.off_ring = (int)off;
  const int nst_max = (a.rows_max + a.rc - 1) / a.rc;
  int S = std::min(kMaxStages, nst_max);
  while (S > 1 && off + (size_t)S * a.stage_bytes > kSmemLimit) S--;
  SF_UNSUPPORTED(off + (size_t)S * a.stage_bytes <= kSmemLimit,
                 "n=%d, k=%d, %d selected channels: %zu bytes of shared memory needed", N, K, n_sel,
                 off + (size_t)S * a.stage_bytes);
  a.stages = S;
  P.smem = off + (size_t)S * a.stage_bytes;
  return SF_OK;
}

template <int BITS, int ZW>
void* kernel_for(int rpw) {
  return rpw == 4 ? (void*)gemv_kernel<BITS, ZW, 4> : (void*)gemv_kernel<BITS, ZW, 2>;
}

void* pick_kernel(int b, int zw, int rpw) {
  if (b == 2) return zw == 1 ? kernel_for<2, 1>(rpw) : kernel_for<2, 2>(rpw);
  if (b == 3) return zw == 1 ? kernel_for<3, 1>(rpw) : kernel_for<3, 2>(rpw);
  return zw == 1 ? kernel_for<4, 1>(rpw) : kernel_for<4, 2>(rpw);
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
  Plan P;
  st = make_plan(w, n_sel, P);
  if (st != SF_OK) return st;

  // the selection (when not given), then the GEMV, which waits for it (and for
  // x) through programmatic dependent launch while its first code copies fly
  const int32_t* sel = sel_in;
  if (kch > 0 && !sel_in) {
    st = launch_select(x, batch, w->k, chunk, kch, sel_out, s, true);
    if (st != SF_OK) return st;
    sel = sel_out;
  }
  void* kern = pick_kernel(w->b, P.zw, P.rpw);
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.grid);
  cfg.blockDim = dim3(P.threads);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one launch per batch row: each streams the codes once for its row
  for (int b = 0; b < batch; b++) {
    GemvArgs a = P.a;
    a.base = (const uint8_t*)w->base;
    a.sz = (const uint32_t*)w->sz;
    a.staged = refine_rows != nullptr;
    a.refine = refine_rows ? (const uint32_t*)refine_rows + (size_t)b * n_sel * a.row_words
                           : (const uint32_t*)w->refine;
    a.x = x + (size_t)b * w->k;
    a.sel = sel ? sel + (size_t)b * n_sel : nullptr;
    a.y = y + (size_t)b * w->n;
    a.y_corr = y_corr ? y_corr + (size_t)b * w->n : nullptr;
    void* args[] = {&a};
    SF_CUDA(cudaLaunchKernelExC(&cfg, kern, args));
  }
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

extern "C" sf_status sf_device_wait_timeouts(unsigned int* count, int reset) {
  SF_REQUIRE(count, "count must be non-null");
  SF_CUDA(cudaMemcpyFromSymbol(count, g_wait_timeouts, sizeof(unsigned int)));
  if (reset) {
    const unsigned int zero = 0;
    SF_CUDA(cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(unsigned int)));
  }
  if (*count) {
    set_error("%u bounded device wait(s) ran out", *count);
    return SF_ERR_TIMEOUT;
  }
  return SF_OK;
}
