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
// Two forms, both with one CTA per SM over a contiguous range of rows (a
// multiple of 4) and a producer warp that streams the CTA's codes through a
// ring of shared-memory stages with 1-D bulk copies (cp.async.bulk, one per
// stage and plane, completion counted on an mbarrier per stage) and copies
// the rows' (s, m) words once.  The weights do not depend on earlier kernels,
// so these copies start before the grid dependency wait and overlap the
// previous kernel's tail.  Packed rows store their 16-byte units permuted by
// row mod 8 (wqlayout.cuh); a lane reads whole units either way.
//
// Batch 1 (gemv_kernel, CUDA cores).  After the grid dependency wait the
// compute warps build the correction tables (selected channel, x_c, group;
// the refinement words of the CTA's rows copied with cp.async) and the
// activation planes (four threads per 64-channel block) together.  Warp w
// owns the 2,048-channel segment w % segs (lane L: 64 consecutive channels,
// one 16-byte unit of a 2-bit row) for every row whose index in its stage is
// congruent to w / segs.  Its activations are turned once into fixed point
// x = x_fix * 2^e per 64-channel lane block (e from the block's largest |x|,
// |x_fix| < 2^20: every value within 2^9 of the block's largest is exact, the
// rest round to 2^-20 of it) held as three byte planes in registers, in the
// order of the code byte vectors: a 32-bit word of 2-bit codes gives four byte
// vectors with one AND each (the codes at bit offsets 2 and 6 of a byte carry
// a factor 4 that is folded into the scale), dp4a takes four code x byte
// products per instruction, and the planes are combined in 32-bit integers:
// the lane's partial dot product over its block is exact for its fixed-point
// x.  Per row: s * 2^e * dot + m * sum(x), summed over the warp with a
// transposed butterfly into a per-(row, segment) slot.  Correction (after the
// base pass, all threads): a thread owns 4 consecutive rows (the r bits of 4
// rows never straddle a 32-bit word) and a share of the selected channels; per
// channel it reads one refinement word and adds x_c * (1 + rho/2^r) to a
// per-row run, and every run of channels in one scale group is scaled once,
// s * (run - sum x_c (1 - off/2^r)) with off = 1/2 - 2^(r-1).  The base pass
// leaves the scales group-major for it.  Every partial has its own slot, so
// the sums are deterministic.
//
// Batch 2 to 8 (gemv_mma_kernel, tensor cores, then corr_only_kernel).  The
// same fixed point, per scale group, as three balanced byte digits; the codes
// of 16 rows x 32 channels are the A operand of an integer mma.m16n8k32 and
// the eight B columns are two batch rows x their digit planes, so every
// decoded code serves two batch rows per instruction and up to four per
// launch.  The correction of every batch row follows in corr_only_kernel.
#include "common.cuh"
#include "internal.cuh"
#include "wqlayout.cuh"

#include <algorithm>

namespace sf {
namespace {

constexpr int kLaneCh = 64;                 // input channels per lane
constexpr int kSegCh = 32 * kLaneCh;        // channels per warp segment
constexpr int kMaxSegs = 16;                // k <= 32,768
constexpr int kMaxWarps = 15;               // compute warps per CTA (plus the producer: 16 warps)
constexpr int kXP = 3;                      // byte planes of the fixed-point activations
constexpr int kXW = 16 * kXP + 4;           // shared words per lane block: planes, sum0, sum1, scale, pad
// x_fix = x * 2^(kXE - ilogb(max |x| of the block)): |x_fix| < 2^(kXE + 1), so
// 4 * sum code * x_fix over 64 channels fits an int32 for every base width
constexpr int kXE = 19;
constexpr int kRowUnit = 4;                 // CTA row ranges start at multiples of 4
constexpr size_t kSmemLimit = 227 * 1024;   // dynamic shared memory of one CTA
constexpr size_t kStageTarget = 36 * 1024;  // bytes of codes per ring stage, at most
constexpr size_t kStageMax = 56 * 1024;     // batch form: bytes per stage above one row block, at most
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
// cw: the row's 16 bytes of codes of this lane (plane L; b = 4: cw and cw2,
// the block's two 16-byte units), hw: its 8 bytes of plane H (b = 3), zw:
// the row's (s, m) word(s) for the lane's group(s).
template <int BITS, int ZW>
__device__ __forceinline__ float lane_row(const uint8_t* __restrict__ cw, const uint8_t* __restrict__ cw2,
                                          const uint8_t* __restrict__ hw, const uint32_t (&xr)[16 * kXP],
                                          float xs0, float xs1, float xsc, uint32_t z0, uint32_t z1) {
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
    const uint4 q0 = *reinterpret_cast<const uint4*>(cw), q1 = *reinterpret_cast<const uint4*>(cw2);
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
          // 16-byte unit u of a packed row sits at unit u ^ (row mod 8)
          const int sw = (n0 + lr) & 7;
          const uint8_t* rowp = sl + (size_t)rr * a.rowL;
          const uint8_t* cw = rowp + ((BITS == 4 ? (2 * lg) ^ sw : lg ^ sw) << 4);
          const uint8_t* cw2 = rowp + ((BITS == 4 ? (2 * lg + 1) ^ sw : 0) << 4);
          const uint8_t* hw = sl + (size_t)a.rc * a.rowL + (size_t)rr * a.rowH + ((((lg >> 1) ^ sw) << 4) | (8 * (lg & 1)));
          pv[t] = lane_row<BITS, ZW>(cw, cw2, hw, xr, xs0, xs1, xsc, z0, z1);
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
      const int j0 = q * a.n_sel / Q, j1 = (q + 1) * a.n_sel / Q;
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
          const uint4 z = *reinterpret_cast<const uint4*>(szt + gcur * a.szt_pitch + 4 * blk);
          const uint32_t zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
          for (int t = 0; t < 4; t++)
            acc[t] = fmaf(__low2float(*reinterpret_cast<const __half2*>(&zz[t])), run[t] - C, acc[t]);
        }
      };
      // channel j + 1's table entry and refinement word are read while j is summed
      uint2 d = j0 < j1 ? jd[j0] : make_uint2(0u, 0u);
      uint32_t w = j0 < j1 ? wt[j0 * a.wt_pitch + wi] : 0u;
      for (int j = j0; j < j1; j++) {
        const uint2 dn = j + 1 < j1 ? jd[j + 1] : make_uint2(0u, 0u);
        const uint32_t wn = j + 1 < j1 ? wt[(j + 1) * a.wt_pitch + wi] : 0u;
        if ((int)d.y != gcur) {
          flush();
          gcur = (int)d.y, C = 0.f;
#pragma unroll
          for (int t = 0; t < 4; t++) run[t] = 0.f;
        }
        const float xc = __uint_as_float(d.x);
        // f = 1 + rho / 2^r; sum x f - sum x (1 - off/2^r) = sum x (rho + off) / 2^r
#pragma unroll
        for (int t = 0; t < 4; t++)
          run[t] = fmaf(__uint_as_float(0x3F800000u | (__funnelshift_l(w, w, rot[t]) & fmask)), xc, run[t]);
        C = fmaf(xc, cfac, C);
        d = dn, w = wn;
      }
      flush();
      *reinterpret_cast<float4*>(cpart + (size_t)q * a.rows_max + 4 * blk) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    bar_sync(2, blockDim.x);
  }

  // ---------------- output: T = 2^k threads per row (as many as the block
  // has for its rows, at most 32) sum the row's partials (base pass ranges,
  // correction shares), then combine over their lanes
  {
    int T = 1;
    while (T < 32 && 2 * T * rows <= (int)blockDim.x) T *= 2;
    const int sub = threadIdx.x & (T - 1);
    for (int lr0 = 0; lr0 < rows; lr0 += (int)blockDim.x / T) {
      const int lr = lr0 + (int)threadIdx.x / T;
      const bool in = lr < rows;
      float base = 0.f, c = 0.f;
      if (in) {
        for (int q = sub; q < a.segs; q += T) base += part[lr * a.segs + q];
        if (corr)
          for (int q = sub; q < a.cparts; q += T) c += cpart[(size_t)q * a.rows_max + lr];
      }
      for (int o = T / 2; o > 0; o >>= 1) {
        base += __shfl_xor_sync(0xffffffffu, base, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
      if (in && sub == 0) {
        if (a.y_corr) {
          a.y[n0 + lr] = base;
          a.y_corr[n0 + lr] = c;
        } else {
          a.y[n0 + lr] = base + c;
        }
      }
    }
  }
}


// ---- activations -------------------------------------------------------------

// The activations of one batch row as the B operand of mma.m16n8k32 (s8).
// Per scale group, x = x_fix * 2^(e - kXE) with e = ilogb(max |x| of the
// group) and |x_fix| < 2^(kXE + 1); x_fix is split into balanced byte digits
// x_fix = d0 + 2^8 d1 + 2^16 d2 (d0, d1 in [-128, 127], |d2| <= 16), one
// digit plane per B column.  Unit u = 4 s + t (s: 64-channel block, t: quad
// lane) holds 16 channels; for each plane one uint4 of byte vectors in the
// order the main loop's A fragments take the codes:
//   b = 2, 3: word k, byte L <- channel 64 s + 16 t + 4 L + {0, 2, 1, 3}[k]
//             (the code byte vectors w & 0x03.., (w >> 4) & 0x03.. (set 0),
//             w & 0x0C.., (w >> 4) & 0x0C.. (set 1, codes times 4) of the
//             lane's 2-bit word 4 s + t);
//   b = 4:    word k, byte L <- channel 64 s + 32 (k >> 1) + 8 t + 2 L + (k & 1)
//             (the nibble vectors of the lane's words 8 s + t and 8 s + 4 + t).
// Batch rows go in pairs to the eight columns of an mma: row br's plane p is
// column 4 (br & 1) + p of row pair br / 2 (columns 3 and 7 are not used), and
// its uint4 sits at xb[((s nbp + br / 2) 8 + column) 4 + t], so the eight
// lanes of each quarter-warp read 128 consecutive bytes.  gt[g] (the row's table) =
// (2^(e - kXE) / 4 (b = 2, 3) or 2^(e - kXE) (b = 4), sum of x over group g).
// SPLIT (b = 4 with 32-channel groups): the unit's two halves lie in two
// groups.  rw: units per group (SPLIT: 4, the units of one block).
template <int BITS, bool SPLIT>
__device__ __forceinline__ void build_unit(const uint16_t* __restrict__ x, int u, int rw, int gshift, int nbp,
                                           int br, uint4* __restrict__ xb, float2* __restrict__ gt) {
  const int s = u >> 2, t = u & 3;
  uint32_t h[8];
  {
    const uint16_t* p0 = BITS == 4 ? x + 64 * s + 8 * t : x + 16 * u;
    const uint16_t* p1 = BITS == 4 ? p0 + 32 : p0 + 8;
    const uint4 a0 = *reinterpret_cast<const uint4*>(p0), a1 = *reinterpret_cast<const uint4*>(p1);
    h[0] = a0.x, h[1] = a0.y, h[2] = a0.z, h[3] = a0.w, h[4] = a1.x, h[5] = a1.y, h[6] = a1.z, h[7] = a1.w;
  }
  // the largest |x| (fp16 bits order like magnitudes) and the sum, per half
  uint32_t m2[2] = {0u, 0u};
  float sm[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 8; i++) {
    m2[i >> 2] = __vmaxu2(m2[i >> 2], h[i] & 0x7fff7fffu);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    sm[i >> 2] += f.x + f.y;
  }
  uint32_t mx[2] = {max(m2[0] & 0xffffu, m2[0] >> 16), max(m2[1] & 0xffffu, m2[1] >> 16)};
  if (!SPLIT) mx[0] = mx[1] = max(mx[0], mx[1]), sm[0] += sm[1];
  for (int o = 1; o < rw; o <<= 1) {
#pragma unroll
    for (int hh = 0; hh < 2; hh++) {
      mx[hh] = max(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], o));
      sm[hh] += __shfl_xor_sync(0xffffffffu, sm[hh], o);
    }
  }
  float scale[2], fac[2];
#pragma unroll
  for (int hh = 0; hh < 2; hh++) {
    const int eb = mx[hh] ? ((__float_as_int(h2f((uint16_t)mx[hh])) >> 23) & 0xff) - 127 : 0;  // ilogb
    scale[hh] = mx[hh] ? __int_as_float((127 + kXE - eb) << 23) : 0.f;
    fac[hh] = mx[hh] ? __int_as_float((127 + eb - kXE - (BITS == 4 ? 0 : 2)) << 23) : 1.f;
  }
  // x_fix of the 16 channels in load order (c = 0..15; b = 4: halves of 8)
  int q[16];
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    const float sc = scale[BITS == 4 ? (i >> 2) : 0];
    // round to nearest even through the float mantissa: 1.5 * 2^23 + x_fix
    q[2 * i] = __float_as_int(fmaf(f.x, sc, 12582912.0f)) - 0x4B400000;
    q[2 * i + 1] = __float_as_int(fmaf(f.y, sc, 12582912.0f)) - 0x4B400000;
  }
  uint32_t wd[3][4];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    uint32_t acc[3] = {0u, 0u, 0u};
#pragma unroll
    for (int L = 0; L < 4; L++) {
      constexpr int perm[4] = {0, 2, 1, 3};
      const int c = BITS == 4 ? 8 * (k >> 1) + 2 * L + (k & 1) : 4 * L + perm[k];
      const int v = q[c];
      const int d0 = ((v + 128) & 255) - 128;
      const int v1 = (v - d0) >> 8;
      const int d1 = ((v1 + 128) & 255) - 128;
      const int d2 = (v1 - d1) >> 8;
      acc[0] |= (uint32_t)(d0 & 255) << (8 * L);
      acc[1] |= (uint32_t)(d1 & 255) << (8 * L);
      acc[2] |= (uint32_t)(d2 & 255) << (8 * L);
    }
#pragma unroll
    for (int p = 0; p < 3; p++) wd[p][k] = acc[p];
  }
#pragma unroll
  for (int p = 0; p < 3; p++)
    xb[((s * nbp + (br >> 1)) * 8 + 4 * (br & 1) + p) * 4 + t] = make_uint4(wd[p][0], wd[p][1], wd[p][2], wd[p][3]);
  if (SPLIT) {
    if (t == 0) gt[2 * s] = make_float2(fac[0], sm[0]), gt[2 * s + 1] = make_float2(fac[1], sm[1]);
  } else if ((u & (rw - 1)) == 0) {
    gt[(u * 16) >> gshift] = make_float2(fac[0], sm[0]);
  }
}

// ---- the tensor-core product ----------------------------------------------------

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// The four code byte vectors of one 16-channel word of 2-bit codes (b = 3:
// with the high bits of its 32-channel block word H merged in; par: which
// half of the block the word is): c[0] = codes of channels 0, 4, 8, 12 of
// the word, c[2] of 2, 6, 10, 14 (set 0), c[1] of 1, 5, 9, 13 and c[3] of
// 3, 7, 11, 15, each times 4 (set 1).
template <int BITS>
__device__ __forceinline__ void code_vectors(uint32_t w, uint32_t H, int par, uint32_t (&c)[4]) {
  const uint32_t w4 = w >> 4;
  c[0] = w & 0x03030303u, c[1] = w & 0x0C0C0C0Cu, c[2] = w4 & 0x03030303u, c[3] = w4 & 0x0C0C0C0Cu;
  if constexpr (BITS == 3) {
    // the high bit of channel 4 L + m (+16 in the block's second half) sits at
    // bit 8 L + m (+4) of H; it joins at bit 2 (set 0) or bit 4 (set 1)
    if (par == 0) {
      c[0] |= (H << 2) & 0x04040404u, c[1] |= (H << 3) & 0x10101010u;
      c[2] |= H & 0x04040404u, c[3] |= (H << 1) & 0x10101010u;
    } else {
      c[0] |= (H >> 2) & 0x04040404u, c[1] |= (H >> 1) & 0x10101010u;
      c[2] |= (H >> 4) & 0x04040404u, c[3] |= (H >> 3) & 0x10101010u;
    }
  }
}

// D = A B (the accumulator starts from zero).
__device__ __forceinline__ void mma_s8_zero(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// Row sums per digit plane: acc[0], acc[1] (row gid, the lane's C columns 2t,
// 2t + 1), acc[2], acc[3] (row gid + 8), and the offset terms am[0], am[1].
struct RowAcc {
  float acc[4], am[2];
};

// One group's integer dot products (J[i]: 4 sum code x_fix for b = 2, 3 or
// sum code x_fix for b = 4, per digit plane = C column) into the rows' sums:
// s * fac * dot per column, m * sum(x) once per row.
__device__ __forceinline__ void group_epilogue(const int (&J)[4], float2 fx, uint32_t z0, uint32_t z1,
                                               RowAcc& ra) {
  const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&z0));
  const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&z1));
  const float f0 = s0.x * fx.x, f1 = s1.x * fx.x;
  ra.acc[0] = fmaf(f0, (float)J[0], ra.acc[0]);
  ra.acc[1] = fmaf(f0, (float)J[1], ra.acc[1]);
  ra.acc[2] = fmaf(f1, (float)J[2], ra.acc[2]);
  ra.acc[3] = fmaf(f1, (float)J[3], ra.acc[3]);
  ra.am[0] = fmaf(s0.y, fx.y, ra.am[0]);
  ra.am[1] = fmaf(s1.y, fx.y, ra.am[1]);
}

// The two rows' sums from the per-plane columns: plane 0 and 1 are the
// columns of quad lane 0, plane 2 column 2 (quad lane 1).  Valid in quad lane 0.
__device__ __forceinline__ void combine_planes(const RowAcc& ra, float& y0, float& y1) {
  const float p2a = __shfl_down_sync(0xffffffffu, ra.acc[0], 1);
  const float p2b = __shfl_down_sync(0xffffffffu, ra.acc[2], 1);
  y0 = fmaf(65536.0f, p2a, fmaf(256.0f, ra.acc[1], ra.acc[0])) + ra.am[0];
  y1 = fmaf(65536.0f, p2b, fmaf(256.0f, ra.acc[3], ra.acc[2])) + ra.am[1];
}

// The sums of the lane's rows (gid, gid + 8) of one 16-row block for NBP pairs
// of batch rows over blocks [b0, b1) of max(G, 64) channels, per digit plane
// (acc[p]: row pair p; the lane's columns are batch row 2 p + t / 2).  ra, rb:
// the rows' codes (plane L) in shared memory; ha, hb: their plane H rows
// (b = 3); sw: the rows' unit permutation (row mod 8).  xbl: the lane's column
// of the B operand (xb + 4 gid + t).  gtl: the group table of the lane's batch
// row for each pair (gt + (2 p + t / 2) gpr).  za, zb: the rows' (s, m) words,
// group-major (group j at j zp).  GM = G / 64 (0: G = 32).
template <int BITS, int GM, int NBP>
__device__ __forceinline__ void row_pairs(const uint8_t* __restrict__ ra, const uint8_t* __restrict__ rb,
                                          const uint8_t* __restrict__ ha, const uint8_t* __restrict__ hb, int sw,
                                          const uint4* __restrict__ xbl, const float2* const (&gtl)[NBP],
                                          const uint32_t* __restrict__ za, const uint32_t* __restrict__ zb, int zp,
                                          int b0, int b1, int t, RowAcc (&acc)[NBP]) {
  const int swt = sw << 4, t4 = 4 * t;
  // the A fragments of 64-channel block s: set 0 (codes) and set 1 (codes
  // times 4; b = 4: the block's second k-step); 16-byte unit u of a row sits
  // at unit u ^ sw
  auto frags = [&](int s, uint32_t (&f0)[4], uint32_t (&f1)[4]) {
    if constexpr (BITS == 4) {
      const int o1 = ((s << 5) ^ swt) | t4, o2 = o1 ^ 16;
      const uint32_t wa = lds32(ra + o1), wb = lds32(rb + o1), va = lds32(ra + o2), vb = lds32(rb + o2);
      f0[0] = wa & 0x0F0F0F0Fu, f0[1] = wb & 0x0F0F0F0Fu, f0[2] = (wa >> 4) & 0x0F0F0F0Fu, f0[3] = (wb >> 4) & 0x0F0F0F0Fu;
      f1[0] = va & 0x0F0F0F0Fu, f1[1] = vb & 0x0F0F0F0Fu, f1[2] = (va >> 4) & 0x0F0F0F0Fu, f1[3] = (vb >> 4) & 0x0F0F0F0Fu;
    } else {
      // word 4 s + t of plane L; word 2 s + t / 2 of plane H (its block's high bits)
      const int o = ((s << 4) ^ swt) | t4;
      const int oh = (((s >> 1) << 4) ^ swt) | (4 * ((2 * s + (t >> 1)) & 3));
      uint32_t ca[4], cb[4];
      code_vectors<BITS>(lds32(ra + o), BITS == 3 ? lds32(ha + oh) : 0u, t & 1, ca);
      code_vectors<BITS>(lds32(rb + o), BITS == 3 ? lds32(hb + oh) : 0u, t & 1, cb);
      f0[0] = ca[0], f0[1] = cb[0], f0[2] = ca[2], f0[3] = cb[2];
      f1[0] = ca[1], f1[1] = cb[1], f1[2] = ca[3], f1[3] = cb[3];
    }
  };
  auto finish = [&](int g, const int (&C0)[NBP][4], const int (&C1)[NBP][4]) {
    const uint32_t z0 = za[g * zp], z1 = zb[g * zp];
#pragma unroll
    for (int p = 0; p < NBP; p++) {
      int J[4];
#pragma unroll
      for (int i = 0; i < 4; i++) J[i] = BITS == 4 ? C0[p][i] + C1[p][i] : 4 * C0[p][i] + C1[p][i];
      group_epilogue(J, gtl[p][g], z0, z1, acc[p]);
    }
  };
  if constexpr (GM >= 1) {
    for (int g = b0; g < b1; g++) {
      int C0[NBP][4], C1[NBP][4];
#pragma unroll
      for (int m = 0; m < GM; m++) {
        const int s = g * GM + m;
        uint32_t f0[4], f1[4];
        frags(s, f0, f1);
#pragma unroll
        for (int p = 0; p < NBP; p++) {
          const uint4 xv = xbl[(s * NBP + p) * 32];
          if (m == 0) {
            mma_s8_zero(C0[p], f0[0], f0[1], f0[2], f0[3], xv.x, xv.y);
            mma_s8_zero(C1[p], f1[0], f1[1], f1[2], f1[3], xv.z, xv.w);
          } else {
            mma_s8(C0[p], f0[0], f0[1], f0[2], f0[3], xv.x, xv.y);
            mma_s8(C1[p], f1[0], f1[1], f1[2], f1[3], xv.z, xv.w);
          }
        }
      }
      finish(g, C0, C1);
    }
  } else {
    // 32-channel groups: block s holds groups 2 s and 2 s + 1
    for (int s = b0; s < b1; s++) {
      uint32_t f0[4], f1[4];
      frags(s, f0, f1);
      int Ca0[NBP][4], Ca1[NBP][4], Cb0[NBP][4], Cb1[NBP][4];  // group 2 s: Ca, group 2 s + 1: Cb
#pragma unroll
      for (int p = 0; p < NBP; p++) {
        const uint4 xv = xbl[(s * NBP + p) * 32];
        if constexpr (BITS == 4) {
          // the block's two k-steps are the two groups
          mma_s8_zero(Ca0[p], f0[0], f0[1], f0[2], f0[3], xv.x, xv.y);
          mma_s8_zero(Cb0[p], f1[0], f1[1], f1[2], f1[3], xv.z, xv.w);
#pragma unroll
          for (int i = 0; i < 4; i++) Ca1[p][i] = Cb1[p][i] = 0;
        } else {
          // quad lanes 0, 1 hold group 2 s, lanes 2, 3 group 2 s + 1: each
          // group's products take the other lanes' activations as zero
          const bool lo = t < 2;
          mma_s8_zero(Ca0[p], f0[0], f0[1], f0[2], f0[3], lo ? xv.x : 0u, lo ? xv.y : 0u);
          mma_s8_zero(Ca1[p], f1[0], f1[1], f1[2], f1[3], lo ? xv.z : 0u, lo ? xv.w : 0u);
          mma_s8_zero(Cb0[p], f0[0], f0[1], f0[2], f0[3], lo ? 0u : xv.x, lo ? 0u : xv.y);
          mma_s8_zero(Cb1[p], f1[0], f1[1], f1[2], f1[3], lo ? 0u : xv.z, lo ? 0u : xv.w);
        }
      }
      finish(2 * s, Ca0, Ca1);
      finish(2 * s + 1, Cb0, Cb1);
    }
  }
}

struct MmaArgs {
  const uint8_t* base;      // codes; b = 3: plane L then plane H (hi_off bytes in)
  const uint32_t* sz;       // [N][gpr] words: fp16 (s, m)
  const uint16_t* x;        // [nb][K] fp16
  float* y;                 // [nb][N]
  size_t hi_off;
  int N, K, gpr, gshift, nb;  // nb: batch rows of this launch (at most 2 NBP)
  int nblk, nseg, rb, W;    // blocks of max(G, 64) channels, group ranges, row blocks per stage, compute warps
  int rc, stages;           // rows per stage (16 rb), ring depth
  int rowL, rowH;           // bytes per row of plane L (all codes for b = 2, 4) and of plane H
  int stage_bytes, rows_max;
  int off_ring, off_szt, off_szs, off_xb, off_gt, off_part;  // shared memory offsets
  int szt_pitch;
};

// The batch form of the base product: one CTA per SM over a contiguous range
// of rows (a multiple of 4), the codes streamed once for up to 2 NBP batch
// rows, which share every decoded A fragment.  A producer warp streams
// 16-row stages with one bulk copy per stage and plane (and the rows' (s, m)
// words once, transposed group-major in shared memory before the grid
// dependency wait); each compute warp owns one (16-row block, range of
// groups) item per stage.  No correction: gemv_launch adds it with
// corr_only_kernel.
constexpr int kMmaWarps = 16;  // compute warps (plus the producer: 17 warps)
constexpr int kMmaRegs = 96;
static_assert(((kMmaWarps + 1 + 3) / 4) * kMmaRegs * 32 + kSideRegs / 4 <= 65536 / 4,
              "batch GEMV registers leave no room for a staging CTA");
template <int BITS, int GM, int NBP>
__global__ void __maxnreg__(kMmaRegs) gemv_mma_kernel(MmaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  uint64_t* szbar = empty + kMaxStages;
  uint8_t* ring = smem + a.off_ring;
  uint32_t* szs = reinterpret_cast<uint32_t*>(smem + a.off_szs);  // [rows][gpr], as copied
  uint32_t* szt = reinterpret_cast<uint32_t*>(smem + a.off_szt);  // [gpr][szt_pitch]
  uint4* xb = reinterpret_cast<uint4*>(smem + a.off_xb);
  float2* gt = reinterpret_cast<float2*>(smem + a.off_gt);        // [2 NBP][gpr]
  float* part = reinterpret_cast<float*>(smem + a.off_part);      // [2 NBP][rows_max][nseg]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int units = a.N / kRowUnit;
  const int n0 = (int)((long)blockIdx.x * units / gridDim.x) * kRowUnit;
  const int n1 = (int)((long)(blockIdx.x + 1) * units / gridDim.x) * kRowUnit;
  const int rows = n1 - n0;
  const int nst = (rows + a.rc - 1) / a.rc;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; s++) mbar_init(&full[s], 1), mbar_init(&empty[s], a.W);
    mbar_init(szbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  pdl_trigger();  // the next kernel of the stream may be scheduled; it waits for this grid

  if (warp == a.W) {
    // ---------------- producer warp (lane 0)
    auto issue = [&](int i) {
      const int slot = i % S;
      const int r0 = i * a.rc, nr = min(a.rc, rows - r0);
      const uint32_t bl = (uint32_t)(nr * a.rowL), bh = (uint32_t)(nr * a.rowH);
      uint8_t* dst = ring + (size_t)slot * a.stage_bytes;
      mbar_expect_tx(&full[slot], bl + bh);
      bulk_g2s(dst, a.base + (size_t)(n0 + r0) * a.rowL, bl, &full[slot]);
      if (BITS == 3) bulk_g2s(dst + (size_t)a.rc * a.rowL, a.base + a.hi_off + (size_t)(n0 + r0) * a.rowH, bh, &full[slot]);
    };
    int issued = 0;
    if (lane == 0) {
      const uint32_t zbytes = (uint32_t)(rows * a.gpr * 4);
      mbar_expect_tx(szbar, zbytes);
      bulk_g2s(szs, a.sz + (size_t)n0 * a.gpr, zbytes, szbar);
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
    const int ntc = a.W * 32;
    const int t = lane & 3, gid = lane >> 2;
    // the scale table does not depend on earlier kernels: transposed before
    // the grid dependency wait
    bool ok = mbar_wait(szbar, 0);
    for (int r = warp; r < rows; r += a.W)
      for (int g = lane; g < a.gpr; g += 32) szt[g * a.szt_pitch + r] = szs[r * a.gpr + g];
    pdl_wait();  // x is complete
    {
      const int nu = a.K / 16;
      const int rw = (BITS == 4 && GM == 0) ? 4 : (1 << (a.gshift - 4));
      for (int br = 0; br < a.nb; br++)
        for (int u0 = warp * 32; u0 < nu; u0 += ntc) {
          if (BITS == 4 && GM == 0)
            build_unit<BITS, true>(a.x + (size_t)br * a.K, u0 + lane, rw, a.gshift, NBP, br, xb, gt + br * a.gpr);
          else
            build_unit<BITS, false>(a.x + (size_t)br * a.K, u0 + lane, rw, a.gshift, NBP, br, xb, gt + br * a.gpr);
        }
    }
    bar_sync(1, a.W * 32);  // B operand, group tables and scale table complete
    // the warp's item, the same in every stage (rb nseg <= W): row block rbk
    // of the stage, blocks [b0, b1) of the channels
    const bool has_item = warp < a.rb * a.nseg;
    const int rbk = warp / a.nseg, sg = warp % a.nseg;
    const int b0 = sg * a.nblk / a.nseg, b1 = (sg + 1) * a.nblk / a.nseg;
    const uint32_t ra_off = (uint32_t)(16 * rbk + gid) * a.rowL;
    const uint32_t ha_off = (uint32_t)a.rc * a.rowL + (uint32_t)(16 * rbk + gid) * a.rowH;
    const uint4* xbl = xb + 4 * gid + t;
    const float2* gtl[NBP];
#pragma unroll
    for (int p = 0; p < NBP; p++) gtl[p] = gt + min(2 * p + (t >> 1), a.nb - 1) * a.gpr;
    for (int i = 0; i < nst && ok; i++) {
      const int slot = i % S;
      if (!mbar_wait(&full[slot], (i / S) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* sl = ring + (size_t)slot * a.stage_bytes;
      const int lr0 = i * a.rc + 16 * rbk;
      if (has_item && lr0 < rows) {
        const uint8_t* ra = sl + ra_off;
        const uint8_t* ha = sl + ha_off;
        // rows past the end read the last row's scales (their sums are not stored)
        const int la = min(lr0 + gid, rows - 1), lb = min(lr0 + gid + 8, rows - 1);
        RowAcc acc[NBP];
#pragma unroll
        for (int p = 0; p < NBP; p++) acc[p] = RowAcc{{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f}};
        row_pairs<BITS, GM, NBP>(ra, ra + 8 * a.rowL, ha, ha + 8 * a.rowH, (n0 + lr0 + gid) & 7, xbl, gtl,
                                 szt + la, szt + lb, a.szt_pitch, b0, b1, t, acc);
#pragma unroll
        for (int p = 0; p < NBP; p++) {
          float y0, y1;
          combine_planes(acc[p], y0, y1);
          const int br = 2 * p + (t >> 1);
          if ((t & 1) == 0 && br < a.nb) {
            float* pr = part + (size_t)br * a.rows_max * a.nseg;
            if (lr0 + gid < rows) pr[(lr0 + gid) * a.nseg + sg] = y0;
            if (lr0 + gid + 8 < rows) pr[(lr0 + gid + 8) * a.nseg + sg] = y1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  }
  __syncthreads();  // every partial is in place

  // ---------------- output: T = 2^k threads per (batch row, row) sum its
  // range partials, then combine over their lanes
  {
    const int items = a.nb * rows;
    int T = 1;
    while (T < 16 && 2 * T * items <= (int)blockDim.x) T *= 2;
    const int sub = threadIdx.x & (T - 1);
    for (int e0 = 0; e0 < items; e0 += (int)blockDim.x / T) {
      const int e = e0 + (int)threadIdx.x / T;
      const bool in = e < items;
      const int br = in ? e / rows : 0, lr = in ? e - br * rows : 0;
      float v = 0.f;
      if (in)
        for (int q = sub; q < a.nseg; q += T) v += part[((size_t)br * a.rows_max + lr) * a.nseg + q];
      for (int o = T / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (in && sub == 0) a.y[(size_t)br * a.N + n0 + lr] = v;
    }
  }
}


// ---------------------------------------------------------------------------
// the correction on its own (fetch lag), added into y
//
// A warp owns 8 consecutive output rows of one batch row; its lanes walk
// consecutive shares of the selected channels in order: per channel a lane
// reads the refinement word that covers the rows, adds x_c f_t,
// f_t = 1 + rho_t / 2^r, into a per-row run, and scales each run of channels
// that share a scale group once, s (run - sum x_c cfac) = s sum x_c
// (rho + off) / 2^r.  The lanes' sums are combined by a fixed butterfly, so
// the result is deterministic.  CTAs of 64 threads, at most 64 registers and
// no shared memory fit in the room every whole-SM kernel of the library
// leaves free, so on a staging stream the correction neither waits for them
// nor delays them.

constexpr int kCorrThreads = 64;
constexpr int kCorrRows = 8;
static_assert(kCorrThreads * 64 <= kSideRegs, "a correction CTA must fit in the room left for staging");

struct CorrArgs {
  const uint32_t* refine;  // channel-major rows [K][row_words], or staged rows [batch][n_sel][row_words]
  const uint16_t* sz;
  const uint16_t* x;
  const int32_t* sel;
  float* y;
  int N, K, gshift, r, n_sel, row_words, staged, units;  // units (one warp each) = batch * N / kCorrRows
  int overwrite;           // y = correction (else y += correction)
};

template <int R>
__global__ void __maxnreg__(64) corr_only_kernel(CorrArgs a) {
  const int lane = threadIdx.x & 31;
  const int u = (blockIdx.x * kCorrThreads + (int)threadIdx.x) >> 5;
  if (u >= a.units) return;  // whole warps
  const int per_b = a.N / kCorrRows;
  const int b = u / per_b, row0 = (u - b * per_b) * kCorrRows;
  const int bit0 = row0 * a.r, wi = bit0 >> 5;
  // the rows' bits start at bit sh of the word (a multiple of 8); the word is
  // shifted down first, so row t's field sits at bit R t
  const int sh = bit0 & 31;
  constexpr uint32_t fmask = ((1u << R) - 1u) << (23 - R);
  const float cfac = 1.0f - (0.5f - 0.5f * (float)(1 << R)) / (float)(1 << R);
  const int gpr = a.K >> a.gshift;
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
        const uint32_t zw = __ldg(zrow + (t * gpr + gcur));
        acc[t] = fmaf(__low2float(*reinterpret_cast<const __half2*>(&zw)), run[t] - C, acc[t]);
      }
    }
  };
  // entry j: channel, activation (-1 - c: selected, not refined now: x = 0)
  // and the rows' refinement word, from one load of the selection
  auto entry = [&](int j, int& c, float& xc, uint32_t& w) {
    const int raw = __ldg(sel + j);
    c = min(max(raw < 0 ? -1 - raw : raw, 0), a.K - 1);
    xc = raw < 0 ? 0.f : h2f(__ldg(xb + c));
    const size_t row = a.staged ? (size_t)b * a.n_sel + j : (size_t)c;
    w = __ldg(a.refine + row * a.row_words + wi) >> sh;
  };
  // the lane's share [j0, j1); channel j + 1's index, activation and word are
  // loaded while j is summed
  const int j0 = lane * a.n_sel / 32, j1 = (lane + 1) * a.n_sel / 32;
  int c = 0;
  float xc = 0.f;
  uint32_t w = 0u;
  if (j0 < j1) entry(j0, c, xc, w);
  for (int j = j0; j < j1; j++) {
    int cn = 0;
    float xn = 0.f;
    uint32_t wn = 0u;
    if (j + 1 < j1) entry(j + 1, cn, xn, wn);
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
  // the 8 rows' sums over the warp, reduced and scattered at once: each round
  // keeps the half of the rows that the lane's bit selects and adds the
  // partner's copy; lane l ends with row (l >> 2) & 7 (a fixed order)
  static_assert(kCorrRows == 8, "the reduction below is written for 8 rows");
#pragma unroll
  for (int n = 8, o = 16; n > 1; n >>= 1, o >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int t = 0; t < n / 2; t++) {
      const float keep = up ? acc[t + n / 2] : acc[t], send = up ? acc[t] : acc[t + n / 2];
      acc[t] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float v = acc[0];
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  if ((lane & 3) != 0) return;
  float* yr = a.y + (size_t)b * a.N + row0 + ((lane >> 2) & 7);
  *yr = a.overwrite ? v : *yr + v;
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
  // channel shares of the correction: every thread busy when the CTA has few
  // rows (the output sums a row's shares on the lanes of a warp)
  a.cparts = n_sel > 0 ? std::max(1, std::min(std::min(n_sel, 64), P.threads / nb_max)) : 0;
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

// The batch form's split and shared memory layout for nbp row pairs: 16-row
// blocks per stage and group ranges per row block (each compute warp takes one
// (row block, range) item per stage; the split with the least work for the
// busiest warp), the ring depth that fits.
struct MmaPlan {
  MmaArgs a;
  int grid, threads, gm;
  size_t smem;
};

sf_status make_mma_plan(const sf_wq* w, int nbp, MmaPlan& P) {
  MmaArgs& a = P.a;
  a = MmaArgs{};
  const int N = w->n, K = w->k, G = w->group;
  a.N = N, a.K = K;
  a.gpr = K / G;
  a.gshift = 0;
  while ((1 << a.gshift) < G) a.gshift++;
  P.gm = G / 64;  // 0: 32-channel groups
  a.nblk = K / std::max(G, 64);
  a.rowL = K * (w->b == 4 ? 4 : 2) / 8;
  a.rowH = w->b == 3 ? K / 8 : 0;
  a.hi_off = w->b == 3 ? (size_t)N * K / 4 : 0;
  const size_t rowB = (size_t)a.rowL + a.rowH;
  const int units = N / kRowUnit;
  P.grid = std::min(num_sms(), units);
  a.rows_max = ((units + P.grid - 1) / P.grid) * kRowUnit;
  a.W = kMmaWarps;
  {
    const int blocks = (a.rows_max + 15) / 16;
    long best = -1;
    for (int rb = 1; rb <= std::min(blocks, 4); rb++) {
      if (rb > 1 && (size_t)rb * 16 * rowB > kStageMax) break;
      const int nseg = std::max(1, std::min(a.nblk, a.W / rb));
      const long cost = (long)((blocks + rb - 1) / rb) * ((a.nblk + nseg - 1) / nseg);
      if (best < 0 || cost < best) best = cost, a.rb = rb, a.nseg = nseg;
    }
  }
  a.rc = 16 * a.rb;
  a.stage_bytes = (int)(a.rc * rowB);
  a.szt_pitch = (a.rows_max + 3) & ~3;
  P.threads = (a.W + 1) * 32;
  size_t off = align128((2 * kMaxStages + 1) * sizeof(uint64_t));
  a.off_szt = (int)off;
  off += align128((size_t)a.gpr * a.szt_pitch * 4);
  a.off_szs = (int)off;
  off += align128((size_t)a.rows_max * a.gpr * 4);
  a.off_xb = (int)off;
  off += align128((size_t)K / 64 * nbp * 8 * 4 * 16);
  a.off_gt = (int)off;
  off += align128((size_t)2 * nbp * a.gpr * 8);
  a.off_part = (int)off;
  off += align128((size_t)2 * nbp * a.rows_max * a.nseg * 4);
  a.off_ring = (int)off;
  const int nst_max = (a.rows_max + a.rc - 1) / a.rc;
  int S = std::min(kMaxStages, nst_max);
  while (S > 1 && off + (size_t)S * a.stage_bytes > kSmemLimit) S--;
  SF_UNSUPPORTED(off + (size_t)S * a.stage_bytes <= kSmemLimit,
                 "n=%d, k=%d, %d batch rows: %zu bytes of shared memory needed", N, K, 2 * nbp,
                 off + (size_t)S * a.stage_bytes);
  a.stages = S;
  P.smem = off + (size_t)S * a.stage_bytes;
  return SF_OK;
}

template <int BITS, int NBP>
void* mma_kernel_for(int gm) {
  switch (gm) {
    case 0: return (void*)gemv_mma_kernel<BITS, 0, NBP>;
    case 1: return (void*)gemv_mma_kernel<BITS, 1, NBP>;
    case 2: return (void*)gemv_mma_kernel<BITS, 2, NBP>;
    default: return (void*)gemv_mma_kernel<BITS, 4, NBP>;
  }
}

template <int NBP>
void* pick_mma_kernel_n(int b, int gm) {
  if (b == 2) return mma_kernel_for<2, NBP>(gm);
  if (b == 3) return mma_kernel_for<3, NBP>(gm);
  return mma_kernel_for<4, NBP>(gm);
}

void* pick_mma_kernel(int b, int gm, int nbp) {
  return nbp == 1 ? pick_mma_kernel_n<1>(b, gm) : pick_mma_kernel_n<2>(b, gm);
}

// The batch form's base products for batch rows [0, batch): launches of up to
// 4 rows (2 row pairs: the accumulators of more pairs do not fit the
// registers), one pair when two do not leave room for a ring of two stages.
sf_status launch_mma(const sf_wq* w, const uint16_t* x, int batch, float* y, cudaStream_t s) {
  int done = 0;
  while (done < batch) {
    int nbp = std::min(2, (batch - done + 1) / 2);
    MmaPlan P;
    sf_status st = SF_ERR_UNSUPPORTED;
    for (; nbp >= 1; nbp /= 2) {
      st = make_mma_plan(w, nbp, P);
      if (st == SF_OK && (P.a.stages >= 2 || nbp == 1)) break;
    }
    if (st != SF_OK) return st;
    const int nb = std::min(2 * nbp, batch - done);
    MmaArgs a = P.a;
    a.base = (const uint8_t*)w->base;
    a.sz = (const uint32_t*)w->sz;
    a.x = x + (size_t)done * w->k;
    a.y = y + (size_t)done * w->n;
    a.nb = nb;
    void* kern = pick_mma_kernel(w->b, P.gm, nbp);
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
    void* args[] = {&a};
    SF_CUDA(cudaLaunchKernelExC(&cfg, kern, args));
    done += nb;
  }
  return SF_OK;
}

// corr_only_kernel over batch rows [0, batch): y (+)= the corrections of the
// selected channels (a plain launch: on a staging stream it follows an event
// wait; after the batch form's base products it follows them in order).
sf_status launch_corr(const sf_wq* w, const uint16_t* x, int batch, int chunk, int kch, const int32_t* sel,
                      const void* refine_rows, float* y, bool overwrite, cudaStream_t s) {
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
  a.overwrite = overwrite;
  const int blocks = (a.units * 32 + kCorrThreads - 1) / kCorrThreads;
  if (a.r == 2)
    corr_only_kernel<2><<<blocks, kCorrThreads, 0, s>>>(a);
  else
    corr_only_kernel<1><<<blocks, kCorrThreads, 0, s>>>(a);
  SF_LAUNCHED();
  return SF_OK;
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
  // the selection (when not given), then the GEMV, which waits for it (and for
  // x) through programmatic dependent launch while its first code copies fly
  const int32_t* sel = sel_in;
  if (kch > 0 && !sel_in) {
    st = launch_select(x, batch, w->k, chunk, kch, sel_out, s, true);
    if (st != SF_OK) return st;
    sel = sel_out;
  }
  if (batch > 1) {
    // batch form: the base products of every row on the tensor cores, then
    // the corrections (into y_corr, or added into y)
    st = launch_mma(w, x, batch, y, s);
    if (st != SF_OK) return st;
    if (n_sel > 0) return launch_corr(w, x, batch, chunk, kch, sel, refine_rows, y_corr ? y_corr : y, y_corr != nullptr, s);
    return SF_OK;
  }
  Plan P;
  st = make_plan(w, n_sel, P);
  if (st != SF_OK) return st;
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
  // batch 1 (the loop keeps the per-row addressing general)
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
  return launch_corr(w, x, batch, chunk, kch, sel, refine_rows, y, false, as_stream(stream));
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
