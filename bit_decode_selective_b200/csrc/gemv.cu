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
// Producer warp: streams the CTA's codes through a ring of shared memory
// stages of 16-row blocks with 1-D bulk copies (cp.async.bulk; completion
// counted on an mbarrier per stage; one copy per stage and plane), and copies
// the rows' (s, m) words once.  The packed rows are stored with their 16-byte
// units permuted by row mod 8 (wqlayout.cuh), so the eight rows a quad-lane
// load touches fall in distinct banks.  The weights do not depend on earlier
// kernels, so these copies start before the grid dependency wait and overlap
// the previous kernel's tail.
//
// Compute warps: the inner sums run on the tensor cores as integer products,
// mma.sync m16n8k32 with s8 operands and s32 accumulation: A = 16 rows x 32
// channels of codes (byte vectors cut from the packed words with one AND,
// or a shift and an AND), B = the activations of the same channels in fixed
// point, one balanced byte digit per column (x_fix = d0 + 2^8 d1 + 2^16 d2,
// x = x_fix * 2^(e - 19) per scale group, e from the group's largest |x|:
// every value within 2^9 of the group's largest is exact, the rest round to
// 2^-20 of it).  A k-step's 32 channels all lie in one scale group, so each
// group's dot product per row and digit is exact in the s32 accumulator; the
// digits are combined in fp32 and the group scaled once: s * 2^(e-19) * dot
// + m * sum(x).  Work items are (16-row block, range of groups) of a stage;
// their partial sums go to per-(row, range) slots.
//
// Correction (after the base pass, all threads): a thread owns 4 consecutive
// rows (the r bits of 4 rows never straddle a 32-bit word) and a share of the
// selected channels; per channel it reads one refinement word and adds
// x_c * (1 + rho/2^r) to a per-row run, and every run of channels in one scale
// group is scaled once, s * (run - sum x_c (1 - off/2^r)) with
// off = 1/2 - 2^(r-1).  Every partial has its own slot, so the sums are
// deterministic.
#include "common.cuh"
#include "internal.cuh"
#include "wqlayout.cuh"

#include <algorithm>

namespace sf {
namespace {

constexpr int kMaxWarps = 24;               // compute warps per CTA (plus the producer: 25 warps)
constexpr int kXE = 19;                     // |x_fix| < 2^(kXE + 1): three byte digits
constexpr int kRowUnit = 4;                 // CTA row ranges start at multiples of 4
constexpr size_t kSmemLimit = 227 * 1024;   // dynamic shared memory of one CTA
constexpr size_t kStageMax = 56 * 1024;     // bytes of codes per ring stage, at most (above: one row block)
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
  int nseg, nblk, rb, W;    // group ranges, blocks of max(G, 64) channels, row blocks per stage, compute warps
  int rc, stages;           // rows per stage (16 rb), ring depth
  int rowL, rowH;           // bytes per row of plane L (all codes for b = 2, 4) and of plane H
  int stage_bytes;
  int row_words, staged, rows_max;
  int off_ring, off_szt, off_xb, off_gt, off_part, off_jd, off_jrow, off_wt, off_cpart;  // shared memory offsets
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
// Stored at xb[(s * 4 + p) * 4 + t] (p: plane; slot 3 is not used), so the
// eight lanes of each quarter-warp read 128 consecutive bytes.  gt[g] =
// (2^(e - kXE) / 4 (b = 2, 3) or 2^(e - kXE) (b = 4), sum of x over group g).
// SPLIT (b = 4 with 32-channel groups): the unit's two halves lie in two
// groups.  rw: units per group (SPLIT: 4, the units of one block).
template <int BITS, bool SPLIT>
__device__ __forceinline__ void build_unit(const uint16_t* __restrict__ x, int u, int rw, int gshift,
                                           uint4* __restrict__ xb, float2* __restrict__ gt) {
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
  for (int p = 0; p < 3; p++) xb[(s * 4 + p) * 4 + t] = make_uint4(wd[p][0], wd[p][1], wd[p][2], wd[p][3]);
  if (SPLIT) {
    if (t == 0) gt[2 * s] = make_float2(fac[0], sm[0]), gt[2 * s + 1] = make_float2(fac[1], sm[1]);
  } else if ((u & (rw - 1)) == 0) {
    gt[(u * 16) >> gshift] = make_float2(fac[0], sm[0]);
  }
}

// ---- the tensor-core base pass ---------------------------------------------------

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

// The sums of the lane's rows of NB 16-row blocks (rows gid + 8 h, h < 2 NB)
// over blocks [b0, b1) of max(G, 64) channels, per digit plane (acc[k]: row
// block k).  rl: the item's first row (gid) of plane L in shared memory, rh:
// of plane H (b = 3); sw: the rows' unit permutation (row mod 8, the same for
// all of them).  xbl: the lane's column of the B operand (xb + 4 p + t).  z:
// the rows' (s, m) words, group-major (row h, group j at z[h][j * zp]).
// GM = G / 64 (0: G = 32).
template <int BITS, int GM, int NB>
__device__ __forceinline__ void row_blocks(const uint8_t* __restrict__ rl, int rowL, const uint8_t* __restrict__ rh,
                                           int rowH, int sw, const uint4* __restrict__ xbl,
                                           const float2* __restrict__ gt, const uint32_t* const (&z)[2 * NB], int zp,
                                           int b0, int b1, int t, RowAcc (&acc)[NB]) {
  constexpr int NR = 2 * NB;
  const uint8_t* rp[NR];
  const uint8_t* hp[NR];
#pragma unroll
  for (int h = 0; h < NR; h++) rp[h] = rl + h * 8 * rowL, hp[h] = rh + h * 8 * rowH;
  const int swt = sw << 4, t4 = 4 * t;
  // The raw words of 64-channel block s: the lane's plane-L word of each row
  // (b = 4: its two words), its plane-H word (b = 3), its B fragments.  16-byte
  // unit u of a row sits at unit u ^ sw.
  struct Raw {
    uint32_t w[NR], v[NR];
    uint4 xv;
  };
  auto load = [&](int s, Raw& r) {
    r.xv = xbl[s * 16];
    if constexpr (BITS == 4) {
      const int o1 = ((s << 5) ^ swt) | t4, o2 = o1 ^ 16;
#pragma unroll
      for (int h = 0; h < NR; h++) r.w[h] = lds32(rp[h] + o1), r.v[h] = lds32(rp[h] + o2);
    } else {
      // word 4 s + t of plane L; word 2 s + t / 2 of plane H (its block's high bits)
      const int o = ((s << 4) ^ swt) | t4;
#pragma unroll
      for (int h = 0; h < NR; h++) r.w[h] = lds32(rp[h] + o);
      if constexpr (BITS == 3) {
        const int oh = (((s >> 1) << 4) ^ swt) | (4 * ((2 * s + (t >> 1)) & 3));
#pragma unroll
        for (int h = 0; h < NR; h++) r.v[h] = lds32(hp[h] + oh);
      }
    }
  };
  // the A fragments for row block k: set 0 (codes) and set 1 (codes times 4;
  // b = 4: the block's second k-step)
  auto decode = [&](const Raw& r, uint32_t (&f0)[NB][4], uint32_t (&f1)[NB][4]) {
    if constexpr (BITS == 4) {
#pragma unroll
      for (int k = 0; k < NB; k++) {
        const uint32_t wa = r.w[2 * k], wb = r.w[2 * k + 1], va = r.v[2 * k], vb = r.v[2 * k + 1];
        f0[k][0] = wa & 0x0F0F0F0Fu, f0[k][1] = wb & 0x0F0F0F0Fu;
        f0[k][2] = (wa >> 4) & 0x0F0F0F0Fu, f0[k][3] = (wb >> 4) & 0x0F0F0F0Fu;
        f1[k][0] = va & 0x0F0F0F0Fu, f1[k][1] = vb & 0x0F0F0F0Fu;
        f1[k][2] = (va >> 4) & 0x0F0F0F0Fu, f1[k][3] = (vb >> 4) & 0x0F0F0F0Fu;
      }
    } else {
      uint32_t c[NR][4];
#pragma unroll
      for (int h = 0; h < NR; h++) code_vectors<BITS>(r.w[h], BITS == 3 ? r.v[h] : 0u, t & 1, c[h]);
#pragma unroll
      for (int k = 0; k < NB; k++) {
        f0[k][0] = c[2 * k][0], f0[k][1] = c[2 * k + 1][0], f0[k][2] = c[2 * k][2], f0[k][3] = c[2 * k + 1][2];
        f1[k][0] = c[2 * k][1], f1[k][1] = c[2 * k + 1][1], f1[k][2] = c[2 * k][3], f1[k][3] = c[2 * k + 1][3];
      }
    }
  };
  auto frags = [&](int s, uint32_t (&f0)[NB][4], uint32_t (&f1)[NB][4], uint4& xv) {
    Raw r;
    load(s, r);
    decode(r, f0, f1);
    xv = r.xv;
  };
  // a group's epilogue: its scale words and factor are loaded with its codes
  struct Ep {
    uint32_t z[NR];
    float2 fx;
  };
  auto load_ep = [&](int g, Ep& e) {
    e.fx = gt[g];
    const int col = g * zp;
#pragma unroll
    for (int h = 0; h < NR; h++) e.z[h] = z[h][col];
  };
  auto finish = [&](const Ep& e, const int (&C0)[NB][4], const int (&C1)[NB][4]) {
#pragma unroll
    for (int k = 0; k < NB; k++) {
      int J[4];
#pragma unroll
      for (int i = 0; i < 4; i++) J[i] = BITS == 4 ? C0[k][i] + C1[k][i] : 4 * C0[k][i] + C1[k][i];
      group_epilogue(J, e.fx, e.z[2 * k], e.z[2 * k + 1], acc[k]);
    }
  };
  if constexpr (GM >= 1) {
    for (int g = b0; g < b1; g++) {
      int C0[NB][4], C1[NB][4];
#pragma unroll
      for (int m = 0; m < GM; m++) {
        uint4 xv;
        uint32_t f0[NB][4], f1[NB][4];
        frags(g * GM + m, f0, f1, xv);
#pragma unroll
        for (int k = 0; k < NB; k++) {
          if (m == 0) {
            mma_s8_zero(C0[k], f0[k][0], f0[k][1], f0[k][2], f0[k][3], xv.x, xv.y);
            mma_s8_zero(C1[k], f1[k][0], f1[k][1], f1[k][2], f1[k][3], xv.z, xv.w);
          } else {
            mma_s8(C0[k], f0[k][0], f0[k][1], f0[k][2], f0[k][3], xv.x, xv.y);
            mma_s8(C1[k], f1[k][0], f1[k][1], f1[k][2], f1[k][3], xv.z, xv.w);
          }
        }
      }
      Ep e;
      load_ep(g, e);
      finish(e, C0, C1);
    }
  } else {
    // 32-channel groups: block s holds groups 2 s and 2 s + 1
    for (int s = b0; s < b1; s++) {
      uint4 xv;
      uint32_t f0[NB][4], f1[NB][4];
      frags(s, f0, f1, xv);
      int Ca0[NB][4], Ca1[NB][4], Cb0[NB][4], Cb1[NB][4];  // group 2 s: Ca, group 2 s + 1: Cb
#pragma unroll
      for (int k = 0; k < NB; k++) {
        if constexpr (BITS == 4) {
          // the block's two k-steps are the two groups
          mma_s8_zero(Ca0[k], f0[k][0], f0[k][1], f0[k][2], f0[k][3], xv.x, xv.y);
          mma_s8_zero(Cb0[k], f1[k][0], f1[k][1], f1[k][2], f1[k][3], xv.z, xv.w);
#pragma unroll
          for (int i = 0; i < 4; i++) Ca1[k][i] = Cb1[k][i] = 0;
        } else {
          // quad lanes 0, 1 hold group 2 s, lanes 2, 3 group 2 s + 1: each
          // group's products take the other lanes' activations as zero
          const bool lo = t < 2;
          mma_s8_zero(Ca0[k], f0[k][0], f0[k][1], f0[k][2], f0[k][3], lo ? xv.x : 0u, lo ? xv.y : 0u);
          mma_s8_zero(Ca1[k], f1[k][0], f1[k][1], f1[k][2], f1[k][3], lo ? xv.z : 0u, lo ? xv.w : 0u);
          mma_s8_zero(Cb0[k], f0[k][0], f0[k][1], f0[k][2], f0[k][3], lo ? 0u : xv.x, lo ? 0u : xv.y);
          mma_s8_zero(Cb1[k], f1[k][0], f1[k][1], f1[k][2], f1[k][3], lo ? 0u : xv.z, lo ? 0u : xv.w);
        }
      }
      Ep e0, e1;
      load_ep(2 * s, e0);
      load_ep(2 * s + 1, e1);
      finish(e0, Ca0, Ca1);
      finish(e1, Cb0, Cb1);
    }
  }
}

// ---- the kernel -----------------------------------------------------------------

// A CTA's warps are spread over the SM's four schedulers, each with a quarter
// of the register file: seven warps of 64 registers a thread leave kSideRegs
// / 4 of every quarter free for a staging CTA.
constexpr int kGemvRegs = 64;
static_assert(((kMaxWarps + 1 + 3) / 4) * kGemvRegs * 32 + kSideRegs / 4 <= 65536 / 4,
              "GEMV registers leave no room for a staging CTA");
template <int BITS, int GM, int NB>
__global__ void __maxnreg__(kGemvRegs) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  uint64_t* szbar = empty + kMaxStages;
  uint8_t* ring = smem + a.off_ring;
  // the rows' (s, m) words: copied row-major into the region the correction
  // partials take at the end, then transposed group-major (szt) for the
  // epilogue and the correction, whose reads then take consecutive rows of
  // one group
  uint32_t* szs = reinterpret_cast<uint32_t*>(smem + a.off_cpart);  // [rows][gpr]
  uint32_t* szt = reinterpret_cast<uint32_t*>(smem + a.off_szt);  // [gpr][szt_pitch]
  uint4* xb = reinterpret_cast<uint4*>(smem + a.off_xb);
  float2* gt = reinterpret_cast<float2*>(smem + a.off_gt);
  float* part = reinterpret_cast<float*>(smem + a.off_part);
  uint2* jd = reinterpret_cast<uint2*>(smem + a.off_jd);
  uint32_t* wt = reinterpret_cast<uint32_t*>(smem + a.off_wt);
  int* jrow = reinterpret_cast<int*>(smem + a.off_jrow);
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
    // ---------------- producer warp (lane 0): one bulk copy per stage and
    // plane, the rows' (s, m) words in one copy
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
      // the scale table and the first two stages are needed first: the other
      // stages are requested once the table has landed, so that they do not
      // compete with it for the memory system
      const uint32_t zbytes = (uint32_t)(rows * a.gpr * 4);
      mbar_expect_tx(szbar, zbytes);
      bulk_g2s(szs, a.sz + (size_t)n0 * a.gpr, zbytes, szbar);
      for (; issued < min(min(S, nst), 2); issued++) issue(issued);
      mbar_wait(szbar, 0);
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
    const int tc = threadIdx.x, ntc = a.W * 32;
    const int t = lane & 3, gid = lane >> 2, p = gid & 3;
    // the scale table does not depend on earlier kernels: transposed before
    // the grid dependency wait
    bool ok = mbar_wait(szbar, 0);
    for (int r = warp; r < rows; r += a.W)
      for (int g = lane; g < a.gpr; g += 32) szt[g * a.szt_pitch + r] = szs[r * a.gpr + g];
    pdl_wait();  // x, the selection and the staged rows are complete
    // correction tables, entries tc, tc + ntc, ...: the selection's loads are
    // issued first, their activations after the B operand (every load of a
    // round in flight together)
    constexpr int kJ = 2;
    int rawj[kJ];
    if (corr)
#pragma unroll
      for (int u = 0; u < kJ; u++) rawj[u] = tc + u * ntc < a.n_sel ? __ldg(a.sel + tc + u * ntc) : 0;
    {
      const int nu = a.K / 16;
      const int rw = (BITS == 4 && GM == 0) ? 4 : (1 << (a.gshift - 4));
      for (int u0 = warp * 32; u0 < nu; u0 += ntc) {
        if (BITS == 4 && GM == 0)
          build_unit<BITS, true>(a.x, u0 + lane, rw, a.gshift, xb, gt);
        else
          build_unit<BITS, false>(a.x, u0 + lane, rw, a.gshift, xb, gt);
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
          jrow[j] = a.staged ? j : c;
        }
      }
    }
    bar_sync(1, a.W * 32);  // B operand, group table, channel table and scale table complete
    if (corr) {
      // the refinement words of the CTA's rows, (entry, word) pairs spread
      // over the threads; they land during the base pass
      for (int e = tc; e < a.n_sel * nwr; e += ntc) {
        const int j = e / nwr, k = e - j * nwr;
        cp_async4(wt + (size_t)j * a.wt_pitch + k, a.refine + (size_t)jrow[j] * a.row_words + w_lo + k);
      }
      cp_async_commit();
    }
    // the warp's item, the same in every stage ((rb / NB) nseg <= W): row
    // blocks rbk .. rbk + NB - 1 of the stage, blocks [b0, b1) of the channels
    const bool has_item = warp < (a.rb / NB) * a.nseg;
    const int rbk = (warp / a.nseg) * NB, sg = warp % a.nseg;
    const int b0 = sg * a.nblk / a.nseg, b1 = (sg + 1) * a.nblk / a.nseg;
    const uint32_t rl_off = (uint32_t)(16 * rbk + gid) * a.rowL;
    const uint32_t rh_off = (uint32_t)a.rc * a.rowL + (uint32_t)(16 * rbk + gid) * a.rowH;
    const uint4* xbl = xb + 4 * p + t;
    for (int i = 0; i < nst && ok; i++) {
      const int slot = i % S;
      if (!mbar_wait(&full[slot], (i / S) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* sl = ring + (size_t)slot * a.stage_bytes;
      const int lr0 = i * a.rc + 16 * rbk;
      if (has_item && lr0 < rows) {
        // the rows' (s, m) words; rows past the end read the last row's (their
        // sums are not stored)
        const uint32_t* z[2 * NB];
#pragma unroll
        for (int h = 0; h < 2 * NB; h++) z[h] = szt + min(lr0 + gid + 8 * h, rows - 1);
        RowAcc acc[NB];
#pragma unroll
        for (int k = 0; k < NB; k++) acc[k] = RowAcc{{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f}};
        row_blocks<BITS, GM, NB>(sl + rl_off, a.rowL, sl + rh_off, a.rowH, (n0 + lr0 + gid) & 7, xbl, gt, z,
                                 a.szt_pitch, b0, b1, t, acc);
#pragma unroll
        for (int k = 0; k < NB; k++) {
          float y0, y1;
          combine_planes(acc[k], y0, y1);
          const int r0 = lr0 + 16 * k + gid;
          if (t == 0) {
            if (r0 < rows) part[r0 * a.nseg + sg] = y0;
            if (r0 + 8 < rows) part[(r0 + 8) * a.nseg + sg] = y1;
          }
        }
      }
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
        for (int q = sub; q < a.nseg; q += T) base += part[lr * a.nseg + q];
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
  int grid, threads, gm;
  size_t smem;
};

// Work split and shared memory layout of one GEMV shape: 16-row blocks per
// stage and group ranges per row block (each compute warp takes one (row
// block, range) item per stage), the ring depth that fits.
sf_status make_plan(const sf_wq* w, int n_sel, Plan& P) {
  GemvArgs& a = P.a;
  a = GemvArgs{};
  const int N = w->n, K = w->k, G = w->group;
  a.N = N, a.K = K, a.r = w->r, a.n_sel = n_sel;
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
  a.W = kMaxWarps;
  // row blocks per stage (rb) and group ranges (nseg = W / rb, one item per
  // warp and stage): the split with the least work for the busiest warp,
  // stages ceil(rows / 16 rb) x blocks ceil(nblk / nseg); among equal ones the
  // smaller stage (a deeper ring)
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
  a.row_words = N * w->r / 32;
  a.wt_pitch = ((a.rows_max * w->r + 31) >> 5) + 1;
  P.threads = (a.W + 1) * 32;
  const int nb_max = a.rows_max / 4;
  // channel shares of the correction: every thread busy when the CTA has few
  // rows (the output sums a row's shares on the lanes of a warp)
  a.cparts = n_sel > 0 ? std::max(1, std::min(std::min(n_sel, 64), P.threads / nb_max)) : 0;
  size_t off = align128((2 * kMaxStages + 1) * sizeof(uint64_t));
  a.szt_pitch = (a.rows_max + 3) & ~3;
  a.off_szt = (int)off;
  off += align128((size_t)a.gpr * a.szt_pitch * 4);
  a.off_gt = (int)off;
  off += align128((size_t)a.gpr * 8);
  a.off_part = (int)off;
  off += align128((size_t)a.rows_max * a.nseg * 4);
  a.off_xb = (int)off;
  off += align128((size_t)K * 4);
  // one region for the row-major scale copy (until it is transposed) and the
  // correction partials (after the base pass)
  a.off_cpart = (int)off;
  off += align128(std::max((size_t)a.cparts * a.rows_max * 4, (size_t)a.rows_max * a.gpr * 4));
  if (n_sel > 0) {
    a.off_jd = (int)off;
    off += align128((size_t)n_sel * 8);
    a.off_jrow = (int)off;
    off += align128((size_t)n_sel * 4);
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

template <int BITS>
void* kernel_for(int gm) {
  switch (gm) {
    case 0: return (void*)gemv_kernel<BITS, 0, 1>;
    case 1: return (void*)gemv_kernel<BITS, 1, 1>;
    case 2: return (void*)gemv_kernel<BITS, 2, 1>;
    default: return (void*)gemv_kernel<BITS, 4, 1>;
  }
}

void* pick_kernel(int b, int gm) {
  if (b == 2) return kernel_for<2>(gm);
  if (b == 3) return kernel_for<3>(gm);
  return kernel_for<4>(gm);
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
  void* kern = pick_kernel(w->b, P.gm);
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
