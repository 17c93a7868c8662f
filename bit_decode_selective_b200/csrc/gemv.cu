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
//
// Decomposition, per output row i (fp32 accumulation):
//   y_i = sum_groups [ s_ig * sum_{c in g} x_c q_ic + m_ig * sum_{c in g} x_c ]
//       + sum_{c selected} x_c * s_i,g(c) * (2 rho_ic + 1 - 2^r) / 2^(r+1)
//
// Base pass (HBM-bound; every resident code is read once): each CTA owns a
// contiguous range of rows; each warp owns one 2,048-channel segment of K and
// keeps that segment's activations in registers as exact fixed point (per
// 32-channel block, x = x_fix * 2^e with |x_fix| < 2^23, split into three
// bytes).  A lane reads 64 channels of a row (16 B of 2-bit codes) per step,
// expands them to byte vectors with shifts and masks and takes the integer
// dot products with dp4a (4 code x byte products per instruction); the three
// byte planes are recombined, scaled by 2^e, s and m in fp32.
//
// Correction pass: after griddepcontrol.wait (the selection kernel may still
// be running while the base pass streams), one warp per row sums the
// selected channels' corrections from the channel-major refinement rows.
#include "common.cuh"
#include "internal.cuh"

namespace sf {
namespace {

constexpr int kSegChannels = 2048;  // 32 lanes x 2 blocks x 32 channels
constexpr int kMaxWarps = 16;
constexpr int kUnroll = 4;          // rows in flight per warp

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
};

// ---- dp4a wrappers (inline PTX: unsigned codes times unsigned/signed bytes)
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

// Words of packed codes per lane per row (two 32-channel blocks).
template <int BITS>
struct Lane;
template <>
struct Lane<2> {
  static constexpr int W = 4;
};
template <>
struct Lane<3> {
  static constexpr int W = 6;
};
template <>
struct Lane<4> {
  static constexpr int W = 8;
};

template <int BITS>
__device__ __forceinline__ void load_codes(const GemvParams& p, int row, int blk0,
                                           uint32_t (&w)[Lane<BITS>::W]) {
  if constexpr (BITS == 2) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p.base + (size_t)row * (p.K / 16) + blk0 * 2));
    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
  } else if constexpr (BITS == 3) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p.base + (size_t)row * (p.K / 16) + blk0 * 2));
    uint2 h = __ldg(reinterpret_cast<const uint2*>(p.base + (size_t)p.N * p.K / 16 +
                                                   (size_t)row * (p.K / 32) + blk0));
    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w, w[4] = h.x, w[5] = h.y;
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(p.base + (size_t)row * (p.K / 8) + blk0 * 4);
    uint4 a = __ldg(src), b = __ldg(src + 1);
    w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
  }
}

// Code byte-vector v (0..7) of block k (0,1) of the lane's words.  Byte L of
// vector v holds the code of channel chan_of(v, L) (see prep_x).
template <int BITS>
__device__ __forceinline__ uint32_t code_vec(const uint32_t (&w)[Lane<BITS>::W], int k, int v) {
  if constexpr (BITS == 4) {
    int wi = v >> 1, j = v & 1;
    return (w[k * 4 + wi] >> (4 * j)) & 0x0F0F0F0Fu;
  } else {
    int wi = v >> 2, j = v & 3;  // wi: channels 0-15 (A) or 16-31 (B) of the block
    uint32_t c = (w[k * 2 + wi] >> (2 * j)) & 0x03030303u;
    if constexpr (BITS == 3) {
      uint32_t h = w[4 + k];
      c |= ((h >> (4 * wi + j)) << 2) & 0x04040404u;
    }
    return c;
  }
}

// Channel (0..31 within the block) held in byte L of vector v.
template <int BITS>
__host__ __device__ __forceinline__ int chan_of(int v, int L) {
  if (BITS == 4) return 8 * (v >> 1) + (v & 1) + 2 * L;
  return 16 * (v >> 2) + (v & 3) + 4 * L;
}

// Integer dot product of one block's codes with the x byte planes, as fp32.
template <int BITS>
__device__ __forceinline__ float block_dot(const uint32_t (&w)[Lane<BITS>::W], int k,
                                           const uint32_t* xv) {
  uint32_t lo = 0, mid = 0;
  int32_t hi = 0;
#pragma unroll
  for (int v = 0; v < 8; v++) {
    uint32_t c = code_vec<BITS>(w, k, v);
    lo = dp4a_uu(c, xv[v * 3 + 0], lo);
    mid = dp4a_uu(c, xv[v * 3 + 1], mid);
    hi = dp4a_us(c, xv[v * 3 + 2], hi);
  }
  return fmaf((float)hi, 65536.0f, (float)((mid << 8) + lo));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Shared-memory image of x for one batch row: per 32-channel block, 8 vectors
// x 3 byte planes (lo, mid, hi), two floats (sum of x, 2^e) and two words of
// padding so that every block starts on a 16-byte boundary.
constexpr int kXWords = 28;

template <int BITS>
__device__ void prep_x(const uint16_t* __restrict__ x, int K, uint32_t* xs) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  uint8_t* xb = reinterpret_cast<uint8_t*>(xs);
  for (int blk = warp; blk < K / 32; blk += nwarps) {
    float xv = h2f(x[blk * 32 + lane]);
    float mx = fabsf(xv);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    // scale so that |x_fix| < 2^23: e = floor(log2 max|x|) - 22
    int e = mx > 0.f ? ilogbf(mx) - 22 : 0;
    int xf = mx > 0.f ? __float2int_rn(ldexpf(xv, -e)) : 0;  // exact power-of-2 scaling
    // lane = channel c; find its (vector, byte) slot
    int v, L;
    if (BITS == 4) {
      v = 2 * (lane >> 3) + (lane & 1);
      L = (lane & 7) >> 1;
    } else {
      v = 4 * (lane >> 4) + (lane & 3);
      L = (lane & 15) >> 2;
    }
    uint8_t* dst = xb + (size_t)blk * kXWords * 4 + v * 12 + L;
    dst[0] = (uint8_t)(xf & 0xff);
    dst[4] = (uint8_t)((xf >> 8) & 0xff);
    dst[8] = (uint8_t)((xf >> 16) & 0xff);
    float s = warp_sum(xv);
    if (lane == 0) {
      reinterpret_cast<float*>(xs)[blk * kXWords + 24] = s;
      reinterpret_cast<float*>(xs)[blk * kXWords + 25] = ldexpf(1.0f, e);
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) gemv_kernel(GemvParams p) {
  extern __shared__ __align__(16) uint32_t smem[];
  const int nblk = p.K / 32;
  uint32_t* xs = smem;                                        // nblk * kXWords
  float* part = reinterpret_cast<float*>(smem + nblk * kXWords);  // rows x segs

  const int n0 = (int)((long)blockIdx.x * p.N / gridDim.x);
  const int n1 = (int)((long)(blockIdx.x + 1) * p.N / gridDim.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = warp % p.segs, rw = warp / p.segs;
  const bool warp_active = rw < p.row_warps;
  const int blk0 = seg * (kSegChannels / 32) + 2 * lane;  // first of the lane's two blocks
  const bool lane_active = warp_active && blk0 < nblk;
  const int gpb = p.G / 32;  // blocks per group

  for (int b = 0; b < p.batch; b++) {
    prep_x<BITS>(p.x + (size_t)b * p.K, p.K, xs);
    __syncthreads();
    uint32_t xr[2][24];
    float xsum[2] = {0.f, 0.f}, xscale[2] = {0.f, 0.f};
    if (lane_active) {
#pragma unroll
      for (int k = 0; k < 2; k++) {
        const uint4* src = reinterpret_cast<const uint4*>(xs + (blk0 + k) * kXWords);
#pragma unroll
        for (int i = 0; i < 6; i++) {
          uint4 v = src[i];
          xr[k][4 * i + 0] = v.x, xr[k][4 * i + 1] = v.y, xr[k][4 * i + 2] = v.z,
          xr[k][4 * i + 3] = v.w;
        }
        xsum[k] = __uint_as_float(xs[(blk0 + k) * kXWords + 24]);
        xscale[k] = __uint_as_float(xs[(blk0 + k) * kXWords + 25]);
      }
    }
    if (warp_active) {
      for (int i0 = n0 + rw * kUnroll; i0 < n1; i0 += p.row_warps * kUnroll) {
        uint32_t w[kUnroll][Lane<BITS>::W];
        uint32_t zs[kUnroll][2];
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
          int row = i0 + u;
          if (lane_active && row < n1) {
            load_codes<BITS>(p, row, blk0, w[u]);
            const uint32_t* szw = reinterpret_cast<const uint32_t*>(p.sz) + (size_t)row * (p.K / p.G);
            zs[u][0] = __ldg(szw + blk0 / gpb);
            zs[u][1] = __ldg(szw + (blk0 + 1) / gpb);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
          int row = i0 + u;
          float acc = 0.f;
          if (lane_active && row < n1) {
#pragma unroll
            for (int k = 0; k < 2; k++) {
              float2 sm = __half22float2(*reinterpret_cast<const __half2*>(&zs[u][k]));
              float d = block_dot<BITS>(w[u], k, xr[k]) * xscale[k];
              acc = fmaf(sm.x, d, acc);
              acc = fmaf(sm.y, xsum[k], acc);
            }
          }
          acc = warp_sum(acc);
          if (lane == 0 && row < n1) part[(row - n0) * p.segs + seg] = acc;
        }
      }
    }
    __syncthreads();

    // correction for the selected channels of batch row b
    if (p.n_sel > 0) {
      pdl_wait();  // selection (and staged rows) complete and visible
      const int32_t* sel = p.sel + (size_t)b * p.n_sel;
      const uint16_t* xb = p.x + (size_t)b * p.K;
      const int nwarps = blockDim.x >> 5;
      // (2 rho + 1 - 2^r) / 2^(r+1) = (rho + 1/2 - 2^(r-1)) / 2^r
      const float half = 0.5f * (float)(1 << p.r);
      const float inv = 1.0f / (float)(1 << p.r);
      for (int row = n0 + warp; row < n1; row += nwarps) {
        float corr = 0.f;
        const int rbit = row * p.r;
        for (int j = lane; j < p.n_sel; j += 32) {
          int c = __ldg(sel + j);
          const uint32_t* rrow = p.staged ? p.refine + ((size_t)b * p.n_sel + j) * p.refine_row_words
                                          : p.refine + (size_t)c * p.refine_row_words;
          uint32_t rho = (__ldg(rrow + (rbit >> 5)) >> (rbit & 31)) & ((1u << p.r) - 1);
          float s = h2f(__ldg(p.sz + ((size_t)row * (p.K / p.G) + c / p.G) * 2));
          float cf = ((float)rho + 0.5f - half) * inv;
          corr = fmaf(h2f(__ldg(xb + c)) * s, cf, corr);
        }
        corr = warp_sum(corr);
        if (lane == 0) part[(row - n0) * p.segs] += corr;
      }
      __syncthreads();
    }
    for (int row = n0 + threadIdx.x; row < n1; row += blockDim.x) {
      float acc = 0.f;
      for (int s = 0; s < p.segs; s++) acc += part[(row - n0) * p.segs + s];
      p.y[(size_t)b * p.N + row] = acc;
    }
    __syncthreads();
  }
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
  sf_status st = check_wq_public(w, false);
  if (st != SF_OK) return st;
  SF_REQUIRE(x && aligned16(x), "x must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(y && aligned16(y), "y must be a non-null 16-byte aligned device pointer");
  SF_UNSUPPORTED(batch >= 1 && batch <= 8, "batch=%d outside [1, 8]", batch);
  SF_REQUIRE(kch >= 0, "kch=%d < 0", kch);
  cudaStream_t s = as_stream(stream);
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
  }
  GemvParams p;
  p.base = (const uint32_t*)w->base;
  p.refine = (const uint32_t*)(refine_rows ? refine_rows : w->refine);
  p.sz = w->sz;
  p.x = x;
  p.sel = sel;
  p.y = y;
  p.N = w->n, p.K = w->k, p.G = w->group, p.r = w->r, p.batch = batch, p.n_sel = n_sel;
  p.segs = (w->k + kSegChannels - 1) / kSegChannels;
  SF_UNSUPPORTED(p.segs <= kMaxWarps, "k=%d too large", w->k);
  p.refine_row_words = w->n * w->r / 32;
  p.staged = refine_rows != nullptr;
  int grid = num_sms();
  if (grid > w->n / 8) grid = w->n / 8;
  int rows_per_cta = (w->n + grid - 1) / grid;
  p.row_warps = kMaxWarps / p.segs;
  int needed = (rows_per_cta + kUnroll - 1) / kUnroll;
  if (p.row_warps > needed) p.row_warps = needed;
  int threads = p.segs * p.row_warps * 32;
  if (threads < 128) threads = 128;  // the correction pass uses every warp
  size_t smem = (size_t)(w->k / 32) * kXWords * 4 + (size_t)rows_per_cta * p.segs * 4;
  SF_UNSUPPORTED(smem <= 200 * 1024, "k=%d needs too much shared memory", w->k);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (kch > 0 && !sel_in) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void (*kern)(GemvParams) = w->b == 2 ? gemv_kernel<2> : w->b == 3 ? gemv_kernel<3> : gemv_kernel<4>;
  SF_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
  SF_CUDA(cudaLaunchKernelEx(&cfg, kern, p));
  return SF_OK;
}
