// fit.cu -- fitted weight refinements on calibration activations.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// nested-quantization paragraph: for weights the refinement values are fitted
// on a small calibration set, so that the channels a step refines partly make
// up for the error of the channels it leaves at base precision.  Per chunk J of
// input channels (the unit of the chunked top-k selection), with A the
// calibration activations X masked to the channels the selection picks for
// each calibration row and e = weight minus base value:
//   G = A_J^T A_J,  lam = alpha * trace(G) / |J|  (1 where the trace is 0),
//   P = (G + lam I)^-1 (A_J^T X_J + lam I),   d_i[J] = P e_i[J],
// which minimises sum_n (X_nJ . e_iJ - A_nJ . d)^2 + lam |d - e_iJ|^2: on every
// calibration row the selected channels reproduce the whole chunk's base
// error, and the ridge term pulls the channels calibration rarely selects
// towards their plain refinement.  Each refinement code is then rewritten to
// the sub-bin of its base bin that holds base + d,
//   rho = clamp(floor((d / s + 1/2) 2^r), 0, 2^r - 1)   (0 where s = 0),
// so the packed format and the decode kernels are unchanged.
//
// Everything is fp64.  The Gram products, the left-looking blocked Cholesky
// factorisation of G + lam I, the two blocked triangular solves and the
// application of P are one strided fp64 tile kernel plus three small kernels
// on the 64 x 64 diagonal blocks, each launch batched over the chunks.  This is
// a one-off preparation step, not part of a decode step.
#include <cmath>

#include "common.cuh"
#include "internal.cuh"
#include "wqlayout.cuh"

namespace sf {
namespace {

constexpr int kT = 64;   // output tile and diagonal block size
constexpr int kBK = 16;  // k step of the tile kernel
constexpr int kGemmThreads = 256;

// C = beta C + alpha A B for a batch of z problems; A(m, k) = A[m sam + k sak],
// B(k, n) = B[k sbk + n sbn], C(m, n) = C[m scm + n scn]; problem z starts at
// A + z bza, B + z bzb, C + z bzc.  Each output sums over k in ascending order.
struct GemmArgs {
  int M, N, K;
  const double* A;
  long sam, sak, bza;
  const double* B;
  long sbk, sbn, bzb;
  double* C;
  long scm, scn, bzc;
  double alpha;
  int beta;  // 0 or 1
};

__global__ void __launch_bounds__(kGemmThreads) gemm_f64_kernel(GemmArgs g) {
  __shared__ double As[kBK][kT + 1];
  __shared__ double Bs[kBK][kT + 1];
  const double* A = g.A + (long)blockIdx.z * g.bza;
  const double* B = g.B + (long)blockIdx.z * g.bzb;
  double* C = g.C + (long)blockIdx.z * g.bzc;
  const int m0 = blockIdx.y * kT, n0 = blockIdx.x * kT;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 4; j++) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < g.K; k0 += kBK) {
    for (int e = threadIdx.x; e < kBK * kT; e += kGemmThreads) {
      // consecutive threads walk the operand's contiguous index
      int kk, mm;
      if (g.sak == 1) kk = e % kBK, mm = e / kBK;
      else kk = e / kT, mm = e % kT;
      const int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < g.M && k < g.K) ? A[(long)m * g.sam + (long)k * g.sak] : 0.0;
      int nn;
      if (g.sbk == 1) kk = e % kBK, nn = e / kBK;
      else kk = e / kT, nn = e % kT;
      const int n = n0 + nn, k2 = k0 + kk;
      Bs[kk][nn] = (n < g.N && k2 < g.K) ? B[(long)k2 * g.sbk + (long)n * g.sbn] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; kk++) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[kk][ty + 16 * i], b[i] = Bs[kk][tx + 16 * i];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < g.M && n < g.N) {
        double* c = C + (long)m * g.scm + (long)n * g.scn;
        const double v = g.alpha * acc[i][j];
        *c = g.beta ? *c + v : v;
      }
    }
}

sf_status gemm(const GemmArgs& g, int batch, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return SF_OK;
  const dim3 grid((g.N + kT - 1) / kT, (g.M + kT - 1) / kT, batch);
  gemm_f64_kernel<<<grid, kGemmThreads, 0, s>>>(g);
  SF_LAUNCHED();
  return SF_OK;
}

// Cholesky factor of the 64 x 64 diagonal block at (i0, i0) of every chunk's
// matrix (C x C, row-major, lower triangle), in place; the block's upper part
// is set to 0.  A pivot that is not positive sets *bad.
__global__ void __launch_bounds__(256) chol_diag_kernel(double* H, int C, int i0, int* bad) {
  __shared__ double L[kT][kT + 1];
  double* Hz = H + (long)blockIdx.x * C * C;
  for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) L[e / kT][e % kT] = Hz[(long)(i0 + e / kT) * C + i0 + e % kT];
  __syncthreads();
  for (int j = 0; j < kT; j++) {
    if (threadIdx.x == 0) {
      const double d = L[j][j];
      if (!(d > 0.0)) atomicExch(bad, 1);
      L[j][j] = d > 0.0 ? sqrt(d) : 1.0;
    }
    __syncthreads();
    for (int i = j + 1 + threadIdx.x; i < kT; i += blockDim.x) L[i][j] = L[i][j] / L[j][j];
    __syncthreads();
    const int w = kT - 1 - j;  // trailing block rows/cols j+1 .. 63
    for (int e = threadIdx.x; e < w * w; e += blockDim.x) {
      const int i = j + 1 + e / w, k = j + 1 + e % w;
      if (k <= i) L[i][k] = fma(-L[i][j], L[k][j], L[i][k]);
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) {
    const int i = e / kT, k = e % kT;
    Hz[(long)(i0 + i) * C + i0 + k] = k <= i ? L[i][k] : 0.0;
  }
}

__device__ __forceinline__ void load_diag(const double* Hz, int C, int i0, double (*L)[kT + 1]) {
  for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) L[e / kT][e % kT] = Hz[(long)(i0 + e / kT) * C + i0 + e % kT];
  __syncthreads();
}

// Panel below the diagonal block: rows m >= i0 + 64, columns i0 .. i0+63 of
// every chunk's matrix become H[m][cols] L_dd^-T (one thread per row).
__global__ void __launch_bounds__(128) trsm_panel_kernel(double* H, int C, int i0) {
  __shared__ double L[kT][kT + 1];
  double* Hz = H + (long)blockIdx.y * C * C;
  load_diag(Hz, C, i0, L);
  const int m = i0 + kT + blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= C) return;
  double* row = Hz + (long)m * C + i0;
  double x[kT];
#pragma unroll
  for (int j = 0; j < kT; j++) {
    double v = row[j];
    for (int t = 0; t < j; t++) v = fma(-x[t], L[j][t], v);
    x[j] = v / L[j][j];
  }
#pragma unroll
  for (int j = 0; j < kT; j++) row[j] = x[j];
}

// Rows i0 .. i0+63 of every chunk's right-hand sides R (C columns): forward
// (L_dd y = r) or backward (L_dd^T y = r) substitution with the diagonal block
// of the factor; one thread per column.
template <bool FWD>
__global__ void __launch_bounds__(128) trsm_rows_kernel(const double* H, double* R, int C, int i0) {
  __shared__ double L[kT][kT + 1];
  const double* Hz = H + (long)blockIdx.y * C * C;
  double* Rz = R + (long)blockIdx.y * C * C;
  load_diag(Hz, C, i0, L);
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= C) return;
  double y[kT];
  if (FWD) {
#pragma unroll
    for (int j = 0; j < kT; j++) {
      double v = Rz[(long)(i0 + j) * C + n];
      for (int t = 0; t < j; t++) v = fma(-L[j][t], y[t], v);
      y[j] = v / L[j][j];
    }
  } else {
#pragma unroll
    for (int j = kT - 1; j >= 0; j--) {
      double v = Rz[(long)(i0 + j) * C + n];
      for (int t = j + 1; t < kT; t++) v = fma(-L[t][j], y[t], v);
      y[j] = v / L[j][j];
    }
  }
#pragma unroll
  for (int j = 0; j < kT; j++) Rz[(long)(i0 + j) * C + n] = y[j];
}

// X[n][c] = x as fp64 (one thread per element).
__global__ void fit_convert_kernel(const uint16_t* __restrict__ x, long total, double* __restrict__ X) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < total) X[i] = h2d(x[i]);
}

// A[n][c] = X[n][c] for every selected channel c of calibration row n (A zeroed
// before); one thread per selection entry.
__global__ void fit_scatter_kernel(const int32_t* __restrict__ sel, int n_cal, int K, int chunks, int kch,
                                   const double* __restrict__ X, double* __restrict__ A) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)n_cal * chunks * kch) return;
  const long n = i / ((long)chunks * kch);
  const int c = sel[i];
  A[n * K + c] = X[n * K + c];
}

// lam = alpha * trace(G) / C per chunk (1 where the trace is 0), added to the
// diagonals of G and of the right-hand sides.
__global__ void fit_ridge_kernel(double* H, double* R, int C, double alpha) {
  __shared__ double lam;
  double* Hz = H + (long)blockIdx.x * C * C;
  double* Rz = R + (long)blockIdx.x * C * C;
  if (threadIdx.x == 0) {
    double tr = 0.0;
    for (int i = 0; i < C; i++) tr = __dadd_rn(tr, Hz[(long)i * C + i]);
    const double l = __ddiv_rn(__dmul_rn(alpha, tr), (double)C);
    lam = l == 0.0 ? 1.0 : l;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    Hz[(long)i * C + i] = __dadd_rn(Hz[(long)i * C + i], lam);
    Rz[(long)i * C + i] = __dadd_rn(Rz[(long)i * C + i], lam);
  }
}

// E[n][c] = w - (m + s q): the base error (fp64, each operation rounded once).
__global__ void fit_error_kernel(const float* __restrict__ wf, const uint32_t* __restrict__ base,
                                 const uint16_t* __restrict__ sz, int N, int K, int b, int G,
                                 double* __restrict__ E) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)N * K) return;
  const long n = i / K, c = i % K;
  const int q = packed_base_code(base, N, K, b, n, c);
  const long zi = (n * (K / G) + c / G) * 2;
  const double S = h2d(sz[zi]), M = h2d(sz[zi + 1]);
  E[i] = __dsub_rn((double)wf[i], __dadd_rn(M, __dmul_rn(S, (double)q)));
}

// Refinement words: word widx of the channel-major stream holds 32/r codes of
// one channel c, rows n0 .. n0 + 32/r - 1; each code is the sub-bin of the
// fitted value d (one thread per word).
__global__ void fit_codes_kernel(const double* __restrict__ D, const uint16_t* __restrict__ sz, int N, int K,
                                 int G, int r, uint32_t* __restrict__ refine) {
  const long widx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per = 32 / r;
  if (widx >= (long)K * N / per) return;
  const long first = widx * per;
  const long c = first / N, n0 = first % N;
  const double scale = (double)(1 << r), top = (double)((1 << r) - 1);
  uint32_t word = 0;
  for (int i = 0; i < per; i++) {
    const long n = n0 + i;
    const double S = h2d(sz[(n * (K / G) + c / G) * 2]);
    uint32_t rho = 0;
    if (S != 0.0) {
      double f = floor(__dmul_rn(__dadd_rn(__ddiv_rn(D[n * K + c], S), 0.5), scale));
      f = fmin(fmax(f, 0.0), top);
      rho = (uint32_t)f;
    }
    word |= rho << (i * r);
  }
  refine[widx] = word;
}

inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct FitLayout {
  size_t sel, A, X, H, R, E, D, flag, total;
};

FitLayout fit_layout(int n, int k, int n_cal, int chunk, int kch) {
  FitLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  L.sel = take((size_t)n_cal * (k / chunk) * kch * 4);
  L.A = take((size_t)n_cal * k * 8);
  L.X = take((size_t)n_cal * k * 8);
  L.H = take((size_t)k * chunk * 8);
  L.R = take((size_t)k * chunk * 8);
  L.E = take((size_t)n * k * 8);
  L.D = take((size_t)n * k * 8);
  L.flag = take(sizeof(int));
  L.total = off;
  return L;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" size_t sf_fit_refinements_workspace_bytes(int n, int k, int n_cal, int chunk, int kch) {
  if (n <= 0 || k <= 0 || n_cal <= 0 || chunk <= 0 || kch <= 0 || k % chunk != 0) return 0;
  return fit_layout(n, k, n_cal, chunk, kch).total;
}

extern "C" sf_status sf_fit_refinements(const float* wf, const sf_wq* w, const uint16_t* x_cal, int n_cal,
                                        int chunk, int kch, double alpha, double* delta, void* ws,
                                        size_t ws_bytes, sf_stream_t stream) {
  sf_status st = check_wq_public(w, true);
  if (st != SF_OK) return st;
  SF_REQUIRE(wf && aligned16(wf), "wf must be a non-null 16-byte aligned device pointer");
  SF_REQUIRE(n_cal >= 1, "n_cal=%d < 1", n_cal);
  SF_REQUIRE(std::isfinite(alpha) && alpha > 0.0, "alpha must be positive and finite");
  SF_REQUIRE(!delta || aligned16(delta), "delta must be 16-byte aligned");
  st = check_select_args(x_cal, 1, w->k, chunk, kch);
  if (st != SF_OK) return st;
  const int N = w->n, K = w->k, C = chunk, chunks = K / C;
  const FitLayout L = fit_layout(N, K, n_cal, C, kch);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) {
    set_error("workspace: need %zu bytes (16-byte aligned), got %zu", L.total, ws_bytes);
    return SF_ERR_WORKSPACE;
  }
  cudaStream_t s = as_stream(stream);
  char* base = (char*)ws;
  int32_t* sel = (int32_t*)(base + L.sel);
  double *A = (double*)(base + L.A), *X = (double*)(base + L.X);
  double *H = (double*)(base + L.H), *R = (double*)(base + L.R);
  double *E = (double*)(base + L.E), *D = delta ? delta : (double*)(base + L.D);
  int* bad = (int*)(base + L.flag);
  const long nx = (long)n_cal * K;
  SF_CUDA(cudaMemsetAsync(A, 0, nx * sizeof(double), s));
  SF_CUDA(cudaMemsetAsync(bad, 0, sizeof(int), s));
  // the decode step's selection on every calibration row
  for (int b0 = 0; b0 < n_cal; b0 += 64) {
    const int nb = n_cal - b0 < 64 ? n_cal - b0 : 64;
    st = launch_select(x_cal + (size_t)b0 * K, nb, K, C, kch, sel + (size_t)b0 * chunks * kch, s, false);
    if (st != SF_OK) return st;
  }
  fit_convert_kernel<<<(unsigned)((nx + 255) / 256), 256, 0, s>>>(x_cal, nx, X);
  SF_LAUNCHED();
  const long nsel = (long)n_cal * chunks * kch;
  fit_scatter_kernel<<<(unsigned)((nsel + 255) / 256), 256, 0, s>>>(sel, n_cal, K, chunks, kch, X, A);
  SF_LAUNCHED();
  // G = A_J^T A_J and the right-hand sides A_J^T X_J, per chunk
  GemmArgs g{};
  g.M = C, g.N = C, g.K = n_cal;
  g.A = A, g.sam = 1, g.sak = K, g.bza = C;
  g.sbk = K, g.sbn = 1, g.bzb = C;
  g.scm = C, g.scn = 1, g.bzc = (long)C * C;
  g.alpha = 1.0, g.beta = 0;
  g.B = A, g.C = H;
  if ((st = gemm(g, chunks, s)) != SF_OK) return st;
  g.B = X, g.C = R;
  if ((st = gemm(g, chunks, s)) != SF_OK) return st;
  fit_ridge_kernel<<<chunks, 256, 0, s>>>(H, R, C, alpha);
  SF_LAUNCHED();
  // Cholesky factor of G + lam I (left-looking, 64-column blocks)
  const int nb = C / kT;
  for (int I = 0; I < nb; I++) {
    const int i0 = I * kT;
    if (i0 > 0) {
      GemmArgs u{};
      u.M = C - i0, u.N = kT, u.K = i0;
      u.A = H + (long)i0 * C, u.sam = C, u.sak = 1, u.bza = (long)C * C;
      u.B = H + (long)i0 * C, u.sbk = 1, u.sbn = C, u.bzb = (long)C * C;
      u.C = H + (long)i0 * C + i0, u.scm = C, u.scn = 1, u.bzc = (long)C * C;
      u.alpha = -1.0, u.beta = 1;
      if ((st = gemm(u, chunks, s)) != SF_OK) return st;
    }
    chol_diag_kernel<<<chunks, 256, 0, s>>>(H, C, i0, bad);
    SF_LAUNCHED();
    if (i0 + kT < C) {
      trsm_panel_kernel<<<dim3((C - i0 - kT + 127) / 128, chunks), 128, 0, s>>>(H, C, i0);
      SF_LAUNCHED();
    }
  }
  // P = L^-T L^-1 (A^T X + lam I), in place in R: forward, then backward
  for (int I = 0; I < nb; I++) {
    const int i0 = I * kT;
    if (i0 > 0) {
      GemmArgs u{};
      u.M = kT, u.N = C, u.K = i0;
      u.A = H + (long)i0 * C, u.sam = C, u.sak = 1, u.bza = (long)C * C;
      u.B = R, u.sbk = C, u.sbn = 1, u.bzb = (long)C * C;
      u.C = R + (long)i0 * C, u.scm = C, u.scn = 1, u.bzc = (long)C * C;
      u.alpha = -1.0, u.beta = 1;
      if ((st = gemm(u, chunks, s)) != SF_OK) return st;
    }
    trsm_rows_kernel<true><<<dim3((C + 127) / 128, chunks), 128, 0, s>>>(H, R, C, i0);
    SF_LAUNCHED();
  }
  for (int I = nb - 1; I >= 0; I--) {
    const int i0 = I * kT;
    if (i0 + kT < C) {
      GemmArgs u{};
      u.M = kT, u.N = C, u.K = C - i0 - kT;
      u.A = H + (long)(i0 + kT) * C + i0, u.sam = 1, u.sak = C, u.bza = (long)C * C;
      u.B = R + (long)(i0 + kT) * C, u.sbk = C, u.sbn = 1, u.bzb = (long)C * C;
      u.C = R + (long)i0 * C, u.scm = C, u.scn = 1, u.bzc = (long)C * C;
      u.alpha = -1.0, u.beta = 1;
      if ((st = gemm(u, chunks, s)) != SF_OK) return st;
    }
    trsm_rows_kernel<false><<<dim3((C + 127) / 128, chunks), 128, 0, s>>>(H, R, C, i0);
    SF_LAUNCHED();
  }
  // d = E_J P^T per chunk, then the refinement codes
  const long nw = (long)N * K;
  fit_error_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, s>>>(wf, (const uint32_t*)w->base, w->sz, N, K, w->b,
                                                                 w->group, E);
  SF_LAUNCHED();
  GemmArgs ap{};
  ap.M = N, ap.N = C, ap.K = C;
  ap.A = E, ap.sam = K, ap.sak = 1, ap.bza = C;
  ap.B = R, ap.sbk = 1, ap.sbn = C, ap.bzb = (long)C * C;
  ap.C = D, ap.scm = K, ap.scn = 1, ap.bzc = C;
  ap.alpha = 1.0, ap.beta = 0;
  if ((st = gemm(ap, chunks, s)) != SF_OK) return st;
  const long words = (long)K * N * w->r / 32;
  fit_codes_kernel<<<(unsigned)((words + 255) / 256), 256, 0, s>>>(D, w->sz, N, K, w->group, w->r,
                                                                   (uint32_t*)w->refine);
  SF_LAUNCHED();
  int h_bad = 0;
  SF_CUDA(cudaMemcpyAsync(&h_bad, bad, sizeof(int), cudaMemcpyDeviceToHost, s));
  SF_CUDA(cudaStreamSynchronize(s));
  SF_REQUIRE(h_bad == 0, "the calibration system G + lam I is not positive definite in fp64");
  return SF_OK;
}
