/*
 * sf_oracle.c -- CPU oracle for the selective-precision decode path.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never links, imports or calls it, and
 * this file shares no code, header or table with the product path.
 *
 * It is deliberately plain and slow: every value is computed in fp64, loops run
 * in the order the method is described, and there is no blocking, fusion or
 * reordering.  OpenMP pragmas only spread independent outer iterations (rows,
 * heads, batch rows) across cores; each output is computed by exactly one
 * thread in the same sequential order, so results do not depend on the thread
 * count.
 *
 * Sources (web pages describing StrataFlux; cited by title and paragraph):
 *   [EXPL] "StrataFlux -- Selective precision streaming -- What does it mean?"
 *          paragraphs: "which tiles count" (channel chunks, token scoring),
 *          "nested quantization" (fetched bits subdivide the resident bin),
 *          "the map app also loads tiles" (fetch lead / fetch lag),
 *          "worked example" (bits-per-weight arithmetic).
 *   [ABS]  "StrataFlux: Memory-Hierarchy-Native Low-Bit LLM Inference",
 *          abstract (2-4-bit weights, 2-3-bit KV cache, Llama-3.1-8B).
 *
 * Readings taken where the pages are silent are stated beside each function.
 * The packed byte formats (or_pack_*) follow the format text in the library
 * header; the pages fix no format, so those are this project's definitions,
 * re-implemented here independently from the text.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_API __attribute__((visibility("default")))

OR_API int or_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* IEEE 754 binary16, written from the definition: 1 sign bit, 5 exponent bits
 * (bias 15), 10 fraction bits; exponent field 0 encodes subnormals f * 2^-24. */

OR_API double or_f16_to_f64(uint16_t h) {
  int sign = h >> 15;
  int e = (h >> 10) & 31;
  int f = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25);
  return sign ? -v : v;
}

/* nearest integer to q >= 0, ties to the even integer */
static double round_half_even(double q) {
  double fl = floor(q);
  double diff = q - fl;
  if (diff > 0.5) return fl + 1.0;
  if (diff < 0.5) return fl;
  return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;
}

/* fp64 -> binary16, round to nearest, ties to even (one rounding). */
OR_API uint16_t or_f16_from_f64(double x) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7C00;
  int e2;
  frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) */
  int E = e2 - 1;         /* a in [2^E, 2^(E+1)) */
  if (E < -14) {
    /* subnormal binade: the representable values are n * 2^-24 */
    double n = round_half_even(ldexp(a, 24));
    return sign | (uint16_t)n; /* n == 1024 encodes the smallest normal */
  }
  /* normal binade: representable values n * 2^(E-10), n in [1024, 2048) */
  double n = round_half_even(ldexp(a, 10 - E));
  if (n == 2048.0) {
    n = 1024.0;
    E += 1;
  }
  if (E > 15) return sign | 0x7C00;
  return sign | (uint16_t)(((E + 15) << 10) | ((int)n - 1024));
}

/* ------------------------------------------------------------------------- */
/* Nested quantisation of one group.  [EXPL] "nested quantization": the
 * resident b-bit code names a bin; r fetched bits split that bin into 2^r equal
 * parts, so base + refinement has the resolution of a (b+r)-bit code.
 *
 * Readings (the pages give no formula):
 *  - the base is ordinary asymmetric round-to-nearest over the group's range:
 *    step s = fp16((hi - lo) / (2^b - 1)), offset m = fp16(lo), each rounded
 *    once from fp64; the base bin of code q is [q - 1/2, q + 1/2) steps
 *    around m + s*q;
 *  - rounding is half-up: q = floor(u + 1/2) with u = (w - m) / s;
 *  - the refinement index is the sub-bin of that interval:
 *    Q = floor((u + 1/2) * 2^r) clamped to [0, 2^(b+r) - 1], base code
 *    q = Q >> r, refinement rho = Q & (2^r - 1);
 *  - a group whose fp16 step is 0 gets all codes 0 (it reconstructs to m).
 * All arithmetic is fp64 with a single rounding per operation. */
OR_API void or_quant_group(const double* w, int n, int b, int r, uint16_t* s16,
                           uint16_t* m16, uint8_t* qb, uint8_t* rho) {
  double lo = w[0], hi = w[0];
  for (int i = 1; i < n; i++) {
    if (w[i] < lo) lo = w[i];
    if (w[i] > hi) hi = w[i];
  }
  *s16 = or_f16_from_f64((hi - lo) / (double)((1 << b) - 1));
  *m16 = or_f16_from_f64(lo);
  double S = or_f16_to_f64(*s16);
  double M = or_f16_to_f64(*m16);
  int qmax = (1 << (b + r)) - 1;
  for (int i = 0; i < n; i++) {
    int Q = 0;
    if (S != 0.0) {
      double u = (w[i] - M) / S;
      double t = u + 0.5;
      double f = floor(t * (double)(1 << r));
      if (f < 0.0) f = 0.0;
      if (f > (double)qmax) f = (double)qmax;
      Q = (int)f;
    }
    qb[i] = (uint8_t)(Q >> r);
    rho[i] = (uint8_t)(Q & ((1 << r) - 1));
  }
}

/* Reconstruction ([EXPL] "nested quantization").  Base value: the centre of
 * bin q.  Refined value: the centre of sub-bin rho of bin q, i.e.
 * m + s * (q + (2*rho + 1 - 2^r) / 2^(r+1)). */
OR_API double or_dequant_base(uint16_t s16, uint16_t m16, int q) {
  return or_f16_to_f64(m16) + or_f16_to_f64(s16) * (double)q;
}

OR_API double or_dequant_refined(uint16_t s16, uint16_t m16, int q, int rho, int r) {
  double sub = (double)(2 * rho + 1 - (1 << r)) / (double)(1 << (r + 1));
  return or_f16_to_f64(m16) + or_f16_to_f64(s16) * ((double)q + sub);
}

/* Weights W[N][K] (fp32), groups of G consecutive input channels of one row.
 * Outputs: qb[N][K], rho[N][K] (one code per byte), sz[N][K/G][2] fp16 bits
 * (step, offset). */
OR_API void or_quant_weights(const float* w, int N, int K, int b, int r, int G,
                             uint8_t* qb, uint8_t* rho, uint16_t* sz) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; n++) {
    double* buf = (double*)malloc(sizeof(double) * (size_t)G);
    for (int j = 0; j < K / G; j++) {
      size_t off = (size_t)n * K + (size_t)j * G;
      for (int i = 0; i < G; i++) buf[i] = (double)w[off + i];
      size_t zo = ((size_t)n * (K / G) + j) * 2;
      or_quant_group(buf, G, b, r, &sz[zo], &sz[zo + 1], &qb[off], &rho[off]);
    }
    free(buf);
  }
}

/* KV cache values k[B][H][T][D] (fp16 bits), groups of G consecutive
 * head-dim elements of one token.  [EXPL] "nested quantization" applies the
 * same nesting to the KV cache.  Outputs qb/rho [B][H][T][D] and
 * sz[B][H][T][D/G][2]. */
OR_API void or_quant_kv(const uint16_t* x, int B, int H, int T, int D, int b, int r,
                        int G, uint8_t* qb, uint8_t* rho, uint16_t* sz) {
  long rows = (long)B * H * T;
#pragma omp parallel for schedule(static)
  for (long row = 0; row < rows; row++) {
    double buf[1024];
    for (int j = 0; j < D / G; j++) {
      size_t off = (size_t)row * D + (size_t)j * G;
      for (int i = 0; i < G; i++) buf[i] = or_f16_to_f64(x[off + i]);
      size_t zo = ((size_t)row * (D / G) + j) * 2;
      or_quant_group(buf, G, b, r, &sz[zo], &sz[zo + 1], &qb[off], &rho[off]);
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Packed byte formats (this project's definition; see the library header).
 * A "natural w-bit stream" stores element e at bit (w*e) of a little-endian
 * byte string: byte (w*e)/8, bit offset (w*e)%8.                            */

static void put_bits(uint8_t* dst, long e, int w, int v) {
  long bit = (long)w * e;
  dst[bit >> 3] |= (uint8_t)((v & ((1 << w) - 1)) << (bit & 7));
}

/* Position of channel c' (0..31 within a 32-channel block) in the block's
 * 32-bit high-bit word of a 3-bit base: channels 0..15 at bit 8*(c'/4)+c'%4,
 * channels 16..31 at bit 8*((c'-16)/4)+4+(c'-16)%4. */
static int hi_plane_bit(int cp) {
  if (cp < 16) return 8 * (cp / 4) + cp % 4;
  cp -= 16;
  return 8 * (cp / 4) + 4 + cp % 4;
}

/* Weight base codes, row n of N, channel c of K:
 *   b = 2, 4: per row a natural b-bit stream (K*b/8 bytes), rows consecutive;
 *   b = 3:    plane L (per row the natural 2-bit stream of the low 2 bits,
 *             K/4 bytes) followed by plane H (per row K/8 bytes: per
 *             32-channel block one little-endian 32-bit word laid out by
 *             hi_plane_bit).
 *   Every row of a plane is then cut into 16-byte units and unit u is stored
 *   at unit (u XOR (n mod 8)) of the row (the units move only inside their
 *   aligned 128-byte block).
 * Refinement codes: channel-major natural r-bit streams, R[c] holds rho[n][c]
 * for n = 0..N-1 (K rows of N*r/8 B). */
static void store_row_units(uint8_t* dst_row, const uint8_t* natural, long bytes, long n) {
  for (long u = 0; u < bytes / 16; u++) {
    long to = u ^ (n % 8);
    memcpy(dst_row + 16 * to, natural + 16 * u, 16);
  }
}

OR_API void or_pack_weights(const uint8_t* qb, const uint8_t* rho, int N, int K, int b,
                            int r, uint8_t* base, uint8_t* refine) {
  size_t base_bytes = (size_t)N * K * b / 8;
  memset(base, 0, base_bytes);
  memset(refine, 0, (size_t)K * N * r / 8);
  const long rowL = (long)K * (b == 3 ? 2 : b) / 8, rowH = K / 8;
  uint8_t* lo = (uint8_t*)calloc((size_t)rowL, 1);
  uint8_t* hi = (uint8_t*)calloc((size_t)rowH, 1);
  for (long n = 0; n < N; n++) {
    memset(lo, 0, (size_t)rowL);
    memset(hi, 0, (size_t)rowH);
    for (long c = 0; c < K; c++) {
      int q = qb[n * K + c];
      if (b == 2 || b == 4) {
        put_bits(lo, c, b, q);
      } else { /* b == 3 */
        put_bits(lo, c, 2, q & 3);
        long blk = c / 32;
        int bit = hi_plane_bit((int)(c % 32));
        hi[blk * 4 + bit / 8] |= (uint8_t)(((q >> 2) & 1) << (bit % 8));
      }
      put_bits(refine, c * N + n, r, rho[n * K + c]);
    }
    store_row_units(base + (size_t)n * rowL, lo, rowL, n);
    if (b == 3) store_row_units(base + (size_t)N * rowL + (size_t)n * rowH, hi, rowH, n);
  }
  free(lo);
  free(hi);
}

/* KV codes and refinements: pair-slot layout.  A little-endian 32-bit word
 * holds 16/w pairs of w-bit codes; pair slot j keeps its first code at bits
 * [w*j, w*j+w) and its second at bits [16+w*j, 16+w*j+w).
 * Keys: per token, 4 chunks c of w words; pair p = 2s+e of chunk c holds dims
 * 16s+2c+8e (first) and 16s+2c+8e+1 (second).
 * Values: per tile of 16 tokens, 32 chunks l = 4g+c of 2w words; pair
 * p = 16h+2m+e of chunk l holds dim 16m+g+8e of tile tokens 2c+8h (first) and
 * 2c+8h+1 (second).  D must be 128. */
static void put_pair(uint8_t* chunk, int w, int p, int second, int v) {
  int per_word = 16 / w;
  int word = p / per_word, slot = p % per_word;
  int bit = 32 * word + 16 * second + w * slot;
  chunk[bit >> 3] |= (uint8_t)((v & ((1 << w) - 1)) << (bit & 7));
}

/* (chunk, pair, second) of head-dim element d of a key token */
static void key_place(int d, int* c, int* p, int* second) {
  int s = d / 16, within = d % 16;
  int e = within / 8;
  *c = (within % 8) / 2;
  *second = within % 2;
  *p = 2 * s + e;
}

/* (chunk, pair, second) of element (token tt of its 16-token tile, dim d) of
 * a value tile */
static void value_place(int tt, int d, int* l, int* p, int* second) {
  int m = d / 16, within = d % 16;
  int e = within / 8, g = within % 8;
  int h = tt / 8, c = (tt % 8) / 2;
  *second = tt % 2;
  *l = 4 * g + c;
  *p = 16 * h + 2 * m + e;
}

/* Bits [shift, shift + w) of every code go to a w-bit pair-slot plane that
 * starts `off` bytes into each token's (keys) or tile's (values) `stride`
 * bytes of the output. */
static void pack_keys(const uint8_t* x, int w, int shift, size_t stride, size_t off, int B, int H, int T,
                      int Tmax, int D, uint8_t* out) {
  for (long bh = 0; bh < (long)B * H; bh++)
    for (long t = 0; t < T; t++)
      for (int d = 0; d < D; d++) {
        int c, p, second;
        key_place(d, &c, &p, &second);
        uint8_t* chunk = out + ((size_t)bh * Tmax + t) * stride + off + (size_t)c * 4 * w;
        put_pair(chunk, w, p, second, x[((size_t)bh * T + t) * D + d] >> shift);
      }
}

static void pack_values(const uint8_t* x, int w, int shift, size_t stride, size_t off, int B, int H, int T,
                        int Tmax, int D, uint8_t* out) {
  for (long bh = 0; bh < (long)B * H; bh++)
    for (long t = 0; t < T; t++)
      for (int d = 0; d < D; d++) {
        int l, p, second;
        value_place((int)(t % 16), d, &l, &p, &second);
        uint8_t* chunk = out + ((size_t)bh * (Tmax / 16) + t / 16) * stride + off + (size_t)l * 8 * w;
        put_pair(chunk, w, p, second, x[((size_t)bh * T + t) * D + d] >> shift);
      }
}

/* One kind (keys or values) of w-bit codes.  w = 2 and 4 divide the 16 bits of
 * a word half and use the pair-slot layout directly; 3-bit codes are stored as
 * two planes of that layout, the low two bits of every code (w = 2) followed by
 * the high bit (w = 1): 32 + 16 bytes per key token, 512 + 256 bytes per value
 * tile. */
static void pack_kind(const uint8_t* x, int which, int w, int B, int H, int T, int Tmax, int D,
                      uint8_t* out) {
  const size_t stride = (size_t)(which == 0 ? 16 : 256) * w;
  memset(out, 0, (size_t)B * H * (which == 0 ? Tmax : Tmax / 16) * stride);
  void (*pk)(const uint8_t*, int, int, size_t, size_t, int, int, int, int, int, uint8_t*) =
      which == 0 ? pack_keys : pack_values;
  if (w == 3) {
    pk(x, 2, 0, stride, 0, B, H, T, Tmax, D, out);
    pk(x, 1, 2, stride, (size_t)(which == 0 ? 32 : 512), B, H, T, Tmax, D, out);
  } else {
    pk(x, w, 0, stride, 0, B, H, T, Tmax, D, out);
  }
}

/* which = 0: keys, 1: values.  Writes base (b bits) and refinement (r bits)
 * buffers of a cache with token capacity Tmax; only the first T tokens of each
 * head are written, everything else is zero. */
OR_API void or_pack_kv(const uint8_t* qb, const uint8_t* rho, int which, int B, int H, int T,
                       int Tmax, int D, int b, int r, uint8_t* base, uint8_t* refine) {
  pack_kind(qb, which, b, B, H, T, Tmax, D, base);
  pack_kind(rho, which, r, B, H, T, Tmax, D, refine);
}

/* ------------------------------------------------------------------------- */
/* Chunked channel selection.  [EXPL] "which tiles count": a projection's input
 * channels are split into chunks of C (1,024 on the pages); in each chunk the
 * k channels with the largest activation magnitude at this step are refined.
 * Readings: magnitude is the fp16 magnitude (bits & 0x7fff compared as an
 * unsigned integer, so +0 and -0 are equal); equal magnitudes go to the lower
 * channel index; each batch row selects on its own; indices are absolute
 * channel numbers, ascending within each chunk.
 * sel[B][K/C][k]. */
OR_API void or_select_chunks(const uint16_t* x, int B, int K, int C, int k, int32_t* sel) {
  for (int bb = 0; bb < B; bb++) {
    for (int ch = 0; ch < K / C; ch++) {
      const uint16_t* xc = x + (size_t)bb * K + (size_t)ch * C;
      char* taken = (char*)calloc((size_t)C, 1);
      int32_t* out = sel + ((size_t)bb * (K / C) + ch) * k;
      for (int j = 0; j < k; j++) {
        int best = -1;
        for (int i = 0; i < C; i++) {
          if (taken[i]) continue;
          if (best < 0 || (xc[i] & 0x7fff) > (xc[best] & 0x7fff)) best = i;
        }
        taken[best] = 1;
      }
      int m = 0;
      for (int i = 0; i < C; i++)
        if (taken[i]) out[m++] = ch * C + i;
      free(taken);
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Refined GEMV.  [EXPL] "which tiles count": the projection uses the refined
 * value for the selected input channels and the base value everywhere else
 * ("everything not selected still takes part in the computation at low
 * precision").  y[b][n] = sum_c x[b][c] * w~[n][c], fp64, c ascending.
 * sel[B][K/C][k] (k = 0 means base only; sel may then be NULL). */
OR_API void or_gemv_refined(const uint8_t* qb, const uint8_t* rho, const uint16_t* sz,
                            int N, int K, int r, int G, const uint16_t* x, int B,
                            const int32_t* sel, int C, int k, double* y) {
  for (int bb = 0; bb < B; bb++) {
    char* selected = (char*)calloc((size_t)K, 1);
    for (int j = 0; j < (K / C) * k; j++) selected[sel[(size_t)bb * (K / C) * k + j]] = 1;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
      double acc = 0.0;
      for (int c = 0; c < K; c++) {
        size_t e = (size_t)n * K + c;
        size_t zo = ((size_t)n * (K / G) + c / G) * 2;
        double wv = selected[c] ? or_dequant_refined(sz[zo], sz[zo + 1], qb[e], rho[e], r)
                                : or_dequant_base(sz[zo], sz[zo + 1], qb[e]);
        acc += or_f16_to_f64(x[(size_t)bb * K + c]) * wv;
      }
      y[(size_t)bb * N + n] = acc;
    }
    free(selected);
  }
}

/* ------------------------------------------------------------------------- */
/* KV token scoring.  [EXPL] "which tiles count": every cached token is scored by
 * the attention it receives, computed from the resident low-bit keys, and the
 * highest-scoring tokens are refined for each KV head (the keys and values a
 * group of query heads shares).
 * Readings: query head h reads KV head h / (Hq/H); logits use the base keys and
 * the usual 1/sqrt(D) scale; a token's score for KV head g is the sum over the
 * group's query heads of that head's softmax probability over all T tokens.
 *
 * logits[B][Hq][T] (fp64). */
OR_API void or_kv_logits(const uint8_t* kqb, const uint16_t* ksz, int B, int H, int T,
                         int D, int G, const uint16_t* q, int Hq, double* logits) {
  int grp = Hq / H;
  double scale = 1.0 / sqrt((double)D);
#pragma omp parallel for collapse(2) schedule(static)
  for (int bb = 0; bb < B; bb++)
    for (int h = 0; h < Hq; h++) {
      int g = h / grp;
      for (int t = 0; t < T; t++) {
        size_t row = ((size_t)bb * H + g) * T + t;
        double acc = 0.0;
        for (int d = 0; d < D; d++) {
          size_t zo = (row * (D / G) + d / G) * 2;
          double kv = or_dequant_base(ksz[zo], ksz[zo + 1], kqb[row * D + d]);
          acc += or_f16_to_f64(q[((size_t)bb * Hq + h) * D + d]) * kv;
        }
        logits[((size_t)bb * Hq + h) * T + t] = acc * scale;
      }
    }
}

/* score[B][H][T] = sum over the group's query heads of softmax_t(logits). */
OR_API void or_kv_scores(const double* logits, int B, int Hq, int H, int T, double* score) {
  int grp = Hq / H;
  memset(score, 0, sizeof(double) * (size_t)B * H * T);
  for (int bb = 0; bb < B; bb++)
    for (int h = 0; h < Hq; h++) {
      const double* l = logits + ((size_t)bb * Hq + h) * T;
      double M = l[0];
      for (int t = 1; t < T; t++)
        if (l[t] > M) M = l[t];
      double Z = 0.0;
      for (int t = 0; t < T; t++) Z += exp(l[t] - M);
      double* s = score + ((size_t)bb * H + h / grp) * T;
      for (int t = 0; t < T; t++) s[t] += exp(l[t] - M) / Z;
    }
}

typedef struct {
  double v;
  int32_t t;
} scored_token;

static int by_score_then_index(const void* a, const void* b) {
  const scored_token* x = (const scored_token*)a;
  const scored_token* y = (const scored_token*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->t > y->t) - (x->t < y->t);
}

static int ascending_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* Per KV head, the k_tok highest scores (equal scores: lower token first),
 * written in ascending token order.  sel[B][H][k_tok]. */
OR_API void or_kv_select(const double* score, int B, int H, int T, int k_tok, int32_t* sel) {
  scored_token* buf = (scored_token*)malloc(sizeof(scored_token) * (size_t)T);
  for (long bh = 0; bh < (long)B * H; bh++) {
    for (int t = 0; t < T; t++) {
      buf[t].v = score[bh * T + t];
      buf[t].t = t;
    }
    qsort(buf, (size_t)T, sizeof(scored_token), by_score_then_index);
    int32_t* out = sel + bh * k_tok;
    for (int j = 0; j < k_tok; j++) out[j] = buf[j].t;
    qsort(out, (size_t)k_tok, sizeof(int32_t), ascending_i32);
  }
  free(buf);
}

/* Refined attention.  [EXPL] "which tiles count" and "nested quantization":
 * softmax(q.k~ / sqrt(D)) . v~ over all T cached tokens, where k~ and v~ are the
 * refined (b+r-bit) values for the tokens selected for the query head's KV head
 * and the base values for every other token.  Reading: one selection per KV
 * head refines both its keys and its values.  Single pass, no split.
 * out[B][Hq][D] (fp64). */
OR_API void or_kv_attention(const uint8_t* kqb, const uint8_t* krho, const uint16_t* ksz,
                            const uint8_t* vqb, const uint8_t* vrho, const uint16_t* vsz,
                            int B, int H, int T, int D, int G, int r, const uint16_t* q,
                            int Hq, const int32_t* sel, int k_tok, double* out) {
  int grp = Hq / H;
  double scale = 1.0 / sqrt((double)D);
#pragma omp parallel for collapse(2) schedule(static)
  for (int bb = 0; bb < B; bb++)
    for (int h = 0; h < Hq; h++) {
      int g = h / grp;
      char* selected = (char*)calloc((size_t)T, 1);
      for (int j = 0; j < k_tok; j++) selected[sel[((size_t)bb * H + g) * k_tok + j]] = 1;
      double* l = (double*)malloc(sizeof(double) * (size_t)T);
      for (int t = 0; t < T; t++) {
        size_t row = ((size_t)bb * H + g) * T + t;
        double acc = 0.0;
        for (int d = 0; d < D; d++) {
          size_t e = row * D + d;
          size_t zo = (row * (D / G) + d / G) * 2;
          double kv = selected[t] ? or_dequant_refined(ksz[zo], ksz[zo + 1], kqb[e], krho[e], r)
                                  : or_dequant_base(ksz[zo], ksz[zo + 1], kqb[e]);
          acc += or_f16_to_f64(q[((size_t)bb * Hq + h) * D + d]) * kv;
        }
        l[t] = acc * scale;
      }
      double M = l[0];
      for (int t = 1; t < T; t++)
        if (l[t] > M) M = l[t];
      double Z = 0.0;
      for (int t = 0; t < T; t++) Z += exp(l[t] - M);
      double* o = out + ((size_t)bb * Hq + h) * D;
      for (int d = 0; d < D; d++) o[d] = 0.0;
      for (int t = 0; t < T; t++) {
        double p = exp(l[t] - M) / Z;
        size_t row = ((size_t)bb * H + g) * T + t;
        for (int d = 0; d < D; d++) {
          size_t e = row * D + d;
          size_t zo = (row * (D / G) + d / G) * 2;
          double vv = selected[t] ? or_dequant_refined(vsz[zo], vsz[zo + 1], vqb[e], vrho[e], r)
                                  : or_dequant_base(vsz[zo], vsz[zo + 1], vqb[e]);
          o[d] += p * vv;
        }
      }
      free(l);
      free(selected);
    }
}

/* ------------------------------------------------------------------------- */
/* Decoder-step glue.  The pages run StrataFlux inside llama.cpp on
 * Llama-3.1-8B and leave the rest of the decoder as it is; these are the
 * standard Llama operations, in fp64, with activations rounded to fp16
 * where the decode step hands them from one operation to the next.
 * Readings: RMSNorm weights are 1 and eps = 1e-5; rotary embedding pairs
 * element i with i + d/2 and turns it by pos * theta^(-2i/d), theta = 500000,
 * no frequency rescaling; the MLP is SiLU(gate) * up. */

OR_API void or_rmsnorm_f16(const double* h, int n, double eps, uint16_t* x) {
  double ss = 0.0;
  for (int i = 0; i < n; i++) ss += h[i] * h[i];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int i = 0; i < n; i++) x[i] = or_f16_from_f64(h[i] * inv);
}

OR_API void or_rope(double* v, int heads, int d, int pos, double theta) {
  int half = d / 2;
  for (int h = 0; h < heads; h++) {
    double* x = v + (size_t)h * d;
    for (int i = 0; i < half; i++) {
      double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
      double c = cos(ang), s = sin(ang);
      double x0 = x[i], x1 = x[i + half];
      x[i] = x0 * c - x1 * s;
      x[i + half] = x0 * s + x1 * c;
    }
  }
}

OR_API void or_silu_mul_f16(const double* gu, int inter, uint16_t* out) {
  for (int i = 0; i < inter; i++) {
    double g = gu[i], u = gu[inter + i];
    out[i] = or_f16_from_f64(g / (1.0 + exp(-g)) * u);
  }
}

/* y[n] = sum_c w[n][c] x[c], fp16 weights and activations (the LM head). */
OR_API void or_gemv_f16(const uint16_t* w, const uint16_t* x, int N, int K, double* y) {
  double* xv = (double*)malloc(sizeof(double) * (size_t)K);
  for (int c = 0; c < K; c++) xv[c] = or_f16_to_f64(x[c]);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; n++) {
    double acc = 0.0;
    for (int c = 0; c < K; c++) acc += or_f16_to_f64(w[(size_t)n * K + c]) * xv[c];
    y[n] = acc;
  }
  free(xv);
}

/* The refinement correction alone ([EXPL] "the map app also loads tiles":
 * with fetch lag it is applied after the base product):
 * y[n] = sum over the n_sel selected channels c of x[c] * (w~[n][c] - w^[n][c]). */
OR_API void or_gemv_correction(const uint8_t* qb, const uint8_t* rho, const uint16_t* sz, int N,
                               int K, int r, int G, const uint16_t* x, const int32_t* sel,
                               int n_sel, double* y) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; n++) {
    double acc = 0.0;
    for (int j = 0; j < n_sel; j++) {
      int c = sel[j];
      size_t e = (size_t)n * K + c;
      size_t zo = ((size_t)n * (K / G) + c / G) * 2;
      double d = or_dequant_refined(sz[zo], sz[zo + 1], qb[e], rho[e], r) -
                 or_dequant_base(sz[zo], sz[zo + 1], qb[e]);
      acc += or_f16_to_f64(x[c]) * d;
    }
    y[n] = acc;
  }
}
