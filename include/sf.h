/*
 * sf.h -- C ABI of the selective-precision (nested refinement) decode path.
 *
 * The operations follow the StrataFlux pages, cited by title and paragraph:
 *   [EXPL] "StrataFlux -- Selective precision streaming -- What does it mean?"
 *          - "nested quantization": fetched bits subdivide the bin the resident
 *            code already names (a 2-bit code + 2 fetched bits = 4-bit
 *            resolution);
 *          - "which tiles count": weights refine the k input channels with the
 *            largest |activation| in each chunk of 1,024 channels; the KV cache
 *            scores every cached token by the attention it receives from the
 *            resident low-bit keys and refines the highest-scoring tokens per
 *            KV head; everything not selected still takes part at low
 *            precision;
 *          - "the map app also loads tiles": refinements are fetched early
 *            (fetch lead) and applied late (fetch lag), overlapping transfers
 *            with compute;
 *          - "where it earns its keep": KV refinement is a step that cannot
 *            overlap the attention around it, because the selection depends on
 *            the attention scores.
 *   [ABS]  "StrataFlux: Memory-Hierarchy-Native Low-Bit LLM Inference",
 *          abstract: 2-4-bit weights and 2-3-bit KV caches.
 *
 * Conventions
 *   - Every pointer is a DEVICE pointer unless its comment says "host".
 *   - All memory is owned and allocated by the caller.  No entry point
 *     allocates device memory.  Scratch space is passed as (ws, ws_bytes); the
 *     matching *_workspace_bytes() function gives the size needed.
 *   - Every entry point that takes a stream only enqueues work on it and
 *     returns without waiting for the device.  Arguments are validated on the
 *     host before anything is enqueued; on a validation error nothing is
 *     enqueued.
 *   - fp16 values are IEEE binary16 bit patterns in uint16_t.
 *   - Errors are returned as sf_status; sf_last_error() gives a message for
 *     the calling thread's most recent failure.  The library never aborts,
 *     prints, traps or asserts on the device.
 *   - Device pointers must be 16-byte aligned.
 *
 * Quantisation (shared by weights and KV), for one group of values w:
 *   s = fp16((max w - min w) / (2^b - 1)),  m = fp16(min w)   (one rounding each)
 *   u = (w - m) / s,  Q = clamp(floor((u + 1/2) * 2^r), 0, 2^(b+r) - 1)
 *   base code q = Q >> r,  refinement code rho = Q & (2^r - 1)
 *   base value    = m + s * q
 *   refined value = m + s * (q + (2*rho + 1 - 2^r) / 2^(r+1))
 * (all in fp64, one rounding per operation; a group whose s is 0 gets all
 * codes 0).  q alone is the ordinary b-bit round-to-nearest code; q and rho
 * together are the (b+r)-bit round-to-nearest code on the grid with step
 * s/2^r and offset m + s(1 - 2^r)/2^(r+1).
 *
 * "Natural w-bit stream": element e sits at bit w*e of a little-endian byte
 * string (byte (w*e)/8, bit offset (w*e)%8).
 */
#ifndef SF_H_
#define SF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SF_ABI_VERSION 1

#if defined(__GNUC__)
#define SF_API __attribute__((visibility("default")))
#else
#define SF_API
#endif

typedef struct CUstream_st* sf_stream_t; /* same type as cudaStream_t */
typedef struct CUevent_st* sf_event_t;   /* same type as cudaEvent_t */

typedef enum {
  SF_OK = 0,
  SF_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or range      */
  SF_ERR_UNSUPPORTED = 2, /* valid request this build does not implement     */
  SF_ERR_CUDA = 3,        /* a CUDA call or launch failed (see sf_last_error) */
  SF_ERR_TIMEOUT = 4,     /* a bounded host-side wait ran out                */
  SF_ERR_WORKSPACE = 5    /* ws too small (or NULL with ws_bytes needed > 0) */
} sf_status;

SF_API int sf_abi_version(void);
SF_API const char* sf_status_string(sf_status st);
/* Message of the calling thread's last failure ("" if none).  The pointer
 * stays valid until the thread's next failing call. */
SF_API const char* sf_last_error(void);


/* ======================================================================== */
/* Weights                                                                   */
/* ======================================================================== */

/* A quantised weight matrix W[n][k] (n output rows, k input channels), in
 * groups of `group` consecutive input channels of one row.
 *   b in {2,3,4}, r in {1,2}, group in {32,64,128,256}, k % 1024 == 0 and
 *   k % group == 0, n % 128 == 0.
 * base (n*k*b/8 bytes):
 *   b = 2, 4 : one natural b-bit stream of the k codes per row, rows in order.
 *   b = 3    : plane L = the low 2 bits of every code, a natural 2-bit stream
 *              per row (n*k/4 bytes), then plane H = the high bit (n*k/8
 *              bytes): per row, per block of 32 channels, one little-endian
 *              32-bit word in which channel c (0..31 within the block) sits at
 *              bit 8*(c/4) + c%4 for c < 16 and at bit 8*((c-16)/4) + 4 +
 *              (c-16)%4 for c >= 16.
 *   Each row of a plane is then cut into 16-byte units, and unit u of row i
 *   is stored at unit u XOR (i mod 8) of the row (units move only inside
 *   their aligned 128-byte block; rows of eight consecutive indices hold a
 *   unit in eight different shared-memory bank groups).
 * refine (k*n*r/8 bytes): channel-major, one natural r-bit stream of the n
 *   refinement codes of each input channel ("one contiguous run per channel",
 *   so a selected channel's refinement is one row); may be NULL when
 *   refinements only ever arrive as staged rows.
 * sz (n * k/group * 2 fp16): (s, m) of row i's group j at sz[(i*(k/group)+j)*2]. */
typedef struct {
  int32_t n, k, b, r, group;
  void* base;
  void* refine;
  uint16_t* sz;
} sf_wq;

/* Byte sizes of the three buffers of an sf_wq; any out pointer may be NULL. */
SF_API sf_status sf_wq_bytes(int n, int k, int b, int r, int group, size_t* base_bytes,
                      size_t* refine_bytes, size_t* sz_bytes);

/* Quantise w[n][k] (fp32, device) into the buffers of *out (nested
 * quantisation above, [EXPL] "nested quantization").  Bit-exact with the
 * definition: the fp64 decisions are made with IEEE operations and no
 * contraction.  out->refine must be non-NULL. */
SF_API sf_status sf_pack_nested(const float* w, const sf_wq* out, sf_stream_t stream);

/* Inverse of the packing, for checking: qb[n][k] and rho[n][k] (one code per
 * byte).  rho may be NULL (or out->refine NULL: rho is then not written). */
SF_API sf_status sf_unpack_codes(const sf_wq* w, uint8_t* qb, uint8_t* rho, sf_stream_t stream);

/* Fitted refinement values ([EXPL] "nested quantization": for weights the
 * refinement values are fitted on a small calibration set, so that the
 * channels a step refines partly make up for the error of the channels it
 * leaves at base precision).  Rewrites w->refine of a matrix that
 * sf_pack_nested(wf, w) packed; the base codes, steps and offsets stay.
 *   wf    [n][k] fp32 device: the full-precision weights w was packed from;
 *   x_cal [n_cal][k] fp16 device: calibration activations (16-byte aligned);
 *   chunk, kch: the channel selection the decode step uses (as
 *         sf_select_channels), applied to every calibration row;
 *   alpha > 0: ridge weight;
 *   delta (nullable) [n][k] fp64 device: receives the fitted corrections d.
 * Per chunk J of input channels, with A = x_cal masked to each row's selected
 * channels and e = wf minus the base value (m + s q):
 *   G = A_J^T A_J,  lam = alpha * trace(G) / chunk  (1 where the trace is 0),
 *   d_i[J] = (G + lam I)^-1 (A_J^T X_J + lam I) e_i[J],
 * the minimiser of sum_n (X_nJ . e_iJ - A_nJ . d)^2 + lam |d - e_iJ|^2, and
 *   rho = clamp(floor((d / s + 1/2) * 2^r), 0, 2^r - 1)  (0 where s = 0),
 * the sub-bin of the base bin that holds base + d.  All arithmetic is fp64.
 * ws: sf_fit_refinements_workspace_bytes(n, k, n_cal, chunk, kch) bytes,
 * 16-byte aligned (about 16 (n + n_cal + chunk) k bytes).  A one-off
 * preparation step: it synchronises with the stream before returning
 * (SF_ERR_INVALID_ARG if G + lam I did not factor in fp64). */
SF_API sf_status sf_fit_refinements(const float* wf, const sf_wq* w, const uint16_t* x_cal, int n_cal, int chunk,
                                    int kch, double alpha, double* delta, void* ws, size_t ws_bytes,
                                    sf_stream_t stream);
SF_API size_t sf_fit_refinements_workspace_bytes(int n, int k, int n_cal, int chunk, int kch);

/* Chunked channel selection ([EXPL] "which tiles count"): for every batch row
 * and every chunk of `chunk` input channels, the kch channels with the
 * largest fp16 magnitude |x| (bits & 0x7fff; +0 == -0), equal magnitudes to
 * the lower index, written as absolute channel indices in ascending order.
 *   x   [batch][k] fp16;  sel [batch][k/chunk][kch] int32.
 *   1 <= batch <= 64, k % chunk == 0, chunk in {256, 512, 1024, 2048},
 *   1 <= kch <= chunk. */
SF_API sf_status sf_select_channels(const uint16_t* x, int batch, int k, int chunk, int kch,
                             int32_t* sel, sf_stream_t stream);

/* Refined GEMV ([EXPL] "which tiles count"):
 *   y[b][i] = sum_c x[b][c] * w~[i][c],
 * where w~ is the refined value for the channels selected for batch row b and
 * the base value for every other channel.  Accumulation is fp32.
 *   x [batch][k] fp16, y [batch][n] fp32, 1 <= batch <= 8.
 *   kch = 0: base only (sel_in, sel_out, refine_rows ignored).
 *   sel_in (nullable): a selection made earlier ([batch][k/chunk][kch],
 *     ascending per chunk), e.g. from the previous layer's activation (fetch
 *     lead).  NULL: the call selects from x itself and writes sel_out.  A
 *     negative entry -1 - c names channel c as selected but not refined in
 *     this call (its refinement did not arrive: base precision, no correction;
 *     see sf_stage_refinements_cached).
 *   sel_out (nullable when sel_in is given): receives the selection used.
 *   refine_rows (nullable): staged refinement rows [batch][k/chunk*kch][n*r/8];
 *     row j of batch row b holds the refinement of channel sel[b][j]
 *     (flattened over chunks).  NULL: rows are read from w->refine.
 *   ws/ws_bytes: sf_gemv_workspace_bytes(); currently 0 (ws may be NULL).
 * The call enqueues the selection (when sel_in is NULL) and the GEMV, which is
 * launched with programmatic serialization: its CTAs start copying codes
 * while the previous kernel of the stream drains, and wait for it before
 * reading x, the selection or the staged rows. */
SF_API sf_status sf_gemv_refined(const sf_wq* w, const uint16_t* x, int batch, int chunk, int kch,
                          const int32_t* sel_in, int32_t* sel_out, const void* refine_rows,
                          float* y, void* ws, size_t ws_bytes, sf_stream_t stream);
SF_API size_t sf_gemv_workspace_bytes(const sf_wq* w, int batch, int chunk, int kch);

/* The refinement correction of a GEMV on its own, ADDED into y:
 *   y[b][i] += sum_{c in sel[b]} x[b][c] * (w~[i][c] - w^[i][c]).
 * This is the fetch-lag form ([EXPL] "the map app also loads tiles": the
 * correction is applied one or more layers later than the base product, so
 * the refinement transfer has longer to land): run sf_gemv_refined with
 * kch = 0 for the base product, and this call once the rows are resident.
 * Arguments as sf_gemv_refined; sel is required (kch = 0: no-op). */
SF_API sf_status sf_gemv_correction(const sf_wq* w, const uint16_t* x, int batch, int chunk,
                                    int kch, const int32_t* sel, const void* refine_rows,
                                    float* y, sf_stream_t stream);

/* Base product and correction of one refined GEMV in one launch, written to
 * separate outputs (both overwritten):
 *   y_base[b][i] = sum_c x[b][c] * w^[i][c],
 *   y_corr[b][i] = sum_{c in sel[b]} x[b][c] * (w~[i][c] - w^[i][c]).
 * This serves fetch lag ([EXPL] "the map app also loads tiles") when the rows
 * are already resident: the base product goes on at once and the correction
 * is kept aside until the point of the residual stream where the lag applies
 * it.  Arguments as sf_gemv_refined; kch >= 1, sel_in is required, y_corr is
 * [batch][n] fp32 (16-byte aligned, not overlapping y_base). */
SF_API sf_status sf_gemv_refined_split(const sf_wq* w, const uint16_t* x, int batch, int chunk, int kch,
                                const int32_t* sel_in, const void* refine_rows, float* y_base,
                                float* y_corr, sf_stream_t stream);

/* Number of bounded device-side waits that ran out on the current device
 * (*count), optionally reset to 0 (reset != 0).  The refined GEMV waits on
 * shared-memory barriers for its bulk copies; each such wait gives up after one
 * second, counts itself here and lets the kernel finish without its result
 * (the output is then undefined), so a fault in the memory system shows up as
 * a count, not as a hung GPU.  A nonzero count makes this call return
 * SF_ERR_TIMEOUT.  The call synchronises with the device (it reads the counter
 * with cudaMemcpyFromSymbol). */
SF_API sf_status sf_device_wait_timeouts(unsigned int* count, int reset);

/* ======================================================================== */
/* KV cache                                                                  */
/* ======================================================================== */

/* `batch` independent caches of h_kv heads with room for t_max tokens of d
 * elements, quantised per token in groups of `group` consecutive elements.
 *   d == 128, group == 32, b in {2,3,4}, r in {1,2}, t_max % 16 == 0.
 * Codes (w = b bits) and refinements (w = r bits) use a pair-slot layout laid
 * out for the tensor-core fragments that consume them: a little-endian 32-bit
 * word holds 16/w pairs of w-bit codes; pair slot j keeps its first code at
 * bits [w*j, w*j + w) and its second at bits [16 + w*j, 16 + w*j + w).
 *   kb, kr: per token (16*w bytes), 4 chunks c = 0..3 of w words each; pair
 *     p = 2*s + e (s = 0..7, e = 0..1) of chunk c (word p/(16/w) of the chunk,
 *     slot p%(16/w)) holds dims 16*s + 2*c + 8*e (first) and 16*s + 2*c + 8*e + 1
 *     (second).  Tokens are consecutive: [batch][h_kv][t_max][16*w bytes].
 *   vb, vr: per tile of 16 consecutive tokens 16*u .. 16*u + 15 (256*w bytes),
 *     32 chunks l = 4*g + c (g = 0..7, c = 0..3) of 2*w words each; pair
 *     p = 16*h + 2*m + e (h, e = 0..1, m = 0..7) of chunk l holds dim
 *     16*m + g + 8*e of tokens 16*u + 2*c + 8*h (first) and 16*u + 2*c + 8*h + 1
 *     (second).  [batch][h_kv][t_max/16][256*w bytes].
 *   b = 3: 3 does not divide the 16 bits of a word half, so the codes are two
 *     planes of this layout in the same 48 bytes per token (kb) or 768 bytes
 *     per tile (vb): the low two bits of every code in the w = 2 layout (a key
 *     token's words 0..7, a value tile's words 0..127), then the high bit in
 *     the w = 1 layout (words 8..11, words 128..191).
 * ksz, vsz: [batch][h_kv][t_max][d/group][2] fp16 (s, m) per token and group. */
typedef struct {
  int32_t batch, h_kv, d, t_max, b, r, group;
  void *kb, *kr, *vb, *vr;
  uint16_t *ksz, *vsz;
} sf_kv;

SF_API sf_status sf_kv_bytes(int batch, int h_kv, int d, int t_max, int b, int r, int group,
                      size_t* code_bytes, size_t* refine_bytes, size_t* sz_bytes);

/* Quantise and store tokens t0 .. t0+nt-1 of every head (nested quantisation
 * applied to the KV cache, [EXPL] "nested quantization").
 *   k, v: [batch][h_kv][nt][d] fp16 (either may be NULL to skip it). */
SF_API sf_status sf_kv_pack_tokens(const sf_kv* kv, const uint16_t* k, const uint16_t* v, int t0,
                            int nt, sf_stream_t stream);

/* The decode step's new token from its qkv projection row, in one launch:
 * the rotary embedding of q and k (as sf_rope_split: pairs (i, i + d/2),
 * angle pos * theta^(-2i/d) in fp64), q written to q [batch][h_q][d] fp16,
 * and k and v rounded to fp16 and stored at token t of every head exactly as
 * sf_kv_pack_tokens stores them.  The same results as sf_rope_split followed
 * by sf_kv_pack_tokens(kv, k, v, t, 1).
 *   qkv [batch][(h_q + 2 h_kv) d] fp32; 0 <= t < t_max; h_q % h_kv == 0. */
SF_API sf_status sf_kv_append_rope(const sf_kv* kv, const float* qkv, int h_q, int pos, float theta, int t,
                                   uint16_t* q, sf_stream_t stream);

/* Codes of tokens 0..t-1, for checking: which = 0 keys, 1 values;
 * qb, rho: [batch][h_kv][t][d] (rho nullable). */
SF_API sf_status sf_kv_unpack_codes(const sf_kv* kv, int which, int t, uint8_t* qb, uint8_t* rho,
                             sf_stream_t stream);

/* Token scoring and selection ([EXPL] "which tiles count"):
 *   logit[h][t] = q[h] . k^_base[h / (h_q/h_kv)][t] / sqrt(d)
 *   score[g][t] = sum over the query heads h of KV head g of
 *                 exp(logit[h][t] - max_t logit[h]) / sum_t exp(...)
 *   sel[g] = the k_tok tokens with the highest score (equal scores: lower
 *            token first), ascending.
 *   q [batch][h_q][d] fp16;  sel [batch][h_kv][k_tok] int32.
 *   logits (nullable): receives the base logits [batch][h_q][t] fp32.
 *   scores (nullable): receives score [batch][h_kv][t] fp32.
 *   1 <= t <= min(t_max, 262144), 1 <= k_tok <= min(t, 4096),
 *   h_q % h_kv == 0, h_q / h_kv <= 8 (SF_ERR_UNSUPPORTED above the caps: the
 *   CTA that finishes a head's selection keeps a bitmap of the head's tokens
 *   in shared memory). */
/* The base logits of sf_kv_score_select computed on the CUDA cores (fp32 FMAs,
 * a thread per token) instead of the tensor cores, kept to compare the two
 * forms of the key contraction ([EXPL] "which tiles count": the scores come
 * from the resident low-bit keys).  logits [batch][h_q][t] fp32, as
 * sf_kv_score_select writes them; 2-bit keys and h_q / h_kv <= 4 only
 * (SF_ERR_UNSUPPORTED otherwise).  ws: sf_kv_logits_fma_workspace_bytes(kv, t,
 * h_q) bytes, 16-byte aligned (the per-split softmax records). */
SF_API sf_status sf_kv_logits_fma(const sf_kv* kv, int t, const uint16_t* q, int h_q, float* logits, void* ws,
                                  size_t ws_bytes, sf_stream_t stream);
SF_API size_t sf_kv_logits_fma_workspace_bytes(const sf_kv* kv, int t, int h_q);

SF_API sf_status sf_kv_score_select(const sf_kv* kv, int t, const uint16_t* q, int h_q, int k_tok,
                             int32_t* sel, float* logits, float* scores, void* ws,
                             size_t ws_bytes, sf_stream_t stream);
SF_API size_t sf_kv_score_select_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                          int logits_given);

/* Refined attention for a given selection ([EXPL] "which tiles count",
 * "nested quantization"):
 *   out[h] = sum_t softmax_t(q[h] . k~[t] / sqrt(d)) v~[t]
 * over all t tokens, where k~, v~ are the refined values for the tokens in
 * sel[g] (g the KV head of h) and the base values for every other token.
 * One pass over the cache computes the base attention split over the
 * context (n_splits parts, 0 = automatic); the selected tokens' base
 * contributions are then replaced by their refined ones and the parts are
 * merged by log-sum-exp.  The result does not depend on n_splits beyond fp32
 * rounding.
 *   sel [batch][h_kv][k_tok] (k_tok may be 0: base attention);
 *   out [batch][h_q][d] fp32;
 *   t, k_tok, h_q within the limits of sf_kv_score_select (k_tok >= 0). */
SF_API sf_status sf_kv_attn_refined(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                    const int32_t* sel, int k_tok, int n_splits, float* out,
                                    void* ws, size_t ws_bytes, sf_stream_t stream);
SF_API size_t sf_kv_attn_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                         int n_splits);

/* Score, select and attend in one call (the decode-step form of the two calls
 * above): the base pass over the cache yields the base logits, the softmax
 * statistics and the base attention at once; the tokens are then scored and
 * selected exactly as sf_kv_score_select does, and the selected tokens'
 * contributions are swapped for their refined ones as in sf_kv_attn_refined.
 * The cache is read once.  sel, logits (nullable) and out as above. */
SF_API sf_status sf_kv_attend_selective(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                        int k_tok, int32_t* sel, float* logits, float* out,
                                        void* ws, size_t ws_bytes, sf_stream_t stream);
SF_API size_t sf_kv_attend_selective_workspace_bytes(const sf_kv* kv, int t, int h_q, int k_tok,
                                                     int logits_given);

/* sf_kv_attend_selective with out [batch][h_q][d] rounded to fp16 (nearest
 * even) by the attention kernel itself: the decode step hands the attention
 * output to the next projection in fp16.  Same workspace and errors. */
SF_API sf_status sf_kv_attend_selective_f16(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                            int k_tok, int32_t* sel, float* logits, uint16_t* out,
                                            void* ws, size_t ws_bytes, sf_stream_t stream);

/* Largest workspace sf_kv_attend_selective_static can serve (32 MiB). */
#define SF_KV_STATIC_WS_BYTES (32u << 20)

/* sf_kv_attend_selective with a library-owned workspace: the same kernels and
 * results, but the scratch is a file-scope device array of
 * SF_KV_STATIC_WS_BYTES inside the library instead of (ws, ws_bytes).  The
 * pages have no counterpart of this entry point; it serves callers that cannot
 * allocate device memory per call: a plain C program or an embedding runtime
 * without a caching allocator would need cudaMalloc/cudaFree around every call,
 * and cudaFree synchronises the device, which a latency-bound decode loop
 * cannot afford.  This call allocates nothing.
 *   - The first call on each device does set-up (looks up the array's device
 *     address, which loads the library's module on that device); make it before
 *     any stream capture.
 *   - The workspace sf_kv_attend_selective_workspace_bytes(kv, t, h_q, k_tok,
 *     logits != NULL) gives must not exceed SF_KV_STATIC_WS_BYTES; a larger
 *     request returns SF_ERR_WORKSPACE (with a message) and enqueues nothing.
 *     Passing logits lowers the need by batch*h_q*t*4 bytes.
 *   - All calls on one device share the one array: calls that overlap on the
 *     GPU (streams or threads with no ordering between them) race and give
 *     wrong results.  Order them on one stream or with events.
 * Arguments, layouts and the other errors as sf_kv_attend_selective. */
SF_API sf_status sf_kv_attend_selective_static(const sf_kv* kv, int t, const uint16_t* q, int h_q,
                                               int k_tok, int32_t* sel, float* logits, float* out,
                                               sf_stream_t stream);

/* ======================================================================== */
/* Refinement staging ([EXPL] "the map app also loads tiles": fetch lead)    */
/* ======================================================================== */

/* Copy the rows host_rows[sel[j]] (j < n_sel, each row_bytes long) into
 * dst[j] on `stream`, reading pinned host memory directly from the GPU, and
 * record `done` (nullable) on `stream` after the copy.  sel is a DEVICE array
 * (a selection made on the GPU, e.g. by sf_select_channels one layer early),
 * so no host round trip is needed.  host_rows must be page-locked host memory
 * mapped into the device address space (cudaHostAlloc with
 * cudaHostAllocMapped, or cudaHostRegister with cudaHostRegisterMapped) that
 * holds n_rows rows of row_bytes; row_bytes % 16 == 0.
 * Since the indices are only known on the device, they are checked there: an
 * index outside [0, n_rows) is not read; its destination row is filled with
 * zeros and, when `bad` (nullable, a device int32) is given, *bad is
 * incremented once per such index (the caller zeroes it and reads it back). */
SF_API sf_status sf_stage_refinements(const void* host_rows, size_t row_bytes, int n_rows,
                                      const int32_t* sel, int n_sel, void* dst, int32_t* bad,
                                      sf_stream_t stream, sf_event_t done);

/* Same copy with a HOST index array: one cudaMemcpyAsync per run of
 * consecutive indices.  host_rows must be pinned and hold n_rows rows; every
 * index is checked against [0, n_rows) before anything is enqueued
 * (SF_ERR_INVALID_ARG otherwise). */
SF_API sf_status sf_stage_refinements_host(const void* host_rows, size_t row_bytes, int n_rows,
                                           const int32_t* sel_host, int n_sel, void* dst,
                                           sf_stream_t stream, sf_event_t done);

/* A device-resident cache of refinement rows, reused across decode steps
 * ([EXPL] "the map app also loads tiles": fetched bits are kept and reused
 * while the selections repeat from token to token; on a miss the runtime
 * either waits for the transfer or runs the channel at its resident precision
 * for the moment).  Every array is device memory owned by the caller.
 *   capacity    rows held, n_sel <= capacity <= 8192;
 *   n_channels  the channel index space (the rows of host_rows);
 *   row_bytes   bytes per row (a multiple of 16);
 *   slot_of     [n_channels] int32: slot holding the channel's row, -1 if none;
 *   channel_of  [capacity] int32: channel held by the slot, -1 if free;
 *   stamp       [capacity] uint32: step of the slot's last use;
 *   state       [4] uint32: step counter, clock hand, cumulative hits,
 *               cumulative misses (readable for statistics);
 *   work        [max_sel] int32: scratch of one call;
 *   max_sel     the most entries one call stages (<= 4096);
 *   rows        [capacity][row_bytes].
 * sf_row_cache_reset() empties it (enqueued on `stream`).  Calls that share a
 * cache must not overlap on the GPU. */
typedef struct {
  int32_t capacity, n_channels, row_bytes;
  int32_t* slot_of;
  int32_t* channel_of;
  uint32_t* stamp;
  uint32_t* state;
  int32_t* work;
  int32_t max_sel;
  void* rows;
} sf_row_cache;

SF_API sf_status sf_row_cache_reset(const sf_row_cache* cache, sf_stream_t stream);

/* sf_stage_refinements through row caches, one per batch row.  The selected
 * channels a cache holds are copied from its device rows (no host-link
 * traffic); every other channel gets the cache's slot least recently used and
 * not needed now, and its row is read from host_rows (mapped pinned memory, as
 * for sf_stage_refinements) into that slot.
 *   sel      [batch][n_sel] DEVICE, distinct channels per batch row;
 *   caches   HOST array of `batch` caches (1 <= batch <= 8);
 *   dst      [batch][n_sel][row_bytes] DEVICE;
 *   sel_eff  [batch][n_sel] DEVICE, receives the selection the GEMV is to use:
 *            sel[b][j], or -1 - sel[b][j] for a channel that stays at base
 *            precision in this step (sf_gemv_refined adds no correction for a
 *            negative entry);
 *   skip_missing = 0: missing rows are read into dst too, and sel_eff == sel;
 *   skip_missing = 1: missing channels are marked in sel_eff and their rows go
 *            only to the cache, after `done`, on the same stream: a GEMV that
 *            waits for `done` does not wait for the host link (skip on miss);
 *   `done` (nullable) is recorded once dst and sel_eff are complete.
 * An entry of sel outside [0, n_rows) is not staged (sel_eff marks it
 * skipped). */
SF_API sf_status sf_stage_refinements_cached(const void* host_rows, size_t row_bytes, int n_rows,
                                             const int32_t* sel, int n_sel, int batch,
                                             const sf_row_cache* caches, int skip_missing, void* dst,
                                             int32_t* sel_eff, sf_stream_t stream, sf_event_t done);

/* ======================================================================== */
/* Decoder-step glue (standard Llama operations around the refined ones)     */
/* ======================================================================== */

/* h[b] += add0[b] + add1[b] (each nullable), then x[b] = fp16(h[b] /
 * sqrt(mean(h[b]^2) + eps)) (RMSNorm with unit weights).  h [batch][n] fp32,
 * x [batch][n] fp16. */
SF_API sf_status sf_rmsnorm_residual(float* h, const float* add0, const float* add1, int batch,
                                     int n, float eps, uint16_t* x, sf_stream_t stream);

/* qkv [batch][(h_q + 2 h_kv) d] fp32 -> q [batch][h_q][d], k, v [batch][h_kv][d]
 * fp16; q and k turned by the rotary embedding (pairs (i, i + d/2), angle
 * pos * theta^(-2i/d), computed in fp64). */
SF_API sf_status sf_rope_split(const float* qkv, int batch, int h_q, int h_kv, int d, int pos,
                               float theta, uint16_t* q, uint16_t* k, uint16_t* v,
                               sf_stream_t stream);

/* out[b][i] = fp16(silu(gu[b][i]) * gu[b][inter + i]). */
SF_API sf_status sf_silu_mul(const float* gu, int batch, int inter, uint16_t* out,
                             sf_stream_t stream);

/* y = fp16(x) and y = fp32(x) element-wise. */
SF_API sf_status sf_cast_f16(const float* x, size_t n, uint16_t* y, sf_stream_t stream);
SF_API sf_status sf_widen_f16(const uint16_t* x, size_t n, float* y, sf_stream_t stream);

/* y[b][i] = sum_c w[i][c] x[b][c] with fp16 w [n][k] and x [batch][k], fp32
 * accumulation (the LM head).  1 <= batch <= 8, k % 8 == 0. */
SF_API sf_status sf_gemv_f16(const uint16_t* w, const uint16_t* x, int batch, int n, int k,
                             float* y, sf_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SF_H_ */
