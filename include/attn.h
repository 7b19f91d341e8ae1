/*
 * attn.h -- C ABI of the B200 (sm_100a) fused attention forward library.
 *
 * The operation is scaled-dot-product attention, O = softmax(scale*Q K^T + mask) V,
 * computed flash-style (key/value tiles streamed through shared memory, an
 * online softmax, no score matrix in global memory).  Sources for the problem
 * statement:
 *   - "perf(metal): widen four-row flash KV tiles - #89", section "Performance
 *     evidence": query rows, n_head query heads over n_kv key/value heads,
 *     head_dim, kv_len, the start position `pos` of query row 0, f16 K/V and a
 *     causal mask; section "Summary": a sliding-window lower bound on the keys.
 *   - "Shmoosh update", sections "The measured changes" and "An explicit
 *     fast-mode policy": an exact default precision and an opt-in fast mode
 *     that is never switched on silently.
 *   - "Ядра attention на домашней RTX 5080", table of section "1 · Только
 *     ядро": the opt-in mode's form, INT8 Q K^T with FP8 P V.
 *   - "round 21 track b -- qsa2" (the qsa2 audit), section "implementation and
 *     review": chunked (split-KV) attention whose partial results are merged
 *     with cached per-chunk maxima and weights and one denominator.
 *
 * Conventions
 *   - Layout: Q and O are [batch, n_q_heads, q_len, head_dim]; K and V are
 *     [batch, n_kv_heads, kv_len, head_dim]; all contiguous, head_dim fastest.
 *     lse is [batch, n_q_heads, q_len] float32.
 *   - GQA: query head h reads key/value head h / (n_q_heads / n_kv_heads).
 *   - Query row i sits at absolute position start_pos + i.  With causal != 0
 *     it sees keys j <= start_pos + i.  Keys j < window_lo are never seen.  With
 *     window_size W > 0 it sees only keys j >= start_pos + i - W + 1 as well (the
 *     last W positions up to its own when causal).
 *     A row that sees no key gets O = 0 and lse = -inf.
 *   - All tensor pointers are DEVICE pointers owned by the caller and must be
 *     16-byte aligned; the library never frees them.  A buffer of zero length
 *     (q_len or kv_len 0) may be NULL.  `stream` is a
 *     cudaStream_t passed as void*.  Every call is asynchronous on that stream;
 *     argument errors are reported synchronously, before anything is launched.
 *   - Keys of a loaded 128-key tile that a row cannot see get a zero weight in P.V;
 *     they must hold finite values (an Inf or NaN there reaches O).  Key tiles that
 *     no row of a CTA sees are not loaded at all.
 *   - A context is not safe for concurrent use from several host threads.  Its
 *     workspace (split-KV partials, V channel maxima) is shared by all of its
 *     calls: calls on different streams that use it must be ordered by the caller.
 *   - Device-side waits are bounded (about 1.5 s).  A wait that runs out
 *     records an error word in the context; attn_get_error() reports it.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* a parameter or pointer is invalid */
  ATTN_ERR_UNSUPPORTED = 2, /* valid but not supported (e.g. head_dim, alignment) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  ATTN_ERR_OOM = 4,         /* workspace allocation failed */
  ATTN_ERR_TIMEOUT = 5      /* a device-side wait ran out (see attn_get_error) */
} attn_status;

typedef enum { ATTN_BF16 = 0, ATTN_FP16 = 1 } attn_dtype;

/* ATTN_EXACT is the default: 16-bit inputs, f32 accumulation.
 * ATTN_INT8QK_FP8PV is opt-in: Q/K quantised to INT8 per 128-token block with
 * FP32 scales, P and V in FP8 E4M3 (V with one FP32 scale per head and channel).
 * ATTN_MIXED_DIAG is opt-in too: diagonal-tiled mixed precision ("Transformers
 * Get a Turbo Boost with Mixed-Precision Magic": two kinds of computation chosen
 * per tile).  It is ATTN_INT8QK_FP8PV except that the key tiles of the causal
 * diagonal band -- the tiles some row of a 256-row query tile must partly mask --
 * get Q K^T from the 16-bit inputs (float32 scores); P and V stay FP8 E4M3.
 * Without a causal mask there is no band and it computes what ATTN_INT8QK_FP8PV
 * does.  It always runs the single-pass kernel (num_splits 0 or 1).
 * ATTN_MXFP4QK_FP8PV is opt-in: the FP4 microscaled mode.  Q and K are quantised to
 * MXFP4 (OCP Microscaling: E2M1 elements, one E8M0 power-of-two scale per 32
 * channels of a row) and Q K^T runs on the block-scaled tensor-core MMA; P and V
 * stay FP8 E4M3 as in ATTN_INT8QK_FP8PV.  FP4 attention and the MXFP formats on B200
 * are named on the pages "Ядра attention на домашней RTX 5080" (table of section
 * "1 · Только ядро", SageAttention 3) and "Transformers Get a Turbo Boost with
 * Mixed-Precision Magic".  head_dim 64 only: the scale factors live in tensor
 * memory, which the head_dim-128 kernel fills with its scores and outputs.  Single-
 * pass kernel only (num_splits 0 or 1); no RoPE. */
typedef enum {
  ATTN_EXACT = 0,
  ATTN_INT8QK_FP8PV = 1,
  ATTN_MIXED_DIAG = 2,
  ATTN_MXFP4QK_FP8PV = 3
} attn_precision;

typedef struct {
  int batch;       /* B >= 1 */
  int n_q_heads;   /* Hq >= 1, a multiple of n_kv_heads */
  int n_kv_heads;  /* Hkv >= 1 */
  int q_len;       /* Sq >= 0 (0: nothing to do) */
  int kv_len;      /* Skv >= 0 (0: every row sees no key) */
  int head_dim;    /* 64 or 128 */
  int start_pos;   /* absolute position of query row 0, >= 0 */
  int causal;      /* 0 or 1 */
  int window_lo;   /* first visible key index, >= 0 (0: no window) */
  float scale;     /* multiplier of Q K^T; <= 0 selects 1/sqrt(head_dim) */
  int dtype;       /* attn_dtype of Q, K, V and O */
  int precision;   /* attn_precision */
  int num_splits;  /* key/value splits: 0 = chosen by the library, 1 = none, >1 = forced */
  int window_size; /* sliding window W >= 0: row i sees keys j >= start_pos + i - W + 1
                      (0: none); combined with window_lo, the larger bound applies */
  /* Rotary position embedding (RoPE), applied to Q and K before Q K^T.  Planned
   * "with NTK / YaRN scaling" inside the kernel instead of a separate pass on the
   * page "Ядра attention на домашней RTX 5080", section "Планы · Rigsy Kernel".
   * Query row i rotates by position start_pos + i, key j by position j, with the
   * cos/sin table given by attn_set_rope_table (built by attn_rope_table). */
  int rope_dim;          /* rotated channels R: 0 (no RoPE) or a multiple of 16 <= head_dim;
                            channels R .. head_dim-1 are not rotated */
  int rope_interleaved;  /* 0: channel i pairs with i + R/2; 1: channel 2i pairs with 2i + 1 */
  int rope_keys_rotated; /* 1: k already holds rotated keys (a key cache written through
                            attn_rope_apply); only q is rotated.  0: both are rotated */
} attn_params;

/* Frequencies of the rotary table: theta_i = base^(-2i/R), i < R/2.
 *   ATTN_ROPE_PLAIN: as is.
 *   ATTN_ROPE_NTK:   base becomes base * factor^(R / (R - 2)) (NTK-aware scaling).
 *   ATTN_ROPE_YARN:  with r_i = original_len * theta_i / (2 pi) and the ramp
 *                    g_i = clamp((r_i - beta_slow) / (beta_fast - beta_slow), 0, 1),
 *                    theta_i becomes (1 - g_i) theta_i / factor + g_i theta_i, and
 *                    cos and sin are multiplied by 0.1 ln(factor) + 1 (factor > 1). */
typedef enum { ATTN_ROPE_PLAIN = 0, ATTN_ROPE_NTK = 1, ATTN_ROPE_YARN = 2 } attn_rope_scaling;

typedef struct {
  float base;        /* > 0, e.g. 10000 */
  int scaling;       /* attn_rope_scaling */
  float factor;      /* NTK / YaRN context-extension factor (>= 1; 1 = none) */
  int original_len;  /* YaRN: the original context length */
  float beta_fast;   /* YaRN ramp bounds (e.g. 32 and 1), beta_fast > beta_slow */
  float beta_slow;
} attn_rope_freq;

/* Caller-owned device buffers of the quantised modes (all 16-byte aligned):
 *   q       int8   [B, Hq,  Sq,  D]          q_scale float [B, Hq,  ceil(Sq/128)]
 *   k       int8   [B, Hkv, Skv, D]          k_scale float [B, Hkv, ceil(Skv/128)]
 *   v_t     uint8  [B, Hkv, D, ceil(Skv/128)*128]  E4M3 codes of V, transposed,
 *                                            zero padded;  v_scale float [B, Hkv, D]
 * In the FP4 mode (ATTN_MXFP4QK_FP8PV) q and k hold packed E2M1 codes instead, two
 * per byte (channel 2i in the low nibble): q [B, Hq, Sq, D/2], k [B, Hkv, Skv, D/2];
 * q_scale and k_scale are unused (may be NULL); and q_sf, k_sf hold the E8M0 scale
 * bytes in the tensor core's layout: one 512-byte chunk per 128-row tile, row r of
 * the tile and channel block b (of 32) at byte (r % 32) * 16 + (r / 32) * 4 + b
 * (b = 2, 3 unused).  Q's tiles run over the rows of a (batch, kv head) unit, its
 * query heads stacked (G * Sq rows), rounded up to an even tile count:
 * q_sf [B * Hkv][2 * ceil(G * Sq / 256)][512]; K's over each (batch, kv head)'s
 * keys: k_sf [B * Hkv][ceil(Skv / 128)][512] (attn_qbufs_sf_sizes gives the sizes). */
typedef struct {
  int8_t *q;
  int8_t *k;
  float *q_scale;
  float *k_scale;
  uint8_t *v_t;
  float *v_scale;
  uint8_t *q_sf;  /* FP4 mode only (else ignored, may be NULL) */
  uint8_t *k_sf;
} attn_qbufs;

typedef struct attn_ctx attn_ctx;

/* Validates `p`, picks the kernel variant and the key/value split for the
 * current CUDA device, and allocates the context's workspace (split partial
 * results, the V channel maxima, the device error word, and in the exact mode
 * with RoPE on unrotated keys a buffer of K's size for the rotated keys).  On
 * success *out owns that workspace until attn_destroy().  Launches nothing.
 * Errors: ATTN_ERR_INVALID_ARG (bad field or NULL), ATTN_ERR_UNSUPPORTED
 * (head_dim not 64/128; the FP4 mode at head_dim 128 or with RoPE; the diagonal
 * band mode with RoPE; more than 2^30 stacked rows per kv head or positions past
 * 2^30; batch * n_kv_heads above 65535 in a quantised mode; a problem whose CTA or
 * 128-token block count passes 2^31 - 1; a device other than sm_100),
 * ATTN_ERR_CUDA (no device), ATTN_ERR_OOM. */
attn_status attn_create(const attn_params *p, attn_ctx **out);

/* Quantised, diagonal band and FP4 modes, step 1 (the quantisers): reads q, k, v (dtype of
 * the context) and writes every buffer of *qb.  Q and K: per (b, h, 128-token
 * block) s = max|x| / 127 and code = clamp(round_half_even(x / s), +-127), s = 0
 * for an all-zero block.  V: per (b, hkv, channel) s = max|v| / 448 and code =
 * E4M3(v / s) rounded to nearest-even and saturated.  Each step is one
 * correctly rounded float32 operation, so the bytes are reproducible.  FP4 mode,
 * Q and K: per row and block of 32 channels, the E8M0 scale 2^e with
 * e = floor(log2(max|x|)) - 2 (clamped to [-127, 127]; an all-zero block takes
 * e = -127) and codes = E2M1(x / 2^e) rounded to nearest-even and saturated to +-6
 * (the OCP MX conversion; x / 2^e is exact).  With
 * RoPE, Q and K (K unless rope_keys_rotated) are rotated in float32 first and
 * the codes are those of the rotated values.
 * Errors: ATTN_ERR_INVALID_ARG (NULL or misaligned pointer, context not in the
 * quantised mode, RoPE without a table), ATTN_ERR_CUDA (launch failure). */
attn_status attn_quantize_qk(attn_ctx *c, const void *q, const void *k, const void *v,
                             const attn_qbufs *qb, void *stream);

/* ATTN_INT8QK_FP8PV with a paged key/value cache (the qsa2 audit's decode workload
 * runs on a 32768-cell KV cache; the paging is as in attn_forward_paged below):
 * attn_quantize_qk with K and V read from the pools of attn_forward_paged
 * ([num_blocks][n_kv_heads][128][head_dim], 16-bit; block_table
 * [batch][ceil(kv_len / 128)] int32, device) and Q dense as usual.  The buffers *qb
 * it writes are those of the dense layout, bit-identical to attn_quantize_qk's on
 * the gathered keys and values (positions past kv_len in a block are not read);
 * attn_forward(c, NULL, NULL, NULL, qb, o, lse, stream) then runs the quantised
 * attention.  V's scale is per channel over the whole sequence, so each call
 * quantises the whole cache.  A table entry outside [0, num_blocks) is read as
 * block 0 and makes the next attn_get_error return ATTN_ERR_INVALID_ARG.  With RoPE
 * the pool's keys must be rotated already (rope_keys_rotated).
 * Errors: ATTN_ERR_INVALID_ARG (as attn_quantize_qk; NULL or misaligned
 * block_table, num_blocks < 1), ATTN_ERR_UNSUPPORTED (another precision, or RoPE on
 * unrotated keys), ATTN_ERR_CUDA (launch failure). */
attn_status attn_quantize_qk_paged(attn_ctx *c, const void *q, const void *k_pool,
                                   const void *v_pool, const int32_t *block_table,
                                   int num_blocks, const attn_qbufs *qb, void *stream);

/* The attention forward.  Exact mode: q, k, v are read and qb must be NULL.
 * Quantised mode: q, k, v are ignored (may be NULL) and qb holds the output of
 * attn_quantize_qk.  Diagonal band mode: qb as in the quantised mode, and q and k
 * (the 16-bit inputs) are read for the band tiles; v is ignored.  Writes o ([B, Hq, Sq, D], the context's dtype) and, if
 * lse is not NULL, the natural-log sum of exp(scale * q.k) over each row's
 * visible keys.  Few-row (decode-shaped) problems are split along the keys and
 * merged by a second kernel into the same outputs.
 * With RoPE (rope_dim > 0) the table must have been set (attn_set_rope_table).
 * Errors: ATTN_ERR_INVALID_ARG (NULL or misaligned pointer, qb presence not
 * matching the mode, RoPE without a table), ATTN_ERR_CUDA (tensor-map encode or
 * launch failure). */
attn_status attn_forward(attn_ctx *c, const void *q, const void *k, const void *v,
                         const attn_qbufs *qb, void *o, float *lse, void *stream);

/* End-to-end forward from host memory.
 * No counterpart on the source pages: it is for callers whose Q, K and V sit in
 * host memory.  It copies q, k and v from the host into the caller's device
 * buffers, runs the forward (preceded by the quantiser in the quantised mode)
 * and copies o, and lse if asked for, back to the host, overlapping the copies
 * with the kernels.  The problem's units (one per batch entry and kv head, with
 * that head's query heads) are independent and every tensor is unit-major, so
 * the call cuts the units into `chunks` contiguous ranges.  For each range the
 * host-to-device copies, the kernels and the device-to-host copies run in that
 * order, on four streams that the context owns: while one range computes, the
 * next range's inputs arrive and the previous range's outputs leave, each
 * direction on its own copy engine.  The kernels of consecutive ranges go to
 * two streams, so the last wave of one range overlaps the first of the next.
 * A range's outputs leave once the next range's inputs are in, in pieces of 1
 * to 8 MiB sized from the problem's output/input byte ratio, so that the
 * inputs, the larger stream, keep most of the link.
 * Every result is bit-identical to attn_forward's (and attn_quantize_qk's) on
 * the same inputs.  All of the work is ordered after the work already queued on
 * `stream`, and work queued on `stream` afterwards waits for all of it:
 * synchronise `stream` before reading o_host.
 *
 * Arguments: q_host, k_host, v_host (read) and o_host, lse_host (written) are
 * host pointers in the layouts above.  lse_host may be NULL, and must be NULL
 * exactly when lse_dev is.  Page-locked host memory (cudaHostAlloc or
 * cudaHostRegister) lets the copies overlap the kernels; pageable memory gives
 * the same results with the copies serialised by the driver.  q_dev, k_dev,
 * v_dev, o_dev and lse_dev are device buffers of the full sizes, 16-byte
 * aligned, which the call uses as staging (q_dev, k_dev and v_dev hold the
 * 16-bit inputs in both modes).  qb: in the quantised mode, the quantiser's
 * output buffers as for attn_forward (filled by this call); NULL in exact mode.
 * chunks: 0 lets the library choose (about 24 MiB of inputs per range, at most
 * 64 ranges); 1 to 64 asks for that many ranges; either is capped at the number
 * of units.
 * A problem on the split-KV path runs as one range.  Every buffer must stay
 * valid until the work completes.  The first call creates the context's streams
 * and events on the current device, which must be the context's.
 * Errors: ATTN_ERR_INVALID_ARG (NULL host pointer, NULL or misaligned device
 * pointer, lse_host and lse_dev not both given or both NULL, qb presence not
 * matching the mode, chunks out of range), ATTN_ERR_CUDA (stream or event
 * creation, copy, tensor-map encode or launch failure). */
attn_status attn_forward_host(attn_ctx *c, const void *q_host, const void *k_host,
                              const void *v_host, void *o_host, float *lse_host, void *q_dev,
                              void *k_dev, void *v_dev, void *o_dev, float *lse_dev,
                              const attn_qbufs *qb, int chunks, void *stream);

/* Paged key/value cache (exact mode).
 * No counterpart on the source pages beyond the decode workload of the qsa2
 * audit (its 32768-cell KV cache): keys and values live in fixed blocks of 128
 * positions in a pool shared by all batch entries, as a serving engine keeps
 * them, and a block table maps each batch entry's positions to blocks.
 * k_pool, v_pool: [num_blocks, n_kv_heads, 128, head_dim] (the context's dtype,
 * 16-byte aligned).  block_table: int32 [batch, ceil(kv_len / 128)] (4-byte
 * aligned, device memory); entry [b][t] is the block that holds positions
 * 128 t .. 128 t + 127 of batch entry b.  Everything else is as attn_forward
 * (q, o and lse dense; kv_len is every batch entry's number of positions), and
 * the result equals attn_forward on K and V gathered through the table.  An
 * entry outside [0, num_blocks) reads zeros (the copy engine's bounds), never
 * memory outside the pool.  The positions past kv_len in a batch entry's last
 * block must hold finite values.
 * Errors: ATTN_ERR_INVALID_ARG (NULL or misaligned pointer, num_blocks < 1),
 * ATTN_ERR_UNSUPPORTED (a quantised mode: the INT8 mode reads a paged cache through
 * attn_quantize_qk_paged, then attn_forward), ATTN_ERR_CUDA (tensor-map encode or
 * launch failure). */
attn_status attn_forward_paged(attn_ctx *c, const void *q, const void *k_pool,
                               const void *v_pool, const int32_t *block_table, int num_blocks,
                               void *o, float *lse, void *stream);

/* Host-side RoPE table: table_host[p][0][i] = cos(p theta_i) * m and
 * table_host[p][1][i] = sin(p theta_i) * m for p < n_pos, i < rope_dim / 2
 * (float32, n_pos * rope_dim floats), with theta_i and the factor m from `f`
 * (m = 1 except for YaRN).  Each entry is computed in double precision and
 * rounded once.  Pure host arithmetic; copy the table to device memory and pass
 * it to attn_set_rope_table.
 * Errors: ATTN_ERR_INVALID_ARG (NULL pointer, rope_dim not a positive even
 * number, n_pos < 1, base <= 0, factor < 1, YaRN with beta_fast <= beta_slow or
 * original_len < 1, unknown scaling). */
attn_status attn_rope_table(int rope_dim, int n_pos, const attn_rope_freq *f, float *table_host);

/* Gives a context with rope_dim > 0 its cos/sin table: a DEVICE pointer (16-byte
 * aligned, caller-owned, valid while the context uses it) to float32
 * [n_pos][2][rope_dim / 2] as attn_rope_table writes it.  n_pos must cover every
 * position the context rotates: max(start_pos + q_len, kv_len) (and the
 * positions passed to attn_rope_apply).  Launches nothing.
 * How the rotation runs: in the quantised mode the Q/K quantiser rotates each
 * block in float32 before taking its maximum (no extra pass: the codes are those
 * of the rotated values, reproducible bit for bit).  In the exact mode the
 * attention kernel rotates its staged Q tile in shared memory, and K (unless
 * rope_keys_rotated) is rotated by a pass into the context's workspace before
 * the kernel.  Rotated 16-bit values are rounded to nearest-even.  The rotation
 * of a pair (a, b) with table entries (c, s) is a' = RN(RN(a c) - RN(b s)),
 * b' = RN(RN(a s) + RN(b c)) in float32.
 * Errors: ATTN_ERR_INVALID_ARG (NULL context or table, misaligned table, the
 * context has rope_dim 0, n_pos too small). */
attn_status attn_set_rope_table(attn_ctx *c, const float *table_dev, int n_pos);

/* Rotates x [batch, n_heads, len, head_dim] (the context's dtype, batch and
 * head_dim; device memory) into y (same shape; y may equal x) with the
 * context's table and pair layout; row t of every head sits at position
 * pos0 + t.  For writing keys into a cache once, so that later forwards can run
 * with rope_keys_rotated = 1.  Asynchronous on `stream`.
 * Errors: ATTN_ERR_INVALID_ARG (NULL or misaligned pointer, n_heads < 1,
 * len < 0, pos0 < 0, no table set, positions past the table),
 * ATTN_ERR_CUDA (launch failure). */
attn_status attn_rope_apply(attn_ctx *c, const void *x, void *y, int n_heads, int len, int pos0,
                            void *stream);

/* Synchronises `stream`, reads and clears the context's device error word.
 * Returns ATTN_ERR_INVALID_ARG if attn_quantize_qk_paged met a block-table entry
 * outside the pool since the last call, ATTN_ERR_TIMEOUT if a kernel gave up on a
 * wait, ATTN_ERR_CUDA if the stream reports an error, else ATTN_OK. */
attn_status attn_get_error(attn_ctx *c, void *stream);

/* Waits for the context's own work (its last call, recorded on that call's
 * stream, and the streams of attn_forward_host's pipeline), then frees the
 * workspace.  Work of other contexts or libraries on the device is not waited
 * for by this call (the CUDA runtime's cudaFree may still synchronise the
 * device).  Calls captured into a CUDA graph are not waited for: destroy the
 * context only after every launch of such a graph has finished (the graph
 * refers to the workspace).  NULL is ignored. */
void attn_destroy(attn_ctx *c);

/* Static string naming a status code. */
const char *attn_status_string(attn_status s);

/* Sizes, in bytes, of the caller-owned buffers of the quantised modes for `p`,
 * in the order of attn_qbufs (q, k, q_scale, k_scale, v_t, v_scale); in the FP4
 * mode q and k are the packed codes and the two scale sizes are 0.  Pure host
 * arithmetic.  Errors: ATTN_ERR_INVALID_ARG. */
attn_status attn_qbufs_sizes(const attn_params *p, size_t sizes[6]);

/* FP4 mode: sizes in bytes of q_sf and k_sf for `p` (0 in the other modes).
 * Pure host arithmetic.  Errors: ATTN_ERR_INVALID_ARG. */
attn_status attn_qbufs_sf_sizes(const attn_params *p, size_t sizes[2]);

/* Number of key/value splits the context uses (1 = no split), 0 for NULL. */
int attn_num_splits(const attn_ctx *c);

/* The kernel a context runs, fixed by attn_create:
 *   ATTN_PATH_SINGLE_PASS  the tensor-core kernel, 256 query rows per CTA, every key;
 *   ATTN_PATH_SPLIT_MERGE  one 128-row query tile per CTA, the keys split across
 *                          CTAs, then a merge kernel (few rows per kv head, or too few
 *                          CTAs to fill the GPU);
 *   ATTN_PATH_SINGLE_PASS_TAIL  the single-pass kernel, whose grid would end in a
 *                          last wave at most half full: those last CTAs' rows run
 *                          instead on the split kernel (keys split across CTAs) and a
 *                          merge, so that every wave is full (non-causal, exact or
 *                          INT8 mode, Hq/Hkv * q_len a multiple of 256, num_splits 0);
 *   ATTN_PATH_DECODE       exact mode with at most 16 stacked rows per unit
 *                          (Hq/Hkv * q_len <= 16, e.g. decode steps) and num_splits
 *                          0 or 2..16: one thread-block cluster of num_splits CTAs per
 *                          (batch, kv head); each CTA streams an equal run of the
 *                          rows' visible keys, and the CTAs merge their partial
 *                          results through distributed shared memory in the same
 *                          launch.  The split key range is the union of the rows'
 *                          visible ranges; the merge is the qsa2 audit's ("round 21
 *                          track b -- qsa2", "implementation and review": cached
 *                          per-split maxima and weights, one denominator).
 * Returns 0 for NULL. */
typedef enum {
  ATTN_PATH_SINGLE_PASS = 1,
  ATTN_PATH_SPLIT_MERGE = 2,
  ATTN_PATH_DECODE = 3,
  ATTN_PATH_SINGLE_PASS_TAIL = 4
} attn_kernel_path_kind;
int attn_kernel_path(const attn_ctx *c);

/* The kernel choice attn_create makes for `p` on a GPU with `num_sms` SMs, as plain
 * host arithmetic (no device is touched).  attn_create makes the same choice, except
 * that on the device it may lower a decode cluster's size (`splits`) until every
 * (batch, kv head)'s cluster fits at once.
 *   path             attn_kernel_path_kind
 *   splits           key splits (1: none; ATTN_PATH_DECODE: CTAs per cluster)
 *   tiles_per_split  ATTN_PATH_SPLIT_MERGE: 128-key tiles per split (else 0)
 *   ctas             CTAs of the main launch
 *   tail_items       ATTN_PATH_SINGLE_PASS_TAIL: 256-row CTAs moved to the split kernel
 *   tail_splits      their key splits
 *   decode_chunk     ATTN_PATH_DECODE: keys per chunk (32 at head_dim 128, 64 at 64)
 *   decode_chunks    ATTN_PATH_DECODE: chunks covering the rows' visible keys
 * Errors: those of attn_create's validation of `p`; ATTN_ERR_INVALID_ARG for a NULL
 * `out` or num_sms < 1. */
typedef struct {
  int path;
  int splits;
  int tiles_per_split;
  int ctas;
  int tail_items;
  int tail_splits;
  int decode_chunk;
  int decode_chunks;
} attn_plan;
attn_status attn_plan_for(const attn_params *p, int num_sms, attn_plan *out);

/* TEST HOOK.  Bit 0 of `flags` makes the next attn_forward's loader skip the
 * second key tile of every CTA (ATTN_PATH_DECODE: the second key chunk of the
 * first warp of the first CTA), so that the waits on it run out: the kernel then
 * records ATTN_ERR_TIMEOUT in the context and returns without hanging.  Bit 1
 * does the same to attn_quantize_qk: the first CTA of the Q quantiser never
 * loads its second block.  The hook exists only to test that error path; 0
 * restores normal operation. */
attn_status attn_debug_set(attn_ctx *c, unsigned flags);

/* TEST HOOK.  y[i] = 2^x[i] (device pointers, n floats) computed by the
 * polynomial exponential that the softmax runs on the FMA pipe for part of its
 * exponentials (range reduction to [-1/2, 1/2] and a degree-3 fit of 2^f; max
 * relative error 7.5e-5 for -125 <= x <= 126; inputs below -125 are treated as -125).
 * Errors: ATTN_ERR_INVALID_ARG (NULL pointer with n > 0), ATTN_ERR_CUDA. */
attn_status attn_debug_exp2(const float *x, float *y, size_t n, void *stream);

/* Split-KV forward that allocates nothing (exact mode only).
 * No counterpart on the source pages: it is a convenience for callers that
 * cannot call cudaMalloc.  Examples are code whose device memory is owned by
 * another allocator (a serving engine that reserves HBM up front and forbids
 * stray allocations), and a latency-critical decode step that cannot afford
 * cudaMalloc's implicit device synchronisation.  It takes the problem
 * description directly (no context, so no attn_create) and computes the same
 * result as attn_forward does on the split-KV path: key/value splits in one
 * kernel, then the merge.  The split partials live in a fixed device array
 * inside the library, which every GPU that loads the library holds until the
 * process exits: up to 2^20 floats (4 MiB) of partial outputs
 * (splits x B x Hq x Sq x head_dim) and 2^15 floats (128 KiB) of per-row
 * statistics (2 x splits x B x Hq x Sq).
 *
 * Arguments: as attn_forward, with `p` in place of a context; p->precision must
 * be ATTN_EXACT; p->num_splits 0 (library's choice) or > 1 (forced); 1 is
 * rejected with ATTN_ERR_INVALID_ARG (this entry point always splits).  `err` is
 * an optional device word (4-byte aligned) into which a device-side wait that
 * runs out ORs 1; pass NULL to ignore such errors.  The array is shared by
 * every call: calls that overlap on the GPU (several streams, or several host
 * threads) race on it and must be serialised by the caller.  Every value the
 * kernels read from it is first written by the same call, so nothing needs
 * clearing between calls.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture.
 * Errors: ATTN_ERR_INVALID_ARG (bad field, num_splits 1, NULL or misaligned
 * pointer), ATTN_ERR_UNSUPPORTED (quantised mode, RoPE, head_dim, or partials larger than the
 * array; use attn_forward then), ATTN_ERR_CUDA (no sm_100 device, lookup,
 * tensor-map encode or launch failure). */
attn_status attn_forward_splitkv_noalloc(const attn_params *p, const void *q, const void *k,
                                         const void *v, void *o, float *lse, unsigned *err,
                                         void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
