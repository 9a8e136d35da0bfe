/*
 * iskv.h -- C ABI of the B200 (sm_100a) iS-KV cache: basis-synchronized online
 * low-rank KV compression.
 *
 * Method source: "iS-KV -- Basis-synchronized online low-rank KV compression
 * -- What does it mean?" (learnaivisually.com explainer).  Per KV head the
 * newest W tokens stay exact; every 64-row block that leaves that window is
 * folded into a rank-r factorization (coefficients C, n x r; orthonormal basis
 * B, d x r; singular values S) by Brand's block-incremental SVD, and every old
 * coefficient row is rewritten in the new basis at the same update (Jargon:
 * Block-incremental SVD; the body paragraph on basis synchronization and
 * drift).  Keys are stored before RoPE and rotated when read (Jargon:
 * Pre-RoPE keys).  Decode attention reads the mixed cache directly, without
 * rebuilding values (ASKV design report, Design requirements: no
 * reconstruction on the decode path).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Return value: ISKV_OK (0) or a negative ISKV_ERR_* code.  Nothing throws
 *    across the ABI.  iskv_strerror() names a code.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Work is enqueued on it and the call returns without
 *    waiting, except iskv_status, iskv_get_counts, iskv_kv_bytes and
 *    iskv_destroy (host only or synchronizing).  Calls on
 *    one cache must be ordered on one stream (or ordered by the caller).
 *  - Caller buffers (k, v, q, out, ...): contiguous, row-major, owned by the
 *    caller and borrowed only for the stream-ordered duration of the call.
 *    They may be memory of the current device, host memory (pinned or
 *    pageable) or another GPU's memory; the kind is detected with
 *    cudaPointerGetAttributes.  In iskv_append and iskv_decode_attention,
 *    page-locked host buffers are read and written in place over PCIe by the
 *    library's kernels: k, v (16-byte aligned) by the append kernel, q
 *    (16-byte aligned) by a copy kernel into the cache's staging buffer, out
 *    (4-byte aligned) by the decode's own stores.  Every other non-device
 *    buffer, and device buffers off those boundaries, are staged through the
 *    cache's own device buffers with cudaMemcpyAsync on `stream`.  Either way
 *    the call does not wait: a host buffer must stay valid, and an output
 *    unread, until `stream` has passed the call.
 *  - Counters: T (tokens appended) and n_c (tokens folded, a multiple of 64)
 *    are kept per layer on the host and are shared by the whole batch; they
 *    advance when a call is enqueued, so they are exact integers at all times.
 *  - The cache owns all of its device memory, allocated once in iskv_create
 *    for `max_tokens`; no entry point allocates after that.
 */
#ifndef ISKV_H
#define ISKV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ISKV_API __attribute__((visibility("default")))
#else
#define ISKV_API
#endif

/* ---- status codes ------------------------------------------------------ */
#define ISKV_OK                 0
#define ISKV_ERR_INVALID_ARG   -1  /* bad pointer, shape, layer or config   */
#define ISKV_ERR_CAPACITY      -2  /* T would exceed max_tokens, or the exact
                                      window would overflow its ring        */
#define ISKV_ERR_STATE         -3  /* no ready block to fold, decode of an
                                      empty cache, postponed rewrites pending,
                                      or too many postponed folds           */
#define ISKV_ERR_CUDA          -4  /* a CUDA runtime call failed            */
#define ISKV_ERR_NOCONVERGE    -5  /* a core SVD hit its sweep limit (sticky;
                                      results are finite but less accurate) */
#define ISKV_ERR_NOMEM         -6  /* device allocation failed in create    */
#define ISKV_ERR_UNSUPPORTED   -7  /* shape outside the compiled kernels    */
#define ISKV_ERR_DEVICE_TIMEOUT -8 /* a bounded device-side wait gave up (sticky;
                                      the results of that call are incomplete;
                                      destroy the cache: its decode bookkeeping
                                      may be left inconsistent)             */
#define ISKV_ERR_RANGE         -9  /* a score of the tensor-core decode was not
                                      finite: a value its MMAs take as fp16
                                      went beyond fp16's range (|x| >=
                                      65504) -- a rotated key or a query in
                                      the rotation kernel (r_K g > 128), a
                                      query-basis product in the query-side
                                      RoPE kernel -- or an input was inf or
                                      NaN (sticky; that call's outputs are
                                      not finite)                           */

/* ---- element types ----------------------------------------------------- */
#define ISKV_F32   0
#define ISKV_BF16  1

/* ---- selectors and flags ----------------------------------------------- */
#define ISKV_WHICH_K 0
#define ISKV_WHICH_V 1
#define ISKV_ALL_LAYERS (-1)
/* iskv_compress_block flag: fold now, postpone the rewrite of the rows that
 * are already stored (step (e)) until iskv_sync.  Meant for prefill, where
 * nothing reads the cache between folds: the postponed rewrites are applied
 * in fold order by one pass over the stored rows.                          */
#define ISKV_FOLD_DEFER_SYNC 1

typedef struct iskv_cache* iskv_t;

/* Low-bit coefficient codes in latent channels: the SVDq page ("SVDq:
 * 1.25-bit and 410x Key Cache Compression for LLM Attention", Abstract) keeps
 * a key cache in SVD latent channels and gives the more significant channels
 * more bits; the iS-KV explainer (body paragraph on GQA and quantization)
 * calls iS-KV combined with low-bit storage untried.  Here column c of a
 * factor's coefficients C is latent channel c (columns are kept in
 * descending singular-value order), and each coefficient row is stored per
 * group of channels: group g covers `channels[g]` channels from the end of
 * the previous group, with `bits[g]` bits per code (0: the channels are
 * dropped and read as zero; 2, 4 or 8 otherwise).  Per row and group, in
 * fp32: scale = max |x| / (2^(b-1) - 1) (0 for an all-zero group), code =
 * x / scale rounded half to even into [-(2^(b-1) - 1), 2^(b-1) - 1], stored
 * as code + 2^(b-1) - 1 in b bits, packed from the lowest bit of 32-bit words
 * upward, each group starting a new word; the stored value is code * scale.
 * Channels per group are multiples of 16, their sum is the factor's rank.   */
typedef struct {
    int32_t groups;         /* 1..4 groups, from latent channel 0 on        */
    int32_t channels[4];    /* channels of each group (multiples of 16)     */
    int32_t bits[4];        /* bits per code: 0, 2, 4 or 8                  */
} iskv_quant_format;

/* Shape and format of one cache (a batch of equal-length sequences, every
 * layer of a model).  head_dim must be 128 and block 64 in this build.      */
typedef struct {
    int32_t batch;          /* sequences                                    */
    int32_t layers;         /* model layers held by this cache (<= 128)     */
    int32_t kv_heads;       /* KV heads per layer                           */
    int32_t q_heads;        /* query heads; a multiple of kv_heads (GQA)    */
    int32_t head_dim;       /* d = 128                                      */
    int32_t rank_k;         /* r_K: multiple of 16, 16 <= r_K <= d          */
    int32_t rank_v;         /* r_V: multiple of 16, 16 <= r_V <= d          */
    int32_t window;         /* W: exact recent tokens, multiple of 64       */
    int32_t block;          /* rows folded at once: 64                      */
    int32_t max_tokens;     /* capacity of T per layer                      */
    int32_t kv_dtype;       /* ISKV_F32 or ISKV_BF16: k, v and q elements    */
    int32_t coef_dtype;     /* ISKV_F32 or ISKV_BF16: stored coefficients C  */
    int32_t use_rope;       /* 1: keys are rotated by RoPE when read         */
    double  rope_theta;     /* RoPE base (1e6 for Qwen3-shaped caches)       */
    int32_t sync;           /* 1: rewrite old rows at every fold (the method);
                               0: no-synchronization ablation               */
    int32_t max_deferred;   /* folds whose rewrite may be postponed before an
                               iskv_sync is required (0: no postponing)     */
    int32_t jacobi_max_sweeps; /* sweep limit of the core SVD (0: 40)        */
    int32_t ring_extra;     /* exact-window ring rows beyond W + 64 (0: 64)  */
    int32_t protect;        /* P: leading positions (the prompt's protected
                               rows) kept exact and never folded (0: none).
                               Positions 0..P-1 stay exact, P..P+n_c-1 are
                               folded rows, P+n_c..T-1 the exact window.
                               The iS-KV explainer ("What does it mean?",
                               the paint-shop section) leaves some prompt
                               positions uncompressed, besides the recent
                               window.                                      */
    int32_t coef_quant;     /* 1: coefficients stored as low-bit latent-channel
                               codes (quant_k, quant_v) instead of coef_dtype;
                               every new row and every rewrite is coded again,
                               and decode reads the codes (CUDA-core path)   */
    iskv_quant_format quant_k;  /* code groups of the K factor (ranks sum to r_K) */
    iskv_quant_format quant_v;  /* code groups of the V factor (ranks sum to r_V) */
    int32_t joint;          /* 1: one K and one V factor per sequence and layer
                               over all its KV heads, whose rows sit side by
                               side (D = kv_heads * 128 <= 1024; the reading
                               of the explainer's worked-example ranks 64, 96
                               and 128 as layer-wide ranks); coefficients are
                               then shared by the heads and each head decodes
                               with its 128 rows of the basis.  0: one factor
                               per KV head.                                 */
} iskv_config;

/* Fill `cfg` with the defaults of the one-layer Qwen3-8B-shaped cache
 * (8 KV / 32 query heads, d 128, r_K 32, r_V 64, W 1024, bf16 K/V, fp32 C,
 * RoPE theta 1e6).  Returns ISKV_OK, or ISKV_ERR_INVALID_ARG for NULL.     */
ISKV_API int iskv_config_default(iskv_config* cfg);

/* Create a cache: validates `cfg`, allocates every device buffer for
 * max_tokens on `stream`, sets B = I_d[:, :r], S = 0, T = n_c = 0 (the
 * explainer's empty factorization before the first block, Jargon:
 * Block-incremental SVD).  On success *out owns the cache; on failure *out
 * is NULL and nothing leaks.                                               */
ISKV_API int iskv_create(const iskv_config* cfg, void* stream, iskv_t* out);

/* Synchronize the cache's streams, free everything.  NULL is a no-op.      */
ISKV_API int iskv_destroy(iskv_t h);

/* Append t tokens to every sequence of `layer`: k, v are
 * [batch, kv_heads, t, head_dim] in kv_dtype, PRE-RoPE (explainer, Jargon:
 * Pre-RoPE keys; the newest W tokens stay exact).  T += t.  Never folds.
 * *ready_blocks (may be NULL) receives floor((T - P - n_c - W) / 64), at
 * least 0 (P = protected positions): the whole blocks that have left the
 * exact window and may be folded.  Positions below P go to the protected
 * rows.  Errors: CAPACITY if T + t > max_tokens or the ring would hold more
 * than W + 64 + ring_extra rows (fold first).                              */
ISKV_API int iskv_append(iskv_t h, int layer, const void* k, const void* v, int t,
                void* stream, int* ready_blocks);

/* Fold the oldest ready block of `layer` (or of every layer that has one,
 * for ISKV_ALL_LAYERS), K and V factors of every (sequence, KV head) -- the
 * explainer's block update (Jargon: Block-incremental SVD; steps as in
 * Brand's update): (a) P = X B; (b) residual and Householder QR of the complement;
 * (c) one-sided Jacobi SVD of the (r+64) x (r+k) core, truncated to r;
 * (d) B' = [B, Q] W_r, S' and the block's coefficient rows; (e) unless
 * ISKV_FOLD_DEFER_SYNC is set, every old row is rewritten, C <- C W_r[0:r,:].
 * n_c += 64.  Errors: STATE if the layer has no ready block (for
 * ISKV_ALL_LAYERS: if no layer has one) or if a deferred fold would exceed
 * max_deferred.                                                           */
ISKV_API int iskv_compress_block(iskv_t h, int layer, int flags, void* stream);

/* The same block update (fold and, unless postponed, rewrite) enqueued on a
 * second stream, `stream`, so that it runs while the caller's stream `after`
 * keeps decoding other layers.  It starts after everything enqueued so far on
 * `after` (the appended rows); the next call that touches a folded layer, on
 * whatever stream, is ordered after the update -- the swap to the updated
 * factors happens at that call, and until the update completes nothing reads
 * the layer.  Host counters (T, n_c) advance at once, as for
 * iskv_compress_block.  All other calls on the cache stay on one stream.
 * This answers the ASKV design report (Design requirements, the item on
 * maintenance and the critical path): decoding should not have to wait for
 * compression work.  With one layer updated per call, its fold and rewrite
 * overlap the other layers' decode.
 * Errors: as iskv_compress_block, plus CUDA for event failures.            */
ISKV_API int iskv_compress_block_async(iskv_t h, int layer, int flags, void* stream,
                                       void* after);

/* Apply the postponed rewrites of `layer` (or ISKV_ALL_LAYERS) in fold order:
 * one pass over the stored rows, each row multiplied by the product of the
 * W_r[0:r,:] of the folds that came after it was written -- the explainer's
 * basis synchronization (body paragraph on drift: old coefficients follow
 * every basis update), applied late but in the same order.  No-op if
 * nothing is pending.                                                      */
ISKV_API int iskv_sync(iskv_t h, int layer, void* stream);

/* Decode attention of `layer` over the mixed cache (explainer, Jargon:
 * Pre-RoPE keys -- folded keys rotated at their positions when read; ASKV
 * design report, Design requirements -- values never rebuilt): q is
 * [batch, q_heads, head_dim] in kv_dtype, already rotated for position T - 1;
 * out is [batch, q_heads, head_dim] fp32.  Query head j reads KV head j / (q_heads / kv_heads).  Scores over
 * all T tokens (folded rows rebuilt as C_K B_K^T and rotated at their absolute
 * positions, exact rows rotated likewise), scale 1/sqrt(d), one softmax; the
 * value side is (p^T C_V) B_V^T + p_win^T V_win.  Errors: STATE if T = 0 or
 * rewrites are pending.                                                    */
ISKV_API int iskv_decode_attention(iskv_t h, int layer, const void* q, float* out,
                          void* stream);

/* Rebuild the folded rows of one factor before RoPE (explainer, Jargon:
 * Block-incremental SVD: the stored form is C B^T): out is
 * [batch, kv_heads, n_c, head_dim] fp32 = C B^T.  `which` is ISKV_WHICH_K or
 * ISKV_WHICH_V.  With n_c = 0 nothing is written and `out` may be NULL.
 * Errors: STATE if rewrites are pending.                                   */
ISKV_API int iskv_reconstruct(iskv_t h, int layer, int which, float* out, void* stream);

/* Copy out one factor: basis [batch, kv_heads, head_dim, r] fp32 (row i of a
 * head is basis row i), sigma [batch, kv_heads, r] fp32, coef
 * [batch, kv_heads, n_c, r] row-major in coef_dtype (fp32 values code * scale
 * for a coef_quant cache).  Any pointer may be NULL.                       */
ISKV_API int iskv_get_factors(iskv_t h, int layer, int which, float* basis, float* sigma,
                     void* coef, void* stream);

/* Host counters of `layer`: tokens appended and tokens folded.             */
ISKV_API int iskv_get_counts(iskv_t h, int layer, int64_t* T, int64_t* n_c);

/* Persistent-KV bytes (the iS-KV explainer, Jargon: Persistent-KV
 * compression): what the cache keeps between decode steps for every layer,
 * sequence and KV head at the current T and n_c -- coefficient rows
 * (n_c x (r_K + r_V) in coef_dtype), bases and singular values (fp32,
 * (d + 1)(r_K + r_V)), exact window and protected rows (K and V in kv_dtype)
 * -- and the bytes of the uncompressed K/V cache of the same T in kv_dtype.
 * Neither counts preallocated capacity, the exact-window ring's spare rows
 * or temporary buffers.  Either pointer may be NULL.  Host only, no GPU work.
 * Errors: INVALID_ARG for a NULL cache.                                    */
ISKV_API int iskv_kv_bytes(iskv_t h, int64_t* persistent_bytes, int64_t* full_bytes);

/* The kernel the next iskv_decode_attention of `layer` runs, given the
 * configuration, the environment read at creation and the layer's current
 * n_c: ISKV_DECODE_CUDA_CORE (split fp32 CUDA-core kernel plus combine: fp32
 * coefficients or K/V, or tensor cores switched off with
 * ISKV_TENSOR_CORES=0), ISKV_DECODE_ROTATE (tensor cores; folded keys
 * rebuilt, rotated and scored per tile), ISKV_DECODE_QUERY_ROPE (tensor
 * cores; RoPE folded into the queries, scores from a position table times
 * per-head query-basis products; only where r_K * g <= 128).  Between the
 * two tensor-core kernels the default takes the query-side one when the
 * call's folded 128-row tiles number at least 200 per SM;
 * ISKV_DECODE_KERNEL=u or =rot fixes the choice.  Host only.
 * Errors: INVALID_ARG (NULL pointers, layer out of range).                */
#define ISKV_DECODE_CUDA_CORE  0
#define ISKV_DECODE_ROTATE     1
#define ISKV_DECODE_QUERY_ROPE 2
ISKV_API int iskv_decode_kernel(iskv_t h, int layer, int* kernel);

/* Code `n` fp32 rows of `rank` coefficients with the latent-channel format
 * `fmt` (see iskv_quant_format): rows [n][rank] fp32, codes [n][words]
 * uint32 (words = iskv_quant_words(fmt)), scales [n][4] fp32 (unused groups
 * 0).  Device pointers; enqueued on `stream`.  The same device routine codes
 * a cache's new rows and rewrites, so callers can prepare or check codes
 * outside a cache.  Errors: INVALID_ARG (format, rank or pointers), CUDA.   */
ISKV_API int iskv_quantize_rows(const iskv_quant_format* fmt, int rank, const float* rows,
                                int64_t n, uint32_t* codes, float* scales, void* stream);

/* 32-bit code words per row of a format (host only); -1 if invalid.        */
ISKV_API int iskv_quant_words(const iskv_quant_format* fmt);

/* Synchronize the device and return the cache's sticky device status, the
 * most severe first: ISKV_ERR_CUDA, ISKV_ERR_DEVICE_TIMEOUT, ISKV_ERR_RANGE,
 * ISKV_ERR_NOCONVERGE, else ISKV_OK.  Clears nothing.                      */
ISKV_API int iskv_status(iskv_t h);

/* Static string naming a status code.                                     */
ISKV_API const char* iskv_strerror(int code);

/* ---- decode attention without any device allocation --------------------
 * The method's pages have no counterpart to this entry point: it is a
 * packaging of the decode above for callers that cannot call cudaMalloc,
 * such as a serving engine that owns and plans all of its device memory
 * (and forbids allocations after start-up), or a latency-critical path that
 * must avoid cudaMalloc's device-wide synchronization.  Such a caller keeps
 * the factors in its own buffers, row-major as iskv_get_factors returns
 * them (not the cache's internal 8 x 8 blocked bf16 layout), and passes them
 * here; nothing is allocated and nothing is staged.  The
 * operands describe a cache without protected rows (iskv_config.protect 0);
 * caches with protected rows decode through iskv_decode_attention.
 *
 * All pointers are device memory of the current device (or managed
 * memory), owned by the caller, borrowed for the stream-ordered duration of
 * the call:
 *   coef_k, coef_v  [batch*kv_heads][coef_rows][r] in coef_dtype (rows 0..n_c-1
 *                   are read);
 *   basis_k, basis_v [batch*kv_heads][head_dim][r] fp32;
 *   ring_k, ring_v  [batch*kv_heads][ring_rows][head_dim] in kv_dtype, pre-RoPE;
 *                   exact row j (n_c <= j < T) sits at slot j % ring_rows;
 *   rope            [T][head_dim/2] (cos, sin) float pairs of j * theta^(-2i/d),
 *                   or NULL for no RoPE;
 *   q [batch][q_heads][head_dim] kv_dtype, out [batch][q_heads][head_dim] fp32.
 * The split-K partial results live in a library-owned device array of 4 MiB
 * (2^20 floats), present on every GPU that loads the library until the
 * process exits; a call needs batch * q_heads * (2 + rank_v + head_dim)
 * floats per split and is rejected with ISKV_ERR_CAPACITY when even one split
 * does not fit.  The first call on a device looks up that array's device
 * address (cudaGetSymbolAddress) and keeps it; make that first call before
 * any stream capture, and do not use this entry point across a
 * cudaDeviceReset (the array may move).  Calls share the array: calls that
 * overlap on the GPU race and must be serialized by the caller.
 * Errors: INVALID_ARG (null or host pointer, memory of another device,
 * inconsistent sizes), UNSUPPORTED (shape), CAPACITY, CUDA.                */
typedef struct {
    int32_t batch, kv_heads, q_heads, head_dim, rank_k, rank_v;
    int32_t kv_dtype, coef_dtype;
    int64_t T;            /* tokens, >= 1                                   */
    int64_t n_c;          /* folded rows, a multiple of 64, <= T            */
    int64_t coef_rows;    /* row capacity per head of coef_k / coef_v       */
    int64_t ring_rows;    /* row capacity per head of ring_k / ring_v       */
    const void* coef_k;
    const float* basis_k;
    const void* coef_v;
    const float* basis_v;
    const void* ring_k;
    const void* ring_v;
    const float* rope;
} iskv_decode_operands;

ISKV_API int iskv_decode_attention_noalloc(const iskv_decode_operands* ops, const void* q,
                                           float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ISKV_H */
