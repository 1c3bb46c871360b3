/*
 * basiskv.h -- C ABI of the B200 (sm_100a) BasisKV decode-attention library.
 *
 * The operation: one decode step of attention over a compressed, paged KV
 * cache in the form of "BasisKV: Value Latents for Communication and Key
 * Routing" (English abstract):
 *   - Values are stored only as rank-r latents Z; a per-KV-head basis B_v
 *     expands a latent back to a value (V ~ Z.B_v).
 *   - Routing: the Value latents predict part of each key and a rank-s
 *     Key-specific residual R holds what they cannot, so the routing key is
 *     Khat = Z.W_zk + R.B_r.  A page's score is the largest q_h.Khat_t over
 *     the G query heads of the KV head's group and the page's valid tokens.
 *   - Selection: the k pages of largest score per (sequence, KV head); equal
 *     scores go to the lower page index.
 *   - Exact attention: the original keys K are read only for the selected
 *     pages; softmax(scale * q_h.K_t) over their valid tokens weights the
 *     latents, and the weighted latent is expanded by B_v.
 *
 * Layouts (row-major, element type = the pool dtype unless stated):
 *   z_pool [num_slots][Hkv][P][r]     value latents Z
 *   r_pool [num_slots][Hkv][P][s]     key residuals R (NULL when s = 0)
 *   k_pool [num_slots][Hkv][P][d]     original keys K, in the pool dtype or,
 *                                     with k_format = BASISKV_KEYS_INT8, as
 *                                     int8 codes with
 *   k_scale [num_slots][Hkv][P] fp32  one scale per token: K_t = k_scale_t *
 *                                     code_t (see basiskv_quantize_keys)
 *   w_zk   [Hkv][r][d]  fp32          latent-to-key basis
 *   b_r    [Hkv][s][d]  fp32          residual-to-key basis (NULL when s = 0)
 *   b_v    [Hkv][r][d]  fp32          latent-to-value basis
 *   q      [batch][Hkv*G][d]          query; head h of KV head kvh is kvh*G + h
 *   out    [batch][Hkv*G][d] fp32
 *   sel    [batch][Hkv][topk] int32   selected pages, ascending, -1 padded
 * A "slot" holds one page (P tokens) of every KV head.  Logical page j of
 * sequence b (tokens j*P .. j*P+P-1) lives in slot page_table[b][j].  Rows
 * past a sequence's length in its last page are never read into a result
 * (their contents are ignored, whatever they hold).
 *
 * Pointers are DEVICE pointers unless a comment says "host".  The library
 * never frees or writes caller memory other than the outputs named in each
 * call.  Every call returns BASISKV_OK (0) or a negative error code and, on
 * error, leaves a message for basiskv_last_error().  Calls taking a stream
 * enqueue on it and return without waiting unless the comment says otherwise.
 * A handle is not thread-safe: one host thread (or external locking) per
 * handle.
 */
#ifndef BASISKV_H
#define BASISKV_H

#include <stdint.h>

#if defined(__GNUC__)
#define BASISKV_API __attribute__((visibility("default")))
#else
#define BASISKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                          /* cudaStream_t is CUstream_st* */
typedef struct CUstream_st *basiskv_stream_t;

enum {
    BASISKV_OK = 0,
    BASISKV_ERR_INVALID_ARG = -1, /* bad argument, shape or alignment      */
    BASISKV_ERR_OOM = -2,         /* device allocation failed (create)      */
    BASISKV_ERR_CUDA = -3,        /* a CUDA runtime call failed             */
    BASISKV_ERR_UNSUPPORTED = -4, /* no sm_100 device, or unsupported shape */
    BASISKV_ERR_CAPACITY = -5,    /* page table row full                    */
    BASISKV_ERR_STATE = -6        /* e.g. appending a page after a partial  */
};

/* Device-side status bits (basiskv_get_status).  Kernels never trap: a
 * detected fault sets a bit and the kernel completes with garbage output for
 * the affected unit. */
enum {
    BASISKV_STATUS_BAD_SLOT = 1u,   /* a page-table entry outside [0, num_slots) */
    BASISKV_STATUS_TIMEOUT = 2u,    /* a bounded wait on a copy expired          */
    BASISKV_STATUS_BAD_PAGE = 4u,   /* a selected page outside [0, n_b)          */
    BASISKV_STATUS_PART_OVERFLOW = 8u, /* a unit met more split partials than its
                                          slots; that unit's output is invalid  */
    BASISKV_STATUS_BAD_LENGTH = 16u, /* a sequence length needing more pages than
                                       a page-table row holds (device lengths of
                                       basiskv_decode_attn_noalloc only): the
                                       sequence is cut to the row              */
    BASISKV_STATUS_DEBUG_BOUNDS = 32u /* debug build (BASISKV_DEBUG) only: an index
                                       the kernels keep in range by construction
                                       (ring stage, unit, KV head, pool row,
                                       score or selection entry) was not; the
                                       access went to index 0 instead          */
};

enum { BASISKV_DTYPE_BF16 = 0, BASISKV_DTYPE_F32 = 1 };

/* How the original keys are stored.  NATIVE: in the pool dtype.  INT8: int8
 * codes with an fp32 scale per token, the lossy key compression of "PackKV:
 * Reducing KV Cache Memory Footprint through LLM-Aware Lossy Compression"
 * (abstract) read as symmetric per-token int8; the attention kernels read
 * the codes and apply the scale to each token's dot product, so no
 * dequantised copy exists.  Halves the key bytes the exact-attention step
 * reads.  On the tensor-core path the query meets the codes in f16 (the
 * query is rounded to f16: exact for |q| in [2^-14, 65504]). */
enum { BASISKV_KEYS_NATIVE = 0, BASISKV_KEYS_INT8 = 1 };

/* Creation parameters.  Shapes: Hkv = num_kv_heads, G = gqa_group (1..8),
 * d = head_dim, P = page_size, r = rank_r (1..d), s = rank_s (0 allowed).
 * The fast bf16 path needs d % 32 == 0, P % 16 == 0, r % 8 == 0,
 * s % 8 == 0 and (G, d, r, s) among the compiled shapes; every other shape
 * runs the generic CUDA-core kernels (also the fp32 path); int8 keys on the
 * fast path also need d % 64 == 0.  All pools, bases and k_scale must be
 * 16-byte aligned; pool row strides follow from the shapes. */
typedef struct basiskv_params {
    int32_t max_batch;          /* sequences addressable by the page table   */
    int32_t num_kv_heads;
    int32_t gqa_group;
    int32_t head_dim;
    int32_t page_size;
    int32_t rank_r;
    int32_t rank_s;
    int32_t max_pages_per_seq;  /* page-table row length                     */
    int32_t max_topk;           /* largest topk a decode call may ask for    */
    int32_t num_slots;          /* pages the pools hold                      */
    int32_t dtype;              /* BASISKV_DTYPE_*                           */
    int32_t k_format;           /* BASISKV_KEYS_* (0: keys in the pool dtype) */
    const void *z_pool;         /* caller-owned; written only by encode_rows
                                   (k_pool also by quantize_keys)            */
    const void *r_pool;
    const void *k_pool;
    const float *w_zk;
    const float *b_r;
    const float *b_v;
    const float *k_scale;       /* [num_slots][Hkv][P] with BASISKV_KEYS_INT8,
                                   else NULL; caller-owned                   */
} basiskv_params;

typedef struct basiskv_handle basiskv_handle;

/* Validate *p and allocate the library-owned state on the current device:
 * the device page table [max_batch][max_pages_per_seq], sequence lengths, and
 * the decode workspace (page scores, selection, split partials, arrival
 * counters, status word).  Pools and bases stay caller-owned and must outlive
 * the handle.  Errors: INVALID_ARG (shape, null or misaligned pointer),
 * UNSUPPORTED (device is not compute capability 10.x), OOM, CUDA. */
BASISKV_API int basiskv_create(const basiskv_params *p, basiskv_handle **out);

/* Free the library-owned state (never the caller's pools).  Synchronises the
 * device first.  NULL is accepted. */
BASISKV_API int basiskv_destroy(basiskv_handle *h);

/* Append pool slot `slot`, holding n_tokens (1..P) valid tokens, as the next
 * logical page of sequence `seq`.  Only a sequence's last page may be
 * partial, so appending after a partial page is STATE.  Stream-ordered
 * (a one-thread kernel writes the entry); the host mirror used for launch
 * sizing is updated immediately.  Errors: INVALID_ARG, CAPACITY, STATE. */
BASISKV_API int basiskv_append_page(basiskv_handle *h, int seq, int slot, int n_tokens,
                        basiskv_stream_t stream);

/* basiskv_append_page that first copies the page's rows into the slot:
 * z [Hkv][n_tokens][r], r [Hkv][n_tokens][s] (NULL when s = 0) and
 * k [Hkv][n_tokens][d], in the pool dtype (k: int8 codes with int8 keys,
 * then also k_scale [Hkv][n_tokens] fp32; NULL otherwise), all device
 * memory, go to rows [0, n_tokens) of slot `slot`, every KV head (one
 * strided device-to-device copy per pool, on `stream`).  Nothing is copied
 * when the append would fail.  Errors: those of basiskv_append_page,
 * INVALID_ARG for a missing pointer, CUDA. */
BASISKV_API int basiskv_append_page_copy(basiskv_handle *h, int seq, int slot, int n_tokens, const void *z,
                             const void *r, const void *k, const float *k_scale,
                             basiskv_stream_t stream);

/* Grow the last (partial) page of `seq` by n_tokens; the new rows must
 * already be written in its slot.  Errors: INVALID_ARG, STATE (no page, or
 * the page would overflow P). */
BASISKV_API int basiskv_append_tokens(basiskv_handle *h, int seq, int n_tokens,
                          basiskv_stream_t stream);

/* Forget every page of `seq` (length 0).  Stream-ordered. */
BASISKV_API int basiskv_reset_seq(basiskv_handle *h, int seq, basiskv_stream_t stream);

/* Replace the page table of sequences [0, batch) from HOST arrays:
 * page_table [batch][ld] (entries past ceil(seq_lens[b]/P) ignored) and
 * seq_lens [batch].  Validates every entry, then copies and waits for the
 * copy (synchronous w.r.t. the host: a set-up call, not for the decode
 * loop).  Errors: INVALID_ARG, CAPACITY, CUDA. */
BASISKV_API int basiskv_load_page_table(basiskv_handle *h, int batch, const int32_t *page_table,
                            int ld, const int32_t *seq_lens, basiskv_stream_t stream);

/* One decode step for sequences [0, batch):
 *   q        [batch][Hkv*G][d] in the pool dtype (device)
 *   topk     pages kept per (sequence, KV head), 1..max_topk; when
 *            topk >= n_b every page of sequence b is used and its routing
 *            is skipped
 *   out      [batch][Hkv*G][d] fp32 (device)
 *   sel_out  [batch][Hkv][topk] int32 or NULL (device)
 * Enqueues the routing grid (page scores), the selection grid (top-k; on
 * the CUDA-core path the routing grid selects itself) and the attention
 * grid (exact QK on the selected pages, softmax, latent sum, merge of the
 * split partials and B_v) on `stream`, the later grids by programmatic
 * dependent launch; no allocation, no host synchronisation.  A sequence of
 * length 0 gets out = 0 and sel = -1.  Device-detected faults set status
 * bits.  Calls on one handle share its scratch: keep them in one stream
 * order (one stream, or events between streams).  A call is not meant for
 * CUDA-graph capture: its work plan and a per-call tag travel in the kernel
 * parameters, which a replayed graph would repeat unchanged.
 * Errors: INVALID_ARG. */
BASISKV_API int basiskv_decode_attn(basiskv_handle *h, int batch, const void *q, int topk,
                        float softmax_scale, float *out, int32_t *sel_out,
                        basiskv_stream_t stream);

/* The same step, returning the weighted latent instead of the value
 * ("BasisKV: Value Latents for Communication and Key Routing", English
 * abstract: values stay rank-r latents, and their compression is tied to
 * the output projection, so a caller may fold B_v into its own W_o and keep
 * the rank-r form until then):
 *   zbar_out [batch][Hkv*G][r] fp32 (device): zbar_h = sum_t p_t Z_t, the
 *            softmax-weighted latent of each query head (out = zbar . B_v)
 * Arguments, selection, errors and stream behaviour as basiskv_decode_attn;
 * a sequence of length 0 gets zbar = 0. */
BASISKV_API int basiskv_decode_attn_latent(basiskv_handle *h, int batch, const void *q, int topk,
                               float softmax_scale, float *zbar_out, int32_t *sel_out,
                               basiskv_stream_t stream);

/* The same step with HOST buffers: copies q_host (pinned or pageable) to a
 * library-owned device buffer, runs basiskv_decode_attn and waits for the
 * stream.  out_host (and sel_host when not NULL) are written by the kernels
 * through their device mapping when they are pinned, else copied back from
 * library-owned buffers. */
BASISKV_API int basiskv_decode_attn_host(basiskv_handle *h, int batch, const void *q_host, int topk,
                             float softmax_scale, float *out_host, int32_t *sel_host,
                             basiskv_stream_t stream);

/* Encode rows [row0, row0 + n_rows) of pool slot `slot`, every KV head,
 * from incoming keys and values k, v [Hkv][n_rows][d] (pool dtype, device)
 * ("BasisKV: Value Latents for Communication and Key Routing", English
 * abstract: values kept as rank-r latents, and a Key-specific residual
 * storing what the Value latent cannot predict; least-squares reading):
 *   K rows stored as given (int8 keys: quantised as basiskv_quantize_keys
 *   does, codes and scale);
 *   Z = V . pinv(B_v), rounded to the pool dtype;
 *   R = (K - Z . W_zk) . pinv(B_r), from the rounded Z, rounded.
 * With basiskv_encode_tokens and basiskv_quantize_keys, the only calls that
 * write the caller's pools
 * (and k_scale).  The first call computes
 * the pseudo-inverses of the bases on the host (synchronous); later calls
 * only enqueue on `stream`.  The page table is not touched: follow with
 * basiskv_append_page or basiskv_append_tokens.  Errors: INVALID_ARG (slot
 * or rows out of range, NULL k or v, bases with linearly dependent rows),
 * CUDA. */
BASISKV_API int basiskv_encode_rows(basiskv_handle *h, int slot, int row0, int n_rows, const void *k,
                        const void *v, basiskv_stream_t stream);

/* The same encode for a list of n tokens at arbitrary pool positions, in
 * one launch: the decode-time append of one new token per sequence.  Token
 * i, every KV head, goes to row rows[i] of pool slot slots[i] (slots, rows:
 * device int32 [n]); k, v [n][Hkv][d] (pool dtype, device: the layout of a
 * layer's new keys and values).  Entries outside the pool (slot not in
 * [0, num_slots) or row not in [0, P)) set BASISKV_STATUS_BAD_SLOT and are
 * skipped.  Arithmetic, rounding and the page table as basiskv_encode_rows.
 * Errors: INVALID_ARG (n < 0, NULL pointer; bases with linearly dependent
 * rows), CUDA. */
BASISKV_API int basiskv_encode_tokens(basiskv_handle *h, int n, const int32_t *slots, const int32_t *rows,
                          const void *k, const void *v, basiskv_stream_t stream);

/* Store keys into an int8 key pool (k_format = BASISKV_KEYS_INT8): rows
 * [row0, row0 + n_rows) of the pool in its flat row order, row =
 * (slot * Hkv + kvh) * P + token, from k [n_rows][d] (pool dtype, device,
 * 16-byte aligned).
 * Per row, in float32 with IEEE division ("PackKV: Reducing KV Cache Memory
 * Footprint through LLM-Aware Lossy Compression", abstract; symmetric
 * per-token int8 reading):
 *   k_scale[row] = max_c |k_c| / 127,  code_c = rint(k_c / k_scale[row])
 * (ties to even); a row of zeros gets scale 0 and codes 0.  Quantising a
 * whole native pool into an int8 one is one call with row0 = 0 and n_rows =
 * num_slots * Hkv * P.  Enqueued on `stream`.  Errors: INVALID_ARG (the
 * handle's keys are not int8, NULL or misaligned k, rows outside the
 * pool), CUDA. */
BASISKV_API int basiskv_quantize_keys(basiskv_handle *h, const void *k, int64_t row0, int64_t n_rows,
                          basiskv_stream_t stream);

/* Routing alone (steps route-prep, route-score, top-k) for every sequence
 * with at least one page, whether or not topk >= n_b.  scores_out
 * [batch][Hkv][max_pages_per_seq] fp32 (device, nullable) receives the page
 * scores (-inf past n_b); sel_out [batch][Hkv][topk] (device, nullable). */
BASISKV_API int basiskv_route(basiskv_handle *h, int batch, const void *q, int topk,
                  float *scores_out, int32_t *sel_out, basiskv_stream_t stream);

/* Read (and optionally clear) the device status bits.  Synchronises the
 * device.  Clearing a nonzero status also zeroes the handle's arrival
 * counters, which a call that gave up part way (a wait that ran out) can
 * leave behind, so the next call on the handle starts clean. */
BASISKV_API int basiskv_get_status(basiskv_handle *h, uint32_t *status, int clear);

/* Kernel timing: after basiskv_profile_begin(h, n), the next n decode calls
 * record CUDA events on their stream around each grid (the events keep the
 * grids from overlapping, so profiled calls run a little slower).
 * basiskv_profile_end waits for them and writes, per recorded call i,
 * ms[5*i + 0..4] = prep grid, routing grid, selection grid, attention grid,
 * whole call, in milliseconds (host array of >= 5*n floats, nullable), and
 * the number of recorded calls into *ncalls. */
BASISKV_API int basiskv_profile_begin(basiskv_handle *h, int max_calls);
BASISKV_API int basiskv_profile_end(basiskv_handle *h, float *ms, int *ncalls);

/* Launch shape chosen for the last decode call (for reports): routing pages
 * per CTA and CTA count, attention splits per unit and CTA count, whether
 * the tensor-core routing kernel ran (1) or the generic one (0), and which
 * attention kernel ran: 0 generic, 1 tensor-core with a copy ring per warp,
 * 2 tensor-core with one shared copy ring per CTA (units of 64 stages and
 * more). */
BASISKV_API int basiskv_last_launch(basiskv_handle *h, int info[6]);

/* Allocation-free decode step.  The BasisKV paper has no counterpart to
 * this call: it exists for callers that must not allocate device memory,
 * for instance code running under a framework that owns every device
 * allocation, or inside a region where cudaMalloc is not permitted (and so
 * cannot call basiskv_create).  It computes the same step as
 * basiskv_decode_attn, without a handle:
 *   p           pools, bases and shapes (host struct, as for basiskv_create);
 *               p->max_batch bounds batch, p->max_pages_per_seq is the row
 *               length of page_table, p->max_topk bounds topk
 *   page_table  [batch][p->max_pages_per_seq] int32 (device), seq_lens
 *               [batch] int32 (device); q, topk, softmax_scale, out, sel_out
 *               as for basiskv_decode_attn
 * The page table and lengths stay on the device, so they are checked there:
 * a length needing more than p->max_pages_per_seq pages is cut to the row
 * and sets BASISKV_STATUS_BAD_LENGTH; an entry outside [0, num_slots) reads
 * slot 0 and sets BASISKV_STATUS_BAD_SLOT.  Those bits are read with
 * basiskv_noalloc_status; nothing else reports them.
 * It allocates nothing.  Its scratch (page scores, selection, split
 * partials, arrival counters, status word) lives in one 16 MiB __device__
 * array inside the library, held by every GPU that loads the library until
 * the process exits.  A call needs, rounded up to 256-byte pieces,
 *   batch * Hkv * (8 + 4 * max_pages_per_seq + 4 * topk
 *                  + 4 * min(16, topk) * G * (r + 2))  bytes,
 * and one that would exceed 16 MiB is rejected with BASISKV_ERR_CAPACITY and
 * a message naming the size.  The first call on each device resolves the
 * array's device address (cudaGetSymbolAddress, with that device current);
 * make that first call before any stream capture.  Every call clears the
 * counters and status word it needs on `stream`, then reuses the same
 * array, which keeps the last call's contents: calls that may overlap on the
 * GPU (other streams, other host threads) race on it and must be serialised
 * by the caller.  It runs the CUDA-core kernels, not the persistent
 * tensor-core ones.  Errors: INVALID_ARG, CAPACITY, CUDA, UNSUPPORTED. */
BASISKV_API int basiskv_decode_attn_noalloc(const basiskv_params *p, int batch,
                                            const int32_t *page_table, const int32_t *seq_lens,
                                            const void *q, int topk, float softmax_scale,
                                            float *out, int32_t *sel_out, basiskv_stream_t stream);

/* Device status bits (BASISKV_STATUS_*) of the last basiskv_decode_attn_noalloc
 * call on the current device, read from the library's scratch array without
 * allocating.  Synchronises the device first.  The next call clears them.
 * Before any call on this device *status is 0.  Errors: INVALID_ARG (NULL
 * status), CUDA, UNSUPPORTED. */
BASISKV_API int basiskv_noalloc_status(uint32_t *status);

/* Thread-local message for the last non-zero return of this thread. */
BASISKV_API const char *basiskv_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch: BASISKV_VERSION
 * of the header the library was built with.  0.2.0 added int8 key pages
 * (k_format, k_scale in basiskv_params), basiskv_quantize_keys,
 * basiskv_encode_tokens and basiskv_append_page_copy. */
#define BASISKV_VERSION 200
BASISKV_API int basiskv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BASISKV_H */
