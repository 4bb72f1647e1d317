/*
 * lsa.h -- C ABI of the Lookahead Sparse Attention (LSA) decode hot path on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via
 * Lookahead Sparse Attention", gist.science technical summary, section 2.1):
 *   - Periodic Triggering: every tau decode steps (tau = 64) the memory
 *     indexer is evaluated on the current hidden state;
 *   - Scoring Mechanism: a lookahead index score I_{t,s} between the current
 *     indexer queries and every preceding compressed entry s, a head-fused
 *     gated matching score through a sigmoid, fixed here as
 *         I_{t,s} = sigmoid( sum_j w_{t,j} * ReLU(q_{t,j} . k_s) );
 *   - Dynamic Fetching: every entry with I_{t,s} >= 0.5 is fetched from the
 *     CPU cold pool into GPU memory (no rigid top-k at this stage);
 *   - Tiered Selection: a fine-grained top-k inside that fetched subset feeds
 *     the final core attention.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless its comment says host.
 *     The caller owns every buffer; no entry point allocates or frees memory,
 *     except lsa_ctx_create / lsa_ctx_destroy, which own the context's
 *     internal buffers.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).  No entry point synchronises
 *     the host, except where its comment says so.
 *   - Argument validation happens on the host before anything is enqueued.  A
 *     failed validation returns LSA_ERR_INVALID or LSA_ERR_UNSUPPORTED,
 *     launches nothing and sets the message returned by lsa_last_error().
 *   - Conditions only the device can see (kept entries beyond a buffer's
 *     capacity, a bounded wait that gave up) are written to the caller's
 *     device word `err` (int32, first error wins: LSA_ERR_CAPACITY or
 *     LSA_ERR_TIMEOUT).  The caller zeroes it and reads it after the stream
 *     has completed.  `err` may be NULL where the comment allows it.
 *   - Ragged batches use CSR offsets: sequence b owns entries
 *     [seq_off[b], seq_off[b+1]) of a flat entry axis of n_total entries.
 *     Entry indices in kept and top-k lists are local to their sequence.
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lsa_status {
    LSA_OK = 0,
    LSA_ERR_INVALID = 1,      /* bad argument: nothing was launched */
    LSA_ERR_CUDA = 2,         /* a CUDA runtime call failed */
    LSA_ERR_CAPACITY = 3,     /* more kept entries than the output can hold */
    LSA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up */
    LSA_ERR_UNSUPPORTED = 5   /* valid, but not a shape/dtype this library runs */
} lsa_status;

typedef enum lsa_dtype {
    LSA_F32 = 0,   /* IEEE binary32 */
    LSA_BF16 = 1,  /* bfloat16 */
    LSA_E4M3 = 2   /* OCP FP8 E4M3 ("fn"): bias 7, no infinities, max 448 */
} lsa_dtype;

/* Library version, major*10000 + minor*100 + patch. */
/* sizeof(lsa_params) for which = 0, sizeof(lsa_ctx_view) for 1, else -1: lets a
 * binding that mirrors the structs check its layout.  Needs no GPU. */
int64_t lsa_struct_size(int32_t which);
int32_t lsa_version(void);

/* Message of the last failing call on this host thread ("" if none). */
const char *lsa_last_error(void);

/* Static name of a status code. */
const char *lsa_status_name(lsa_status s);

/* Name of the last kernel this host thread launched through the library ("" if
 * none), e.g. "scan_tc e4m3 d64" for the tensor-core index scan of e4m3 keys
 * with d = 64: lets a caller or a test see which implementation ran.  A static
 * string; it needs no GPU to call. */
const char *lsa_last_kernel(void);

/* ------------------------------------------------------------------------
 * lsa_index_score -- the lookahead index score (section 2.1, "Scoring
 * Mechanism"; the interaction is a plain dot product, section 5).
 *
 *   z_s = sum_{j<H} w[b,j] * max(0, q[b,j,:] . k[s,:])     I_s = 1/(1+exp(-z_s))
 *
 * q        [B, H, d]   q_dtype LSA_F32 or LSA_BF16, row-major.
 * w        [B, H]      fp32 gate weights (may be negative).
 * k        [n_total, d] indexer keys K^{IComp}, row-major; k_dtype LSA_F32,
 *                      LSA_BF16 or LSA_E4M3.  Rows start 16-byte aligned
 *                      (d * element size is a multiple of 16).
 * k_scale  [n_total]   fp32, one positive scale per row, required for E4M3
 *                      keys (value = code * scale; rows of d <= 128), else NULL.
 * seq_off  [B+1]       int64 CSR offsets; seq_off[B] == n_total (host value).
 * Listed mode (idx != NULL): only entries idx[idx_off[b] .. idx_off[b+1])
 *   of each sequence (indices local to the sequence) are scored, and z / I
 *   are written at the list position.  idx_off [B+1] int64 on the device;
 *   list_capacity (host) bounds idx_off[B].
 * Full mode (idx == NULL): z / I are written for every entry, [n_total].
 * z        fp32 output (required).   I  fp32 output or NULL.
 * flags    0, or LSA_SCORE_CUDA_CORE.  Scans (full or listed) of bf16 q (16-byte
 *          aligned) over bf16 or e4m3 keys with d in {64, 128} and H in
 *          {16, 32, 64}, B <= 512 and n_total >= 128 (bf16) or >= 256 (e4m3)
 *          run on the tensor cores (tcgen05); every other case, and every call
 *          with LSA_SCORE_CUDA_CORE, runs the CUDA-core kernel
 *          (lsa_last_kernel names the one that ran).
 * err      device error word or NULL (LSA_ERR_TIMEOUT if a bounded wait of the
 *          tensor-core kernel gave up).
 * Shapes run: 1 <= H <= 64, d in {32, 64, 128} (d * element size % 16 == 0).
 * ---------------------------------------------------------------------- */
enum { LSA_SCORE_CUDA_CORE = 1 };
lsa_status lsa_index_score(const void *q, lsa_dtype q_dtype, const float *w,
                           const void *k, lsa_dtype k_dtype, const float *k_scale,
                           const int64_t *seq_off, int64_t n_total,
                           const int32_t *idx, const int64_t *idx_off, int64_t list_capacity,
                           int32_t B, int32_t H, int32_t d,
                           float *z, float *I, int32_t flags, int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * lsa_select -- threshold selection (section 2.1, "Dynamic Fetching"):
 * keep every entry with I >= 0.5.  The decision is taken as z >= 0, which
 * is the same set in exact arithmetic (sigmoid is increasing, sigmoid(0) =
 * 1/2) and cannot be moved by rounding of the sigmoid; -0.0 is kept, NaN is
 * not.
 *
 * z         [n_total] fp32 scores (full mode of lsa_index_score).
 * kept_idx  [capacity] int32 output: kept entries of each sequence, local
 *           indices in ascending order, sequence after sequence.
 * kept_off  [B+1] int64 output: CSR offsets into kept_idx.  kept_off[B] is the
 *           true total even when it exceeds capacity; then only the first
 *           `capacity` indices are written and *err = LSA_ERR_CAPACITY.
 * mask      [ceil(n_total/32)] uint32 output or NULL: bit (s % 32) of word
 *           s / 32 is set iff entry s (flat axis) is kept.
 * workspace device scratch of at least lsa_select_workspace_size(n_total)
 *           bytes, 16-byte aligned; contents need not be initialised.
 * ---------------------------------------------------------------------- */
size_t lsa_select_workspace_size(int64_t n_total);
lsa_status lsa_select(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B,
                      int32_t *kept_idx, int64_t capacity, int64_t *kept_off, uint32_t *mask,
                      void *workspace, size_t ws_bytes, int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * lsa_index_score_select -- the full index scan and the threshold selection in
 * one call (section 2.1, "Scoring Mechanism" then "Dynamic Fetching"): the
 * z of lsa_index_score in full mode (every entry) and the kept lists of
 * lsa_select, bit for bit (same z, same decision z >= 0, same order).
 *
 * On the tensor-core path (the shapes lsa_index_score runs on tcgen05) the
 * selection is fused into the scan: its epilogue takes the z >= 0 ballots of
 * the rows it has just scored, so z is written once and not read again; two
 * short kernels then place the kept entries.  Any other shape runs the
 * CUDA-core scan and lsa_select's kernels.
 *
 * Arguments as lsa_index_score (full mode: no list, no I output, no flags) and
 * lsa_select (kept_idx, capacity, kept_off: kept_off[B] is the true total even
 * when it exceeds capacity, then *err = LSA_ERR_CAPACITY; no mask output).
 * workspace device scratch of at least
 *           lsa_index_score_select_workspace_size(n_total, B) bytes, 16-byte
 *           aligned; contents need not be initialised.
 * ---------------------------------------------------------------------- */
size_t lsa_index_score_select_workspace_size(int64_t n_total, int32_t B);
lsa_status lsa_index_score_select(const void *q, lsa_dtype q_dtype, const float *w,
                                  const void *k, lsa_dtype k_dtype, const float *k_scale,
                                  const int64_t *seq_off, int64_t n_total, int32_t B, int32_t H,
                                  int32_t d, float *z, int32_t *kept_idx, int64_t capacity,
                                  int64_t *kept_off, void *workspace, size_t ws_bytes,
                                  int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * lsa_select_noalloc -- lsa_select without a caller workspace.  The pages
 * have no counterpart: this is a calling convention for callers that cannot
 * allocate device memory when they select (a stream capture that forbids
 * allocation, a runtime whose pool owns all device memory, a plugin host that
 * passes no workspace).  Same arguments and results as lsa_select, minus the
 * workspace; the scratch is a static device array of the library (560 KB on
 * every GPU that loads it, held until the process exits), so n_total is
 * limited to lsa_select_noalloc_max_entries() (4,194,304); larger n_total is
 * rejected with LSA_ERR_INVALID before anything is launched.  The first call
 * on a device is its set-up: it looks the array's device address up
 * (cudaGetSymbolAddress, cached per device and CUDA context) and, with lazy
 * module loading (the CUDA 12 default), loads the library's device code, which
 * creates the array in device memory.  Make that first call early: before any
 * stream capture and before a runtime claims the rest of the device's memory.
 * After it, no call allocates or frees memory (no cudaMalloc, no cudaFree).
 * All calls on a device share the array: calls that overlap on the GPU race.
 * ---------------------------------------------------------------------- */
int64_t lsa_select_noalloc_max_entries(void);
lsa_status lsa_select_noalloc(const float *z, const int64_t *seq_off, int64_t n_total, int32_t B,
                              int32_t *kept_idx, int64_t capacity, int64_t *kept_off, uint32_t *mask,
                              int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * lsa_index_union -- OR-mode union of several indexer layers (section 2.4,
 * "Optimal Configuration": independent Memory Indexers on three layers whose
 * predictions are united at inference to decide what is fetched).  Layer l
 * keeps entry s when z_l[s] >= 0 (I >= 0.5); the union keeps s when any layer
 * does, i.e. when max_l z_l[s] >= 0.  Writes z_union[s] = max_l z_l[s] (exact;
 * a NaN counts as "not kept" by its layer), so lsa_select on z_union gives the
 * union's kept set, and z_union is the union's ranking score for lsa_topk.
 *
 * z_layers   HOST array of n_layers DEVICE pointers, each to n_total fp32
 *            scores on one entry axis (the layers share seq_off)
 * n_layers   1 .. 8
 * n_total    entries (0: nothing is launched)
 * z_union    device fp32 [n_total]; may alias one of the layers' arrays
 * stream     cudaStream_t or NULL
 * Errors: LSA_ERR_INVALID for a null pointer or n_layers outside [1, 8].
 * ---------------------------------------------------------------------- */
lsa_status lsa_index_union(const float *const *z_layers, int32_t n_layers, int64_t n_total, float *z_union,
                           void *stream);

/* ------------------------------------------------------------------------
 * lsa_query_encode -- the indexer's query encoder (section 2.1 "Memory
 * Indexer": the current query token's hidden state h_t is mapped to low-rank
 * indexer queries; section 2.3 "Query Optimization": the encoder's trained
 * part is its low-rank projection matrices).  Read as a rank-r factorisation
 * with the head weights taken from h_t directly, and no norm, activation or
 * positional term (the pages name none):
 *     c = W_dq h,   q_j = rows j*d .. j*d+d-1 of W_uq c,   w = W_w h.
 * Its outputs are lsa_index_score's q and w.
 *
 * h       device bf16 [B, hidden] hidden states
 * W_dq    device bf16 [rank, hidden] down-projection, row-major [out, in]
 * W_uq    device bf16 [H*d, rank] up-projection (rows of head j: j*d .. j*d+d-1)
 * W_w     device bf16 [H, hidden] head-weight projection
 * q_out   device [B, H, d] in q_dtype (BF16: rounded to nearest even from the
 *         fp32 sum; F32)
 * w_out   device fp32 [B, H]
 * c_out   device fp32 [B, rank]: the latent, written by the first pass and
 *         read by the second (the caller's buffer; nothing is allocated)
 * Every sum is an fp32 accumulation of exact bf16 x bf16 (or bf16 x fp32)
 * products; the summation order is fixed, so results are deterministic.
 * Layout rules: hidden and rank multiples of 8 (>= 8); h, the three weight
 * matrices and c_out 16-byte aligned.  Two kernel launches on `stream`.
 * Errors: LSA_ERR_INVALID for a null pointer, a size or an alignment outside
 * these rules; LSA_ERR_UNSUPPORTED for a q_dtype other than BF16 / F32.
 * ---------------------------------------------------------------------- */
lsa_status lsa_query_encode(const void *h, int32_t B, int32_t hidden, const void *W_dq, int32_t rank,
                            const void *W_uq, int32_t H, int32_t d, const void *W_w, void *q_out,
                            lsa_dtype q_dtype, float *w_out, float *c_out, void *stream);

/* ------------------------------------------------------------------------
 * lsa_attn_set_merge -- the merged attention set (section 2.1 "Architectural
 * Design": every Heavily Compressed Attention chunk, 128:1, stays resident for
 * global awareness; section 1 "Problem Statement": the most recent 8K tokens
 * alone answer most long requests).  Per sequence b the core attention runs
 * over the set union of its top-k entries, its last `window` entries and its
 * HCA rows, each row once (a top-k entry inside the window is attended through
 * the window's row).  Writes, per sequence, the row list for lsa_sparse_attn
 * over one KV arena: the top-k slots of entries below the window (ascending
 * entry order), then rows hca_base + hca_off[b] .. hca_base + hca_off[b+1]-1,
 * then rows win_base + b*window + t for t < min(window, N_b) (row t holding
 * entry N_b - min(window, N_b) + t), then -1 up to row_cap.
 *
 * topk_idx, topk_pos, topk_cnt   device, as written by lsa_topk ([B, k], [B, k], [B])
 * seq_off    device int64 [B+1]
 * hca_off    device int64 [B+1] offsets of each sequence's HCA rows, or NULL (none)
 * rows       device int32 [B, row_cap]; count device int32 [B] (rows used) or NULL
 * err        device error word or NULL: LSA_ERR_CAPACITY when a sequence needs more than
 *            row_cap rows (its list is cut at row_cap)
 * One launch (a CTA per sequence) on `stream`.  Row indices are int32: the
 * caller keeps hca_base + hca_off[B] and win_base + B*window below 2^31.
 * Errors: LSA_ERR_INVALID for a null pointer or a negative size.
 * ---------------------------------------------------------------------- */
lsa_status lsa_attn_set_merge(const int32_t *topk_idx, const int32_t *topk_pos, const int32_t *topk_cnt,
                              const int64_t *seq_off, int32_t B, int32_t k, int32_t window, int32_t win_base,
                              const int64_t *hca_off, int32_t hca_base, int32_t *rows, int32_t row_cap,
                              int32_t *count, int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * lsa_topk -- fine-grained top-k inside the kept set (section 2.1, "Tiered
 * Selection").  Per sequence, the k kept entries with the largest z (the
 * sigmoid is monotone, so ranking by z ranks by I); equal z goes to the lower
 * entry index (-0.0 and +0.0 are equal).  The chosen set is written in
 * ascending entry order; if a sequence keeps fewer than k entries, all of
 * them are written and the rest of its row is -1.
 *
 * z            scores.  z_by_entry != 0: z is indexed on the flat entry axis,
 *              z[seq_off[b] + kept_idx[p]] (scores of a full scan; seq_off
 *              required).  z_by_entry == 0: z[p] is the score of kept
 *              position p (a listed scan over the kept set).
 * kept_idx, kept_off  the kept set, as produced by lsa_select.
 * kept_capacity  number of valid kept_idx entries (the capacity given to
 *              lsa_select); kept positions at or past it are ignored.
 * topk_idx     [B, k] int32 output: local entry indices, ascending, -1 padded.
 * topk_pos     [B, k] int32 output or NULL: the kept-list position p of each
 *              chosen entry (= its hot-buffer row after lsa_gather), -1 padded.
 * topk_cnt     [B] int32 output: min(k, kept count).
 * Shapes run: 1 <= k <= 4096.  A sequence may keep any number of entries.
 * ---------------------------------------------------------------------- */
lsa_status lsa_topk(const float *z, int32_t z_by_entry, const int64_t *seq_off,
                    const int32_t *kept_idx, const int64_t *kept_off, int64_t kept_capacity,
                    int32_t B, int32_t k, int32_t *topk_idx, int32_t *topk_pos,
                    int32_t *topk_cnt, void *stream);

/* ------------------------------------------------------------------------
 * lsa_gather -- cold-pool fetch (section 2.1, "Dynamic Fetching": kept
 * entries are fetched from the CPU "Cold Pool" into GPU memory; blog page:
 * "just in time").  Copies the cold row of every kept entry into the HBM hot
 * buffer, in kept order: hot row kept_off[b] + i receives cold row
 * seq_off[b] + kept_idx[kept_off[b] + i].
 *
 * cold_host   HOST pointer to the cold pool [n_total, row_bytes], page-locked
 *             (cudaHostAlloc / cudaHostRegister, or torch pin_memory) so the
 *             device can read it; it is read directly over the host link.
 * row_bytes   bytes per row, a positive multiple of 16.
 * hot         [hot_capacity, row_bytes] device output.  Rows past
 *             hot_capacity are not written and *err = LSA_ERR_CAPACITY.
 * slot_of     [n_total] int32 output or NULL: hot row of each entry, -1 for
 *             entries not kept.
 * ---------------------------------------------------------------------- */
lsa_status lsa_gather(const void *cold_host, int64_t row_bytes, const int64_t *seq_off,
                      int64_t n_total, const int32_t *kept_idx, const int64_t *kept_off, int32_t B,
                      void *hot, int64_t hot_capacity, int32_t *slot_of, int32_t *err,
                      void *stream);

/* ------------------------------------------------------------------------
 * lsa_sparse_attn -- core attention over the selected entries (section 2.1,
 * "Tiered Selection": the top-k feeds "the final core attention
 * computation").  Multi-query attention: all Hq query heads of a sequence
 * attend over the same selected K/V rows.
 *
 *   a_i = scale * Q[b,h,:] . K_i     o[b,h,:] = sum_i softmax(a)_i V_i
 *   lse[b,h] = log sum_i exp(a_i)     (no row selected: o = 0, lse = -inf)
 *
 * Q      [B, Hq, D] dtype LSA_F32 or LSA_BF16.   out  [B, Hq, D] same dtype.
 * kv     rows of the hot buffer, same dtype; row r holds K at element
 *        r * kv_row_stride + k_off and V at r * kv_row_stride + v_off (they
 *        may alias: k_off == v_off for a latent head serving as K and V).
 * rows   [B, k] int32 row indices into kv; negative entries are padding.
 * lse    [B, Hq] fp32 output or NULL.
 * workspace  at least lsa_sparse_attn_workspace_size(B, Hq, D, k) bytes
 *        (fp32 split-K partials); calls that share it must not overlap.
 * err    device error word or NULL (LSA_ERR_TIMEOUT if a bounded wait of the
 *        tensor-core kernel gave up).
 * Shapes run: D % 32 == 0, D <= 512, 1 <= Hq <= 256, 1 <= k <= 65536.  bf16
 * with Hq = 128, D = 512 and K aliasing V (a latent head) runs on the tensor
 * cores (tcgen05); every other shape on the CUDA cores.
 * ---------------------------------------------------------------------- */
size_t lsa_sparse_attn_workspace_size(int32_t B, int32_t Hq, int32_t D, int32_t k);
lsa_status lsa_sparse_attn(const void *Q, lsa_dtype dtype, const void *kv, int64_t kv_row_stride,
                           int64_t k_off, int64_t v_off, const int32_t *rows, int32_t B,
                           int32_t Hq, int32_t D, int32_t k, float scale, void *out, float *lse,
                           void *workspace, size_t ws_bytes, int32_t *err, void *stream);

/* ------------------------------------------------------------------------
 * Decode context and lsa_decode_step -- the tau cadence (section 2.1,
 * "Periodic Triggering", tau = 64).
 *
 * At a refresh step (t % tau == 0): full index scan, selection, cold-pool
 * fetch of the kept rows (on the context's side stream), top-k over the scan's
 * scores, attention.  By default the hot buffer is a cache: a kept entry whose
 * row is already resident keeps its slot and only the others cross the host
 * link (rows no longer kept stay resident until their slot is reused).  The
 * cold pool must not change while the context lives.  At every other step the kept set and hot buffer stay as
 * they are; the kept entries are re-scored with that step's indexer query
 * (listed scan), then top-k and attention.
 * ---------------------------------------------------------------------- */
typedef struct lsa_params {
    int32_t B, H, d;             /* batch, indexer heads, indexer dim */
    lsa_dtype q_dtype, k_dtype;  /* indexer query / key element types */
    int32_t Hq, D;               /* attention query heads, head dim */
    lsa_dtype attn_dtype;        /* Q, K/V rows and output element type */
    int32_t topk;                /* k of the fine-grained top-k */
    int32_t tau;                 /* refresh period; 0 means 64 */
    float scale;                 /* softmax scale; 0 means 1/sqrt(D) */
    int64_t n_total;             /* entries on the flat axis */
    const int64_t *seq_off_host; /* HOST [B+1]; copied at creation */
    const void *k_dev;           /* indexer keys [n_total, d] in HBM (caller-owned) */
    const float *k_scale_dev;    /* [n_total] for E4M3 keys, else NULL */
    const void *cold_host;       /* HOST page-locked cold pool [n_total, row_bytes] */
    int64_t row_bytes;           /* bytes per cold row */
    int64_t kv_row_stride;       /* elements per row (row_bytes / element size) */
    int64_t k_off, v_off;        /* element offsets of K and V inside a row */
    int64_t kept_capacity;       /* hot-buffer rows = max kept entries over the batch */
    int32_t full_fetch;          /* 0: the hot buffer caches rows across refreshes and a refresh
                                    fetches only entries not resident; nonzero: every refresh
                                    fetches every kept row (lsa_gather) into kept order */
    /* Always-resident context merged into the core attention (lsa_attn_set_merge):
     * with window > 0 or hca_rows set, every step attends over the union of its
     * top-k, the last `window` entries of its sequence and the sequence's HCA rows.
     * The context copies both into HBM at creation (window rows from cold_host). */
    int32_t window;              /* recent-window entries per sequence (0: none) */
    const void *hca_rows;        /* HCA rows [hca_off_host[B], row_bytes], host or device memory, same
                                    row format as the cold pool; NULL: none */
    const int64_t *hca_off_host; /* HOST [B+1] offsets of each sequence's HCA rows (with hca_rows) */
    /* OR-mode union of indexer layers in the cadence (lsa_index_union): with n_layers >= 2 every
     * refresh scores each layer's keys with that layer's (q, w) and selects and ranks on the union
     * score max_l z_l; listed steps re-score the kept set in every layer and rank on the union.
     * q and w then carry a leading layer dimension: q [n_layers, B, H, d], w [n_layers, B, H]. */
    int32_t n_layers;                   /* 0 or 1: one layer (k_dev); 2 .. 8: layers 0 .. n_layers-1 */
    const void *const *k_dev_layers;    /* HOST array [n_layers-1] of DEVICE key pointers of layers
                                           1 .. n_layers-1 (layer 0 is k_dev); same dtype and shape */
    const float *const *k_scale_layers; /* HOST array [n_layers-1] of their E4M3 row scales (else NULL) */
    /* Lookahead (blog page: critical chunks fetched from the cold pool "just in time"; section 2.1
     * "Dynamic Fetching"): 0 refreshes at the first step of every window, its fetch on the step's critical
     * path.  L in [1, tau): the kept set of window r >= 1 (steps r*tau .. r*tau + tau-1) is predicted at
     * step r*tau - L with that step's indexer query, after the step's own work; its rows are fetched on the
     * context's side stream while steps r*tau - L .. r*tau - 1 still attend window r-1's set (the fetch never
     * evicts a row that set uses), and at step r*tau the new set becomes current and is re-ranked with that
     * step's query.  Window 0 refreshes at its first step.  Needs full_fetch = 0; the hot buffer must hold
     * both sets' rows (LSA_ERR_CAPACITY otherwise). */
    int32_t lookahead;
} lsa_params;

typedef struct lsa_ctx lsa_ctx;

/* Allocates the context's device buffers (hot buffer, scores, kept list,
 * top-k, workspaces, host staging) and its side stream.  Synchronous. */
lsa_status lsa_ctx_create(const lsa_params *p, lsa_ctx **out);
/* Synchronises the context's streams and frees everything it allocated. */
lsa_status lsa_ctx_destroy(lsa_ctx *ctx);

/* One decode step t >= 0 on device buffers: q [B,H,d], w [B,H], Q [B,Hq,D]
 * in ([n_layers, B, H, d] and [n_layers, B, H] with n_layers >= 2); out
 * [B,Hq,D] and lse [B,Hq] (lse may be NULL) out. */
lsa_status lsa_decode_step(lsa_ctx *ctx, int64_t t, const void *q, const float *w, const void *Q,
                           void *out, float *lse, void *stream);

/* The same step on HOST buffers (page-locked for asynchronous copies).
 * The inputs are copied host->device on an internal copy stream into one of
 * two device staging slots (alternating per call), so a call's input copies
 * overlap the kernels of the call before it; the step's kernels run on
 * `stream` after its inputs have landed, and out and lse are copied
 * device->host before `stream` completes.  Ordering: the input copies are NOT
 * ordered after earlier work on `stream` -- the input host buffers must hold
 * the step's values when the call is made (host program order) and stay
 * unchanged, like out_host and lse_host stay untouched, until `stream` has
 * completed this call's work; out_host and lse_host hold the results once
 * `stream` has completed.  When out_host (and lse_host, if given) are
 * page-locked host memory mapped for the device (cudaHostAlloc, or
 * pinned tensors, on a UVA system), the step's attention writes them
 * directly over the host link; other host memory goes through a device
 * staging buffer and a copy. */
lsa_status lsa_decode_step_host(lsa_ctx *ctx, int64_t t, const void *q_host, const float *w_host,
                                const void *Q_host, void *out_host, float *lse_host, void *stream);

/* Device pointers of the context's internal results, for inspection. */
typedef struct lsa_ctx_view {
    float *z;            /* [n_total] full-scan scores of the last refresh (the union score
                            max_l z_l with n_layers >= 2) */
    float *z_kept;       /* [kept_capacity] listed-scan scores of the last step (union likewise) */
    int32_t *kept_idx;   /* [kept_capacity] */
    int64_t *kept_off;   /* [B+1] */
    int32_t *slot_of;    /* [n_total] hot slot of each entry, or -1 */
    void *hot;           /* [kept_capacity + B * window + HCA rows, row_bytes]: the hot buffer,
                            then the window rows, then the HCA rows */
    int32_t *topk_idx;   /* [B, topk] */
    int32_t *topk_pos;   /* [B, topk] hot slot of each chosen entry, -1 padded */
    int32_t *topk_cnt;   /* [B] */
    int32_t *err;        /* device error word of the context */
    int32_t *kept_slot;  /* [kept_capacity] hot slot of each kept position (NULL with full_fetch) */
    int32_t *owner;      /* [kept_capacity] entry held by each hot slot, or -1 */
    int64_t *fetched;    /* rows fetched from the cold pool by the last refresh */
    int32_t *attn_rows;  /* [B, attn_row_cap] merged attention rows into `hot` (NULL without
                            window / HCA rows): see lsa_attn_set_merge */
    int64_t attn_row_cap;
    int64_t win_base;    /* arena row of sequence 0's first window row (sequence b: + b * window) */
    int64_t hca_base;    /* arena row of the first HCA row */
} lsa_ctx_view;
lsa_status lsa_ctx_get_view(lsa_ctx *ctx, lsa_ctx_view *view);

/* CUDA graphs (on by default): after one eager run of each step kind, a step
 * is captured once per distinct (q, w, Q, out, lse) pointer set and replayed
 * with a single graph launch on the caller's stream (at most 256 cached
 * graphs; the cache is cleared when full).  Captured steps bake in their
 * pointers: the buffers behind them must stay allocated while the context
 * may replay them. */
lsa_status lsa_ctx_set_graphs(lsa_ctx *ctx, int32_t enable);

/* Stage timing.  When enabled, steps run eagerly (no graphs) and CUDA
 * events bracket every stage on the stream it runs on; lsa_ctx_stage_times
 * synchronises on them and returns the
 * accumulated milliseconds and call counts per stage since the last reset
 * (arrays of LSA_STAGE_COUNT).  lsa_ctx_launches returns the number of
 * kernels the context has launched since the last reset. */
enum { LSA_STAGE_SCORE = 0, LSA_STAGE_SELECT, LSA_STAGE_GATHER, LSA_STAGE_TOPK,
       LSA_STAGE_ATTN, LSA_STAGE_RESCORE, LSA_STAGE_COUNT };
lsa_status lsa_ctx_set_timing(lsa_ctx *ctx, int32_t enable);
lsa_status lsa_ctx_stage_times(lsa_ctx *ctx, double *ms, int64_t *calls);
lsa_status lsa_ctx_reset_counters(lsa_ctx *ctx);
int64_t lsa_ctx_launches(lsa_ctx *ctx);

/* Empties the hot-buffer cache (enqueued on `stream`): afterwards no entry counts as resident, so the next
 * refresh or prediction fetches every kept row from the cold pool (a cold start, e.g. a new request or a
 * topic shift).  The current kept set's rows stay in place for the steps that still read them. */
lsa_status lsa_ctx_flush_cache(lsa_ctx *ctx, void *stream);

/* ------------------------------------------------------------------------
 * lsa_selftest_bounded_wait -- checks, on the GPU, the expiry path of the
 * bounded device-side waits that every tcgen05 kernel here uses (the pages
 * have no counterpart: this is failure-handling infrastructure).  One CTA
 * waits on a shared-memory mbarrier that nothing arrives at:
 *   - warp 0 waits with a limit of limit_ns (%globaltimer); when it runs out
 *     the kernel writes LSA_ERR_TIMEOUT into *err (first error wins) and
 *     waited_ns[0] = the time it waited;
 *   - warp 1 waits on the same barrier with a limit of 4 * limit_ns and
 *     returns as soon as warp 0 raises the CTA's abort flag: waited_ns[1] =
 *     its wait (about limit_ns, well below 4 * limit_ns), waited_ns[2] = 1 if
 *     its wait reported success (it must not: 0).
 * The kernel always returns; no fault, trap or hang is involved.
 *
 * limit_ns   1,000 .. 100,000,000 (1 us .. 100 ms), else LSA_ERR_INVALID
 * err        device int32 error word (the caller zeroes it first)
 * waited_ns  device int64[3], written by the kernel
 * stream     cudaStream_t or NULL
 * ---------------------------------------------------------------------- */
lsa_status lsa_selftest_bounded_wait(int64_t limit_ns, int32_t *err, int64_t *waited_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
