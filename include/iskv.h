/*
 * iskv.h - C ABI of the iS-KV hot path on one B200 (sm_100a): block-incremental truncated SVD of
 * each (layer, sequence, kv-head) key and value stream, plus decode attention over the compressed
 * history and an exact recent window.
 *
 * Method: "iS-KV: Online Low-Rank KV Cache Compression via Block-Incremental SVD" (summary page).
 *   - "Architecture Overview": per K/V path an exact window of the most recent tokens and a
 *     low-rank history of rank at most r.
 *   - "Block-Incremental Decoding Updates": each fold takes the pending block F (b rows), forms the
 *     residual E = F - (F B) B^T and an orthonormal residual basis P, the core
 *     Z = [[Sigma, 0], [F B, F P]], its truncated SVD (G, Sigma+, H), and the updated factors
 *     U+ = diag(U, I_b) G, B+ = [B P] H. Old rows' coordinates move with the basis.
 *   - "Reconstruction and Storage": compressed row i is (U Sigma B^T)[i]; window rows are exact;
 *     storage k (n + d + 1) factor scalars per path plus d e exact scalars.
 *
 * Conventions shared by every entry point:
 *   - Return value: ISKV_OK (0) or a negative ISKV_ERR_* code; no C++ exception crosses the ABI.
 *     Argument errors are detected on the host before anything is enqueued.
 *   - Pointers named *_dev are device pointers owned by the caller; they must stay valid until
 *     the work enqueued on `stream` has completed. Pointers to host scalars are written before
 *     the call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). All device work is enqueued on
 *     it asynchronously; nothing synchronises except iskv_sync_status().
 *   - The handle owns all persistent device state, allocated once by iskv_create() and sized by
 *     max_tokens; it is never reallocated. A handle is not thread-safe.
 *   - Each layer keeps its own token count t; layer = -1 addresses all layers at once (they must
 *     then hold the same t).
 *   - Device-side failures (a core SVD that did not converge, a non-finite singular value) set a
 *     sticky status word that iskv_sync_status() returns.
 */
#ifndef ISKV_H
#define ISKV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct iskv_handle iskv_handle;
/* Layout-compatible with cudaStream_t. */
typedef struct CUstream_st *iskv_stream_t;

enum {
    ISKV_OK = 0,
    ISKV_ERR_INVALID_ARG = -1,  /* bad config, NULL pointer, layer out of range, ...        */
    ISKV_ERR_CAPACITY = -2,     /* t + m > max_tokens                                        */
    ISKV_ERR_CUDA = -3,         /* a CUDA runtime call failed (allocation, launch, copy)     */
    ISKV_ERR_NOT_CONVERGED = -4,/* a core SVD hit its sweep cap (sticky, device side)        */
    ISKV_ERR_NONFINITE = -5,    /* a non-finite singular value appeared (sticky, device side) */
    ISKV_ERR_UNSUPPORTED = -6,  /* valid request outside what this build implements          */
    ISKV_ERR_TIMEOUT = -7       /* a device-side wait hit its bound (sticky, device side)    */
};

enum { ISKV_BF16 = 0, ISKV_F32 = 1 };

typedef struct {
    int batch;            /* sequences decoded in lock-step                                  */
    int n_layers;
    int n_kv_heads;
    int n_q_heads;        /* multiple of n_kv_heads; q-head g reads kv-head g / (n_q/n_kv)    */
    int head_dim;         /* d; must be 128                                                  */
    int rank_k, rank_v;   /* rank budgets r_K, r_V (1 .. head_dim)                           */
    int block;            /* b: rows folded per update (1 .. 1024; blocks above 128 rows are  */
                          /*    folded through their 128-row triangular factor)              */
    int window;           /* w: exact rows kept before a fold may take them (>= 0)           */
    long long max_tokens; /* capacity per sequence and layer                                 */
    int kv_dtype;         /* ISKV_BF16 or ISKV_F32: dtype of appended rows and of the window  */
    int rope;             /* 1: rotate keys by RoPE (pairs j, j+d/2) after reconstruction     */
    double rope_theta;    /* RoPE base; angle of pair j at position i is i * theta^(-2j/d)    */
    int rotate_history;   /* 1: iS-KV (old coordinates rotate with the basis).               */
                          /* 0: stale-coordinate ablation (drift study only).                */
    int lookahead_folds;  /* 0: each fold runs on the caller's stream when the window releases  */
                          /*    its block.                                                     */
                          /* 1: each fold starts on an internal stream as soon as its block is */
                          /*    complete (up to window / block + 1 folds ahead) and is joined  */
                          /*    into the caller's stream when the window releases the block;   */
                          /*    every decode sees exactly the state of mode 0. Call            */
                          /*    iskv_join() before ending a stream capture that contains       */
                          /*    appends.                                                       */
    int fixed_basis;      /* 1: fixed-basis ablation ("Ablation Study", bases kept fixed): the   */
                          /*    regular update runs for the first ceil(min(r, d) / block) folds */
                          /*    of a path (they fill its rank budget); after that the path's   */
                          /*    basis and Sigma freeze and each later block is stored as its   */
                          /*    coordinates F B in the frozen basis (old coordinates untouched). */
                          /*    0: iS-KV. Cannot be combined with rotate_history = 0.           */
    int coord_bf16;       /* 1: store the coordinates C = U Sigma (the k n factor scalars that    */
                          /*    grow with the history) in bf16, rounded to nearest even after   */
                          /*    every fold and history rotation; arithmetic stays fp32 and B,    */
                          /*    Sigma stay fp32 ("Reconstruction and Storage": beta_f = 2 for C). */
                          /*    Needs rank_k <= 64, rank_k and rank_v multiples of 8 and a GQA   */
                          /*    group of 1, 2 or 4 (else ISKV_ERR_UNSUPPORTED). 0: fp32.         */
    int prot_cap;         /* 0: iskv_prefill() is not available. >= 1: it is, and the protected */
                          /*    stores hold up to prot_cap exact rows per unit and path        */
                          /*    ("Prefill Compression"; more set ISKV_ERR_CAPACITY, sticky).   */
    int joint_heads;      /* 1: joint per-layer factorisation ("Reconstruction and Storage",     */
                          /*    persistent storage per layer): the rows of all n_kv_heads of a   */
                          /*    (layer, sequence) at one position are concatenated, head by    */
                          /*    head, into one row of length d = n_kv_heads * head_dim, and one  */
                          /*    factorisation per (layer, sequence, path) folds them: one        */
                          /*    coordinate row of rank r per position, shared by the kv-heads,   */
                          /*    and a d x r basis whose rows h*128 .. h*128+127 reconstruct      */
                          /*    kv-head h. The exact window stays per kv-head. Needs            */
                          /*    rank + block <= 128 for both paths, fixed_basis = 0 and          */
                          /*    prot_cap = 0 (else ISKV_ERR_UNSUPPORTED). 0: one factorisation  */
                          /*    per (layer, sequence, kv-head, path).                           */
} iskv_config;

/* Key/value protection of iskv_prefill() ("Prefill Compression", steps 1-2). */
typedef struct {
    int chunk;            /* positions per key chunk (>= 1)                                   */
    int m;                /* outlier chunks protected per kv-head: the m lowest min-cosine     */
                          /*    scores (ties by chunk index) (>= 0)                            */
    int suffix;           /* positions just before the window that are protected too (>= 0)   */
    int rho;              /* value protection radius: P_V = positions within rho of P_K (>= 0) */
} iskv_protect;

/*
 * Creates a cache for `cfg` on the current CUDA device. Allocates every device buffer
 * (coordinates C = U Sigma [max compressed rows x r] in fp32, or bf16 with coord_bf16; bases
 * B [d x r], Sigma [r] and the
 * fold's H_top [r x r] in fp32, each in a ring of 2 buffers, or window / block + 3 with
 * lookahead_folds; the exact ring of window + block rows per path in kv_dtype; a RoPE table
 * [max_tokens x d/2] of (cos, sin); decode split partials; a status word) and, with
 * lookahead_folds, the internal streams and events of the early folds.
 * Errors: ISKV_ERR_INVALID_ARG (cfg out of range), ISKV_ERR_CUDA (allocation failed; nothing
 * leaks). On success *out owns the handle; release it with iskv_destroy().
 */
int iskv_create(const iskv_config *cfg, iskv_handle **out);

/* Frees every device buffer of the handle (synchronises the device first). NULL is a no-op. */
int iskv_destroy(iskv_handle *h);

/*
 * Appends m >= 1 new rows per (sequence, kv-head) to the key and value streams of `layer` and
 * folds every block that the window releases ("Block-Incremental Decoding Updates"): rows enter
 * the exact window one by one; whenever it holds window + block rows its oldest block is folded,
 * so after t tokens n_c(t) = block * floor(max(0, t - window) / block) rows are compressed.
 *   k_rows_dev, v_rows_dev: kv_dtype, row-major [batch][n_kv_heads][m][head_dim] for layer >= 0,
 *                           [n_layers][batch][n_kv_heads][m][head_dim] for layer == -1.
 *                           Keys are pre-RoPE.
 * Errors: ISKV_ERR_INVALID_ARG (NULL rows, m < 1, bad layer, layers with different t for -1),
 *         ISKV_ERR_CAPACITY (t + m > max_tokens), ISKV_ERR_CUDA (launch failed).
 */
int iskv_append_block(iskv_handle *h, int layer, const void *k_rows_dev, const void *v_rows_dev,
                      int m, iskv_stream_t stream);

/*
 * Prefill of an empty layer with T0 rows per (sequence, kv-head) ("Prefill Compression"): the
 * last `window` rows form the exact window; of the rows before it, the protected positions (keys:
 * P_K of step 1; values: P_V of step 2; none when protect is NULL) stay exact for good and the
 * others are factorised by one truncated SVD of rank r (step 3), computed from the rows'
 * triangular factor (Householder QR over 128-row chunks) and a one-sided Jacobi SVD of it; the
 * coordinates of protected positions are zero and decode reads their exact rows. Later appends
 * fold blocks from the window as usual. Chunk scores use keys rotated at their positions.
 *   k_rows_dev, v_rows_dev: kv_dtype [batch][n_kv_heads][T0][head_dim] (keys pre-RoPE).
 *   protect: host pointer or NULL.
 * Synchronises `stream` when protect is given (the largest protected count sizes the decode's
 * protected tiles). Needs cfg.prot_cap >= 1 (else ISKV_ERR_UNSUPPORTED); protection also needs
 * the persistent decode (rank_k <= 32 with fp32 coordinates, <= 64 with bf16; G of 1, 2 or 4).
 * Errors: ISKV_ERR_INVALID_ARG (layer not empty, bad protect values, T0 < 1),
 *         ISKV_ERR_CAPACITY (T0 > max_tokens), ISKV_ERR_UNSUPPORTED, ISKV_ERR_CUDA.
 */
int iskv_prefill(iskv_handle *h, int layer, const void *k_rows_dev, const void *v_rows_dev,
                 long long T0, const iskv_protect *protect, iskv_stream_t stream);

/*
 * Decode attention of `layer` over all t cached positions 0 .. t-1: compressed rows are
 * reconstructed as C B^T ("Reconstruction and Storage"), keys are then rotated by RoPE at their
 * position (when cfg.rope), scores use scale 1/sqrt(d), softmax is exact (fp32, log-sum-exp
 * merge of position splits). Two kernels (position splits, then their merge) on `stream`.
 *   q_dev:   fp32 [batch][n_q_heads][head_dim], already rotated for the query position,
 *            16-byte aligned (the kernels copy it in 16-byte units).
 *   out_dev: fp32 [batch][n_q_heads][head_dim].
 * Errors: ISKV_ERR_INVALID_ARG (NULL pointers, bad layer, t == 0, misaligned q_dev),
 *         ISKV_ERR_CUDA.
 */
int iskv_decode_attn(iskv_handle *h, int layer, const float *q_dev, float *out_dev,
                     iskv_stream_t stream);

/*
 * One decode step of `layer`: appends one new row per (sequence, kv-head) to the key and value
 * streams (with any fold the window releases, as iskv_append_block() with m = 1) and then runs
 * iskv_decode_attn() over positions 0 .. t (the new row included). Same results as those two
 * calls. With the tensor-core decode and window >= 1 the new rows are read by the decode kernel
 * itself, which also stores them in the exact ring, so the step needs no separate append launch;
 * otherwise the two calls are made in turn.
 *   k_row_dev, v_row_dev: kv_dtype [batch][n_kv_heads][1][head_dim] (keys pre-RoPE);
 *   q_dev, out_dev: as iskv_decode_attn().
 * Errors: those of iskv_append_block() and iskv_decode_attn().
 */
int iskv_append_decode(iskv_handle *h, int layer, const void *k_row_dev, const void *v_row_dev,
                       const float *q_dev, float *out_dev, iskv_stream_t stream);

/*
 * Writes the reconstructed cache of one path of `layer` ("Reconstruction and Storage"): row i is
 * (C B^T)[i] for i < n_c and the exact window row otherwise; keys are rotated by RoPE when
 * apply_rope != 0 (ignored for values).
 *   which:   0 = keys, 1 = values.
 *   out_dev: fp32 [batch][n_kv_heads][t][head_dim].
 * Errors: ISKV_ERR_INVALID_ARG, ISKV_ERR_CUDA.
 */
int iskv_reconstruct(iskv_handle *h, int layer, int which, int apply_rope, float *out_dev,
                     iskv_stream_t stream);

/*
 * Copies the factors of one unit (layer, seq, kv_head, path) into caller buffers (device to
 * device, on `stream`) and reports its current rank and compressed-row count.
 *   coords_dev: fp32 [n_c][rank] (row stride = rank budget of the path; bf16-stored coordinates
 *               are widened to fp32 exactly), may be NULL;
 *   basis_dev:  fp32 [head_dim][rank], may be NULL;
 *   sigma_dev:  fp32 [rank], may be NULL (entries >= *k_out are zero);
 *   k_out, n_c_out: host pointers, may be NULL.
 * Errors: ISKV_ERR_INVALID_ARG, ISKV_ERR_CUDA.
 */
int iskv_get_factors(iskv_handle *h, int layer, int seq, int kv_head, int which,
                     float *coords_dev, float *basis_dev, float *sigma_dev, int *k_out,
                     long long *n_c_out, iskv_stream_t stream);

/*
 * Empties every layer (t = n_c = 0, rank 0) and clears the sticky status, keeping all device
 * allocations, so a handle can serve a new batch of sequences. Joins pending early folds into
 * `stream` first (iskv_join); then host bookkeeping plus asynchronous device writes on `stream`;
 * later calls must be ordered after it on a stream.
 * Errors: ISKV_ERR_INVALID_ARG, ISKV_ERR_CUDA.
 */
int iskv_reset(iskv_handle *h, iskv_stream_t stream);

/*
 * Number of kernel launches this handle has enqueued since creation (host counter; launches
 * captured into a CUDA graph are counted once, at capture). Errors: ISKV_ERR_INVALID_ARG.
 */
int iskv_launch_count(const iskv_handle *h, long long *count_out);

/*
 * Statistics of the core SVDs run since creation or the last iskv_reset(): the largest number of
 * Jacobi sweeps one core needed, the total number of sweeps, and the number of cores solved.
 * Synchronises `stream` (a device-to-host copy). Any output pointer may be NULL.
 * Errors: ISKV_ERR_INVALID_ARG, ISKV_ERR_CUDA.
 */
int iskv_fold_stats(iskv_handle *h, iskv_stream_t stream, int *max_sweeps_out,
                    long long *total_sweeps_out, long long *cores_out);

/* Tokens cached in `layer` (host value). Errors: ISKV_ERR_INVALID_ARG. */
int iskv_num_tokens(const iskv_handle *h, int layer, long long *t_out);

/*
 * Persistent bytes of one layer per the storage formula of "Reconstruction and Storage":
 * sum_X [beta_c k_X n_X + 4 k_X (d + 1)] + beta_e * d * sum_X e_X, summed over sequences and
 * kv-heads, with beta_c = 2 (coord_bf16) or 4 bytes per coordinate, fp32 bases and Sigma, and
 * beta_e = bytes of kv_dtype. Host only.
 */
int iskv_storage_bytes(const iskv_handle *h, int layer, long long *bytes_out);

/*
 * Host-only schedule of the fold trigger ("Architecture Overview" window, read as: fold the
 * oldest block whenever window + block rows are exact). For a stream holding t tokens, appending
 * m rows leaves *n_c_out compressed rows and performs *folds_out folds. Needs no GPU.
 * Errors: ISKV_ERR_INVALID_ARG (block < 1, window < 0, t < 0, m < 0).
 */
int iskv_schedule(int block, int window, long long t, long long m, long long *n_c_out,
                  long long *folds_out);

/*
 * Makes `stream` wait for every fold that lookahead_folds started on an internal stream and that
 * no later call has joined yet (those whose blocks the window has not released). Required before
 * ending a stream capture that contains iskv_append_block() calls, so that the capture holds no
 * unjoined work; a no-op without lookahead_folds. Enqueues only event waits.
 * Errors: ISKV_ERR_INVALID_ARG, ISKV_ERR_CUDA.
 */
int iskv_join(iskv_handle *h, iskv_stream_t stream);

/*
 * Joins pending early folds (iskv_join), synchronises `stream` and returns the sticky status: ISKV_OK, ISKV_ERR_NOT_CONVERGED,
 * ISKV_ERR_NONFINITE or ISKV_ERR_TIMEOUT (the first error seen since creation or the last
 * iskv_reset()), or ISKV_ERR_CUDA if the synchronisation itself failed.
 */
int iskv_sync_status(iskv_handle *h, iskv_stream_t stream);

/*
 * Decode attention over caller-owned buffers that allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine, no handle). The paper has no counterpart: this entry point exists
 * for callers that cannot allocate device memory on their decode path - code running inside CUDA
 * stream capture (cudaMalloc is not capturable), engines whose device memory is entirely owned by
 * their own pool allocator, and latency-critical loops where cudaMalloc's implicit device
 * synchronisation is not acceptable.
 *
 * The computation is that of iskv_decode_attn() for one layer, on the CUDA-core decode kernels,
 * with the cache described by `view` instead of a handle. The split partials that
 * iskv_decode_attn() keeps in handle-owned memory live here in a file-scope device array of
 * ISKV_NOALLOC_SCRATCH_FLOATS floats (4 MiB) that every GPU which loads the library holds until the
 * process exits. Required scratch: batch * n_kv_heads * splits * (n_q_heads / n_kv_heads) *
 * (head_dim + 2) floats, with splits = ceil(n_c / 128) + ceil((t - n_c) / 128) at most; larger
 * requests return ISKV_ERR_CAPACITY before anything is enqueued.
 *
 * All calls share that array and it keeps the last call's contents; nothing in it has to start at
 * zero (every split writes its partials before the merge reads them). Calls whose work overlaps
 * on the GPU (different streams, or different host threads) race on the array: order them on one
 * stream. The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that first call before any
 * stream capture.
 *   view:    cache description (layouts below), all pointers device pointers owned by the caller
 *            (one coordinate array per kv-head unit: a joint-factorisation cache, whose kv-heads
 *            share their coordinates, is decoded through iskv_decode_attn instead);
 *   q_dev:   fp32 [batch][n_q_heads][head_dim], already rotated for the query position;
 *   out_dev: fp32 [batch][n_q_heads][head_dim].
 * Errors: ISKV_ERR_INVALID_ARG (NULL pointer, inconsistent sizes), ISKV_ERR_CAPACITY (scratch
 * too small), ISKV_ERR_CUDA (address lookup or launch failed).
 */
#define ISKV_NOALLOC_SCRATCH_FLOATS (1 << 20)

typedef struct {
    long long n_c;        /* compressed rows per unit (positions 0 .. n_c-1)                   */
    long long t;          /* tokens: positions 0 .. t-1 are attended (t >= 1)                  */
    long long n_max;      /* coordinate rows per unit in coords_k / coords_v (>= n_c)          */
    int batch, n_kv_heads, n_q_heads, head_dim;    /* head_dim must be 128                  */
    int rank_k, rank_v;   /* row stride of the coordinate arrays = columns of the bases        */
    int k_k, k_v;         /* ranks in use (1 .. rank) when n_c > 0                             */
    int ring_rows;        /* R: exact row of position i (n_c <= i < t) sits at slot i mod R   */
    int kv_dtype;         /* ISKV_BF16 or ISKV_F32 (exact rows)                                */
    const float *coords_k, *coords_v;  /* [batch*n_kv_heads][n_max][rank] fp32                */
    const float *basis_k, *basis_v;    /* [batch*n_kv_heads][head_dim][rank] fp32             */
    const void *ring_k, *ring_v;       /* [batch*n_kv_heads][R][head_dim] kv_dtype, pre-RoPE */
    const float *rope_cs;              /* [t][head_dim/2] (cos, sin) pairs, or NULL: no RoPE */
} iskv_decode_view;

int iskv_decode_attn_noalloc(const iskv_decode_view *view, const float *q_dev, float *out_dev,
                             iskv_stream_t stream);

/* Static description of an error code. */
const char *iskv_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* ISKV_H */
