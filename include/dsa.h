/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) forward pass on one
 * NVIDIA B200 (sm_100a).  Exported by libdsa.so.
 *
 * What it computes (DeepSeek-V3.2 technical-report summary, ai.flicky.cc,
 * section "DSA: внимание только к важному"):
 *
 *   lightning indexer ("Молниеносный индексатор", equation for I_{t,s}):
 *       I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_I[t,j] . k_I[s])        for s <= t
 *     with q_I and k_I in FP8 e4m3, each token carrying one positive fp32
 *     scale (q_I[t,j] = e4m3 * q_scale[t], k_I[s] = e4m3 * k_scale[s]);
 *   top-k selection and attention ("Отбор и основное внимание", equation for u_t):
 *       u_t = Attn(h_t, { c_s : I[t,s] in Top-k(I[t,:]) }),   k = 2048,
 *     MLA in MQA form: one latent KV row c_s (width d_qk) is shared by all H
 *     query heads; its leading d_v columns are the value.
 *
 * Conventions shared by every entry point:
 *   - Every pointer is caller-owned DEVICE memory, row-major and contiguous,
 *     16-byte aligned.  The library never allocates, frees or synchronises;
 *     it only enqueues kernels on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).
 *   - Query i of batch b sits at sequence position t = q_offset + i and sees
 *     keys 0..t.  Keys 0..Lk-1 exist; q_offset + Lq <= Lk is required.
 *     Decode is Lq = 1, q_offset = Lk - 1; a prefill chunk is
 *     q_offset = chunk start, Lk = q_offset + Lq.
 *   - Argument and shape errors return before anything is enqueued.  A launch
 *     failure returns DSA_ERR_CUDA.  Faults inside a kernel show up at the
 *     caller's next synchronisation.  Kernels never trap: a device-side wait
 *     that exceeds its limit is recorded and reported by dsa_device_status().
 *   - Supported shapes: (H_I, d_I) in {(4, 64), (64, 128)};
 *     (H, d_qk, d_v) in {(16, 192, 128), (128, 576, 512)}; 1 <= k <= 2048;
 *     Lk < 2^31 / 16 per batch.  Anything else returns DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, misaligned pointer, q_offset+Lq > Lk */
    DSA_ERR_UNSUPPORTED = 2, /* a shape outside the supported set */
    DSA_ERR_WORKSPACE = 3,   /* workspace smaller than dsa_workspace_size() */
    DSA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    DSA_ERR_TIMEOUT = 5      /* a device-side wait gave up (see dsa_device_status) */
} dsa_status;

/* Inputs of the lightning indexer (equation for I_{t,s}). */
typedef struct {
    int B, Lq, Lk, q_offset;
    int H_I, d_I;            /* indexer heads and head width */
    const void *q_I;         /* e4m3 codes [B, Lq, H_I, d_I] */
    const float *q_scale;    /* fp32 [B, Lq], > 0; NULL means 1.0 */
    const void *w;           /* bf16 [B, Lq, H_I] */
    const void *k_I;         /* e4m3 codes [B, Lk, d_I] */
    const float *k_scale;    /* fp32 [B, Lk], > 0; NULL means 1.0 */
} dsa_indexer_args;

/* Inputs of the MQA / MLA-absorbed attention (equation for u_t). */
typedef struct {
    int H, d_qk, d_v;        /* query heads, latent row width, value width (d_v <= d_qk) */
    float scale;             /* softmax scale applied to q . c_s */
    const void *q;           /* bf16 [B, Lq, H, d_qk] */
    const void *kv;          /* bf16 [B, Lk, d_qk]: latent rows c_s; value = leading d_v columns */
} dsa_attn_args;

/* Which entry point dsa_workspace_size() is asked about. */
typedef enum {
    DSA_OP_TOPK = 0,
    DSA_OP_SPARSE_ATTN = 1,
    DSA_OP_FORWARD = 2,          /* dsa_forward, staged selection (the faster path) */
    DSA_OP_INDEXER_TOPK = 3,
    DSA_OP_FORWARD_LOWMEM = 4    /* dsa_forward, fused selection (no score matrix) */
} dsa_op;

/*
 * Indexer scores, equation for I_{t,s}.
 *   scores: fp32 [B, Lq, Lk]; scores[b,i,s] = I[q_offset+i, s] for s <= q_offset+i,
 *   and -INFINITY for s > q_offset+i.
 * Accumulation is fp32 over exact FP8 products; the per-token scales are
 * applied after the head sum (they are positive, so they commute with ReLU).
 */
dsa_status dsa_indexer_scores(const dsa_indexer_args *args, float *scores, void *stream);

/*
 * Top-k selection over indexer scores ("Отбор и основное внимание": the k
 * positions with the largest I[t,:]).
 *   scores:  fp32 [B, Lq, Lk] (only entries s <= q_offset+i are read);
 *   indices: int32 [B, Lq, k].  Row (b,i) receives the m = min(k, q_offset+i+1)
 *            positions with the largest scores, ties to the smaller position,
 *            -0.0 equal to +0.0, written in ascending position order in slots
 *            0..m-1; slots m..k-1 receive -1.
 *   workspace: may be NULL when dsa_workspace_size(DSA_OP_TOPK, ...) is 0.
 */
dsa_status dsa_topk(const float *scores, int B, int Lq, int Lk, int q_offset, int k,
                    int32_t *indices, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Indexer and top-k fused: the k positions with the largest I[t,s] per row
 * (equation for I_{t,s} of "Молниеносный индексатор", then the Top-k of the
 * equation for u_t in "Отбор и основное внимание"), selected on chip as the
 * scores are produced, so the [B, Lq, Lk] score matrix is never written.
 *   indices:    int32 [B, Lq, k], exactly as dsa_topk would return for the scores
 *               of dsa_indexer_scores (ties to the smaller position, -0.0 == +0.0,
 *               ascending position order, -1 padding after min(k, t+1) slots);
 *   sel_scores: fp32 [B, Lq, k] or NULL: I[t, indices[...]] for each valid slot,
 *               -INFINITY on padding slots;
 *   workspace:  dsa_workspace_size_args(DSA_OP_INDEXER_TOPK, args, k, 0, 0) bytes
 *               (the per-row candidate lists; a few tens of MB, independent of Lk
 *               for prefill).  Its contents need not be initialised.
 */
dsa_status dsa_indexer_topk(const dsa_indexer_args *args, int k, int32_t *indices, float *sel_scores,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Sparse MQA attention over the selected latent rows (equation for u_t).
 *   indices: int32 [B, Lq, k]; entries outside [0, Lk) are skipped.
 *   out:     bf16 [B, Lq, H, d_v];  out[b,i,h,:] = sum_s p_s kv[b,s,:d_v],
 *            p = softmax over the selected s of scale * q[b,i,h,:] . kv[b,s,:].
 *   lse:     fp32 [B, Lq, H] or NULL; natural-log log-sum-exp of the logits
 *            (-INFINITY and out = 0 for a row with no valid entry).
 * Rows with B*Lq small are split over the k entries across CTAs and merged
 * (split-k); the workspace holds the partial results.
 */
dsa_status dsa_sparse_attn(const dsa_attn_args *args, int B, int Lq, int Lk,
                           const int32_t *indices, int k, void *out, float *lse,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * dsa_sparse_attn without a workspace argument.  The pages have no counterpart
 * to this call: it is for callers that may not allocate device memory at the
 * point of the call yet still reach the split-k path (few query rows, e.g.
 * decode) -- a serving loop that committed all device memory to its own pool up
 * front, or code that must not risk the implicit device synchronisation that
 * freeing memory brings.
 *
 * Arguments, layouts, results and errors are those of dsa_sparse_attn.  The
 * split-k partials (dsa_workspace_size(DSA_OP_SPARSE_ATTN, ...) bytes; 0 when
 * B*Lq is large enough that no row is split) are kept in a fixed array of
 * DSA_NOALLOC_SCRATCH_BYTES that is part of the library's device code, so the
 * call allocates and frees nothing.  A call that needs more returns
 * DSA_ERR_WORKSPACE before launching anything.  Nothing in the array has to
 * start at zero: every partial is written before it is read.
 * Memory: the array is device memory held by every device on which it has been
 * looked up, until the process exits.  It sits in a module of its own, so with
 * the CUDA runtime's default lazy module loading only callers of this entry
 * point reserve it; with eager loading (CUDA_MODULE_LOADING=EAGER) every
 * context that loads libdsa.so does.
 * Set-up: the first call that needs the array in a CUDA context of a device
 * looks its address up (which may make the CUDA runtime load that module); the
 * address is reused until the context changes (e.g. after cudaDeviceReset).
 * Make that first call before any stream capture begins.
 * The array is shared by all calls on a device: calls whose executions overlap
 * (different streams, or host threads with no ordering between them) race on it
 * and produce wrong results.  Order them, e.g. on one stream.
 */
#define DSA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
dsa_status dsa_sparse_attn_noalloc(const dsa_attn_args *args, int B, int Lq, int Lk,
                                   const int32_t *indices, int k, void *out, float *lse,
                                   void *stream);

/*
 * The whole forward pass: indexer -> top-k -> sparse attention.  `iargs` and
 * `aargs` describe the same B, Lq, Lk, q_offset.
 * The selection runs one of two ways, chosen by the workspace the caller gives;
 * both produce identical indices and selected scores:
 *   staged (workspace >= dsa_workspace_size_args(DSA_OP_FORWARD, ...)): the
 *     indexer writes the causal part of the [B, Lq, Lk] fp32 score matrix into
 *     the workspace and a separate top-k kernel selects from it.  The faster
 *     path on every measured shape: the selection then runs on all SMs at full
 *     issue rate instead of competing with the indexer's epilogue.
 *   fused (workspace >= dsa_workspace_size_args(DSA_OP_FORWARD_LOWMEM, ...) but
 *     below the staged size): dsa_indexer_topk; no score matrix, a workspace of
 *     a few tens of MB, slower.
 * A workspace below both sizes is refused with DSA_ERR_WORKSPACE.
 * Short sequences (q_offset + Lq <= k): every row selects all of its positions
 * 0..t whatever the indexer says, so the pass is dense causal MLA attention (the
 * short-sequence mode of the DSA report's "Стоимость" section, where attention
 * falls back to the masked dense form): neither the indexer nor a top-k runs; the
 * attention kernel reads keys 0..t as contiguous tiles (no gathers) and writes
 * the index lists 0..t itself.
 *   indices: int32 [B, Lq, k] (as dsa_topk); out: bf16 [B, Lq, H, d_v];
 *   lse: fp32 [B, Lq, H] or NULL.
 * The workspace holds the score matrix (staged) or the candidate lists (fused),
 * then the split-k partials; its contents need not be initialised.
 */
dsa_status dsa_forward(const dsa_indexer_args *iargs, const dsa_attn_args *aargs, int k,
                       int32_t *indices, void *out, float *lse,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * dsa_forward with two extras.
 *   sel_scores:   fp32 [B, Lq, k] or NULL: the indexer score of every selected
 *                 position (as dsa_indexer_topk), e.g. for dsa_indexer_kl_loss_selected.
 *                 When given, the indexer runs even for short sequences.
 *   stage_events: NULL, or four cudaEvent_t handles (created by the caller)
 *                 recorded on `stream` before the indexer, after the indexer,
 *                 after the top-k (on the fused path the second and third
 *                 coincide: the top-k is part of the indexer) and after the
 *                 attention (including its split-k merge).  For short sequences
 *                 without sel_scores the first three coincide (the attention
 *                 writes the index lists).
 */
dsa_status dsa_forward_timed(const dsa_indexer_args *iargs, const dsa_attn_args *aargs, int k,
                             int32_t *indices, float *sel_scores, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream,
                             void *const *stage_events);

/*
 * Forward of the lightning indexer's training loss (section "Как учили
 * индексатор": the indexer learns the main attention's distribution through a
 * KL divergence; in the sparse stage only over the selected positions).
 * For query row (b,i) with the valid selected positions S (indices entries in
 * [0, Lk); others are padding):
 *   a_h[s]  = exp(scale * q[b,i,h,:] . kv[b,s,:] - lse[b,i,h])   (the attention
 *             probabilities of head h, as dsa_sparse_attn computes them);
 *   p[s]    = sum_h a_h[s] / sum_{s' in S} sum_h a_h[s']          (target, L1-normalised);
 *   kl[b,i] = sum_{s in S} p[s] * (log p[s] - log softmax_S(scores[b,i,:])[s]).
 *   args, B, Lq, Lk, indices, k: as dsa_sparse_attn (same shapes and limits);
 *   lse:    fp32 [B, Lq, H], the natural-log log-sum-exp that dsa_sparse_attn
 *           returned for the same q, kv and indices;
 *   scores: fp32 [B, Lq, Lk], the indexer scores (dsa_indexer_scores layout);
 *           only the selected entries are read, and they must be finite;
 *   target: fp32 [B, Lq, k] or NULL: p at each index slot, 0 on padding slots;
 *   kl:     fp32 [B, Lq]: the per-row loss, 0 for a row with no valid entry.
 * The reduction over rows (sum or mean) is left to the caller.  No workspace.
 */
dsa_status dsa_indexer_kl_loss(const dsa_attn_args *args, int B, int Lq, int Lk,
                               const int32_t *indices, int k, const float *lse,
                               const float *scores, float *target, float *kl, void *stream);

/*
 * dsa_indexer_kl_loss with the indexer scores given per index slot instead of as
 * a full matrix: sel_scores fp32 [B, Lq, k], sel_scores[b,i,j] = I[t, indices[b,i,j]]
 * for every valid slot j (padding slots are not read) -- what dsa_forward_timed
 * and dsa_indexer_topk return.  Everything else is dsa_indexer_kl_loss.
 */
dsa_status dsa_indexer_kl_loss_selected(const dsa_attn_args *args, int B, int Lq, int Lk,
                                        const int32_t *indices, int k, const float *lse,
                                        const float *sel_scores, float *target, float *kl, void *stream);

/*
 * Bytes of device workspace the entry point `op` needs for these sizes (0 = none).
 * For DSA_OP_FORWARD, DSA_OP_FORWARD_LOWMEM and DSA_OP_INDEXER_TOPK it assumes
 * H_I = 64, d_I = 128 and q_offset = Lk - Lq (decode, or a prefill chunk);
 * dsa_workspace_size_args gives the exact figure for any indexer arguments.
 * DSA_OP_FORWARD includes the fp32 score matrix, B * Lq * Lk * 4 bytes (4.3 GB
 * at Lq = Lk = 32768).
 */
size_t dsa_workspace_size(dsa_op op, int B, int Lq, int Lk, int k, int H, int d_v);

/* Exact workspace of `op` for these indexer arguments (pointers are not read; 0 for
 * invalid arguments).  H and d_v describe the attention (ignored for
 * DSA_OP_INDEXER_TOPK and DSA_OP_TOPK). */
size_t dsa_workspace_size_args(dsa_op op, const dsa_indexer_args *iargs, int k, int H, int d_v);

/* Human-readable name of a status code (static storage; never NULL). */
const char *dsa_status_string(dsa_status status);

/*
 * Device-side status of this library on the current device: reads (and, when
 * `clear` is non-zero, resets) the word the kernels write when a bounded wait
 * gives up.  Synchronises the device.  Returns DSA_OK or DSA_ERR_TIMEOUT
 * (DSA_ERR_CUDA if the read itself fails).
 */
dsa_status dsa_device_status(int clear);

/*
 * Self-test of the failure path: launches one CTA that waits, with a limit of
 * about `spin_limit` polls, on a barrier that nothing will ever complete, and
 * returns DSA_ERR_TIMEOUT after synchronising if (and only if) the wait gave
 * up and the kernel returned normally.  Clears the device status first and
 * afterwards.  No fault, trap or hang is involved.
 */
dsa_status dsa_selftest_wait_timeout(uint32_t spin_limit, void *stream);

/* Library version: major * 10000 + minor * 100 + patch. */
int dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
