/*
 * dsa.h -- C ABI of libdsa.so: the DeepSeek-Sparse-Attention hot path of GLM-5.2
 * (lightning indexer -> causal top-k -> absorbed sparse MLA, with IndexShare
 * reuse), as hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section) for what each call computes:
 *  [TM] "GLM-5.2 -- Model techniques map", section "Checked in its code":
 *       row "Indexer-selected sparse attention (DeepSeek Sparse Attention)" --
 *       an indexer scores past tokens per head, each query attends only to the
 *       index_topk = 2048 selected tokens; index_n_heads = 32, index_head_dim =
 *       128; the selection is min(index_topk, n) indices as int32 [B, S, topk];
 *       row "QK normalization" -- one indexer key per token, [B, S, 1, D];
 *       row "Multi-head latent attention" -- a 512-dim kv latent plus a 64-dim
 *       RoPE key per token; row "Learnable attention sink" -- plain float32
 *       softmax, no sink; row "Partial RoPE" -- 192 nope + 64 rope dims.
 *  [HA] "GLM 5.2 -- Hermosa AI", section "MLA + DSA with IndexShare" -- a full
 *       layer selects the top 2048 cached tokens per query, the next three
 *       layers reuse that selection; section "78 layers, IndexShare pattern".
 *  [AE] "GLM-5.2 -- LLM architectures explained", section "Modelled costs" --
 *       93 KiB of BF16 cache per token pins the per-layer row of 576 bf16 and the
 *       128-bf16 indexer key on full layers.
 *  [TM] section "inference & serving", inference quantization -- FP8 inference;
 *  [LA] "GLM-5.2 -- LLM atlas", key facts -- precision fp8.  Neither gives a
 *       format: the FP8 variants below (E4M3 with per-row scales) are this
 *       library's reading.
 *
 * Details the pages leave open, fixed here:
 *  - score(t,s) = sum_h w[t,h] * max(0, q_idx[t,h] . k_idx[s]) (post-RoPE
 *    inputs, no extra scale), w float32;
 *  - query t sees cache rows s = 0..t;
 *  - top-k keeps min(topk, t+1) rows, ties go to the lower position, the kept
 *    positions are written in ascending order and padded with -1;
 *  - absorbed MLA: per head the query is [q_lat (d_latent) | q_rope (d_rope)],
 *    logit = scale * (q_lat . c_s + q_rope . r_s) with cache rows [c_s | r_s],
 *    output o = sum_j softmax_j * c_{s_j} (d_latent values per head); the W_UV
 *    up-projection is applied by the caller.
 *
 * Conventions for every call:
 *  - Memory: the caller owns every buffer.  All tensor pointers are DEVICE
 *    pointers unless stated otherwise; the library never allocates, frees or
 *    synchronises inside a compute call.  `stream` is a cudaStream_t (NULL =
 *    legacy default stream); work is enqueued on it and results are valid in
 *    stream order.  Kernels are launched with programmatic dependent launch:
 *    one may start while the previous kernel on the stream finishes and read
 *    the inputs that no kernel of the call writes (the query positions and
 *    sequences, the attention's query tile) before it waits for that kernel.  A kernel of the
 *    caller's that writes those inputs just before the call must therefore not
 *    release its dependents early (a kernel that never executes
 *    griddepcontrol.launch_dependents does not).
 *  - Workspace: `ws` is a device buffer of at least dsa_workspace_bytes(...)
 *    bytes, 256-byte aligned.  Its first 256 bytes hold a status word that
 *    kernels set on device-detected errors (out-of-range positions or indices,
 *    a bounded wait that ran out) and the counters from which the tensor-core
 *    indexer's CTAs claim their work (zero between calls).  Zero the workspace
 *    once with dsa_workspace_init(); read (and clear) the status with
 *    dsa_check_status().  Calls that share a workspace must run one after
 *    another (one stream, or streams ordered by events), never concurrently.
 *    One workspace of dsa_workspace_bytes(DSA_OP_INDEXSHARE_GROUP, ...) bytes
 *    serves the separate calls of a step (dsa_index_scores, dsa_topk,
 *    dsa_sparse_mla_*) on the same queries: every call's scratch leaves alone
 *    the histograms and tickets that the indexer and top-k keep zero.  The
 *    group call lays its scratch out differently (scores first): a workspace
 *    moved between dsa_indexshare_group and the separate calls must be
 *    re-initialised with dsa_workspace_init() in between.
 *  - Errors: invalid arguments are rejected synchronously, before any launch,
 *    with DSA_ERR_INVALID (null pointer, bad size, misaligned row, workspace too
 *    small -> DSA_ERR_WORKSPACE); a launch failure returns DSA_ERR_CUDA.  A call
 *    with n_q == 0 does nothing and returns DSA_OK.
 *  - Fast paths: bf16 or FP8 (E4M3) indexers with 32 heads x 128 dims run on
 *    tcgen05 tensor cores fed by TMA; MLA with bf16 queries, 64 heads x (512 +
 *    64) and a bf16 or packed FP8 latent cache runs on tcgen05 with TMEM
 *    accumulators.  Other shapes and float32 inputs run generic CUDA-core
 *    kernels; the FP8 forms have no generic path (DSA_ERR_UNSUPPORTED).  There
 *    is no CPU path.
 *  - Thread safety: calls are re-entrant; the only global state is one-time
 *    per-device kernel attribute setup.
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
    DSA_ERR_INVALID = 1,     /* bad argument (host) or bad position/index (device) */
    DSA_ERR_UNSUPPORTED = 2, /* valid but unsupported shape/dtype combination */
    DSA_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
    DSA_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    DSA_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (device) */
} dsa_status;

/* DSA_FP8_E4M3: OCP 8-bit float E4M3 (no infinities) with per-row scales: the
 * indexer's q and k (dsa_indexer.q_scale / k_scale) and the MLA latent cache
 * (dsa_mla.kv_dtype, packed rows with their scale). */
typedef enum { DSA_BF16 = 0, DSA_F32 = 1, DSA_FP8_E4M3 = 2 } dsa_dtype;

/* Flags of dsa_indexer.flags and of dsa_topk. */
enum {
    /* dsa_indexer.flags: dsa_index_scores also leaves, in the workspace, the
     * per-query histogram of the first radix digit of the scores it wrote (the
     * first pass of dsa_topk; on the tensor-core path it is built in the
     * epilogue at no extra pass).  The workspace must then be at least
     * dsa_workspace_bytes(DSA_OP_TOPK, ...) bytes.  Honoured only when
     * queries->seq_run is odd (queries not tiled together); ignored otherwise.
     * The histogram region is expected to be zero on entry (no memset per
     * call): dsa_workspace_init zeroes it and dsa_topk zeroes it again once it
     * has used it, so every dsa_index_scores with this flag must be followed by
     * a dsa_topk on the same workspace before the next one (as
     * dsa_indexshare_group does), or the workspace re-initialised. */
    DSA_INDEXER_TOPK_HIST = 1,
    /* dsa_topk flags: the workspace holds that histogram for these scores (the
     * preceding dsa_index_scores on the same scores, queries and workspace had
     * DSA_INDEXER_TOPK_HIST), so the top-k skips its own histogram pass.
     * Ignored, like the indexer flag, when queries->seq_run is even. */
    DSA_TOPK_HIST_FROM_INDEXER = 1
};

/* Operation ids for dsa_workspace_bytes. */
typedef enum {
    DSA_OP_INDEX_SCORES = 0,
    DSA_OP_TOPK = 1,
    DSA_OP_MLA_DECODE = 2,
    DSA_OP_MLA_PREFILL = 3,
    DSA_OP_INDEXSHARE_GROUP = 4,
    DSA_OP_SHARD_MERGE = 5 /* dsa_shard_merge; dsa_workspace_bytes' last argument = shards */
} dsa_op;

/*
 * The query tokens of one call.
 *   n_q      number of query tokens (>= 0)
 *   n_seq    number of sequences (caches), >= 1
 *   max_ctx  L: rows in every cache; each q_pos must be < L
 *   seq_run  a promise that queries come in runs of `seq_run` consecutive
 *            queries sharing one sequence (run r = queries r*seq_run ...); 1 makes
 *            no promise.  The indexer tiles up to gcd(seq_run, 8) queries that
 *            share a cache into one tensor-core tile.  A broken promise is
 *            reported as DSA_ERR_INVALID in the status word.
 *   q_seq    device int32 [n_q]: sequence of each query, in [0, n_seq)
 *   q_pos    device int32 [n_q]: position t of each query, in [0, L); the query
 *            sees rows 0..t of its sequence
 */
typedef struct {
    int32_t n_q;
    int32_t n_seq;
    int32_t max_ctx;
    int32_t seq_run;
    const int32_t *q_seq;
    const int32_t *q_pos;
} dsa_queries;

/*
 * Lightning indexer of one full layer [TM, Indexer-selected sparse attention].
 *   heads, dim    32 and 128 for GLM-5.2 (any positive values on the generic path)
 *   dtype         DSA_BF16 or DSA_F32, for q and k; or DSA_FP8_E4M3 (32 x 128
 *                 only, tensor cores), where the operands are
 *                   q[i,h,d] = e4m3(q[i,h,d]) * q_scale[i*heads + h]
 *                   k[s,d]   = e4m3(k[s,d]) * k_scale[b*ks_seq_stride + s]
 *                 (the FP8 variant: half the key bytes of bf16)
 *   q             [n_q][heads][dim], contiguous, post-RoPE
 *   w             float32 [n_q][heads], contiguous
 *   k             row s of sequence b at k + b*k_seq_stride + s*k_row_stride
 *                 (strides in elements; k_seq_stride 0 = all sequences share one
 *                 cache).  Tensor-core path: row and sequence strides multiple of
 *                 8 elements (16 for FP8), k and q 16-byte aligned.
 *   q_scale       FP8 only: float32 [n_q][heads], or NULL (all 1); positive
 *   k_scale       FP8 only: float32, sequence b's row s at
 *                 k_scale[b*ks_seq_stride + s] (ks_seq_stride 0 = shared), or
 *                 NULL (all 1); positive.  A positive scale factors out of the
 *                 ReLU, which the kernel uses (non-positive scales are not
 *                 supported and give unspecified scores).
 */
typedef struct {
    int32_t heads;
    int32_t dim;
    int32_t dtype;
    int32_t flags; /* DSA_INDEXER_TOPK_HIST or 0 */
    const void *q;
    const float *w;
    const void *k;
    int64_t k_seq_stride;
    int64_t k_row_stride;
    const float *q_scale;  /* FP8 only */
    const float *k_scale;  /* FP8 only */
    int64_t ks_seq_stride; /* FP8 only, elements */
} dsa_indexer;

/*
 * Absorbed MLA of one layer [TM, Multi-head latent attention; Partial RoPE].
 *   heads              64 for GLM-5.2
 *   d_latent, d_rope   512 and 64 for GLM-5.2
 *   dtype              DSA_BF16 or DSA_F32 for q and out (and kv, see kv_dtype)
 *   scale              softmax scale (1/sqrt(192 + 64) for GLM-5.2)
 *   kv_dtype           0 or `dtype`: the cache holds `dtype` values (below);
 *                      DSA_FP8_E4M3: the cache holds packed 8-bit rows, see
 *                      DSA_MLA_FP8_ROW_BYTES (dtype DSA_BF16, 64 x (512 + 64) only,
 *                      else DSA_ERR_UNSUPPORTED).  Every layer of a call agrees.
 *   q                  [n_q][heads][d_latent + d_rope], contiguous
 *   kv                 cache row s of sequence b at kv + b*kv_seq_stride +
 *                      s*kv_row_stride, laid out [c (d_latent) | r (d_rope)];
 *                      tensor-core path: strides multiple of 8 elements, 16-byte
 *                      aligned base, and the sequence stride a whole number of
 *                      rows (or 0) -- the rows are gathered by TMA from one 2-D
 *                      tensor of every sequence's rows (bf16 caches that miss it
 *                      take the generic path).  Packed FP8 rows: strides in bytes,
 *                      multiples of 16, row stride >= DSA_MLA_FP8_ROW_BYTES, the
 *                      sequence stride a whole number of rows (else
 *                      DSA_ERR_UNSUPPORTED)
 *   out                [n_q][heads][d_latent], dtype `dtype`
 *   lse                float32 [n_q][heads] (natural log of the softmax
 *                      normaliser of the scaled logits), or NULL
 */
/*
 * Packed FP8 latent-cache row (kv_dtype = DSA_FP8_E4M3) [TM, inference
 * quantization: FP8 inference; LA, key facts: precision fp8 -- the pages give no
 * format, this one is the library's]:
 *   bytes [0, 512)     E4M3 codes c8[d] of the latent
 *   bytes [512, 640)   the RoPE key r, 64 bf16 values
 *   bytes [640, 644)   float32 row scale sigma (positive, finite)
 *   bytes [644, 656)   unused
 * The latent attended over is c[d] = sigma * e4m3(c8[d]).  The kernel multiplies
 * the exact codes (E4M3 values are exact in fp16) on fp16 tensor cores and applies
 * sigma in fp32: to the row's logit, and to its softmax weight, rounded to fp16
 * once before the product with the codes.
 */
#define DSA_MLA_FP8_ROW_BYTES 656

typedef struct {
    int32_t heads;
    int32_t d_latent;
    int32_t d_rope;
    int32_t dtype;
    float scale;
    int32_t kv_dtype; /* 0 = dtype, or DSA_FP8_E4M3 */
    const void *q;
    const void *kv;
    int64_t kv_seq_stride;
    int64_t kv_row_stride;
    void *out;
    float *lse;
} dsa_mla;

/*
 * Indexer scores [TM, Indexer-selected sparse attention; QK normalization]:
 *   scores[i*ld_scores + s] = sum_h w[i,h] * max(0, q[i,h,:] . k[q_seq[i], s, :])
 * for s <= q_pos[i]; entries s > q_pos[i] are left unspecified.
 *   scores     float32 [n_q][ld_scores], ld_scores >= max_ctx, multiple of 4,
 *              16-byte aligned base
 *   ws         workspace of dsa_workspace_bytes(DSA_OP_INDEX_SCORES, ...) bytes
 * On integer-valued inputs (see the test recipe) every score is exact in float32.
 */
dsa_status dsa_index_scores(const dsa_queries *queries, const dsa_indexer *indexer, float *scores,
                            int64_t ld_scores, void *ws, size_t ws_bytes, void *stream);

/*
 * Causal top-k [TM, Indexer-selected sparse attention: min(index_topk, n)
 * largest scores, int32 indices]: for query i with n = q_pos[i] + 1 visible
 * rows keep k = min(topk, n) positions with the largest scores (ties -> lower
 * position; -0.0 == +0.0), written ascending to idx[i*topk + 0..k-1], the rest
 * of the row set to -1, cnt[i] = k.  Scores must not be NaN.
 *   scores     float32 [n_q][ld_scores] (only s <= q_pos[i] is read),
 *              ld_scores >= max_ctx, multiple of 4, 16-byte aligned base
 *   topk       1 .. 4096
 *   flags      0, or DSA_TOPK_HIST_FROM_INDEXER (see the flag)
 *   idx        int32 [n_q][topk];  cnt  int32 [n_q]
 */
dsa_status dsa_topk(const dsa_queries *queries, const float *scores, int64_t ld_scores,
                    int32_t topk, int32_t flags, int32_t *idx, int32_t *cnt, void *ws,
                    size_t ws_bytes, void *stream);

/*
 * Sparse absorbed MLA, decode schedule [TM, Indexer-selected sparse attention;
 * Multi-head latent attention; Learnable attention sink]: for each query i and
 * head h, attention over the rows idx[i*topk + 0..cnt[i]-1] of its sequence:
 *   l_j = scale * (q_lat[i,h] . c_{s_j} + q_rope[i,h] . r_{s_j}),
 *   out[i,h,:] = sum_j softmax(l)_j c_{s_j},  lse[i,h] = log sum_j exp(l_j).
 * The selected rows are split over several CTAs per query (split-K over rows,
 * partial results in the workspace, then a log-sum-exp merge): the schedule for
 * few queries.  Entries of idx must lie in [0, max_ctx).
 */
dsa_status dsa_sparse_mla_decode(const dsa_queries *queries, const dsa_mla *mla,
                                 const int32_t *idx, const int32_t *cnt, int32_t topk, void *ws,
                                 size_t ws_bytes, void *stream);

/*
 * Same result as dsa_sparse_mla_decode, prefill schedule: one CTA per query
 * walks all of its selected rows with an online softmax (no partials), the
 * schedule for many queries.
 */
dsa_status dsa_sparse_mla_prefill(const dsa_queries *queries, const dsa_mla *mla,
                                  const int32_t *idx, const int32_t *cnt, int32_t topk, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Sparse absorbed MLA for a multi-token-prediction (speculative) iteration
 * [LA, raw config.json fields: index_share_for_mtp_iteration = true -- the
 * tokens of an MTP iteration share the index selection instead of scoring
 * again; HA, "78 layers, IndexShare pattern": one Multi-Token Prediction layer
 * next to the 78].  The pages give only the flag; the reading here: the n_q
 * queries come in groups of `draft_tokens` consecutive queries of one
 * sequence, and every query of group g attends over the one selection
 * idx[g*topk + 0..cnt[g]-1] -- exactly dsa_sparse_mla_decode with the selection
 * row repeated for each query of the group.  The selection was made for a
 * position no later than any query of the group, so it is causal for all of
 * them.
 *   idx        int32 [n_q / draft_tokens][topk];  cnt  int32 [n_q / draft_tokens]
 *   draft_tokens  >= 1 and dividing n_q (else DSA_ERR_INVALID)
 *   ws         dsa_workspace_bytes(DSA_OP_MLA_DECODE, queries, topk, ...) bytes
 * The decode (split-K) schedule runs up to 256 queries, the prefill schedule
 * above.  The queries of a group gather the same rows, so their CTAs read them
 * from L2 after the first.
 */
dsa_status dsa_sparse_mla_mtp(const dsa_queries *queries, const dsa_mla *mla, const int32_t *idx,
                              const int32_t *cnt, int32_t topk, int32_t draft_tokens, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * dsa_sparse_mla_decode without a workspace.  The pages have no counterpart to
 * this call: it exists for callers that cannot allocate device memory where
 * they run attention (a runtime or plugin that hands over only its input and
 * output tensors, or memory that was planned and fixed up front), so they have
 * no workspace to pass.  Same arguments, checks and result as
 * dsa_sparse_mla_decode (tensor-core shape only: bf16 queries and outputs, 64
 * heads, 512 + 64, a bf16 or packed FP8 cache; other shapes return
 * DSA_ERR_UNSUPPORTED), minus `ws`.
 *  - Scratch: a fixed 32 MiB device array inside the library (status word +
 *    split-K partials), held by every GPU that loads the library until the
 *    process exits.  A call needs 256 + n_q * splits * 131,584 bytes, where
 *    splits is the decode plan's split count (at most SMs / n_q, 1 for 75 or
 *    more queries on 148 SMs, and no partials at all with one split): at most
 *    about 19.5 MB on a B200.  A call whose plan needs more than the array (a
 *    GPU with more than 255 SMs) is rejected with DSA_ERR_WORKSPACE before any
 *    launch.
 *  - Set-up: each call made outside stream capture looks up the array's device
 *    address (cudaGetSymbolAddress) with the current device; calls made while
 *    the stream is capturing reuse the address looked up last on that device,
 *    so make one call on each device before capturing it.
 *  - Every call on a device shares the one array, so calls that overlap on the
 *    GPU (other streams, other host threads) race; serialise them.
 *  - Device-detected errors (an index or count out of range, a bounded wait
 *    that ran out) go to the array's status word, which keeps the first error
 *    until dsa_noalloc_check_status reads and clears it.
 *  - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call.
 */
dsa_status dsa_sparse_mla_decode_noalloc(const dsa_queries *queries, const dsa_mla *mla,
                                         const int32_t *idx, const int32_t *cnt, int32_t topk,
                                         void *stream);

/*
 * Status of the dsa_sparse_mla_decode_noalloc calls made on the current device
 * (no counterpart on the pages): synchronises `stream`, reads the status word of
 * the library's fixed scratch array, clears it, and returns it (DSA_OK when no
 * kernel reported an error since the last read).  Allocates nothing.
 */
dsa_status dsa_noalloc_check_status(void *stream);

/*
 * IndexShare group [HA, MLA + DSA with IndexShare]: layer 0 (the full layer)
 * runs dsa_index_scores -> dsa_topk -> sparse MLA; layers 1..n_layers-1 run
 * sparse MLA with layer 0's idx/cnt on their own queries and caches, without
 * re-scoring.  The scores live in the workspace.
 *   indexer   the full layer's indexer
 *   layers    host array of n_layers (1..4) dsa_mla descriptions (same heads,
 *             dims, dtype and scale)
 *   idx, cnt  outputs as in dsa_topk
 * The decode or prefill MLA schedule is chosen from n_q.
 */
dsa_status dsa_indexshare_group(const dsa_queries *queries, const dsa_indexer *indexer,
                                const dsa_mla *layers, int32_t n_layers, int32_t topk,
                                int32_t *idx, int32_t *cnt, void *ws, size_t ws_bytes,
                                void *stream);

/*
 * dsa_indexshare_group with the step's inputs and outputs in host memory (the
 * call a host-driven decode loop makes each step; the caches, the indexer keys
 * and the workspace stay on the device).  All on `stream`, in this order:
 *   1. in_bytes bytes from h_in (host) to d_in (device),
 *   2. dsa_indexshare_group on the descriptors, which point into d_in and
 *      d_out (or anywhere else on the device),
 *   3. out_bytes bytes from d_out (device) to h_out (host).
 * Every argument is checked before anything is enqueued (same results as
 * dsa_indexshare_group; DSA_ERR_INVALID also for a null buffer with a
 * non-zero size); n_q = 0 enqueues the two copies only.  The call returns once
 * the work is enqueued: synchronise `stream` before reading h_out.  With
 * page-locked (pinned) host buffers the copies are asynchronous; with pageable
 * ones the driver stages them and the call may wait for them.  The caller
 * owns all four buffers; h_in must stay unchanged and h_out unread until the
 * stream has passed the call.
 */
dsa_status dsa_indexshare_group_host(const dsa_queries *queries, const dsa_indexer *indexer,
                                     const dsa_mla *layers, int32_t n_layers, int32_t topk,
                                     int32_t *idx, int32_t *cnt, void *ws, size_t ws_bytes,
                                     const void *h_in, void *d_in, size_t in_bytes,
                                     void *h_out, const void *d_out, size_t out_bytes,
                                     void *stream);

/*
 * Key-range sharding of one long sequence over several GPUs.  The pages name
 * attention data parallelism only ["GLM-5.2 -- Model techniques map",
 * inference & serving]; splitting one sequence's cache by contiguous key
 * ranges is this library's reading of how a 1M-token context
 * ["GLM 5.2 -- Hermosa AI", "MLA + DSA with IndexShare": 1,048,576 tokens]
 * spreads over GPUs, and it computes exactly the single-GPU result:
 *   rank g holds rows [row_begin_g, row_end_g) of the sequence (contiguous,
 *   in rank order) and, per query:
 *   1. dsa_index_scores + dsa_topk on its shard (positions shard-relative);
 *   2. dsa_shard_candidates: its <= topk (score, position) candidates;
 *   3. an all-gather of every rank's candidates (the caller's collective);
 *   4. dsa_shard_merge: the global selection (the top-k of all candidates,
 *      ties to the lower position) and this rank's part of it;
 *   5. dsa_sparse_mla_decode on its shard with that part;
 *   6. an all-gather of the ranks' outputs, lse and part counts;
 *   7. dsa_shard_combine: the log-sum-exp merge of the ranks' attentions.
 * A row of the global top-k that lies in shard g is among shard g's top-k (its
 * rank inside the shard is no worse than its global rank), so step 4 sees
 * every row it needs.  Every query must see at least one row of every shard
 * (decode at the end of the sequence).
 */

/*
 * Step 2: candidates of this rank's local selection.
 *   scores, ld_scores  the local scores (queries->max_ctx = shard rows)
 *   idx, cnt           the local top-k (shard-relative, ascending, -1 padded)
 *   row_offset         the shard's first row in the sequence
 *   cand_score         float32 [n_q][topk]: the selected rows' scores, 0 after cnt
 *   cand_pos           int32 [n_q][topk]: their sequence positions, -1 after cnt
 *   ws                 at least 256 bytes (status word)
 */
dsa_status dsa_shard_candidates(const dsa_queries *queries, const float *scores, int64_t ld_scores,
                                const int32_t *idx, const int32_t *cnt, int32_t topk, int32_t row_offset,
                                float *cand_score, int32_t *cand_pos, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 4: merge of the gathered candidates (n_shards ranks, rank order).
 *   cand_score, cand_pos  [n_shards][n_q][topk] as gathered from step 2
 *   idx, cnt              the global selection: sequence positions, ascending,
 *                         -1 padded; cnt = min(topk, candidates)
 *   row_begin, row_end    this rank's rows
 *   local_idx, local_cnt  [n_q][topk], [n_q]: the selected rows in
 *                         [row_begin, row_end), shard-relative, ascending,
 *                         -1 padded (the selection step 5 attends over)
 *   ws                    dsa_workspace_bytes(DSA_OP_SHARD_MERGE, queries, topk,
 *                         0, 0, n_shards) bytes, initialised once
 */
dsa_status dsa_shard_merge(const dsa_queries *queries, int32_t n_shards, const float *cand_score,
                           const int32_t *cand_pos, int32_t topk, int32_t row_begin, int32_t row_end, int32_t *idx,
                           int32_t *cnt, int32_t *local_idx, int32_t *local_cnt, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * Step 7: o = sum_g exp(lse_g - lse) o_g, lse = log sum_g exp(lse_g), over the
 * parts g with part_cnt[g][i] > 0 (the others are ignored, whatever their
 * out/lse hold).
 *   part_out   bf16 [n_parts][n_q][heads][d_latent] (8-byte aligned)
 *   part_lse   float32 [n_parts][n_q][heads];  part_cnt  int32 [n_parts][n_q]
 *   out        bf16 [n_q][heads][d_latent];  lse  float32 [n_q][heads] or NULL
 *   heads even, d_latent a multiple of 4 up to 512 (else DSA_ERR_UNSUPPORTED)
 */
dsa_status dsa_shard_combine(const dsa_queries *queries, int32_t n_parts, int32_t heads, int32_t d_latent,
                             const void *part_out, const float *part_lse, const int32_t *part_cnt, void *out,
                             float *lse, void *stream);

/*
 * Producers around the path (GLM-5.2 shapes only: latent 512, RoPE key 64,
 * indexer key 128, no-RoPE query part 192, value 256) ["GLM-5.2 -- Model
 * techniques map", "Checked in its code": Multi-head latent attention --
 * kv_a_proj_with_mqa maps the hidden state to the 512-dim latent plus the
 * 64-dim RoPE key, kv_a_layernorm (RMSNorm) normalises the latent, kv_b_proj
 * holds per head a 192-dim no-RoPE key part (W_UK) and a 256-dim value (W_UV);
 * QK normalization -- the indexer key is k_norm(wk(h)), k_norm a LayerNorm;
 * Partial RoPE; "GLM 5.2 -- Hermosa AI", "MLA + DSA with IndexShare": RoPE
 * theta 8e6; "GLM-5.2 -- LLM atlas", raw config.json fields: rope_interleave
 * and indexer_rope_interleave true, rms_norm_eps].  Readings where the pages
 * are silent: RoPE turns adjacent pairs (x[2i], x[2i+1]) of a 64-wide RoPE part
 * by pos * theta^(-2i/64); the indexer key's RoPE part is its last 64 dims;
 * LayerNorm has a weight and a bias, RMSNorm a weight.  Dense contractions run
 * on tcgen05 tensor cores (bf16 operands, fp32 sums), bf16 results.
 */

/* One batch of tokens whose cache rows are written. */
typedef struct {
    int32_t n_tok;            /* tokens (>= 0) */
    int32_t hidden;           /* hidden size (6144 for GLM-5.2), a multiple of 8, >= 64 */
    const void *h;            /* bf16 [n_tok][hidden] hidden states, row stride h_row_stride
                                 (elements, multiple of 8), 16-byte aligned */
    int64_t h_row_stride;
    const void *w;            /* bf16 [704][hidden] weights in the [out][in] layout: rows 0..511
                                 the latent and 512..575 the RoPE key (kv_a_proj_with_mqa), rows
                                 576..703 the indexer key (wk); 16-byte aligned */
    const float *rms_weight;  /* [512] kv_a_layernorm weight */
    const float *ln_weight;   /* [128] k_norm weight */
    const float *ln_bias;     /* [128] k_norm bias */
    const int32_t *tok_seq;   /* device [n_tok]: sequence of each token, in [0, n_seq) */
    const int32_t *tok_pos;   /* device [n_tok]: its position = its cache row and RoPE position */
    int32_t n_seq, max_ctx;
    void *kv;                 /* bf16 latent cache [c | r] (the layout dsa_mla reads), or NULL */
    int64_t kv_seq_stride, kv_row_stride;     /* elements */
    void *k_idx;              /* bf16 indexer-key cache [128] rows, or NULL (not both NULL) */
    int64_t k_seq_stride, k_row_stride;       /* elements */
    float eps;                /* 1e-5 for GLM-5.2 (rms_norm_eps; also the LayerNorm's) */
    float rope_theta;         /* 8e6 for GLM-5.2 */
} dsa_cache_writer;

/*
 * Cache rows of a batch of tokens: y = h . W^T (704 outputs per token), then
 *   kv[seq][pos]    = [ RMSNorm(y[0:512]) * rms_weight | RoPE(y[512:576], pos) ]
 *   k_idx[seq][pos] = LayerNorm(y[576:704]) * ln_weight + ln_bias, its last 64
 *                     dims turned by RoPE(pos)
 *   ws   dsa_cache_writer_workspace_bytes(n_tok, hidden) bytes, 256-byte aligned
 *        (status word + split-K partials of y)
 * Out-of-range tok_seq / tok_pos skip the token and set DSA_ERR_INVALID in the
 * workspace status word.
 */
dsa_status dsa_write_cache_rows(const dsa_cache_writer *writer, void *ws, size_t ws_bytes, void *stream);
size_t dsa_cache_writer_workspace_bytes(int32_t n_tok, int32_t hidden);

/*
 * Absorbed MLA queries: per query i and head h
 *   q_out[i][h][0:512]   = W_UK[h]^T q_nope[i][h]      (the no-RoPE key up-projection
 *                                                      folded into the query)
 *   q_out[i][h][512:576] = RoPE(q_rope[i][h], pos[i])
 *   q_nope  bf16 [n_q][heads][192];  q_rope  bf16 [n_q][heads][64] (before RoPE)
 *   w_uk_t  bf16 [heads][512][192]: W_UK[h] transposed (row j holds the weights
 *           of latent dim j), the K-major layout the tensor cores read
 *   pos     device int32 [n_q];  q_out  bf16 [n_q][heads][576] (the dsa_mla query)
 *   ws      at least 256 bytes (status word)
 */
dsa_status dsa_absorb_queries(int32_t n_q, int32_t heads, const void *q_nope, const void *q_rope, const void *w_uk_t,
                              const int32_t *pos, float rope_theta, void *q_out, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * Value up-projection of the absorbed attention output: per query i and head h
 *   out[i][h][0:256] = W_UV[h] o_lat[i][h]
 *   o_lat  bf16 [n_q][heads][512] (dsa_mla's out);  w_uv  bf16 [heads][256][512]
 *   out    bf16 [n_q][heads][256];  ws  at least 256 bytes (status word)
 */
dsa_status dsa_up_project(int32_t n_q, int32_t heads, const void *o_lat, const void *w_uv, void *out, void *ws,
                          size_t ws_bytes, void *stream);

/*
 * Upper bound of the workspace bytes an operation needs (host only).
 *   op         a dsa_op value
 *   queries    n_q and max_ctx are read (pointers are not)
 *   topk       selection size (ignored for DSA_OP_INDEX_SCORES)
 *   mla_heads, d_latent, n_layers   MLA shape (ignored where no MLA runs)
 * Returns 0 for an unknown op.
 */
size_t dsa_workspace_bytes(int32_t op, const dsa_queries *queries, int32_t topk, int32_t mla_heads,
                           int32_t d_latent, int32_t n_layers);

/* Zero a whole workspace, status word included (async on `stream`).  Call
 * once after allocating it (and after any failed call that may have left it
 * half-updated). */
dsa_status dsa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronise `stream`, read the workspace status word, clear it, and return
 * it (DSA_OK when no kernel reported an error).  The one synchronising call.
 */
dsa_status dsa_check_status(void *ws, void *stream);

/* Human-readable name of a status code (static string). */
const char *dsa_status_str(dsa_status status);

/*
 * Diagnostic (no counterpart on the pages): exercises the device-side bounded
 * wait every kernel of this library uses.  Launches one thread that waits on a
 * shared-memory barrier nothing completes, with the library's wait routine and
 * a limit of `limit_ns` nanoseconds (at most 2 s, the limit the kernels use);
 * when the limit runs out the wait gives up, the thread writes
 * DSA_ERR_TIMEOUT into the workspace status word and exits, and the context
 * stays usable.  Read the result with dsa_check_status().  Nothing else is
 * launched or touched; no copy or tensor-core work is in flight during the
 * wait.  DSA_ERR_INVALID for a null or too-small workspace or a limit above
 * 2 s.
 */
dsa_status dsa_debug_bounded_wait(void *ws, size_t ws_bytes, uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
