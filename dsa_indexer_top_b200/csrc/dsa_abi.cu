// dsa_abi.cu -- the extern "C" entry points declared in include/dsa.h:
// argument validation, workspace layout, TMA descriptor encoding and dispatch to
// the kernels.  No allocation, no synchronisation (except dsa_check_status).
#include <algorithm>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "abi_checks.cuh"
#include "tma_encode.cuh"
#include "dsa.h"
#include "kernels.cuh"

using namespace dsa;

namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kDecodeMaxQueries = 256;  // IndexShare group: split-K MLA up to this many queries

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int64_t round4(int64_t x) { return (x + 3) & ~static_cast<int64_t>(3); }

int num_sms_current() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

EncodeTiledFn encode_fn() { return tma_encode_fn(); }

uint32_t *status_word(void *ws) { return static_cast<uint32_t *>(ws); }

bool ws_ok(void *ws, size_t ws_bytes, size_t need) {
    return ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 && ws_bytes >= need;
}

bool indexer_tc_ok(const dsa_indexer *ix) {
    // TMA strides are multiples of 16 bytes: 8 bf16 or 16 FP8 elements
    const int64_t al = ix->dtype == DSA_FP8_E4M3 ? 16 : 8;
    return (ix->dtype == DSA_BF16 || ix->dtype == DSA_FP8_E4M3) && ix->heads == kIdxHeads && ix->dim == kIdxDim &&
           aligned16(ix->q) && aligned16(ix->k) && ix->k_row_stride % al == 0 && ix->k_seq_stride % al == 0 &&
           ix->k_row_stride >= kIdxDim;
}

size_t ws_index_scores() { return kStatusBytes; }
size_t ws_topk(int n_q, int max_ctx) { return kStatusBytes + align256(topk_scratch_bytes(n_q, max_ctx)); }
int decode_splits(int topk) { return mla_max_splits(topk); }
// The histograms and tickets that dsa_index_scores / dsa_topk keep zero between
// calls head the scratch; the decode attention's partials start after them, so
// the separate calls of a step can share one workspace.
size_t ws_zeroed_head(int n_q) { return align256(topk_zeroed_bytes(n_q)); }
size_t ws_mla_partials(int n_q, int topk, int n_layers) {
    const int ns = decode_splits(topk);
    return ns > 1 ? align256(mla_partial_bytes(n_layers, n_q, ns)) : 0;
}
size_t ws_mla_decode(int n_q, int topk, int n_layers) {
    const size_t part = ws_mla_partials(n_q, topk, n_layers);
    return kStatusBytes + (part ? ws_zeroed_head(n_q) + part : 0);
}
size_t ws_scores(int n_q, int max_ctx) {
    return align256(static_cast<size_t>(n_q) * round4(max_ctx) * sizeof(float));
}
bool group_uses_decode(int n_q) { return n_q <= kDecodeMaxQueries; }
// dsa_shard_merge: [status][merged scores][merged positions][merged counts - 1]
// [top-k of the merged list: indices, counts][top-k scratch of the merged list]
int64_t shard_merged_ld(int n_shards, int topk) { return round4(static_cast<int64_t>(n_shards) * topk); }
struct ShardMergeLayout {
    size_t score, pos, last, sel, sel_cnt, topk_scratch, total;
};
ShardMergeLayout shard_merge_layout(int n_q, int n_shards, int topk) {
    const int64_t ld = shard_merged_ld(n_shards, topk);
    ShardMergeLayout l;
    size_t o = kStatusBytes;
    l.score = o;
    o += align256(static_cast<size_t>(n_q) * ld * sizeof(float));
    l.pos = o;
    o += align256(static_cast<size_t>(n_q) * ld * sizeof(int32_t));
    l.last = o;
    o += align256(static_cast<size_t>(n_q) * sizeof(int32_t));
    l.sel = o;
    o += align256(static_cast<size_t>(n_q) * topk * sizeof(int32_t));
    l.sel_cnt = o;
    o += align256(static_cast<size_t>(n_q) * sizeof(int32_t));
    l.topk_scratch = o;
    o += align256(topk_scratch_bytes(n_q, static_cast<int>(ld)));
    l.total = o;
    return l;
}
size_t ws_group(int n_q, int max_ctx, int topk, int n_layers) {
    size_t b = kStatusBytes + ws_scores(n_q, max_ctx) + align256(topk_scratch_bytes(n_q, max_ctx));
    if (group_uses_decode(n_q)) b += ws_mla_partials(n_q, topk, n_layers);  // after the whole top-k scratch
    return b;
}

// ------------------------------------------------------------------ indexer
dsa_status do_index_generic(const dsa_queries *qs, const dsa_indexer *ix, float *scores, int64_t ld,
                            uint32_t *status, cudaStream_t st);

// ghist: non-null to leave the top-k first-digit histograms there.
dsa_status do_index_scores(const dsa_queries *qs, const dsa_indexer *ix, float *scores, int64_t ld,
                           uint32_t *status, uint32_t *ghist, cudaStream_t st) {
    // the histograms are left only when queries are not tiled together (odd
    // seq_run: one query per tensor-core tile, where the epilogue builds them)
    // (the histograms are zero on entry: see topk_scratch_bytes)
    if ((qs->seq_run & 1) == 0) ghist = nullptr;
    bool hist_done = false;
    dsa_status s = DSA_OK;
    const int n_cache = ix->k_seq_stride == 0 ? 1 : qs->n_seq;
    if (indexer_tc_ok(ix)) {
        EncodeTiledFn enc = encode_fn();
        if (!enc) return DSA_ERR_CUDA;
        CUtensorMap tk, tq;
        // bf16: boxes of 64 values; FP8 (E4M3 bytes, mapped as uint8): boxes of 128
        const bool f8 = ix->dtype == DSA_FP8_E4M3;
        const int esz = f8 ? 1 : 2;
        const CUtensorMapDataType dt = f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const cuuint32_t box_x = f8 ? 128 : 64;
        {
            cuuint64_t dims[3] = {static_cast<cuuint64_t>(kIdxDim), static_cast<cuuint64_t>(qs->max_ctx),
                                  static_cast<cuuint64_t>(n_cache)};
            const int64_t seq_stride = ix->k_seq_stride == 0 ? ix->k_row_stride * qs->max_ctx : ix->k_seq_stride;
            cuuint64_t strides[2] = {static_cast<cuuint64_t>(ix->k_row_stride * esz),
                                     static_cast<cuuint64_t>(seq_stride * esz)};
            cuuint32_t box[3] = {box_x, 128, 1};
            cuuint32_t es[3] = {1, 1, 1};
            if (enc(&tk, dt, 3, const_cast<void *>(ix->k), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return DSA_ERR_INVALID;
        }
        int G = 1;
        while (G < 8 && qs->seq_run % (G * 2) == 0) G *= 2;
        {
            cuuint64_t dims[2] = {static_cast<cuuint64_t>(kIdxDim), static_cast<cuuint64_t>(qs->n_q) * kIdxHeads};
            cuuint64_t strides[1] = {static_cast<cuuint64_t>(kIdxDim * esz)};
            cuuint32_t box[2] = {box_x, static_cast<cuuint32_t>(32 * G)};
            cuuint32_t es[2] = {1, 1};
            if (enc(&tq, dt, 2, const_cast<void *>(ix->q), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return DSA_ERR_INVALID;
        }
        IdxTcArgs a;
        a.w = ix->w;
        a.q_seq = qs->q_seq;
        a.q_pos = qs->q_pos;
        a.scores = scores;
        a.ld = ld;
        a.status = status;
        a.n_q = qs->n_q;
        a.n_seq = qs->n_seq;
        a.L = qs->max_ctx;
        a.k_shared = ix->k_seq_stride == 0 ? 1 : 0;
        a.tiles_per_group = (qs->max_ctx + 127) / 128;
        const long long groups = (qs->n_q + G - 1) / G;
        a.total_items = groups * a.tiles_per_group;
        a.ghist = (ghist && G == 1) ? ghist : nullptr;  // fused into the epilogue
        // Claimed work only where a claim rarely crosses into another query: one
        // bf16 query per tile and at least 4096 key tiles per query.  A query
        // change costs the CTA a pipeline drain for the new query tile and a
        // histogram flush, which outweighs the balance on shorter contexts and on
        // the FP8 form's smaller tiles (measured); those keep contiguous ranges.
        a.work = (!f8 && G == 1 && a.tiles_per_group >= kIdxDynamicMinTiles)
                     ? reinterpret_cast<unsigned long long *>(reinterpret_cast<uint8_t *>(status) + kIdxWorkOffset)
                     : nullptr;
        a.q_scale = f8 ? ix->q_scale : nullptr;
        a.k_scale = f8 ? ix->k_scale : nullptr;
        a.ks_seq_stride = f8 ? ix->ks_seq_stride : 0;
        hist_done = a.ghist != nullptr;
        s = launch_idx_score_tc(G, f8, tk, tq, a, num_sms_current(), st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
    } else if (ix->dtype == DSA_FP8_E4M3) {
        s = DSA_ERR_UNSUPPORTED;  // FP8 runs on the tensor-core path only
    } else {
        s = do_index_generic(qs, ix, scores, ld, status, st);
    }
    if (s != DSA_OK || !ghist || hist_done) return s;
    // histogram pass over the scores just written (generic CUDA-core path)
    TopkArgs t = {};
    t.scores = scores;
    t.ld = ld;
    t.q_pos = qs->q_pos;
    t.status = status;
    t.n_q = qs->n_q;
    t.L = qs->max_ctx;
    t.topk = 0;
    t.ghist = ghist;
    return launch_topk_hist(t, num_sms_current(), st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status do_index_generic(const dsa_queries *qs, const dsa_indexer *ix, float *scores, int64_t ld,
                            uint32_t *status, cudaStream_t st) {
    const size_t smem = sizeof(float) * (static_cast<size_t>(ix->heads) * ix->dim + ix->heads);
    if (smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
    IdxGenericArgs g;
    g.q = ix->q;
    g.w = ix->w;
    g.k = ix->k;
    g.k_seq_stride = ix->k_seq_stride;
    g.k_row_stride = ix->k_row_stride;
    g.q_seq = qs->q_seq;
    g.q_pos = qs->q_pos;
    g.scores = scores;
    g.ld = ld;
    g.status = status;
    g.n_q = qs->n_q;
    g.n_seq = qs->n_seq;
    g.L = qs->max_ctx;
    g.heads = ix->heads;
    g.dim = ix->dim;
    g.is_bf16 = ix->dtype == DSA_BF16;
    return launch_idx_score_generic(g, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status check_indexer(const dsa_queries *qs, const dsa_indexer *ix) {
    if (!ix || !ix->q || !ix->w || !ix->k) return DSA_ERR_INVALID;
    if (ix->heads < 1 || ix->dim < 1 ||
        (ix->dtype != DSA_BF16 && ix->dtype != DSA_F32 && ix->dtype != DSA_FP8_E4M3))
        return DSA_ERR_INVALID;
    if (ix->k_row_stride < ix->dim || ix->k_seq_stride < 0) return DSA_ERR_INVALID;
    if (ix->dtype == DSA_FP8_E4M3) {
        if (ix->ks_seq_stride < 0 || (ix->k_scale && ix->ks_seq_stride != 0 && ix->ks_seq_stride < qs->max_ctx))
            return DSA_ERR_INVALID;
        if (!indexer_tc_ok(ix)) return DSA_ERR_UNSUPPORTED;  // 32 heads x 128 dims, aligned, TMA strides
    }
    if (ix->k_seq_stride != 0 && ix->k_seq_stride < ix->k_row_stride * qs->max_ctx) return DSA_ERR_INVALID;
    return DSA_OK;
}

// ------------------------------------------------------------------ top-k
dsa_status do_topk(const dsa_queries *qs, const float *scores, int64_t ld, int topk, int32_t *idx,
                   int32_t *cnt, uint32_t *status, void *scratch, bool hist_ready, cudaStream_t st,
                   bool pos_early = true) {
    TopkArgs a = {};
    a.scores = scores;
    a.ld = ld;
    a.q_pos = qs->q_pos;
    a.idx = idx;
    a.cnt = cnt;
    a.status = status;
    a.n_q = qs->n_q;
    a.L = qs->max_ctx;
    a.topk = topk;
    a.hist_ready = (hist_ready && (qs->seq_run & 1)) ? 1 : 0;
    a.pos_early = pos_early ? 1 : 0;
    a.ghist = nullptr;
    a.gticket = nullptr;
    a.gcount = nullptr;
    a.gcand = nullptr;
    topk_bind_scratch(a, scratch);
    return launch_topk(a, num_sms_current(), st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

bool scores_ok(const float *scores, int64_t ld, int max_ctx) {
    return scores && aligned16(scores) && ld >= max_ctx && ld % 4 == 0;
}

// ------------------------------------------------------------------ MLA
dsa_status do_mla(const dsa_queries *qs, const dsa_mla *layers, int n_layers, const int32_t *idx,
                  const int32_t *cnt, int topk, bool decode, uint8_t *scratch, uint32_t *status,
                  cudaStream_t st, int sel_group = 1) {
    MlaArgs a;
    std::memset(&a, 0, sizeof(a));
    a.sel_group = sel_group;
    for (int l = 0; l < n_layers; ++l) {
        a.layer[l].q = layers[l].q;
        a.layer[l].kv = layers[l].kv;
        a.layer[l].out = layers[l].out;
        a.layer[l].lse = layers[l].lse;
    }
    const dsa_mla &m = layers[0];
    a.n_layers = n_layers;
    a.kv_seq_stride = m.kv_seq_stride;
    a.kv_row_stride = m.kv_row_stride;
    a.q_seq = qs->q_seq;
    a.idx = idx;
    a.cnt = cnt;
    a.topk = topk;
    a.n_q = qs->n_q;
    a.n_seq = qs->n_seq;
    a.L = qs->max_ctx;
    a.heads = m.heads;
    a.d_lat = m.d_latent;
    a.d_rope = m.d_rope;
    a.scale = m.scale;
    a.is_bf16 = m.dtype == DSA_BF16;
    a.kv_fp8 = mla_kv_fp8(&m) ? 1 : 0;
    a.status = status;
    bool tc = true;
    for (int l = 0; l < n_layers; ++l) tc = tc && mla_tc_ok(&layers[l]);
    tc = tc && mla_tc_rows_ok(&m, qs->n_seq, qs->max_ctx);
    if (a.kv_fp8 && !tc) return DSA_ERR_UNSUPPORTED;  // packed FP8 caches: tensor-core path only
    if (tc) {
        MlaMaps maps;
        std::memset(&maps, 0, sizeof(maps));
        if (!encode_mla_maps(a, maps)) return DSA_ERR_CUDA;
        int n_splits, cpc;
        mla_plan(qs->n_q, n_layers, topk, decode, num_sms_current(), kMlaMaxSplits, n_splits, cpc);
        a.n_splits = n_splits;
        a.chunks_per_cta = cpc;
        if (n_splits > 1) {
            a.part_o = reinterpret_cast<float *>(scratch);
            const size_t rows = static_cast<size_t>(n_layers) * qs->n_q * n_splits * kMlaHeads;
            a.part_ml = reinterpret_cast<float *>(scratch + rows * kLatent * sizeof(float));
            if (launch_mla_tc(a, maps, st) != cudaSuccess) return DSA_ERR_CUDA;
            return launch_mla_combine(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
        }
        return launch_mla_tc(a, maps, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
    }
    const size_t smem = sizeof(float) * (static_cast<size_t>(m.d_latent + m.d_rope) + topk);
    if (smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
    return launch_mla_generic(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

namespace {
// An NVTX range around each compute entry point (header-only NVTX v3: without a
// profiler attached a push/pop is a few nanoseconds of host time).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

namespace {
// Every argument check of the group call (nothing is enqueued before they pass).
dsa_status group_check(const dsa_queries *queries, const dsa_indexer *indexer, const dsa_mla *layers,
                       int32_t n_layers, int32_t topk, const int32_t *idx, const int32_t *cnt, void *ws,
                       size_t ws_bytes) {
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt) return DSA_ERR_INVALID;
    dsa_status s = check_indexer(queries, indexer);
    if (s != DSA_OK) return s;
    s = check_mla_layers(layers, n_layers);
    if (s != DSA_OK) return s;
    if (!ws_ok(ws, ws_bytes, ws_group(queries->n_q, queries->max_ctx, topk, n_layers))) return DSA_ERR_WORKSPACE;
    return DSA_OK;
}

// The group call's launches (arguments already checked, n_q > 0).
dsa_status group_launch(const dsa_queries *queries, const dsa_indexer *indexer, const dsa_mla *layers,
                        int32_t n_layers, int32_t topk, int32_t *idx, int32_t *cnt, void *ws, cudaStream_t st) {
    dsa_status s;
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *scores = reinterpret_cast<float *>(base + kStatusBytes);
    const int64_t ld = round4(queries->max_ctx);
    uint8_t *topk_scratch = base + kStatusBytes + ws_scores(queries->n_q, queries->max_ctx);
    uint8_t *scratch = topk_scratch + align256(topk_scratch_bytes(queries->n_q, queries->max_ctx));
    // the first-digit histograms of top-k come out of the indexer (ghist heads the top-k scratch)
    s = do_index_scores(queries, indexer, scores, ld, status_word(ws), reinterpret_cast<uint32_t *>(topk_scratch), st);
    if (s != DSA_OK) return s;
    s = do_topk(queries, scores, ld, topk, idx, cnt, status_word(ws), topk_scratch, true, st);
    if (s != DSA_OK) return s;
    return do_mla(queries, layers, n_layers, idx, cnt, topk, group_uses_decode(queries->n_q), scratch,
                  status_word(ws), st);
}

}  // namespace

extern "C" {

const char *dsa_status_str(dsa_status s) {
    switch (s) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID: return "DSA_ERR_INVALID";
        case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
        case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    }
    return "DSA_ERR_UNKNOWN";
}

size_t dsa_workspace_bytes(int32_t op, const dsa_queries *qs, int32_t topk, int32_t mla_heads, int32_t d_latent,
                           int32_t n_layers) {
    (void)mla_heads;
    (void)d_latent;
    if (!qs) return 0;
    const int n_q = qs->n_q > 0 ? qs->n_q : 0;
    switch (op) {
        case DSA_OP_INDEX_SCORES: return ws_index_scores();
        case DSA_OP_TOPK: return ws_topk(n_q, qs->max_ctx > 0 ? qs->max_ctx : 1);
        case DSA_OP_MLA_DECODE: return ws_mla_decode(n_q, topk > 0 ? topk : 1, 1);
        case DSA_OP_MLA_PREFILL: return kStatusBytes;
        case DSA_OP_INDEXSHARE_GROUP:
            return ws_group(n_q, qs->max_ctx > 0 ? qs->max_ctx : 1, topk > 0 ? topk : 1,
                            n_layers > 0 ? n_layers : 1);
        case DSA_OP_SHARD_MERGE:  // the last argument is the number of shards
            return shard_merge_layout(n_q, n_layers > 0 ? n_layers : 1, topk > 0 ? topk : 1).total;
    }
    return 0;
}

dsa_status dsa_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws_ok(ws, ws_bytes, kStatusBytes)) return DSA_ERR_WORKSPACE;
    return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK
                                                                                               : DSA_ERR_CUDA;
}

dsa_status dsa_debug_bounded_wait(void *ws, size_t ws_bytes, uint64_t limit_ns, void *stream) {
    if (!ws_ok(ws, ws_bytes, kStatusBytes)) return DSA_ERR_INVALID;
    if (limit_ns > kDeviceWaitLimitNs) return DSA_ERR_INVALID;
    return launch_bounded_wait_probe(status_word(ws), limit_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DSA_OK
               : DSA_ERR_CUDA;
}

dsa_status dsa_check_status(void *ws, void *stream) {
    if (!ws) return DSA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (v != 0 && cudaMemsetAsync(ws, 0, sizeof(v), st) != cudaSuccess) return DSA_ERR_CUDA;
    return static_cast<dsa_status>(v);
}

dsa_status dsa_index_scores(const dsa_queries *queries, const dsa_indexer *indexer, float *scores,
                            int64_t ld_scores, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_index_scores");
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (!ws_ok(ws, ws_bytes, ws_index_scores())) return DSA_ERR_WORKSPACE;
    dsa_status s = check_indexer(queries, indexer);
    if (s != DSA_OK) return s;
    if (!scores_ok(scores, ld_scores, queries->max_ctx)) return DSA_ERR_INVALID;
    const bool hist = (indexer->flags & DSA_INDEXER_TOPK_HIST) != 0;
    if (indexer->flags & ~DSA_INDEXER_TOPK_HIST) return DSA_ERR_INVALID;
    if (hist && !ws_ok(ws, ws_bytes, ws_topk(queries->n_q, queries->max_ctx))) return DSA_ERR_WORKSPACE;
    if (queries->n_q == 0) return DSA_OK;
    uint32_t *ghist = hist ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kStatusBytes) : nullptr;
    return do_index_scores(queries, indexer, scores, ld_scores, status_word(ws), ghist,
                           static_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk(const dsa_queries *queries, const float *scores, int64_t ld_scores, int32_t topk, int32_t flags,
                    int32_t *idx, int32_t *cnt, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_topk");
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (!ws_ok(ws, ws_bytes, ws_topk(queries->n_q, queries->max_ctx))) return DSA_ERR_WORKSPACE;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt) return DSA_ERR_INVALID;
    if (flags & ~DSA_TOPK_HIST_FROM_INDEXER) return DSA_ERR_INVALID;
    if (!scores_ok(scores, ld_scores, queries->max_ctx)) return DSA_ERR_INVALID;
    if (queries->n_q == 0) return DSA_OK;
    return do_topk(queries, scores, ld_scores, topk, idx, cnt, status_word(ws), static_cast<uint8_t *>(ws) + kStatusBytes,
                   (flags & DSA_TOPK_HIST_FROM_INDEXER) != 0, static_cast<cudaStream_t>(stream));
}

static dsa_status mla_entry(const dsa_queries *queries, const dsa_mla *mla, const int32_t *idx, const int32_t *cnt,
                            int32_t topk, void *ws, size_t ws_bytes, void *stream, bool decode, int sel_group = 1) {
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt) return DSA_ERR_INVALID;
    dsa_status s = check_mla_layers(mla, 1);
    if (s != DSA_OK) return s;
    const size_t need = decode ? ws_mla_decode(queries->n_q, topk, 1) : kStatusBytes;
    if (!ws_ok(ws, ws_bytes, need)) return DSA_ERR_WORKSPACE;
    if (queries->n_q == 0) return DSA_OK;
    // partials after the region the indexer / top-k keep zero (see ws_zeroed_head)
    uint8_t *scratch = static_cast<uint8_t *>(ws) + kStatusBytes + ws_zeroed_head(queries->n_q);
    return do_mla(queries, mla, 1, idx, cnt, topk, decode, scratch, status_word(ws),
                  static_cast<cudaStream_t>(stream), sel_group);
}

dsa_status dsa_sparse_mla_decode(const dsa_queries *queries, const dsa_mla *mla, const int32_t *idx,
                                 const int32_t *cnt, int32_t topk, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_sparse_mla_decode");
    return mla_entry(queries, mla, idx, cnt, topk, ws, ws_bytes, stream, true);
}

dsa_status dsa_sparse_mla_prefill(const dsa_queries *queries, const dsa_mla *mla, const int32_t *idx,
                                  const int32_t *cnt, int32_t topk, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_sparse_mla_prefill");
    return mla_entry(queries, mla, idx, cnt, topk, ws, ws_bytes, stream, false);
}

dsa_status dsa_sparse_mla_mtp(const dsa_queries *queries, const dsa_mla *mla, const int32_t *idx,
                              const int32_t *cnt, int32_t topk, int32_t draft_tokens, void *ws, size_t ws_bytes,
                              void *stream) {
    NvtxRange range("dsa_sparse_mla_mtp");
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (draft_tokens < 1 || queries->n_q % draft_tokens != 0) return DSA_ERR_INVALID;
    return mla_entry(queries, mla, idx, cnt, topk, ws, ws_bytes, stream, queries->n_q <= kDecodeMaxQueries,
                     draft_tokens);
}


dsa_status dsa_indexshare_group(const dsa_queries *queries, const dsa_indexer *indexer, const dsa_mla *layers,
                                int32_t n_layers, int32_t topk, int32_t *idx, int32_t *cnt, void *ws,
                                size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_indexshare_group");
    const dsa_status s = group_check(queries, indexer, layers, n_layers, topk, idx, cnt, ws, ws_bytes);
    if (s != DSA_OK || queries->n_q == 0) return s;
    return group_launch(queries, indexer, layers, n_layers, topk, idx, cnt, ws, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_indexshare_group_host(const dsa_queries *queries, const dsa_indexer *indexer, const dsa_mla *layers,
                                     int32_t n_layers, int32_t topk, int32_t *idx, int32_t *cnt, void *ws,
                                     size_t ws_bytes, const void *h_in, void *d_in, size_t in_bytes, void *h_out,
                                     const void *d_out, size_t out_bytes, void *stream) {
    NvtxRange range("dsa_indexshare_group_host");
    dsa_status s = group_check(queries, indexer, layers, n_layers, topk, idx, cnt, ws, ws_bytes);
    if (s != DSA_OK) return s;
    if ((in_bytes > 0 && (!h_in || !d_in)) || (out_bytes > 0 && (!h_out || !d_out))) return DSA_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (in_bytes > 0 && cudaMemcpyAsync(d_in, h_in, in_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (queries->n_q > 0) {
        s = group_launch(queries, indexer, layers, n_layers, topk, idx, cnt, ws, st);
        if (s != DSA_OK) return s;
    }
    if (out_bytes > 0 && cudaMemcpyAsync(h_out, d_out, out_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return DSA_ERR_CUDA;
    return DSA_OK;
}

// ------------------------------------------------------------------ key-range shards
dsa_status dsa_shard_candidates(const dsa_queries *queries, const float *scores, int64_t ld_scores,
                                const int32_t *idx, const int32_t *cnt, int32_t topk, int32_t row_offset,
                                float *cand_score, int32_t *cand_pos, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("dsa_shard_candidates");
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (!ws_ok(ws, ws_bytes, kStatusBytes)) return DSA_ERR_WORKSPACE;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt || !cand_score || !cand_pos || row_offset < 0)
        return DSA_ERR_INVALID;
    if (!scores || ld_scores < queries->max_ctx) return DSA_ERR_INVALID;
    if (queries->n_q == 0) return DSA_OK;
    ShardArgs a = {};
    a.n_q = queries->n_q;
    a.topk = topk;
    a.L = queries->max_ctx;
    a.status = status_word(ws);
    a.scores = scores;
    a.ld = ld_scores;
    a.idx = idx;
    a.cnt = cnt;
    a.row_offset = row_offset;
    a.cand_score = cand_score;
    a.cand_pos = cand_pos;
    return launch_shard_candidates(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_shard_merge(const dsa_queries *queries, int32_t n_shards, const float *cand_score,
                           const int32_t *cand_pos, int32_t topk, int32_t row_begin, int32_t row_end, int32_t *idx,
                           int32_t *cnt, int32_t *local_idx, int32_t *local_cnt, void *ws, size_t ws_bytes,
                           void *stream) {
    NvtxRange range("dsa_shard_merge");
    if (!queries || queries->n_q < 0) return DSA_ERR_INVALID;
    if (n_shards < 1 || n_shards > kMaxShards || topk < 1 || topk > kMaxTopk) return DSA_ERR_INVALID;
    if (!cand_score || !cand_pos || !idx || !cnt || !local_idx || !local_cnt) return DSA_ERR_INVALID;
    if (row_begin < 0 || row_end < row_begin) return DSA_ERR_INVALID;
    const ShardMergeLayout lay = shard_merge_layout(queries->n_q, n_shards, topk);
    if (!ws_ok(ws, ws_bytes, lay.total)) return DSA_ERR_WORKSPACE;
    if (queries->n_q == 0) return DSA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *base = static_cast<uint8_t *>(ws);
    const int64_t ld = shard_merged_ld(n_shards, topk);
    ShardArgs a = {};
    a.n_q = queries->n_q;
    a.topk = topk;
    a.status = status_word(ws);
    a.cand_score = const_cast<float *>(cand_score);
    a.cand_pos = const_cast<int32_t *>(cand_pos);
    a.n_shards = n_shards;
    a.merged_ld = ld;
    a.merged_score = reinterpret_cast<float *>(base + lay.score);
    a.merged_pos = reinterpret_cast<int32_t *>(base + lay.pos);
    a.merged_last = reinterpret_cast<int32_t *>(base + lay.last);
    int32_t *sel = reinterpret_cast<int32_t *>(base + lay.sel);
    int32_t *sel_cnt = reinterpret_cast<int32_t *>(base + lay.sel_cnt);
    a.sel = sel;
    a.sel_cnt = sel_cnt;
    a.out_idx = idx;
    a.out_cnt = cnt;
    a.local_idx = local_idx;
    a.local_cnt = local_cnt;
    a.row_begin = row_begin;
    a.row_end = row_end;
    if (launch_shard_compact(a, st) != cudaSuccess) return DSA_ERR_CUDA;
    // the top-k of each query's merged list (ascending in position), ties to the
    // lower list index = the lower position
    dsa_queries mq;
    mq.n_q = queries->n_q;
    mq.n_seq = 1;
    mq.max_ctx = static_cast<int32_t>(ld);
    mq.seq_run = 1;
    mq.q_seq = a.merged_last;  // not read by the top-k
    mq.q_pos = a.merged_last;
    // (the merged lists' lengths are written by shard_compact, the kernel just before)
    dsa_status s = do_topk(&mq, a.merged_score, ld, topk, sel, sel_cnt, a.status, base + lay.topk_scratch, false, st,
                           false);
    if (s != DSA_OK) return s;
    return launch_shard_map(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_shard_combine(const dsa_queries *queries, int32_t n_parts, int32_t heads, int32_t d_latent,
                             const void *part_out, const float *part_lse, const int32_t *part_cnt, void *out,
                             float *lse, void *stream) {
    NvtxRange range("dsa_shard_combine");
    if (!queries || queries->n_q < 0) return DSA_ERR_INVALID;
    if (n_parts < 1 || n_parts > kMaxShards || !part_out || !part_lse || !part_cnt || !out) return DSA_ERR_INVALID;
    if (heads < 2 || heads % 2 != 0 || d_latent < 4 || d_latent % 4 != 0 || d_latent > 512) return DSA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(part_out) & 7u) || (reinterpret_cast<uintptr_t>(out) & 7u)) return DSA_ERR_INVALID;
    if (queries->n_q == 0) return DSA_OK;
    ShardCombineArgs a;
    a.n_parts = n_parts;
    a.n_q = queries->n_q;
    a.heads = heads;
    a.d_lat = d_latent;
    a.part_out = part_out;
    a.part_lse = part_lse;
    a.part_cnt = part_cnt;
    a.out = out;
    a.lse = lse;
    return launch_shard_combine(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
