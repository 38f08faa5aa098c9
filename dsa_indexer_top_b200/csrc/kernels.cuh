// kernels.cuh -- internal launch interface between the C ABI (dsa_abi.cu) and
// the kernels (indexer.cu, topk.cu, mla.cu).  Not part of the public header.
#pragma once

#include <cstddef>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "dsa.h"

namespace dsa {

// Launch with programmatic stream serialisation (the kernel calls
// griddep_wait() before it reads what earlier work in the stream wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device) and
// size: a launch then pays only a lookup.
template <typename... KArgs>
cudaError_t set_max_dynamic_smem(void (*kernel)(KArgs...), int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const void *key = reinterpret_cast<const void *>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find({key, dev});
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[{key, dev}] = bytes;
    return e;
}

constexpr int kIdxHeads = 32;   // index_n_heads of GLM-5.2
constexpr int kIdxDim = 128;    // index_head_dim of GLM-5.2
constexpr int kMlaHeads = 64;   // num_attention_heads of GLM-5.2
constexpr int kLatent = 512;    // kv_lora_rank
constexpr int kRope = 64;       // qk_rope_head_dim
constexpr int kRow = kLatent + kRope;
// Packed FP8 latent-cache row (bytes): 512 E4M3 codes, the 64 bf16 RoPE values,
// the float32 row scale, 12 bytes of padding -- 41 aligned 16-byte pieces.
constexpr int kFp8RopeOff = kLatent;
constexpr int kFp8ScaleOff = kLatent + 2 * kRope;
constexpr int kFp8Row = kFp8ScaleOff + 16;
constexpr int kRowsPerChunk = 128;  // splits <= ceil(topk / 128): every CTA walks >= 2 chunks of 64 rows
constexpr int kMlaChunk = 64;       // selected rows per tensor-core pipeline chunk
constexpr int kMaxTopk = 4096;
constexpr int kMaxLayers = 4;

// ------------------------------------------------------------------ indexer
// Byte offset, inside the workspace's 256-byte status block, of the indexer's
// two work counters (unsigned 64-bit; zeroed with the workspace).
constexpr size_t kIdxWorkOffset = 128;
constexpr int kIdxDynamicMinTiles = 4096;  // key tiles per query from which work is claimed

struct IdxTcArgs {
    const float *w;
    const int32_t *q_seq;
    const int32_t *q_pos;
    float *scores;
    int64_t ld;
    uint32_t *status;
    int n_q, n_seq, L;
    int k_shared;         // 1: every query reads cache 0
    int tiles_per_group;  // ceil(L / 128)
    long long total_items;
    uint32_t *ghist;      // non-null (one query per tile only): accumulate the top-k
                          // first-digit histogram [n_q][4096] of the scores written
    unsigned long long *work;  // claimed work: [0] next work item, [1] CTAs finished,
                               // zero between launches (the last CTA re-zeroes them);
                               // null: contiguous ranges of items per CTA
    // FP8 (E4M3) operands only: positive per-(query, head) and per-key scales, or null
    const float *q_scale;    // [n_q][32]
    const float *k_scale;    // sequence b's key s at k_scale[b * ks_seq_stride + s]
    int64_t ks_seq_stride;
};

// G = queries per tensor-core tile (1, 2, 4 or 8).  Tensor maps: keys 3-D
// {128, L, n_cache}, queries 2-D {128, n_q*32}, both 128-byte swizzled with
// 128-byte boxes: bf16 boxes {64, 128, 1} / {64, 32*G}, FP8 (uint8) boxes
// {128, 128, 1} / {128, 32*G}.
cudaError_t launch_idx_score_tc(int G, bool fp8, const CUtensorMap &tmap_k, const CUtensorMap &tmap_q,
                                const IdxTcArgs &a, int num_sms, cudaStream_t st);

struct IdxGenericArgs {
    const void *q;
    const float *w;
    const void *k;
    int64_t k_seq_stride, k_row_stride;
    const int32_t *q_seq;
    const int32_t *q_pos;
    float *scores;
    int64_t ld;
    uint32_t *status;
    int n_q, n_seq, L, heads, dim;
    int is_bf16;
};
cudaError_t launch_idx_score_generic(const IdxGenericArgs &a, cudaStream_t st);

// ------------------------------------------------------------------ top-k
constexpr int kTopkBins = 4096;            // first radix digit: 12 bits
constexpr int kTopkSplitMinCtx = 8192;     // contexts above this, with at most
constexpr int kTopkSplitMaxQueries = 64;   // this many queries, split rows over CTAs
constexpr int kSplitMax = 64;              // chunks per query (split schedule)
constexpr int kSplitCap = 1024;            // candidates stored per chunk

struct TopkArgs {
    const float *scores;
    int64_t ld;
    const int32_t *q_pos;
    int32_t *idx;
    int32_t *cnt;
    uint32_t *status;
    int n_q, L, topk;
    int hist_ready;    // ghist already holds the first-digit histograms (indexer epilogue)
    int pos_early;     // q_pos is an input of the call (no kernel of it writes q_pos): the
                       // split schedule reads it before waiting for the previous kernel
    // scratch (workspace)
    uint32_t *ghist;   // [n_q][4096] first-digit histogram
    uint32_t *gticket; // [n_q] chunks of the query done (split schedule), after ghist
    uint32_t *ghist2;  // [n_q][4096] second-digit histogram of the threshold-bin candidates
                       // (split schedule), after the tickets
    uint32_t *gcount;  // [n_q][kSplitMax] candidates per chunk
    uint2 *gcand;      // [n_q][kSplitMax][kSplitCap] (key, position)
};
bool topk_uses_split(int n_q, int max_ctx);
// Bytes at the head of the top-k scratch (histograms, then tickets) that must be
// zero when a top-k launch starts.
size_t topk_zeroed_bytes(int n_q);
size_t topk_scratch_bytes(int n_q, int max_ctx);
void topk_bind_scratch(TopkArgs &a, void *scratch);
cudaError_t launch_topk(const TopkArgs &a, int num_sms, cudaStream_t st);
// First-digit histograms only (into a.ghist, which must be zeroed), every query.
cudaError_t launch_topk_hist(const TopkArgs &a, int num_sms, cudaStream_t st);

// ------------------------------------------------------------------ key-range shards
constexpr int kMaxShards = 64;

struct ShardArgs {
    int n_q, topk, L;
    uint32_t *status;
    // candidates of this rank's local top-k
    const float *scores;
    int64_t ld;
    const int32_t *idx;      // [n_q][topk] local selection (shard rows), ascending, -1 padded
    const int32_t *cnt;      // [n_q]
    int row_offset;          // the shard's first row in the sequence
    float *cand_score;       // [n_q][topk] (one rank) or [n_shards][n_q][topk] (gathered)
    int32_t *cand_pos;       // same layout: sequence positions, -1 padded
    // merge of the gathered candidates
    int n_shards;
    int64_t merged_ld;       // row stride of the merged list (>= n_shards * topk, multiple of 4)
    float *merged_score;     // [n_q][merged_ld]
    int32_t *merged_pos;     // [n_q][merged_ld]
    int32_t *merged_last;    // [n_q] number of merged candidates - 1
    const int32_t *sel;      // [n_q][topk] top-k of the merged list (indices into it)
    const int32_t *sel_cnt;  // [n_q]
    int32_t *out_idx, *out_cnt;      // global selection (sequence positions)
    int32_t *local_idx, *local_cnt;  // this rank's part of it (shard rows)
    int row_begin, row_end;
};
cudaError_t launch_shard_candidates(const ShardArgs &a, cudaStream_t st);
cudaError_t launch_shard_compact(const ShardArgs &a, cudaStream_t st);
cudaError_t launch_shard_map(const ShardArgs &a, cudaStream_t st);

struct ShardCombineArgs {
    int n_parts, n_q, heads, d_lat;
    const void *part_out;     // bf16 [n_parts][n_q][heads][d_lat]
    const float *part_lse;    // [n_parts][n_q][heads]
    const int32_t *part_cnt;  // [n_parts][n_q] rows each part attended over (0: ignored)
    void *out;                // bf16 [n_q][heads][d_lat]
    float *lse;               // [n_q][heads] or null
};
cudaError_t launch_shard_combine(const ShardCombineArgs &a, cudaStream_t st);

// ------------------------------------------------------------------ dense GEMM (producers)
// C[b][m][n] = sum_k A[b][m][k] * B[b][n][k], bf16 operands read by TMA from
// 3-D tensor maps {K, rows, batch} (128-byte swizzle, boxes {64, 128, 1} for A
// and {64, BN, 1} for B), fp32 accumulation in TMEM.  Grid (N tiles, M tiles x
// K splits, batch); split s of batch b writes rows of out_f32 + s * s_split +
// b * s_batch (row stride ldc), or bf16 rows of out_bf16 (one split only).
struct GemmArgs {
    int M, N, K, batch;
    int m_tiles, k_splits, kb_per_split;  // kb: blocks of 64 along K
    float *out_f32;
    void *out_bf16;
    int64_t ldc, s_batch, s_split;        // elements
    int a_batch_inner, b_batch_inner;     // operand map ordered {K, batch, rows} (see encode_gemm_operand)
    uint32_t *status;
};
cudaError_t launch_gemm_tc(int bn, const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &g, cudaStream_t st);

// The same contraction for at most 16 rows of A (decode-sized batches), on CUDA
// cores: B streamed once with 16-byte loads; K split in pieces of k_per_split
// (a multiple of 8, at most 2048); element (m, k) of batch b at a + b * a_batch +
// m * a_row + k, (n, k) at b + b * b_batch + n * b_row + k (elements, 16-byte
// aligned rows); outputs addressed as in GemmArgs.
struct GemmSkinnyArgs {
    int M, N, K, batch, k_per_split;
    const void *a;
    int64_t a_row, a_batch;
    const void *b;
    int64_t b_row, b_batch;
    float *out_f32;
    void *out_bf16;
    int64_t ldc, s_batch, s_split;
};
constexpr int kSkinnyMaxM = 16;
int skinny_rows_per_cta(int M);  // rows of B per CTA of launch_gemm_skinny
cudaError_t launch_gemm_skinny(const GemmSkinnyArgs &g, cudaStream_t st);

// Cache-row writer epilogue: one CTA per token sums the split-K partials of
// y = h . W^T (704 features: latent 512 | RoPE key 64 | indexer key 128) and
// writes RMSNorm(latent) * gamma | RoPE(key) into the latent cache and
// RoPE_last64(LayerNorm(indexer key) * w + b) into the indexer-key cache.
struct CacheWriteArgs {
    const float *y;            // [k_splits][n_tok][704]
    int k_splits, n_tok;
    const float *rms_weight, *ln_weight, *ln_bias;
    const int32_t *tok_seq, *tok_pos;
    void *kv;
    int64_t kv_seq_stride, kv_row_stride;
    void *k_idx;
    int64_t k_seq_stride, k_row_stride;
    int n_seq, L;
    float eps;
    double log2_theta;
    uint32_t *status;
};
constexpr int kProjFeatures = kLatent + kRope + kIdxDim;  // 704
cudaError_t launch_cache_write_epilogue(const CacheWriteArgs &a, cudaStream_t st);

// RoPE of the absorbed queries' RoPE part: q[i][h][512 + d] = RoPE(q_rope[i][h], pos[i]).
struct QueryRopeArgs {
    const void *q_rope;  // bf16 [n][H][64]
    void *q;             // bf16 [n][H][576]
    const int32_t *pos;
    int n, heads;
    double log2_theta;
};
cudaError_t launch_query_rope(const QueryRopeArgs &a, cudaStream_t st);

// ------------------------------------------------------------------ diagnostics
// The limit of every device-side wait (the same value as kWaitLimitNs of the
// PTX wrappers): 2 s.
constexpr uint64_t kDeviceWaitLimitNs = 2000000000ull;
// One thread waits (bounded, limit_ns) on a barrier nothing completes and
// reports DSA_ERR_TIMEOUT into *status.
cudaError_t launch_bounded_wait_probe(uint32_t *status, uint64_t limit_ns, cudaStream_t st);

// ------------------------------------------------------------------ sparse MLA
struct MlaLayerPtrs {
    const void *q;
    const void *kv;
    void *out;
    float *lse;
};

struct MlaArgs {
    MlaLayerPtrs layer[kMaxLayers];
    int n_layers;
    int64_t kv_seq_stride, kv_row_stride;
    const int32_t *q_seq;
    const int32_t *idx;
    const int32_t *cnt;
    int topk;
    int n_q, n_seq, L;
    int heads, d_lat, d_rope;
    float scale;
    int is_bf16;
    int kv_fp8;          // caches are packed FP8 rows (kFp8Row bytes; strides in bytes)
    int sel_group;       // queries per selection row: query i reads idx/cnt row i / sel_group (>= 1)
    uint32_t *status;
    // split-K schedule (tensor-core path)
    int n_splits;        // CTAs per query
    int chunks_per_cta;  // 64-row chunks walked by one CTA
    float *part_o;       // [layers][n_q][n_splits][64][512] unnormalised
    float *part_ml;      // [layers][n_q][n_splits][64][2] (max, sum) in log2 units
};

// TMA descriptors of the tensor-core MLA (one set per layer), over one 2-D
// tensor of every sequence's rows (the row gathers read four rows per op).
// bf16 caches: kv {576, rows}, boxes {64, 1}; q {576, n_q * 64}, boxes {64, 64};
// both 128-byte swizzled.  Packed FP8 caches: kv {656 bytes, rows}, boxes
// {128 bytes, 1}, unswizzled (staging for the widening); kvr the same rows as
// {328 bf16, rows}, boxes {64, 1}, 128-byte swizzled (the RoPE key).
struct MlaMaps {
    CUtensorMap kv[kMaxLayers];   // bf16: the rows; packed FP8: the rows' bytes, boxes {128 B, 1}, unswizzled
    CUtensorMap q[kMaxLayers];    // bf16 only
    CUtensorMap kvr[kMaxLayers];  // packed FP8 only: the rows as bf16, boxes {64, 1} at the RoPE key, swizzled
};

// Tensor-core sparse MLA (bf16 queries and outputs, 64 heads, 512 + 64; bf16 or
// packed FP8 caches).  n_splits == 1 writes the final output; otherwise partials
// followed by launch_mla_combine.  `maps` (bf16 caches; ignored for FP8) come
// from encode_mla_maps.
cudaError_t launch_mla_tc(const MlaArgs &a, const MlaMaps &maps, cudaStream_t st);
bool encode_mla_maps(const MlaArgs &a, MlaMaps &maps);
// Rows of the 2-D tensor the bf16 row gathers read (every sequence's rows, at
// kv_row_stride apart): -1 when the sequence stride is not a whole number of
// rows.  The tensor-core path needs 1 .. INT32_MAX.
int64_t mla_gather_rows(int64_t kv_seq_stride, int64_t kv_row_stride, int n_seq, int max_ctx);
cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t st);
cudaError_t launch_mla_generic(const MlaArgs &a, cudaStream_t st);

// Split-K plan of the tensor-core MLA: n_splits CTAs per query, each walking
// cpc chunks of 64 selected rows.  Decode spreads each query over as many CTAs
// as fill the SMs across the batch (at most max_splits, and at least two
// chunks per CTA: measured on 4 x 1M decode, 16 splits x 2 chunks beat both
// 32 x 1 and 8 x 4); prefill uses one CTA
// per query (n_splits = 1: the final output is written directly).
inline void mla_plan(int n_q, int n_layers, int topk, bool decode, int num_sms, int max_splits, int &n_splits,
                     int &cpc) {
    const int nch = (topk + kMlaChunk - 1) / kMlaChunk;
    int s = 1;
    if (decode) {
        const int work = n_q * n_layers > 0 ? n_q * n_layers : 1;
        s = num_sms / work;
        s = s < 1 ? 1 : (s > max_splits ? max_splits : s);
        const int half = nch / 2 > 0 ? nch / 2 : 1;  // at least two chunks per CTA
        s = s > half ? half : s;
    }
    cpc = (nch + s - 1) / s;
    n_splits = (nch + cpc - 1) / cpc;
}

// Upper bound of the decode splits per query the planner can pick with
// max_splits = kMlaMaxSplits (sizes the workspace).
constexpr int kMlaMaxSplits = 32;
inline int mla_max_splits(int topk) {
    const int nch = (topk + kMlaChunk - 1) / kMlaChunk;
    return nch < kMlaMaxSplits ? nch : kMlaMaxSplits;
}

// Bytes of split-K partials for the tensor-core decode schedule.
inline size_t mla_partial_bytes(int n_layers, int n_q, int n_splits) {
    size_t rows = static_cast<size_t>(n_layers) * n_q * n_splits * kMlaHeads;
    return rows * kLatent * sizeof(float) + rows * 2 * sizeof(float);
}

}  // namespace dsa
