// producers.cu -- what feeds the attention path and what consumes its output:
//   dsa_write_cache_rows  a token's latent-cache row and indexer key from its
//                         hidden state: one GEMM y = h . W^T (704 outputs) and an
//                         epilogue per token:
//                           c = RMSNorm(y[0:512]) * gamma            (kv_a_layernorm)
//                           r = RoPE(y[512:576], pos)                (RoPE key)
//                           k = LayerNorm(y[576:704]) * w + b, RoPE on its last 64
//                                                                    (k_norm(wk(h)))
//   dsa_absorb_queries    q_lat[h] = W_UK[h]^T q_nope[h] per head (batched GEMM over
//                         heads) and the query's RoPE part rotated
//   dsa_up_project        o[h] = W_UV[h] o_lat[h] per head (batched GEMM)
// Batches of up to 16 tokens run the contractions on CUDA cores (the weights
// streamed once, HBM-bound); larger batches on the tcgen05 GEMM.
// ("GLM-5.2 -- Model techniques map", "Checked in its code": Multi-head latent
// attention, QK normalization, Partial RoPE; "GLM 5.2 -- Hermosa AI", "MLA + DSA
// with IndexShare": RoPE theta 8e6; "GLM-5.2 -- LLM atlas", raw config.json
// fields: rope_interleave / indexer_rope_interleave true, rms_norm_eps.)
// RoPE turns each adjacent pair (x[2i], x[2i+1]) of a 64-wide RoPE part by
// pos * theta^(-2i/64); the angle and its sine and cosine are taken in double
// precision (pos * frequency reaches 10^6 radians, past float's resolution).
#include <cuda_bf16.h>

#include "abi_checks.cuh"
#include "dsa.h"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tma_encode.cuh"

namespace dsa {
namespace {

constexpr int kEpiThreads = 256;

__device__ __forceinline__ float block_sum(float v, float *buf) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();  // buf may still be read by a previous call
    if (lane == 0) buf[warp] = v;
    __syncthreads();
    float r = 0.f;
#pragma unroll
    for (int w = 0; w < kEpiThreads / 32; ++w) r += buf[w];
    return r;
}

// (cos, sin) of pos * theta^(-2i/64), i = pair index 0..31.
__device__ __forceinline__ void rope_cs(int pos, int i, double log2_theta, float &c, float &s) {
    const double inv_freq = exp2(-(2.0 * i / 64.0) * log2_theta);
    double sd, cd;
    sincos(static_cast<double>(pos) * inv_freq, &sd, &cd);
    c = static_cast<float>(cd);
    s = static_cast<float>(sd);
}

__global__ void __launch_bounds__(kEpiThreads) cache_write_epilogue_kernel(const CacheWriteArgs a) {
    __shared__ float y[kProjFeatures];
    __shared__ float red[kEpiThreads / 32];
    const int t = blockIdx.x;
    griddep_wait();
    const int seq = a.tok_seq[t], pos = a.tok_pos[t];
    if (seq < 0 || seq >= a.n_seq || pos < 0 || pos >= a.L) {
        if (threadIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
        return;
    }
    {
        // three features per thread (704 = 2.75 x 256), the split partials summed in a
        // fixed order (deterministic) with the loads of four splits in flight at once
        constexpr int kF = (kProjFeatures + kEpiThreads - 1) / kEpiThreads;
        float v[kF];
#pragma unroll
        for (int q = 0; q < kF; ++q) v[q] = 0.f;
        const int64_t split_stride = static_cast<int64_t>(a.n_tok) * kProjFeatures;
        const float *yt = a.y + static_cast<int64_t>(t) * kProjFeatures;
        int s = 0;
        for (; s + 4 <= a.k_splits; s += 4) {
            float x[4][kF];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int q = 0; q < kF; ++q) {
                    const int f = threadIdx.x + q * kEpiThreads;
                    x[u][q] = f < kProjFeatures ? yt[(s + u) * split_stride + f] : 0.f;
                }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int q = 0; q < kF; ++q) v[q] += x[u][q];
        }
        for (; s < a.k_splits; ++s)
#pragma unroll
            for (int q = 0; q < kF; ++q) {
                const int f = threadIdx.x + q * kEpiThreads;
                if (f < kProjFeatures) v[q] += yt[s * split_stride + f];
            }
#pragma unroll
        for (int q = 0; q < kF; ++q) {
            const int f = threadIdx.x + q * kEpiThreads;
            if (f < kProjFeatures) y[f] = v[q];
        }
    }
    __syncthreads();
    // latent: RMSNorm over 512 features, times gamma
    float ss = 0.f;
    for (int f = threadIdx.x; f < kLatent; f += kEpiThreads) ss += y[f] * y[f];
    ss = block_sum(ss, red);
    const float rms = 1.f / sqrtf(ss / kLatent + a.eps);
    // indexer key: LayerNorm over 128 features
    float su = 0.f;
    for (int f = threadIdx.x; f < kIdxDim; f += kEpiThreads) su += y[kLatent + kRope + f];
    const float mu = block_sum(su, red) / kIdxDim;
    float sv = 0.f;
    for (int f = threadIdx.x; f < kIdxDim; f += kEpiThreads) {
        const float d = y[kLatent + kRope + f] - mu;
        sv += d * d;
    }
    const float rstd = 1.f / sqrtf(block_sum(sv, red) / kIdxDim + a.eps);
    if (a.kv) {
        __nv_bfloat16 *row = static_cast<__nv_bfloat16 *>(a.kv) + static_cast<int64_t>(seq) * a.kv_seq_stride +
                             static_cast<int64_t>(pos) * a.kv_row_stride;
        for (int f = threadIdx.x; f < kLatent; f += kEpiThreads)
            row[f] = __float2bfloat16_rn(y[f] * rms * a.rms_weight[f]);
        if (threadIdx.x < kRope / 2) {
            const int i = threadIdx.x;
            float c, s;
            rope_cs(pos, i, a.log2_theta, c, s);
            const float x0 = y[kLatent + 2 * i], x1 = y[kLatent + 2 * i + 1];
            row[kLatent + 2 * i] = __float2bfloat16_rn(x0 * c - x1 * s);
            row[kLatent + 2 * i + 1] = __float2bfloat16_rn(x0 * s + x1 * c);
        }
    }
    if (a.k_idx) {
        __nv_bfloat16 *key = static_cast<__nv_bfloat16 *>(a.k_idx) + static_cast<int64_t>(seq) * a.k_seq_stride +
                             static_cast<int64_t>(pos) * a.k_row_stride;
        const float *yk = y + kLatent + kRope;
        // dims 0..63 keep their normalised value; 64..127 (the RoPE part) are turned in pairs
        for (int f = threadIdx.x; f < kIdxDim - kRope; f += kEpiThreads)
            key[f] = __float2bfloat16_rn((yk[f] - mu) * rstd * a.ln_weight[f] + a.ln_bias[f]);
        if (threadIdx.x < kRope / 2) {
            const int i = threadIdx.x, f0 = kIdxDim - kRope + 2 * i;
            float c, s;
            rope_cs(pos, i, a.log2_theta, c, s);
            const float x0 = (yk[f0] - mu) * rstd * a.ln_weight[f0] + a.ln_bias[f0];
            const float x1 = (yk[f0 + 1] - mu) * rstd * a.ln_weight[f0 + 1] + a.ln_bias[f0 + 1];
            key[f0] = __float2bfloat16_rn(x0 * c - x1 * s);
            key[f0 + 1] = __float2bfloat16_rn(x0 * s + x1 * c);
        }
    }
}

// One thread per (query, head, RoPE pair).
__global__ void __launch_bounds__(256) query_rope_kernel(const QueryRopeArgs a) {
    griddep_wait();
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = static_cast<int64_t>(a.n) * a.heads * (kRope / 2);
    if (e >= total) return;
    const int p = static_cast<int>(e % (kRope / 2));
    const int64_t ih = e / (kRope / 2);  // query * heads + head
    const int i = static_cast<int>(ih / a.heads);
    const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.q_rope) + ih * kRope + 2 * p;
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.q) + ih * kRow + kLatent + 2 * p;
    float c, s;
    rope_cs(a.pos[i], p, a.log2_theta, c, s);
    const float x0 = __bfloat162float(src[0]), x1 = __bfloat162float(src[1]);
    dst[0] = __float2bfloat16_rn(x0 * c - x1 * s);
    dst[1] = __float2bfloat16_rn(x0 * s + x1 * c);
}

}  // namespace

cudaError_t launch_cache_write_epilogue(const CacheWriteArgs &a, cudaStream_t st) {
    return launch_pdl(cache_write_epilogue_kernel, dim3(a.n_tok), dim3(kEpiThreads), 0, st, a);
}

cudaError_t launch_query_rope(const QueryRopeArgs &a, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(a.n) * a.heads * (kRope / 2);
    return launch_pdl(query_rope_kernel, dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256), 0, st, a);
}

}  // namespace dsa

using namespace dsa;

namespace {

constexpr size_t kStatus = 256;
constexpr int kDNope = 192;  // qk_nope_head_dim
constexpr int kDV = 256;     // v_head_dim

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Split-K plan of the cache-row GEMM (M = tokens, N = 704, K = hidden): about
// one CTA per SM on a 148-SM part, at least 4 blocks of 64 along K per split.
void cache_plan(int n_tok, int hidden, int &m_tiles, int &k_splits, int &kb_per_split) {
    const int kb = (hidden + 63) / 64;
    m_tiles = (n_tok + 127) / 128;
    const int tiles = m_tiles * ((kProjFeatures + 127) / 128);
    int s = 144 / tiles;
    s = s < 1 ? 1 : s;
    const int max_s = kb / 4 > 0 ? kb / 4 : 1;
    s = s > max_s ? max_s : s;
    kb_per_split = (kb + s - 1) / s;
    k_splits = (kb + kb_per_split - 1) / kb_per_split;
}

size_t cache_ws_bytes(int n_tok, int hidden) {
    int mt, ks, kbs;
    cache_plan(n_tok, hidden, mt, ks, kbs);
    return kStatus + al256(static_cast<size_t>(ks) * n_tok * kProjFeatures * sizeof(float));
}

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
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

}  // namespace

extern "C" {

size_t dsa_cache_writer_workspace_bytes(int32_t n_tok, int32_t hidden) {
    if (n_tok < 0 || hidden < 1) return 0;
    return cache_ws_bytes(n_tok, hidden);
}

dsa_status dsa_write_cache_rows(const dsa_cache_writer *cw, void *ws, size_t ws_bytes, void *stream) {
    if (!cw || cw->n_tok < 0 || cw->hidden < 64 || cw->hidden % 8 != 0) return DSA_ERR_INVALID;
    if (!cw->h || !cw->w || !cw->rms_weight || !cw->ln_weight || !cw->ln_bias || !cw->tok_seq || !cw->tok_pos)
        return DSA_ERR_INVALID;
    if (!cw->kv && !cw->k_idx) return DSA_ERR_INVALID;
    if (cw->n_seq < 1 || cw->max_ctx < 1 || !(cw->eps > 0.f) || !(cw->rope_theta > 1.f)) return DSA_ERR_INVALID;
    if (cw->h_row_stride < cw->hidden || cw->h_row_stride % 8 != 0 || !a16(cw->h) || !a16(cw->w))
        return DSA_ERR_INVALID;
    if (cw->kv && (cw->kv_row_stride < kRow || cw->kv_seq_stride < 0)) return DSA_ERR_INVALID;
    if (cw->k_idx && (cw->k_row_stride < kIdxDim || cw->k_seq_stride < 0)) return DSA_ERR_INVALID;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < cache_ws_bytes(cw->n_tok, cw->hidden))
        return DSA_ERR_WORKSPACE;
    if (cw->n_tok == 0) return DSA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    GemmArgs g = {};
    g.M = cw->n_tok;
    g.N = kProjFeatures;
    g.K = cw->hidden;
    g.batch = 1;
    cache_plan(cw->n_tok, cw->hidden, g.m_tiles, g.k_splits, g.kb_per_split);
    float *y = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kStatus);
    g.out_f32 = y;
    g.ldc = kProjFeatures;
    g.s_batch = 0;
    g.s_split = static_cast<int64_t>(cw->n_tok) * kProjFeatures;
    g.status = static_cast<uint32_t *>(ws);
    if (cw->n_tok <= kSkinnyMaxM) {
        // decode-sized batch: stream the weights once on CUDA cores (same partials)
        GemmSkinnyArgs k = {};
        k.M = cw->n_tok;
        k.N = kProjFeatures;
        k.K = cw->hidden;
        k.batch = 1;
        // about two CTAs per SM in one wave: K splits for the 704 weight rows,
        // no more than the workspace holds partials for
        const int n_tiles = (kProjFeatures + skinny_rows_per_cta(cw->n_tok) - 1) / skinny_rows_per_cta(cw->n_tok);
        int ks = 2 * sm_count() / n_tiles;
        ks = ks < 1 ? 1 : (ks > g.k_splits ? g.k_splits : ks);
        k.k_per_split = (((cw->hidden + ks - 1) / ks) + 7) / 8 * 8;
        if (k.k_per_split > 2048) return DSA_ERR_UNSUPPORTED;
        g.k_splits = (cw->hidden + k.k_per_split - 1) / k.k_per_split;  // what the epilogue sums
        k.a = cw->h;
        k.a_row = cw->h_row_stride;
        k.b = cw->w;
        k.b_row = cw->hidden;
        k.out_f32 = y;
        k.ldc = kProjFeatures;
        k.s_split = g.s_split;
        if (launch_gemm_skinny(k, st) != cudaSuccess) return DSA_ERR_CUDA;
    } else {
        CUtensorMap ta, tb;
        if (!encode_gemm_operand(&ta, cw->h, cw->hidden, cw->n_tok, 1, cw->h_row_stride, 0, 128, &g.a_batch_inner))
            return DSA_ERR_INVALID;
        if (!encode_gemm_operand(&tb, cw->w, cw->hidden, kProjFeatures, 1, cw->hidden, 0, 128, &g.b_batch_inner))
            return DSA_ERR_INVALID;
        if (launch_gemm_tc(128, ta, tb, g, st) != cudaSuccess) return DSA_ERR_CUDA;
    }
    CacheWriteArgs e;
    e.y = y;
    e.k_splits = g.k_splits;
    e.n_tok = cw->n_tok;
    e.rms_weight = cw->rms_weight;
    e.ln_weight = cw->ln_weight;
    e.ln_bias = cw->ln_bias;
    e.tok_seq = cw->tok_seq;
    e.tok_pos = cw->tok_pos;
    e.kv = cw->kv;
    e.kv_seq_stride = cw->kv_seq_stride;
    e.kv_row_stride = cw->kv_row_stride;
    e.k_idx = cw->k_idx;
    e.k_seq_stride = cw->k_seq_stride;
    e.k_row_stride = cw->k_row_stride;
    e.n_seq = cw->n_seq;
    e.L = cw->max_ctx;
    e.eps = cw->eps;
    e.log2_theta = log2(static_cast<double>(cw->rope_theta));
    e.status = static_cast<uint32_t *>(ws);
    return launch_cache_write_epilogue(e, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_absorb_queries(int32_t n_q, int32_t heads, const void *q_nope, const void *q_rope, const void *w_uk_t,
                              const int32_t *pos, float rope_theta, void *q_out, void *ws, size_t ws_bytes,
                              void *stream) {
    if (n_q < 0 || heads < 1 || heads > 256 || !q_nope || !q_rope || !w_uk_t || !pos || !q_out) return DSA_ERR_INVALID;
    if (!(rope_theta > 1.f) || !a16(q_nope) || !a16(w_uk_t) || !a16(q_out)) return DSA_ERR_INVALID;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < kStatus) return DSA_ERR_WORKSPACE;
    if (n_q == 0) return DSA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // per head h: C[n][j] = sum_k q_nope[n][h][k] * w_uk_t[h][j][k] into q_out[n][h][j], j < 512
    GemmArgs g = {};
    g.M = n_q;
    g.N = kLatent;
    g.K = kDNope;
    g.batch = heads;
    g.m_tiles = (n_q + 127) / 128;
    g.k_splits = 1;
    g.kb_per_split = (kDNope + 63) / 64;
    g.out_bf16 = q_out;
    g.ldc = static_cast<int64_t>(heads) * kRow;
    g.s_batch = kRow;
    g.status = static_cast<uint32_t *>(ws);
    if (n_q <= kSkinnyMaxM) {
        GemmSkinnyArgs k = {};
        k.M = n_q;
        k.N = kLatent;
        k.K = kDNope;
        k.batch = heads;
        k.k_per_split = kDNope;
        k.a = q_nope;
        k.a_row = static_cast<int64_t>(heads) * kDNope;
        k.a_batch = kDNope;
        k.b = w_uk_t;
        k.b_row = kDNope;
        k.b_batch = static_cast<int64_t>(kLatent) * kDNope;
        k.out_bf16 = q_out;
        k.ldc = g.ldc;
        k.s_batch = g.s_batch;
        if (launch_gemm_skinny(k, st) != cudaSuccess) return DSA_ERR_CUDA;
    } else {
        CUtensorMap ta, tb;
        if (!encode_gemm_operand(&ta, q_nope, kDNope, n_q, heads, static_cast<int64_t>(heads) * kDNope, kDNope, 128,
                                 &g.a_batch_inner))
            return DSA_ERR_INVALID;
        if (!encode_gemm_operand(&tb, w_uk_t, kDNope, kLatent, heads, kDNope, static_cast<int64_t>(kLatent) * kDNope,
                                 128, &g.b_batch_inner))
            return DSA_ERR_INVALID;
        if (launch_gemm_tc(128, ta, tb, g, st) != cudaSuccess) return DSA_ERR_CUDA;
    }
    QueryRopeArgs r;
    r.q_rope = q_rope;
    r.q = q_out;
    r.pos = pos;
    r.n = n_q;
    r.heads = heads;
    r.log2_theta = log2(static_cast<double>(rope_theta));
    return launch_query_rope(r, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_up_project(int32_t n_q, int32_t heads, const void *o_lat, const void *w_uv, void *out, void *ws,
                          size_t ws_bytes, void *stream) {
    if (n_q < 0 || heads < 1 || heads > 256 || !o_lat || !w_uv || !out) return DSA_ERR_INVALID;
    if (!a16(o_lat) || !a16(w_uv) || !a16(out)) return DSA_ERR_INVALID;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < kStatus) return DSA_ERR_WORKSPACE;
    if (n_q == 0) return DSA_OK;
    // per head h: out[n][h][v] = sum_l o_lat[n][h][l] * w_uv[h][v][l]
    GemmArgs g = {};
    g.M = n_q;
    g.N = kDV;
    g.K = kLatent;
    g.batch = heads;
    g.m_tiles = (n_q + 127) / 128;
    g.k_splits = 1;
    g.kb_per_split = kLatent / 64;
    g.out_bf16 = out;
    g.ldc = static_cast<int64_t>(heads) * kDV;
    g.s_batch = kDV;
    g.status = static_cast<uint32_t *>(ws);
    if (n_q <= kSkinnyMaxM) {
        GemmSkinnyArgs k = {};
        k.M = n_q;
        k.N = kDV;
        k.K = kLatent;
        k.batch = heads;
        k.k_per_split = kLatent;
        k.a = o_lat;
        k.a_row = static_cast<int64_t>(heads) * kLatent;
        k.a_batch = kLatent;
        k.b = w_uv;
        k.b_row = kLatent;
        k.b_batch = static_cast<int64_t>(kDV) * kLatent;
        k.out_bf16 = out;
        k.ldc = g.ldc;
        k.s_batch = g.s_batch;
        return launch_gemm_skinny(k, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
    }
    CUtensorMap ta, tb;
    if (!encode_gemm_operand(&ta, o_lat, kLatent, n_q, heads, static_cast<int64_t>(heads) * kLatent, kLatent, 128,
                             &g.a_batch_inner))
        return DSA_ERR_INVALID;
    if (!encode_gemm_operand(&tb, w_uv, kLatent, kDV, heads, kLatent, static_cast<int64_t>(kDV) * kLatent, 128,
                             &g.b_batch_inner))
        return DSA_ERR_INVALID;
    return launch_gemm_tc(128, ta, tb, g, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
