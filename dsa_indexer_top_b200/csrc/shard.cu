// shard.cu -- key-range sharding of one long sequence over several GPUs:
// the per-rank candidate list after the local top-k, the merge of every
// rank's candidates into the global selection (and this rank's part of it),
// and the log-sum-exp combine of the ranks' partial attention outputs.
//
// Each rank holds a contiguous range [row_begin, row_end) of the sequence's
// indexer keys and latent rows.  Because the ranges are contiguous and in
// rank order, and every rank's candidates are in ascending position order,
// concatenating the ranks' candidates gives one list in ascending position
// order; selecting the top-k of that list with ties to the lower list index is
// the global top-k with ties to the lower position (a row of the global top-k
// that lies in shard g ranks at least as high inside shard g, so it is among
// shard g's candidates).  Attention over the union of the ranks' parts of the
// selection is the log-sum-exp combine of the ranks' partial attentions.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kShardThreads = 256;

// cand_score[i][j] = scores[i][idx[i][j]], cand_pos[i][j] = idx[i][j] + row_offset
// for j < cnt[i]; -1 positions (and 0 scores) after.
__global__ void __launch_bounds__(kShardThreads) shard_candidates_kernel(const ShardArgs a) {
    const int i = blockIdx.x;
    griddep_wait();
    int c = a.cnt[i];
    if (c < 0 || c > a.topk) {
        if (threadIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
        c = 0;
    }
    const int32_t *idx = a.idx + static_cast<int64_t>(i) * a.topk;
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    float *cs = a.cand_score + static_cast<int64_t>(i) * a.topk;
    int32_t *cp = a.cand_pos + static_cast<int64_t>(i) * a.topk;
    for (int j = threadIdx.x; j < a.topk; j += kShardThreads) {
        float sc = 0.f;
        int32_t pos = -1;
        if (j < c) {
            const int s = idx[j];
            if (s >= 0 && s < a.L) {
                sc = row[s];
                pos = s + a.row_offset;
            } else {
                report_status(a.status, DSA_ERR_INVALID);
            }
        }
        cs[j] = sc;
        cp[j] = pos;
    }
}

// Exclusive scan of one value per thread over the block (256 threads).
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kShardThreads / 32; ++w) {
        const int t = warp_tot[w];
        before += w < warp ? t : 0;
        tot += t;
    }
    __syncthreads();
    total = tot;
    return before + x - v;
}

// Concatenate the shards' valid candidates of query i (shard order = position
// order) into merged_score / merged_pos; merged_last[i] = count - 1.
__global__ void __launch_bounds__(kShardThreads) shard_compact_kernel(const ShardArgs a) {
    __shared__ int warp_tot[kShardThreads / 32];
    __shared__ int base_sh;
    const int i = blockIdx.x;
    griddep_wait();
    const int64_t width = a.merged_ld;
    float *ms = a.merged_score + static_cast<int64_t>(i) * width;
    int32_t *mp = a.merged_pos + static_cast<int64_t>(i) * width;
    if (threadIdx.x == 0) base_sh = 0;
    __syncthreads();
    for (int g = 0; g < a.n_shards; ++g) {
        // shard g's candidates of query i, in the gathered layout [shard][n_q][topk]
        const int64_t off = (static_cast<int64_t>(g) * a.n_q + i) * a.topk;
        const float *cs = a.cand_score + off;
        const int32_t *cp = a.cand_pos + off;
        for (int j0 = 0; j0 < a.topk; j0 += kShardThreads) {
            const int j = j0 + threadIdx.x;
            const int32_t pos = j < a.topk ? cp[j] : -1;
            const bool ok = pos >= 0;
            int total;
            const int slot = block_excl_scan(ok ? 1 : 0, warp_tot, total);
            const int base = base_sh;
            if (ok) {
                ms[base + slot] = cs[j];
                mp[base + slot] = pos;
            }
            __syncthreads();
            if (threadIdx.x == 0) base_sh = base + total;
            __syncthreads();
        }
    }
    if (threadIdx.x == 0) {
        const int n = base_sh;
        a.merged_last[i] = n - 1;
        if (n < 1) report_status(a.status, DSA_ERR_INVALID);  // the query sees no row at all
    }
}

// Global selection from the merged list's top-k (sel: indices into the list,
// ascending) and this rank's part of it, as rows of its shard.
__global__ void __launch_bounds__(kShardThreads) shard_map_kernel(const ShardArgs a) {
    __shared__ int warp_tot[kShardThreads / 32];
    __shared__ int base_sh;
    const int i = blockIdx.x;
    griddep_wait();
    const int64_t width = a.merged_ld;
    const int32_t *mp = a.merged_pos + static_cast<int64_t>(i) * width;
    const int32_t *sel = a.sel + static_cast<int64_t>(i) * a.topk;
    int c = a.sel_cnt[i];
    if (c < 0 || c > a.topk) c = 0;
    int32_t *out = a.out_idx + static_cast<int64_t>(i) * a.topk;
    int32_t *loc = a.local_idx + static_cast<int64_t>(i) * a.topk;
    if (threadIdx.x == 0) base_sh = 0;
    __syncthreads();
    for (int j0 = 0; j0 < a.topk; j0 += kShardThreads) {
        const int j = j0 + threadIdx.x;
        int32_t g = -1;
        if (j < c) {
            const int s = sel[j];
            g = (s >= 0 && s < width) ? mp[s] : -1;
        }
        if (j < a.topk) out[j] = g;
        const bool mine = g >= a.row_begin && g < a.row_end;
        int total;
        const int slot = block_excl_scan(mine ? 1 : 0, warp_tot, total);
        const int base = base_sh;
        if (mine) loc[base + slot] = g - a.row_begin;
        __syncthreads();
        if (threadIdx.x == 0) base_sh = base + total;
        __syncthreads();
    }
    const int nl = base_sh;
    for (int j = nl + threadIdx.x; j < a.topk; j += kShardThreads) loc[j] = -1;
    if (threadIdx.x == 0) {
        a.out_cnt[i] = c;
        a.local_cnt[i] = nl;
    }
}

// o = sum_g exp(lse_g - lse) o_g, lse = log sum_g exp(lse_g) over the parts
// with a non-empty selection.  One CTA per (query, 2 heads); thread t owns 4
// dims of head 2 * blockIdx.x + t / 128.
__global__ void __launch_bounds__(kShardThreads) shard_combine_kernel(const ShardCombineArgs a) {
    __shared__ float wgt[2][kMaxShards];
    const int hp = blockIdx.x, i = blockIdx.y;
    griddep_wait();
    const int hl = threadIdx.x >> 7;
    const int h = hp * 2 + hl;
    if (threadIdx.x < 64) {
        const int wl = threadIdx.x >> 5, g = threadIdx.x & 31;
        const int hh = hp * 2 + wl;
        float m = -INFINITY, wv = 0.f, L = 0.f;
        // up to 64 parts: lanes take g and g + 32
        float l0 = -INFINITY, l1 = -INFINITY;
        if (g < a.n_parts && a.part_cnt[static_cast<int64_t>(g) * a.n_q + i] > 0)
            l0 = a.part_lse[(static_cast<int64_t>(g) * a.n_q + i) * a.heads + hh];
        if (g + 32 < a.n_parts && a.part_cnt[static_cast<int64_t>(g + 32) * a.n_q + i] > 0)
            l1 = a.part_lse[(static_cast<int64_t>(g + 32) * a.n_q + i) * a.heads + hh];
        m = fmaxf(l0, l1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float w0 = l0 == -INFINITY ? 0.f : expf(l0 - m);
        const float w1 = l1 == -INFINITY ? 0.f : expf(l1 - m);
        L = w0 + w1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        wv = L > 0.f ? 1.f / L : 0.f;
        if (g < kMaxShards) wgt[wl][g] = w0 * wv;
        if (g + 32 < kMaxShards) wgt[wl][g + 32] = w1 * wv;
        if (g == 0 && a.lse) a.lse[static_cast<int64_t>(i) * a.heads + hh] = L > 0.f ? m + logf(L) : -INFINITY;
    }
    __syncthreads();
    const int d = (threadIdx.x & 127) * 4;
    if (d >= a.d_lat) return;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    for (int g = 0; g < a.n_parts; ++g) {
        const float wv = wgt[hl][g];
        if (wv == 0.f) continue;
        const __nv_bfloat16 *o =
            static_cast<const __nv_bfloat16 *>(a.part_out) + ((static_cast<int64_t>(g) * a.n_q + i) * a.heads + h) * a.d_lat + d;
        const uint2 raw = *reinterpret_cast<const uint2 *>(o);
        const __nv_bfloat162 x01 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 x23 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        const float2 f01 = __bfloat1622float2(x01), f23 = __bfloat1622float2(x23);
        acc0 = fmaf(wv, f01.x, acc0);
        acc1 = fmaf(wv, f01.y, acc1);
        acc2 = fmaf(wv, f23.x, acc2);
        acc3 = fmaf(wv, f23.y, acc3);
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.out) + (static_cast<int64_t>(i) * a.heads + h) * a.d_lat + d;
    __align__(8) __nv_bfloat16 ob[4] = {__float2bfloat16_rn(acc0), __float2bfloat16_rn(acc1),
                                        __float2bfloat16_rn(acc2), __float2bfloat16_rn(acc3)};
    *reinterpret_cast<uint2 *>(o) = *reinterpret_cast<const uint2 *>(ob);
}

}  // namespace

cudaError_t launch_shard_candidates(const ShardArgs &a, cudaStream_t st) {
    return launch_pdl(shard_candidates_kernel, dim3(a.n_q), dim3(kShardThreads), 0, st, a);
}

cudaError_t launch_shard_compact(const ShardArgs &a, cudaStream_t st) {
    return launch_pdl(shard_compact_kernel, dim3(a.n_q), dim3(kShardThreads), 0, st, a);
}

cudaError_t launch_shard_map(const ShardArgs &a, cudaStream_t st) {
    return launch_pdl(shard_map_kernel, dim3(a.n_q), dim3(kShardThreads), 0, st, a);
}

cudaError_t launch_shard_combine(const ShardCombineArgs &a, cudaStream_t st) {
    return launch_pdl(shard_combine_kernel, dim3(a.heads / 2, a.n_q), dim3(kShardThreads), 0, st, a);
}

}  // namespace dsa
