// topk.cu -- causal top-k selection of indexer scores.
//
// For query i with n = q_pos[i] + 1 visible rows keep k = min(topk, n) rows with
// the largest scores, ties to the lower position, written in ascending position
// order and padded with -1 ("GLM-5.2 -- Model techniques map", "Checked in its
// code", Indexer-selected sparse attention: min(index_topk, n) largest, int32).
//
// One thread-block cluster (1..16 CTAs) per query; CTA r owns a contiguous chunk
// of positions.  No sort: a most-significant-digit radix select over the
// order-preserving 32-bit image of the float scores, three digits (11, 11, 10
// bits).  Each pass builds a shared-memory histogram of the next digit among the
// rows that still match the threshold prefix (warp-aggregated atomics), the
// cluster's histograms are summed through distributed shared memory, and the
// digit holding the k-th largest key is found with a block-wide suffix scan.
// After three passes the threshold key T is exact and `need_eq` rows equal to T
// must be taken.  An ordered compaction follows: per-CTA counts of rows > T and
// == T are exchanged through distributed shared memory, and each CTA writes its
// kept positions at the right slots (rows == T kept first-come in position
// order, which is the lower-position tie rule).  All cross-CTA synchronisation is
// the hardware cluster barrier; nothing spins.  A CTA keeps its chunk of keys in
// shared memory when it fits, else re-reads the scores (L2) every pass.
#include <cooperative_groups.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kBins = 2048;
constexpr int kPerThread = 8;  // consecutive rows per thread in the ordered write

// Order-preserving map float -> uint32 (larger float -> larger key); -0.0 is
// folded onto +0.0 so the two compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t b = __float_as_uint(f);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide scan of a 64-bit value (two packed 32-bit counters);
// also returns the block total.  Every thread of the block must call it.
__device__ __forceinline__ uint64_t block_excl_scan(uint64_t v, uint64_t *buf, uint64_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint64_t t = lane < kTkWarps ? buf[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint64_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kTkWarps) buf[lane] = t;
    }
    __syncthreads();
    const uint64_t before = warp == 0 ? 0 : buf[warp - 1];
    total = buf[kTkWarps - 1];
    __syncthreads();
    return before + x - v;
}

__global__ void __launch_bounds__(kTkThreads, 1) topk_cluster_kernel(const TopkArgs a) {
    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int i = blockIdx.x / C;
    const int tid = threadIdx.x, lane = tid & 31;

    __shared__ uint32_t hist[2][kBins];
    __shared__ uint64_t scan_buf[32];
    __shared__ uint32_t sel_digit, sel_above;
    __shared__ uint32_t cta_counts[2];  // rows > T, rows == T in this CTA's chunk
    __shared__ int32_t cta_plan[2];     // first output slot, quota of rows == T
    extern __shared__ uint32_t cache[];

    int pos = a.q_pos[i];
    if (pos < 0 || pos >= a.L) {
        if (rank == 0 && tid == 0) report_status(a.status, DSA_ERR_INVALID);
        pos = -1;
    }
    const int n = pos + 1;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    if (n <= a.topk) {
        // every visible row is kept (every CTA of the cluster takes this branch)
        for (int p = rank * kTkThreads + tid; p < a.topk; p += C * kTkThreads) out[p] = p < n ? p : -1;
        if (rank == 0 && tid == 0) a.cnt[i] = n;
        return;
    }
    const int k = a.topk;
    const int chunk = (((n + C - 1) / C) + 3) & ~3;
    const int lo = min(n, rank * chunk);
    const int hi = min(n, lo + chunk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    const bool cached = chunk <= a.cache_cap;
    if (cached) {
        for (int e = lo + tid * 4; e < hi; e += kTkThreads * 4) {
            if (e + 3 < hi) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(row + e));
                cache[e - lo] = order_key(v.x);
                cache[e - lo + 1] = order_key(v.y);
                cache[e - lo + 2] = order_key(v.z);
                cache[e - lo + 3] = order_key(v.w);
            } else {
                for (int x = e; x < hi; ++x) cache[x - lo] = order_key(__ldg(row + x));
            }
        }
        __syncthreads();
    }

    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
        uint32_t *h = hist[pass & 1];
        for (int b = tid; b < kBins; b += kTkThreads) h[b] = 0;
        __syncthreads();
        for (int base = lo; base < hi; base += kTkThreads) {
            const int e = base + tid;
            uint32_t d = 0xFFFFFFFFu;
            if (e < hi) {
                const uint32_t u = cached ? cache[e - lo] : order_key(__ldg(row + e));
                if ((u & pmask) == prefix) d = (u >> shift) & dmask;
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (d != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&h[d], __popc(peers));
        }
        cluster.sync();  // every CTA's histogram of this pass is complete
        uint32_t tot[4];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t t = 0;
            for (int r = 0; r < C; ++r) t += cluster.map_shared_rank(h, r)[tid * 4 + j];
            tot[j] = t;
            mine += t;
        }
        uint64_t all;
        const uint64_t before = block_excl_scan(mine, scan_buf, all);
        // rows in bins above this thread's four bins
        uint32_t above = static_cast<uint32_t>(all - before - mine);
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            const uint32_t upto = above + tot[j];  // rows in bins >= tid*4 + j
            if (upto >= static_cast<uint32_t>(remaining) && above < static_cast<uint32_t>(remaining)) {
                sel_digit = tid * 4 + j;
                sel_above = above;
            }
            above = upto;
        }
        __syncthreads();
        remaining -= static_cast<int>(sel_above);
        prefix |= sel_digit << shift;
        pmask |= dmask << shift;
        __syncthreads();  // sel_digit / sel_above are rewritten next pass
    }
    const uint32_t T = prefix;
    const int need_eq = remaining;  // rows equal to T that are kept (>= 1)

    // ----------------------------------------------------------- ordered write
    uint32_t gt = 0, eq = 0;
    for (int e = lo + tid; e < hi; e += kTkThreads) {
        const uint32_t u = cached ? cache[e - lo] : order_key(__ldg(row + e));
        gt += u > T;
        eq += u == T;
    }
    uint64_t tot_pair;
    block_excl_scan((static_cast<uint64_t>(eq) << 32) | gt, scan_buf, tot_pair);
    if (tid == 0) {
        cta_counts[0] = static_cast<uint32_t>(tot_pair & 0xFFFFFFFFu);
        cta_counts[1] = static_cast<uint32_t>(tot_pair >> 32);
    }
    cluster.sync();
    if (tid == 0) {
        int eq_before = 0, sel_before = 0;
        for (int r = 0; r < rank; ++r) {
            const uint32_t *rc = cluster.map_shared_rank(cta_counts, r);
            const int g_r = static_cast<int>(rc[0]), e_r = static_cast<int>(rc[1]);
            sel_before += g_r + max(0, min(need_eq - eq_before, e_r));
            eq_before += e_r;
        }
        cta_plan[0] = sel_before;
        cta_plan[1] = max(0, min(need_eq - eq_before, static_cast<int>(cta_counts[1])));
    }
    cluster.sync();  // remote reads done: shared memory of every CTA may be released
    const int sel_before = cta_plan[0];
    const int quota = cta_plan[1];
    uint32_t g_run = 0, e_run = 0;
    for (int base = lo; base < hi; base += kTkThreads * kPerThread) {
        const int e0 = base + tid * kPerThread;
        uint32_t u[kPerThread];
        uint32_t tg = 0, te = 0;
#pragma unroll
        for (int x = 0; x < kPerThread; ++x) {
            const int e = e0 + x;
            u[x] = 0u;
            if (e < hi) u[x] = cached ? cache[e - lo] : order_key(__ldg(row + e));
            tg += (e < hi) && u[x] > T;
            te += (e < hi) && u[x] == T;
        }
        uint64_t tile_tot;
        const uint64_t ex = block_excl_scan((static_cast<uint64_t>(te) << 32) | tg, scan_buf, tile_tot);
        uint32_t g = g_run + static_cast<uint32_t>(ex & 0xFFFFFFFFu);
        uint32_t q = e_run + static_cast<uint32_t>(ex >> 32);
#pragma unroll
        for (int x = 0; x < kPerThread; ++x) {
            const int e = e0 + x;
            if (e >= hi) break;
            if (u[x] > T) {
                out[sel_before + g + min(q, static_cast<uint32_t>(quota))] = e;
                ++g;
            } else if (u[x] == T) {
                if (q < static_cast<uint32_t>(quota)) out[sel_before + g + q] = e;
                ++q;
            }
        }
        g_run += static_cast<uint32_t>(tile_tot & 0xFFFFFFFFu);
        e_run += static_cast<uint32_t>(tile_tot >> 32);
    }
    if (rank == C - 1) {
        for (int p = k + tid; p < a.topk; p += kTkThreads) out[p] = -1;
    }
    if (rank == 0 && tid == 0) a.cnt[i] = k;
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, int num_sms, cudaStream_t st) {
    // Cluster size: enough CTAs to cover the SMs for small batches, and small
    // enough chunks to stay in shared memory where possible.
    int C = 1;
    while (C < 16 && ((a.L + C - 1) / C > a.cache_cap || static_cast<long long>(a.n_q) * C < 2LL * num_sms))
        C *= 2;
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    cfg.blockDim = dim3(kTkThreads, 1, 1);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Shrink the cluster until the hardware can co-schedule one.
    for (;; C /= 2) {
        const int chunk = (((a.L + C - 1) / C) + 3) & ~3;
        const size_t smem = chunk <= a.cache_cap ? static_cast<size_t>(chunk) * sizeof(uint32_t) : 0;
        e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(static_cast<unsigned>(a.n_q) * C, 1, 1);
        cfg.dynamicSmemBytes = smem;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, topk_cluster_kernel, &cfg);
        if ((e == cudaSuccess && clusters > 0) || C == 1) break;
        (void)cudaGetLastError();
    }
    TopkArgs b = a;
    if ((((a.L + C - 1) / C) + 3 & ~3) > a.cache_cap) b.cache_cap = 0;
    return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, b);
}

}  // namespace dsa
