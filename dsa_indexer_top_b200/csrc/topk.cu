// topk.cu -- causal top-k selection of indexer scores.
//
// For query i with n = q_pos[i] + 1 visible rows keep k = min(topk, n) rows with
// the largest scores, ties to the lower position, written in ascending position
// order and padded with -1 ("GLM-5.2 -- Model techniques map", "Checked in its
// code", Indexer-selected sparse attention: min(index_topk, n) largest, int32).
//
// No sort.  Scores are mapped to order-preserving 32-bit keys and the k-th
// largest key T is found by a most-significant-digit radix select with digits of
// 12, 12 and 8 bits.  Only the first digit is taken over the whole row: every
// row whose first digit is >= the threshold digit is copied, in position order,
// into a candidate list (a few thousand rows), and the last two digits are
// resolved on that list in shared memory.  The output is an ordered filter of the
// candidates: keys > T, then the first `need_eq` keys == T in position order (the
// lower-position tie rule), written at their exclusive-scan slots.  When ties
// make the candidate list too long the same digits are resolved by streaming the
// row again (correct for any input, slower).
//
// Two schedules:
//   row    one CTA per query (contexts up to 64K): histogram pass, candidate
//          pass (L2-hot), refine + write -- a single launch.
//   split  long contexts with few queries: P CTAs per query build a global
//          first-digit histogram (atomics), then collect their chunk's
//          candidates into the workspace, then one CTA per query merges the
//          chunks (in position order) and finishes as above.
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kT = 512;                // threads per CTA
constexpr int kWarps = kT / 32;
constexpr int kBins = 4096;            // first and second digit (12 bits)
constexpr int kBins3 = 256;            // third digit (8 bits)
constexpr int kCap = 10240;            // candidates kept in shared memory
constexpr int kV = 4;                  // consecutive rows per thread per tile

struct TopkSmem {
    uint32_t hist[kBins];
    uint32_t cand_key[kCap];
    int32_t cand_pos[kCap];
    uint64_t scan[kWarps];
    uint32_t sel[4];
};

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t b = __float_as_uint(f);
    if (b == 0x80000000u) b = 0u;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide scan (64-bit); returns the block total in `total`.
__device__ __forceinline__ uint64_t block_scan(uint64_t v, uint64_t *buf, uint64_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint64_t t = lane < kWarps ? buf[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kWarps) buf[lane] = t;
    }
    __syncthreads();
    const uint64_t before = warp == 0 ? 0 : buf[warp - 1];
    total = buf[kWarps - 1];
    __syncthreads();
    return before + x - v;
}

// Add one to hist[d] for every lane with d != ~0u (warp-aggregated).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t d) {
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    if (d != 0xFFFFFFFFu && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[d], __popc(peers));
}

__device__ __forceinline__ void zero_hist(uint32_t *hist, int nbins) {
    for (int b = threadIdx.x; b < nbins; b += kT) hist[b] = 0;
}

// The digit holding the r-th largest key: sel[0] = digit, sel[1] = rows in
// higher bins.  Requires sum(hist) >= r >= 1.
__device__ __forceinline__ void find_digit(const uint32_t *hist, int nbins, uint32_t r, uint64_t *scan,
                                           uint32_t *sel) {
    const int per = nbins / kT > 0 ? nbins / kT : 1;
    const int b0 = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j)
        if (b0 + j < nbins) mine += hist[b0 + j];
    uint64_t all;
    const uint64_t before = block_scan(mine, scan, all);
    uint32_t above = static_cast<uint32_t>(all - before - mine);
    for (int j = per - 1; j >= 0; --j) {
        if (b0 + j >= nbins) continue;
        const uint32_t upto = above + hist[b0 + j];
        if (upto >= r && above < r) {
            sel[0] = b0 + j;
            sel[1] = above;
        }
        above = upto;
    }
    __syncthreads();
}

// Histogram of digit (u >> shift) & dmask over rows [lo, hi) of a score row
// whose key matches `prefix` under `pmask`.
__device__ __forceinline__ void stream_hist(const float *row, int lo, int hi, uint32_t prefix, uint32_t pmask,
                                            int shift, uint32_t dmask, uint32_t *hist) {
    for (int base = lo; base < hi; base += kT * kV) {
        const int e0 = base + threadIdx.x * kV;
        float v[kV];
        if (e0 + kV <= hi) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
            v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
        } else {
#pragma unroll
            for (int x = 0; x < kV; ++x) v[x] = e0 + x < hi ? __ldg(row + e0 + x) : 0.f;
        }
#pragma unroll
        for (int x = 0; x < kV; ++x) {
            const uint32_t u = order_key(v[x]);
            const bool in = e0 + x < hi && (u & pmask) == prefix;
            hist_add(hist, in ? (u >> shift) & dmask : 0xFFFFFFFFu);
        }
    }
    __syncthreads();
}

// Resolve the last two digits on a candidate list (keys in shared memory):
// returns T and the number of rows equal to T to keep.
__device__ __forceinline__ void refine_candidates(TopkSmem &sm, int m, uint32_t d1, uint32_t r2, uint32_t &T,
                                                  uint32_t &need_eq) {
    zero_hist(sm.hist, kBins);
    __syncthreads();
    for (int base = 0; base < m; base += kT) {
        const int c = base + threadIdx.x;
        uint32_t d = 0xFFFFFFFFu;
        if (c < m) {
            const uint32_t u = sm.cand_key[c];
            if ((u >> 20) == d1) d = (u >> 8) & 0xFFFu;
        }
        hist_add(sm.hist, d);
    }
    __syncthreads();
    find_digit(sm.hist, kBins, r2, sm.scan, sm.sel);
    const uint32_t d2 = sm.sel[0];
    const uint32_t r3 = r2 - sm.sel[1];
    __syncthreads();
    zero_hist(sm.hist, kBins3);
    __syncthreads();
    const uint32_t p24 = (d1 << 12) | d2;
    for (int base = 0; base < m; base += kT) {
        const int c = base + threadIdx.x;
        uint32_t d = 0xFFFFFFFFu;
        if (c < m) {
            const uint32_t u = sm.cand_key[c];
            if ((u >> 8) == p24) d = u & 0xFFu;
        }
        hist_add(sm.hist, d);
    }
    __syncthreads();
    find_digit(sm.hist, kBins3, r3, sm.scan, sm.sel);
    T = (p24 << 8) | sm.sel[0];
    need_eq = r3 - sm.sel[1];
    __syncthreads();
}

// Resolve the last two digits by streaming the whole row (tie-heavy fallback).
__device__ __forceinline__ void refine_stream(TopkSmem &sm, const float *row, int n, uint32_t d1, uint32_t r2,
                                              uint32_t &T, uint32_t &need_eq) {
    zero_hist(sm.hist, kBins);
    __syncthreads();
    stream_hist(row, 0, n, d1 << 20, 0xFFF00000u, 8, 0xFFFu, sm.hist);
    find_digit(sm.hist, kBins, r2, sm.scan, sm.sel);
    const uint32_t d2 = sm.sel[0];
    const uint32_t r3 = r2 - sm.sel[1];
    __syncthreads();
    zero_hist(sm.hist, kBins3);
    __syncthreads();
    const uint32_t p24 = (d1 << 12) | d2;
    stream_hist(row, 0, n, p24 << 8, 0xFFFFFF00u, 0, 0xFFu, sm.hist);
    find_digit(sm.hist, kBins3, r3, sm.scan, sm.sel);
    T = (p24 << 8) | sm.sel[0];
    need_eq = r3 - sm.sel[1];
    __syncthreads();
}

// Ordered filter: keep keys > T and the first need_eq keys == T (in list
// order), writing their positions to out[] at exclusive-scan slots.  The list is
// either the candidates in shared memory or the row itself.
template <bool kFromCandidates>
__device__ __forceinline__ void ordered_write(TopkSmem &sm, const float *row, int m, uint32_t T,
                                              uint32_t need_eq, int32_t *out) {
    uint32_t g_run = 0, e_run = 0;
    for (int base = 0; base < m; base += kT * kV) {
        const int e0 = base + threadIdx.x * kV;
        uint32_t u[kV];
        int32_t p[kV];
        uint32_t tg = 0, te = 0;
#pragma unroll
        for (int x = 0; x < kV; ++x) {
            const int e = e0 + x;
            u[x] = 0;
            p[x] = -1;
            if (e < m) {
                if (kFromCandidates) {
                    u[x] = sm.cand_key[e];
                    p[x] = sm.cand_pos[e];
                } else {
                    u[x] = order_key(__ldg(row + e));
                    p[x] = e;
                }
                tg += u[x] > T;
                te += u[x] == T;
            }
        }
        uint64_t tot;
        const uint64_t ex = block_scan((static_cast<uint64_t>(te) << 32) | tg, sm.scan, tot);
        uint32_t g = g_run + static_cast<uint32_t>(ex & 0xFFFFFFFFu);
        uint32_t q = e_run + static_cast<uint32_t>(ex >> 32);
#pragma unroll
        for (int x = 0; x < kV; ++x) {
            if (p[x] < 0) continue;
            if (u[x] > T) {
                out[g + min(q, need_eq)] = p[x];
                ++g;
            } else if (u[x] == T) {
                if (q < need_eq) out[g + q] = p[x];
                ++q;
            }
        }
        g_run += static_cast<uint32_t>(tot & 0xFFFFFFFFu);
        e_run += static_cast<uint32_t>(tot >> 32);
    }
}

// Copy rows [lo, hi) whose first digit is >= d1 into dst (position order).
// Returns the number of such rows (may exceed cap; only cap are stored).
template <bool kToShared>
__device__ __forceinline__ uint32_t collect(const float *row, int lo, int hi, uint32_t d1, TopkSmem &sm,
                                            uint2 *gdst, uint32_t cap) {
    uint32_t run = 0;
    for (int base = lo; base < hi; base += kT * kV) {
        const int e0 = base + threadIdx.x * kV;
        float v[kV];
        if (e0 + kV <= hi) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
            v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
        } else {
#pragma unroll
            for (int x = 0; x < kV; ++x) v[x] = e0 + x < hi ? __ldg(row + e0 + x) : 0.f;
        }
        uint32_t u[kV];
        uint32_t c = 0;
#pragma unroll
        for (int x = 0; x < kV; ++x) {
            u[x] = order_key(v[x]);
            c += (e0 + x < hi) && (u[x] >> 20) >= d1;
        }
        uint64_t tot;
        uint32_t off = run + static_cast<uint32_t>(block_scan(c, sm.scan, tot));
#pragma unroll
        for (int x = 0; x < kV; ++x) {
            if (e0 + x < hi && (u[x] >> 20) >= d1) {
                if (off < cap) {
                    if (kToShared) {
                        sm.cand_key[off] = u[x];
                        sm.cand_pos[off] = e0 + x;
                    } else {
                        gdst[off] = make_uint2(u[x], static_cast<uint32_t>(e0 + x));
                    }
                }
                ++off;
            }
        }
        run += static_cast<uint32_t>(tot);
    }
    __syncthreads();
    return run;
}

__device__ __forceinline__ int visible_rows(const TopkArgs &a, int i) {
    const int pos = a.q_pos[i];
    if (pos < 0 || pos >= a.L) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
        return 0;
    }
    return pos + 1;
}

// Every visible row is kept (n <= topk).
__device__ __forceinline__ void write_all(const TopkArgs &a, int i, int n) {
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    for (int p = threadIdx.x; p < a.topk; p += kT) out[p] = p < n ? p : -1;
    if (threadIdx.x == 0) a.cnt[i] = n;
}

// Shared tail: given the first digit d1 (with `above1` rows above it) and a
// candidate list of m rows in shared memory (or overflow), finish the query.
__device__ __forceinline__ void finish(const TopkArgs &a, TopkSmem &sm, const float *row, int i, int n,
                                       uint32_t d1, uint32_t above1, int m, bool overflow) {
    const uint32_t k = static_cast<uint32_t>(a.topk);
    uint32_t T, need_eq;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    if (!overflow) {
        refine_candidates(sm, m, d1, k - above1, T, need_eq);
        ordered_write<true>(sm, row, m, T, need_eq, out);
    } else {
        refine_stream(sm, row, n, d1, k - above1, T, need_eq);
        ordered_write<false>(sm, row, n, T, need_eq, out);
    }
    if (threadIdx.x == 0) a.cnt[i] = a.topk;
}

// ---------------------------------------------------------------- row schedule
__global__ void __launch_bounds__(kT, 1) topk_row_kernel(const TopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    const int i = blockIdx.x;
    const int n = visible_rows(a, i);
    if (n <= a.topk) {
        write_all(a, i, n);
        return;
    }
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    zero_hist(sm.hist, kBins);
    __syncthreads();
    stream_hist(row, 0, n, 0u, 0u, 20, 0xFFFu, sm.hist);
    find_digit(sm.hist, kBins, static_cast<uint32_t>(a.topk), sm.scan, sm.sel);
    const uint32_t d1 = sm.sel[0], above1 = sm.sel[1];
    const uint32_t m_est = above1 + sm.hist[d1];
    __syncthreads();
    bool overflow = m_est > static_cast<uint32_t>(kCap);
    uint32_t m = 0;
    if (!overflow) m = collect<true>(row, 0, n, d1, sm, nullptr, kCap);
    finish(a, sm, row, i, n, d1, above1, static_cast<int>(m), overflow);
}

// ---------------------------------------------------------------- split schedule
// (1) first-digit histogram of a chunk, added into the query's global histogram.
__global__ void __launch_bounds__(kT, 2) topk_hist_kernel(const TopkArgs a, int chunk) {
    __shared__ uint32_t hist[kBins];
    const int i = blockIdx.y, p = blockIdx.x;
    const int n = visible_rows(a, i);
    if (n <= a.topk) return;
    const int lo = min(n, p * chunk), hi = min(n, lo + chunk);
    if (lo >= hi) return;
    zero_hist(hist, kBins);
    __syncthreads();
    stream_hist(a.scores + static_cast<int64_t>(i) * a.ld, lo, hi, 0u, 0u, 20, 0xFFFu, hist);
    uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
    for (int b = threadIdx.x; b < kBins; b += kT)
        if (hist[b]) atomicAdd(&g[b], hist[b]);
}

// (2) the chunk's candidates (first digit >= the threshold digit), in order.
__global__ void __launch_bounds__(kT, 1) topk_collect_kernel(const TopkArgs a, int chunk) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    const int i = blockIdx.y, p = blockIdx.x;
    const int n = visible_rows(a, i);
    if (n <= a.topk) return;
    const int lo = min(n, p * chunk), hi = min(n, lo + chunk);
    const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
    for (int b = threadIdx.x; b < kBins; b += kT) sm.hist[b] = g[b];
    __syncthreads();
    find_digit(sm.hist, kBins, static_cast<uint32_t>(a.topk), sm.scan, sm.sel);
    const uint32_t d1 = sm.sel[0];
    __syncthreads();
    uint2 *dst = a.gcand + (static_cast<int64_t>(i) * kSplitMax + p) * kSplitCap;
    const uint32_t c = collect<false>(a.scores + static_cast<int64_t>(i) * a.ld, lo, hi, d1, sm, dst, kSplitCap);
    if (threadIdx.x == 0) a.gcount[static_cast<int64_t>(i) * kSplitMax + p] = c;
}

// (3) merge the chunks' candidates in position order and finish the query.
__global__ void __launch_bounds__(kT, 1) topk_merge_kernel(const TopkArgs a, int n_chunks) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    __shared__ uint32_t offs[kSplitMax + 1];
    __shared__ int bad;
    const int i = blockIdx.x;
    const int n = visible_rows(a, i);
    if (n <= a.topk) {
        write_all(a, i, n);
        return;
    }
    const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
    for (int b = threadIdx.x; b < kBins; b += kT) sm.hist[b] = g[b];
    __syncthreads();
    find_digit(sm.hist, kBins, static_cast<uint32_t>(a.topk), sm.scan, sm.sel);
    const uint32_t d1 = sm.sel[0], above1 = sm.sel[1];
    if (threadIdx.x == 0) {
        uint32_t o = 0;
        int ov = 0;
        for (int p = 0; p < n_chunks; ++p) {
            const uint32_t c = a.gcount[static_cast<int64_t>(i) * kSplitMax + p];
            offs[p] = o;
            o += c;
            ov |= c > static_cast<uint32_t>(kSplitCap);
        }
        offs[n_chunks] = o;
        bad = ov || o > static_cast<uint32_t>(kCap);
    }
    __syncthreads();
    const bool overflow = bad != 0;
    const int m = overflow ? 0 : static_cast<int>(offs[n_chunks]);
    if (!overflow) {
        for (int p = 0; p < n_chunks; ++p) {
            const uint2 *src = a.gcand + (static_cast<int64_t>(i) * kSplitMax + p) * kSplitCap;
            const int c = static_cast<int>(offs[p + 1] - offs[p]);
            for (int j = threadIdx.x; j < c; j += kT) {
                const uint2 v = src[j];
                sm.cand_key[offs[p] + j] = v.x;
                sm.cand_pos[offs[p] + j] = static_cast<int32_t>(v.y);
            }
        }
        __syncthreads();
    }
    finish(a, sm, a.scores + static_cast<int64_t>(i) * a.ld, i, n, d1, above1, m, overflow);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

}  // namespace

bool topk_uses_split(int n_q, int max_ctx) { return max_ctx > kTopkRowMaxCtx && n_q <= kTopkSplitMaxQueries; }

cudaError_t launch_topk(const TopkArgs &a, int num_sms, cudaStream_t st) {
    const size_t smem = sizeof(TopkSmem);
    cudaError_t e;
    if (!topk_uses_split(a.n_q, a.L)) {
        if ((e = set_smem(topk_row_kernel, smem)) != cudaSuccess) return e;
        topk_row_kernel<<<a.n_q, kT, smem, st>>>(a);
        return cudaGetLastError();
    }
    int P = (2 * num_sms + a.n_q - 1) / a.n_q;
    P = P < 1 ? 1 : (P > kSplitMax ? kSplitMax : P);
    int chunk = (a.L + P - 1) / P;
    chunk = (chunk + kT * kV - 1) / (kT * kV) * (kT * kV);
    P = (a.L + chunk - 1) / chunk;
    if ((e = cudaMemsetAsync(a.ghist, 0, sizeof(uint32_t) * kBins * a.n_q, st)) != cudaSuccess) return e;
    topk_hist_kernel<<<dim3(P, a.n_q), kT, 0, st>>>(a, chunk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = set_smem(topk_collect_kernel, smem)) != cudaSuccess) return e;
    topk_collect_kernel<<<dim3(P, a.n_q), kT, smem, st>>>(a, chunk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = set_smem(topk_merge_kernel, smem)) != cudaSuccess) return e;
    topk_merge_kernel<<<a.n_q, kT, smem, st>>>(a, P);
    return cudaGetLastError();
}

size_t topk_scratch_bytes(int n_q, int max_ctx) {
    if (!topk_uses_split(n_q, max_ctx)) return 0;
    const size_t hist = sizeof(uint32_t) * kBins * n_q;
    const size_t counts = sizeof(uint32_t) * kSplitMax * n_q;
    const size_t cand = sizeof(uint2) * static_cast<size_t>(kSplitCap) * kSplitMax * n_q;
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    return al(hist) + al(counts) + al(cand);
}

void topk_bind_scratch(TopkArgs &a, void *scratch) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    uint8_t *p = static_cast<uint8_t *>(scratch);
    a.ghist = reinterpret_cast<uint32_t *>(p);
    p += al(sizeof(uint32_t) * kBins * a.n_q);
    a.gcount = reinterpret_cast<uint32_t *>(p);
    p += al(sizeof(uint32_t) * kSplitMax * a.n_q);
    a.gcand = reinterpret_cast<uint2 *>(p);
}

}  // namespace dsa
