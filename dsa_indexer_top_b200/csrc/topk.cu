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
// row whose first digit is at or above a threshold digit is copied, in position
// order, into "warp segments" (each warp owns a contiguous slice of positions),
// and the remaining digits are resolved on those few thousand candidates.  The
// output is an ordered filter of the candidates: keys > T, then the first
// `need_eq` keys == T in position order (the lower-position tie rule); the slot
// of each kept row is its warp's prefix (one 16-entry sum) plus a ballot count
// inside the warp.  When ties make the candidate list too long the digits are
// resolved by streaming the row again (correct for any input, slower).
//
// The threshold digit comes from the first-digit histogram, which is
//   - left by the indexer's epilogue (decode: one query per tensor-core tile), or
//   - built here: a full pass for the split schedule, or, for the row schedule,
//     from a 1/16 sample with a safety margin; the candidates are then counted
//     exactly and the exact first digit is found among them (a sample that
//     overestimates falls back to the exact streaming path).
// Two schedules:
//   row    one CTA per query: threshold digit, one streaming candidate pass,
//          refine and write -- a single launch.
//   split  long contexts with few queries: P CTAs per query collect their
//          chunk's candidates (given the histogram), then one CTA per query
//          walks the chunks' candidates in position order and finishes.
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kT = 512;                // threads per CTA
constexpr int kWarps = kT / 32;
constexpr int kBins = kTopkBins;       // first and second digit (12 bits)
constexpr int kBins3 = 256;            // third digit (8 bits)
constexpr int kWCap = 640;             // candidates per warp segment (row schedule)
constexpr int kU = 8;                  // float4 loads in flight per thread when streaming
constexpr int kSampleEvery = 16;       // row schedule: one 128-row block in 16 is sampled
constexpr int kWarpCap = 128;          // collect kernel: candidates per warp per chunk

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

// Copy a query's first-digit histogram from global memory: every thread's
// eight loads are issued before any is used.
__device__ __forceinline__ void load_hist(uint32_t *hist, const uint32_t *g) {
    uint32_t v[kBins / kT];
#pragma unroll
    for (int j = 0; j < kBins / kT; ++j) v[j] = __ldg(g + threadIdx.x + j * kT);
#pragma unroll
    for (int j = 0; j < kBins / kT; ++j) hist[threadIdx.x + j * kT] = v[j];
}

__device__ __forceinline__ void zero_hist(uint32_t *hist, int nbins) {
    for (int b = threadIdx.x; b < nbins; b += kT) hist[b] = 0;
}

// The digit holding the r-th largest key: sel[0] = digit, sel[1] = rows in
// higher bins.  If the histogram holds fewer than r rows, sel = {0, total}.
// Thread t owns bins [t*per, t*per + per); one barrier: warp totals, then the
// rows above a thread = the warps above + a suffix scan inside its warp.
__device__ __forceinline__ void find_digit(const uint32_t *hist, int nbins, uint32_t r, uint64_t *scan,
                                           uint32_t *sel) {
    uint32_t *wsum = reinterpret_cast<uint32_t *>(scan);  // kWarps entries
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = nbins / kT > 0 ? nbins / kT : 1;
    const int b0 = threadIdx.x * per;
    uint32_t mine = 0;
    for (int j = 0; j < per; ++j)
        if (b0 + j < nbins) mine += hist[b0 + j];
    uint32_t suf = mine;  // rows in this lane's bins and every higher lane's
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
    }
    if (lane == 0) wsum[warp] = suf;
    __syncthreads();
    uint32_t above = suf - mine, total = 0;
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t x = wsum[w];
        total += x;
        if (w > warp) above += x;
    }
    if (threadIdx.x == 0 && total < r) {
        sel[0] = 0;
        sel[1] = total;
    }
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

// Load kU float4 groups of a row: element e = base + (j * kT + tid) * 4 + x.
__device__ __forceinline__ void load_block(const float *row, int base, int hi, float (&v)[kU][4]) {
#pragma unroll
    for (int j = 0; j < kU; ++j) {
        const int e0 = base + (j * kT + threadIdx.x) * 4;
        if (e0 + 4 <= hi) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
            v[j][0] = f.x, v[j][1] = f.y, v[j][2] = f.z, v[j][3] = f.w;
        } else {
#pragma unroll
            for (int x = 0; x < 4; ++x) v[j][x] = e0 + x < hi ? __ldg(row + e0 + x) : 0.f;
        }
    }
}

// Histogram of digit (u >> shift) & dmask over rows [lo, hi) whose key matches
// `prefix` under `pmask` (lo a multiple of 4).
__device__ __forceinline__ void stream_hist(const float *row, int lo, int hi, uint32_t prefix, uint32_t pmask,
                                            int shift, uint32_t dmask, uint32_t *hist) {
    for (int base = lo; base < hi; base += kT * 4 * kU) {
        float v[kU][4];
        load_block(row, base, hi, v);
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int e0 = base + (j * kT + threadIdx.x) * 4;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const uint32_t u = order_key(v[j][x]);
                const bool in = e0 + x < hi && (u & pmask) == prefix;
                hist_add_warp(hist, in ? (u >> shift) & dmask : 0xFFFFFFFFu);
            }
        }
    }
    __syncthreads();
}

// Ordered filter by streaming the row (fallback): keep keys > T and the first
// need_eq keys == T, at exclusive-scan slots.
__device__ __forceinline__ void stream_write(const float *row, int n, uint32_t T, uint32_t need_eq, int32_t *out,
                                             uint64_t *scan) {
    uint32_t g_run = 0, e_run = 0;
    for (int base = 0; base < n; base += kT * 4) {
        const int e0 = base + threadIdx.x * 4;
        uint32_t u[4];
        uint32_t tg = 0, te = 0;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            u[x] = e0 + x < n ? order_key(__ldg(row + e0 + x)) : 0u;
            tg += (e0 + x < n) && u[x] > T;
            te += (e0 + x < n) && u[x] == T;
        }
        uint64_t tot;
        const uint64_t ex = block_scan((static_cast<uint64_t>(te) << 32) | tg, scan, tot);
        uint32_t g = g_run + static_cast<uint32_t>(ex & 0xFFFFFFFFu);
        uint32_t q = e_run + static_cast<uint32_t>(ex >> 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (e0 + x >= n) continue;
            if (u[x] > T) {
                out[g + min(q, need_eq)] = e0 + x;
                ++g;
            } else if (u[x] == T) {
                if (q < need_eq) out[g + q] = e0 + x;
                ++q;
            }
        }
        g_run += static_cast<uint32_t>(tot & 0xFFFFFFFFu);
        e_run += static_cast<uint32_t>(tot >> 32);
    }
}

// Exact path by streaming: first digit d1 (rows above: above1) known.
__device__ __forceinline__ void finish_stream(const float *row, int n, uint32_t k, uint32_t d1, uint32_t above1,
                                              uint32_t *hist, uint64_t *scan, uint32_t *sel, int32_t *out) {
    const uint32_t r2 = k - above1;
    zero_hist(hist, kBins);
    __syncthreads();
    stream_hist(row, 0, n, d1 << 20, 0xFFF00000u, 8, 0xFFFu, hist);
    find_digit(hist, kBins, r2, scan, sel);
    const uint32_t d2 = sel[0];
    const uint32_t r3 = r2 - sel[1];
    __syncthreads();
    zero_hist(hist, kBins3);
    __syncthreads();
    const uint32_t p24 = (d1 << 12) | d2;
    stream_hist(row, 0, n, p24 << 8, 0xFFFFFF00u, 0, 0xFFu, hist);
    find_digit(hist, kBins3, r3, scan, sel);
    const uint32_t T = (p24 << 8) | sel[0];
    const uint32_t need_eq = r3 - sel[1];
    __syncthreads();
    stream_write(row, n, T, need_eq, out, scan);
}

// ------------------------------------------------------------ warp segments
// Candidates as (key, position) pairs in position order; warp w owns pieces
// whose positions all precede those of warp w + 1.
struct RowSegs {  // row schedule: one piece per warp, in shared memory
    const uint2 *wbuf;     // [kWarps][kWCap]
    const uint32_t *wcnt;  // [kWarps]
    __device__ int pieces(int) const { return 1; }
    __device__ const uint2 *ptr(int w, int) const { return wbuf + w * kWCap; }
    __device__ uint32_t count(int w, int) const { return min(wcnt[w], static_cast<uint32_t>(kWCap)); }
};

// Histogram of (u >> shift) & dmask over the candidates matching prefix/pmask.
template <class Segs>
__device__ __forceinline__ void seg_hist(const Segs &sg, uint32_t prefix, uint32_t pmask, int shift, uint32_t dmask,
                                         uint32_t *hist) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = 0; j < sg.pieces(w); ++j) {
        const uint2 *p = sg.ptr(w, j);
        const uint32_t c = sg.count(w, j);
        for (uint32_t b = 0; b < c; b += 32) {
            uint32_t d = 0xFFFFFFFFu;
            if (b + lane < c) {
                const uint32_t u = p[b + lane].x;
                if ((u & pmask) == prefix) d = (u >> shift) & dmask;
            }
            hist_add_warp(hist, d);
        }
    }
    __syncthreads();
}

// Resolve digits 2 and 3 on the candidates: T and the number of rows == T kept.
template <class Segs>
__device__ __forceinline__ void seg_refine(const Segs &sg, uint32_t d1, uint32_t r2, uint32_t *hist, uint64_t *scan,
                                           uint32_t *sel, uint32_t &T, uint32_t &need_eq) {
    zero_hist(hist, kBins);
    __syncthreads();
    seg_hist(sg, d1 << 20, 0xFFF00000u, 8, 0xFFFu, hist);
    find_digit(hist, kBins, r2, scan, sel);
    const uint32_t d2 = sel[0];
    const uint32_t r3 = r2 - sel[1];
    __syncthreads();
    zero_hist(hist, kBins3);
    __syncthreads();
    const uint32_t p24 = (d1 << 12) | d2;
    seg_hist(sg, p24 << 8, 0xFFFFFF00u, 0, 0xFFu, hist);
    find_digit(hist, kBins3, r3, scan, sel);
    T = (p24 << 8) | sel[0];
    need_eq = r3 - sel[1];
    __syncthreads();
}

// Ordered write of the kept candidates: per-warp counts, a 16-entry prefix,
// then ballots inside each warp.
template <class Segs>
__device__ __forceinline__ void seg_write(const Segs &sg, uint32_t T, uint32_t need_eq, int32_t *out,
                                          uint32_t *wg, uint32_t *we) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t g = 0, e = 0;
    for (int j = 0; j < sg.pieces(w); ++j) {
        const uint2 *p = sg.ptr(w, j);
        const uint32_t c = sg.count(w, j);
        for (uint32_t b = 0; b < c; b += 32) {
            const bool ok = b + lane < c;
            const uint32_t u = ok ? p[b + lane].x : 0u;
            g += __popc(__ballot_sync(0xffffffffu, ok && u > T));
            e += __popc(__ballot_sync(0xffffffffu, ok && u == T));
        }
    }
    if (lane == 0) {
        wg[w] = g;
        we[w] = e;
    }
    __syncthreads();
    uint32_t gtb = 0, eqb = 0;
    for (int x = 0; x < w; ++x) {
        gtb += wg[x];
        eqb += we[x];
    }
    const uint32_t lt = (1u << lane) - 1u;
    g = 0;
    e = 0;
    for (int j = 0; j < sg.pieces(w); ++j) {
        const uint2 *p = sg.ptr(w, j);
        const uint32_t c = sg.count(w, j);
        for (uint32_t b = 0; b < c; b += 32) {
            const bool ok = b + lane < c;
            const uint2 v = ok ? p[b + lane] : make_uint2(0u, 0u);
            const bool isg = ok && v.x > T, ise = ok && v.x == T;
            const uint32_t mg = __ballot_sync(0xffffffffu, isg), me = __ballot_sync(0xffffffffu, ise);
            const uint32_t gb = gtb + g + __popc(mg & lt), eb = eqb + e + __popc(me & lt);
            if (isg) out[gb + min(eb, need_eq)] = static_cast<int32_t>(v.y);
            if (ise && eb < need_eq) out[gb + eb] = static_cast<int32_t>(v.y);
            g += __popc(mg);
            e += __popc(me);
        }
    }
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

// ---------------------------------------------------------------- row schedule
struct RowSmem {
    uint32_t hist[kBins];
    uint2 wbuf[kWarps * kWCap];
    uint32_t wcnt[kWarps], wg[kWarps], we[kWarps];
    uint64_t scan[kWarps];
    uint32_t sel[4];
    int flag;
};

__global__ void __launch_bounds__(kT, 2) topk_row_kernel(const TopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem &sm = *reinterpret_cast<RowSmem *>(smem_raw);
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();
    const int n = visible_rows(a, i);
    if (n <= a.topk) {
        write_all(a, i, n);
        return;
    }
    const uint32_t k = static_cast<uint32_t>(a.topk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;

    // ---- 1. a threshold digit d_lo: rows with first digit >= d_lo are candidates
    uint32_t d_lo, above_exact = 0;
    const bool exact = a.hist_ready != 0;
    if (exact) {
        const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
        load_hist(sm.hist, g);
        __syncthreads();
        find_digit(sm.hist, kBins, k, sm.scan, sm.sel);
        d_lo = sm.sel[0];
        above_exact = sm.sel[1];
    } else {
        // sample: the first 128 rows of every kSampleEvery * 128
        zero_hist(sm.hist, kBins);
        __syncthreads();
        const int nblk = (n + 127) / 128;
        for (int bi = warp * kSampleEvery; bi < nblk; bi += kWarps * kSampleEvery) {
            const int e0 = bi * 128 + lane * 4;
            float v[4];
            if (e0 + 4 <= n) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
                v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
            } else {
#pragma unroll
                for (int x = 0; x < 4; ++x) v[x] = e0 + x < n ? __ldg(row + e0 + x) : 0.f;
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
                hist_add_warp(sm.hist, e0 + x < n ? first_digit(order_key(v[x])) : 0xFFFFFFFFu);
        }
        __syncthreads();
        // sampled rows, and the rank to look for among them (k scaled, +25% and +64)
        long long ns = 0;
        for (int bi = 0; bi < nblk; bi += kSampleEvery) ns += min(128, n - bi * 128);
        const long long want = (5LL * k * ns) / (4LL * n) + 64;
        const uint32_t ks = static_cast<uint32_t>(want < ns ? want : ns);
        find_digit(sm.hist, kBins, ks, sm.scan, sm.sel);
        d_lo = sm.sel[0];
    }
    __syncthreads();

    // ---- 2. candidates: each warp streams a contiguous slice of the row
    {
        const int sub = ((n + kWarps - 1) / kWarps + 127) / 128 * 128;
        const int wlo = min(n, warp * sub), whi = min(n, wlo + sub);
        uint2 *mine = sm.wbuf + warp * kWCap;
        uint32_t cnt = 0;
        for (int base = wlo; base < whi; base += 32 * 4 * kU) {
            float v[kU][4];
#pragma unroll
            for (int j = 0; j < kU; ++j) {
                const int e0 = base + (j * 32 + lane) * 4;
                if (e0 + 4 <= whi) {
                    const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
                    v[j][0] = f.x, v[j][1] = f.y, v[j][2] = f.z, v[j][3] = f.w;
                } else {
#pragma unroll
                    for (int x = 0; x < 4; ++x) v[j][x] = e0 + x < whi ? __ldg(row + e0 + x) : 0.f;
                }
            }
#pragma unroll
            for (int j = 0; j < kU; ++j) {
                const int e0 = base + (j * 32 + lane) * 4;
                uint32_t u[4], pick = 0;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    u[x] = order_key(v[j][x]);
                    if (e0 + x < whi && first_digit(u[x]) >= d_lo) pick |= 1u << x;
                }
                const uint32_t c = __popc(pick);
                uint32_t incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                uint32_t slot = cnt + incl - c;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    if (pick & (1u << x)) {
                        if (slot < kWCap) mine[slot] = make_uint2(u[x], static_cast<uint32_t>(e0 + x));
                        ++slot;
                    }
                }
                cnt += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0) sm.wcnt[warp] = cnt;
    }
    if (threadIdx.x == 0) sm.flag = 0;
    __syncthreads();
    if (threadIdx.x < kWarps && sm.wcnt[threadIdx.x] > static_cast<uint32_t>(kWCap)) sm.flag = 1;
    __syncthreads();
    bool overflow = sm.flag != 0;
    const RowSegs sg{sm.wbuf, sm.wcnt};

    // ---- 3. the exact first digit
    uint32_t d1 = d_lo, above1 = above_exact;
    if (!overflow && !exact) {
        zero_hist(sm.hist, kBins);
        __syncthreads();
        seg_hist(sg, 0u, 0u, 20, 0xFFFu, sm.hist);
        find_digit(sm.hist, kBins, k, sm.scan, sm.sel);
        uint32_t m = 0;
        for (int w = 0; w < kWarps; ++w) m += sm.wcnt[w];
        overflow = m < k;  // the sample overestimated the threshold: not enough candidates
        d1 = sm.sel[0];
        above1 = sm.sel[1];
        __syncthreads();
    }
    if (overflow) {
        if (!exact) {
            zero_hist(sm.hist, kBins);
            __syncthreads();
            stream_hist(row, 0, n, 0u, 0u, 20, 0xFFFu, sm.hist);
            find_digit(sm.hist, kBins, k, sm.scan, sm.sel);
            d1 = sm.sel[0];
            above1 = sm.sel[1];
            __syncthreads();
        }
        finish_stream(row, n, k, d1, above1, sm.hist, sm.scan, sm.sel, out);
    } else {
        uint32_t T, need_eq;
        seg_refine(sg, d1, k - above1, sm.hist, sm.scan, sm.sel, T, need_eq);
        seg_write(sg, T, need_eq, out, sm.wg, sm.we);
    }
    if (threadIdx.x == 0) a.cnt[i] = a.topk;
}

// ---------------------------------------------------------------- split schedule
// (1) first-digit histogram of a chunk, added into the query's global histogram.
__global__ void __launch_bounds__(kT, 2) topk_hist_kernel(const TopkArgs a, int chunk) {
    __shared__ uint32_t hist[kBins];
    const int i = blockIdx.y, p = blockIdx.x;
    griddep_wait();
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
// Each warp walks a contiguous slice of the chunk and compacts its candidates
// (warp prefix sums, so position order is kept) into a private buffer; the 16
// warp counts then place the slices in order.
__global__ void __launch_bounds__(kT, 2) topk_collect_kernel(const TopkArgs a, int chunk) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint64_t scan[kWarps];
    __shared__ uint32_t sel[4];
    __shared__ uint2 wbuf[kWarps][kWarpCap];
    __shared__ uint32_t wcount[kWarps], woff[kWarps + 1];
    const int i = blockIdx.y, p = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();
    const int n = visible_rows(a, i);
    if (n <= a.topk) return;
    const int lo = min(n, p * chunk), hi = min(n, lo + chunk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    const int sub = ((hi - lo + kWarps - 1) / kWarps + 127) / 128 * 128;
    const int wlo = min(hi, lo + warp * sub), whi = min(hi, wlo + sub);
    auto load_batch = [&](int base0, float (&v)[kU][4]) {
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int e0 = base0 + j * 128 + lane * 4;
            if (e0 + 4 <= whi) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
                v[j][0] = f.x, v[j][1] = f.y, v[j][2] = f.z, v[j][3] = f.w;
            } else {
#pragma unroll
                for (int x = 0; x < 4; ++x) v[j][x] = e0 + x < whi ? __ldg(row + e0 + x) : 0.f;
            }
        }
    };
    float v[kU][4];
    load_batch(wlo, v);  // in flight while the threshold digit is found
    const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
    load_hist(hist, g);
    __syncthreads();
    find_digit(hist, kBins, static_cast<uint32_t>(a.topk), scan, sel);
    const uint32_t d1 = sel[0];
    if (p == 0 && threadIdx.x == 0) {  // the merge reads the threshold digit from here
        a.gdigit[2 * i] = d1;
        a.gdigit[2 * i + 1] = sel[1];
    }
    uint32_t cnt = 0;
    for (int base0 = wlo; base0 < whi; base0 += 128 * kU) {
        if (base0 != wlo) load_batch(base0, v);
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int e0 = base0 + j * 128 + lane * 4;
            uint32_t u[4], pick = 0;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                u[x] = order_key(v[j][x]);
                if (e0 + x < whi && first_digit(u[x]) >= d1) pick |= 1u << x;
            }
            const uint32_t c = __popc(pick);
            uint32_t incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t slot = cnt + incl - c;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                if (pick & (1u << x)) {
                    if (slot < kWarpCap) wbuf[warp][slot] = make_uint2(u[x], static_cast<uint32_t>(e0 + x));
                    ++slot;
                }
            }
            cnt += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    if (lane == 0) wcount[warp] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t o = 0;
        bool over = false;
        for (int w = 0; w < kWarps; ++w) {
            woff[w] = o;
            o += wcount[w];
            over |= wcount[w] > static_cast<uint32_t>(kWarpCap);
        }
        // a warp buffer that overflowed makes the chunk report more than the
        // per-chunk capacity, which sends the query down the streaming path
        woff[kWarps] = over ? static_cast<uint32_t>(kSplitCap) + 1u : o;
    }
    __syncthreads();
    const uint32_t total = woff[kWarps];
    uint2 *dst = a.gcand + (static_cast<int64_t>(i) * kSplitMax + p) * kSplitCap;
    if (total <= static_cast<uint32_t>(kSplitCap)) {
        const uint32_t c = wcount[warp];
        for (uint32_t j = lane; j < c; j += 32) dst[woff[warp] + j] = wbuf[warp][j];
    }
    if (threadIdx.x == 0) a.gcount[static_cast<int64_t>(i) * kSplitMax + p] = total;
}

// (3) walk the chunks' candidates in position order and finish the query.
// The candidates are first staged in shared memory (independent loads), laid
// out as warp segments: warp w's chunks, in order, at a running offset.
struct MergeSmem {
    uint32_t hist[kBins];
    uint2 cand[kWarps * kWCap];
    uint32_t coff[kSplitMax + 1];
    uint32_t wcnt[kWarps], wg[kWarps], we[kWarps];
    uint64_t scan[kWarps];
    uint32_t sel[4];
};

struct StagedSegs {  // warp w: candidates [wbeg[w], wbeg[w] + wcnt[w]) of one array
    const uint2 *cand;
    const uint32_t *coff;  // chunk offsets
    const int n_chunks;
    __device__ int pieces(int) const { return 1; }
    __device__ const uint2 *ptr(int w, int) const { return cand + coff[w * n_chunks / kWarps]; }
    __device__ uint32_t count(int w, int) const {
        return coff[(w + 1) * n_chunks / kWarps] - coff[w * n_chunks / kWarps];
    }
};

__global__ void __launch_bounds__(kT, 1) topk_merge_kernel(const TopkArgs a, int n_chunks) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    MergeSmem &sm = *reinterpret_cast<MergeSmem *>(smem_raw);
    const int i = blockIdx.x;
    griddep_wait();
    const int n = visible_rows(a, i);
    if (n <= a.topk) {
        write_all(a, i, n);
        return;
    }
    const uint32_t k = static_cast<uint32_t>(a.topk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    const uint32_t d1 = a.gdigit[2 * i], above1 = a.gdigit[2 * i + 1];  // from collect chunk 0
    const uint32_t *counts = a.gcount + static_cast<int64_t>(i) * kSplitMax;
    // chunk counts -> offsets (a block scan; count > cap marks an overflow)
    {
        const uint32_t c = threadIdx.x < n_chunks ? counts[threadIdx.x] : 0u;
        const uint64_t ov = c > static_cast<uint32_t>(kSplitCap) ? 1ull : 0ull;
        uint64_t tot;
        const uint64_t ex = block_scan((ov << 32) | c, sm.scan, tot);
        if (threadIdx.x < n_chunks) sm.coff[threadIdx.x] = static_cast<uint32_t>(ex & 0xFFFFFFFFu);
        if (threadIdx.x == 0) {
            sm.coff[n_chunks] = static_cast<uint32_t>(tot & 0xFFFFFFFFu);
            sm.sel[2] = ((tot >> 32) != 0 || static_cast<uint32_t>(tot) > static_cast<uint32_t>(kWarps * kWCap)) ? 1u
                                                                                                                : 0u;
        }
    }
    __syncthreads();
    const bool overflow = sm.sel[2] != 0;
    if (overflow) {
        finish_stream(row, n, k, d1, above1, sm.hist, sm.scan, sm.sel, out);
    } else {
        // stage: warp w copies chunks w, w + 16, ... (all loads independent)
        const uint2 *src = a.gcand + static_cast<int64_t>(i) * kSplitMax * kSplitCap;
        for (int p = threadIdx.x >> 5; p < n_chunks; p += kWarps) {
            const uint32_t c = sm.coff[p + 1] - sm.coff[p];
            for (uint32_t j = threadIdx.x & 31; j < c; j += 32)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(&sm.cand[sm.coff[p] + j])),
                             "l"(src + static_cast<int64_t>(p) * kSplitCap + j)
                             : "memory");
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        const StagedSegs sg{sm.cand, sm.coff, n_chunks};
        uint32_t T, need_eq;
        seg_refine(sg, d1, k - above1, sm.hist, sm.scan, sm.sel, T, need_eq);
        seg_write(sg, T, need_eq, out, sm.wg, sm.we);
    }
    if (threadIdx.x == 0) a.cnt[i] = a.topk;
}

// P chunks per query so that about two CTAs per SM take part; chunks are
// multiples of 2048 rows.
void split_plan(const TopkArgs &a, int num_sms, int &P, int &chunk) {
    P = (2 * num_sms + a.n_q - 1) / a.n_q;
    P = P < 1 ? 1 : (P > kSplitMax ? kSplitMax : P);
    chunk = (a.L + P - 1) / P;
    chunk = (chunk + 2047) / 2048 * 2048;
    P = (a.L + chunk - 1) / chunk;
}

}  // namespace

bool topk_uses_split(int n_q, int max_ctx) { return max_ctx > kTopkSplitMinCtx && n_q <= kTopkSplitMaxQueries; }

cudaError_t launch_topk_hist(const TopkArgs &a, int num_sms, cudaStream_t st) {
    int P, chunk;
    split_plan(a, num_sms, P, chunk);
    return launch_pdl(topk_hist_kernel, dim3(P, a.n_q), dim3(kT), 0, st, a, chunk);
}

cudaError_t launch_topk(const TopkArgs &a, int num_sms, cudaStream_t st) {
    cudaError_t e;
    if (!topk_uses_split(a.n_q, a.L)) {
        const size_t smem = sizeof(RowSmem);
        if ((e = cudaFuncSetAttribute(topk_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem))) != cudaSuccess)
            return e;
        return launch_pdl(topk_row_kernel, dim3(a.n_q), dim3(kT), smem, st, a);
    }
    int P, chunk;
    split_plan(a, num_sms, P, chunk);
    if (!a.hist_ready) {
        if ((e = cudaMemsetAsync(a.ghist, 0, sizeof(uint32_t) * kBins * a.n_q, st)) != cudaSuccess) return e;
        if ((e = launch_pdl(topk_hist_kernel, dim3(P, a.n_q), dim3(kT), 0, st, a, chunk)) != cudaSuccess) return e;
    }
    if ((e = launch_pdl(topk_collect_kernel, dim3(P, a.n_q), dim3(kT), 0, st, a, chunk)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(sizeof(MergeSmem)))) != cudaSuccess)
        return e;
    return launch_pdl(topk_merge_kernel, dim3(a.n_q), dim3(kT), sizeof(MergeSmem), st, a, P);
}

size_t topk_scratch_bytes(int n_q, int max_ctx) {
    const size_t hist = sizeof(uint32_t) * kBins * n_q;
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    if (!topk_uses_split(n_q, max_ctx)) return al(hist);
    const size_t counts = sizeof(uint32_t) * kSplitMax * n_q;
    const size_t digits = sizeof(uint32_t) * 2 * n_q;
    const size_t cand = sizeof(uint2) * static_cast<size_t>(kSplitCap) * kSplitMax * n_q;
    return al(hist) + al(counts) + al(digits) + al(cand);
}

void topk_bind_scratch(TopkArgs &a, void *scratch) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    uint8_t *p = static_cast<uint8_t *>(scratch);
    a.ghist = reinterpret_cast<uint32_t *>(p);
    if (!topk_uses_split(a.n_q, a.L)) return;
    p += al(sizeof(uint32_t) * kBins * a.n_q);
    a.gcount = reinterpret_cast<uint32_t *>(p);
    p += al(sizeof(uint32_t) * kSplitMax * a.n_q);
    a.gdigit = reinterpret_cast<uint32_t *>(p);
    p += al(sizeof(uint32_t) * 2 * a.n_q);
    a.gcand = reinterpret_cast<uint2 *>(p);
}

}  // namespace dsa
