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
//          chunk's candidates (given the histogram); the last of them to finish
//          walks all the chunks' candidates in position order and writes the
//          query's result -- one launch.
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

__device__ __forceinline__ void zero_hist(uint32_t *hist, int nbins) {
    for (int b = threadIdx.x; b < nbins; b += kT) hist[b] = 0;
}

// The digit holding the r-th largest key: sel[0] = digit, sel[1] = rows in
// higher bins.  If the histogram holds fewer than r rows, sel = {0, total}.
// nbins = 4096: thread t owns bins [8t, 8t + 8) (two 16-byte loads); nbins =
// 256: threads t < 256 own bin t.  One barrier: each warp's suffix total goes to
// shared memory, and every warp adds up the totals of the warps above it with
// lane-parallel loads and four shuffles.
__device__ __forceinline__ void find_digit(const uint32_t *hist, int nbins, uint32_t r, uint64_t *scan,
                                           uint32_t *sel) {
    uint32_t *wsum = reinterpret_cast<uint32_t *>(scan);  // kWarps entries
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kPer = kBins / kT;  // 8
    uint32_t hb[kPer];
    int b0;
    if (nbins == kBins) {
        b0 = threadIdx.x * kPer;
        const uint4 x0 = reinterpret_cast<const uint4 *>(hist)[2 * threadIdx.x];
        const uint4 x1 = reinterpret_cast<const uint4 *>(hist)[2 * threadIdx.x + 1];
        hb[0] = x0.x, hb[1] = x0.y, hb[2] = x0.z, hb[3] = x0.w;
        hb[4] = x1.x, hb[5] = x1.y, hb[6] = x1.z, hb[7] = x1.w;
    } else {  // nbins <= kT: one bin per thread
        b0 = threadIdx.x;
        hb[0] = threadIdx.x < nbins ? hist[threadIdx.x] : 0u;
#pragma unroll
        for (int j = 1; j < kPer; ++j) hb[j] = 0u;
    }
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) mine += hb[j];
    uint32_t suf = mine;  // rows in this lane's bins and every higher lane's
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
    }
    if (lane == 0) wsum[warp] = suf;
    __syncthreads();
    uint32_t ws = lane < kWarps ? wsum[lane] : 0u;  // suffix over warps, lane-parallel
#pragma unroll
    for (int o = 1; o < kWarps; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, ws, o);
        if (lane + o < 32) ws += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, ws, 0);
    uint32_t above = suf - mine + __shfl_sync(0xffffffffu, ws, (warp + 1) & 31);
    if (threadIdx.x == 0 && total < r) {
        sel[0] = 0;
        sel[1] = total;
    }
    const int nb = nbins == kBins ? kPer : 1;
#pragma unroll
    for (int j = kPer - 1; j >= 0; --j) {
        if (j >= nb) continue;
        const uint32_t upto = above + hb[j];
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
                hist_add(hist, in ? (u >> shift) & dmask : 0xFFFFFFFFu);
            }
        }
    }
    __syncthreads();
}

// Ordered filter by streaming the row (fallback): keep keys > T and the first
// need_eq keys == T, at exclusive-scan slots.
__device__ __forceinline__ void stream_write(const float *row, int n, uint32_t T, uint32_t need_eq, uint32_t k,
                                             int32_t *out, uint64_t *scan) {
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
                if (g + min(q, need_eq) < k) out[g + min(q, need_eq)] = e0 + x;
                ++g;
            } else if (u[x] == T) {
                if (q < need_eq && g + q < k) out[g + q] = e0 + x;
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
    stream_write(row, n, T, need_eq, k, out, scan);
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
        for (uint32_t b = lane; b < c; b += 32) {
            const uint32_t u = p[b].x;
            if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
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
__device__ __forceinline__ void seg_write(const Segs &sg, uint32_t T, uint32_t need_eq, uint32_t k, int32_t *out,
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
            if (isg && gb + min(eb, need_eq) < k) out[gb + min(eb, need_eq)] = static_cast<int32_t>(v.y);
            if (ise && eb < need_eq && gb + eb < k) out[gb + eb] = static_cast<int32_t>(v.y);
            g += __popc(mg);
            e += __popc(me);
        }
    }
}

// Refine and write in one go with the candidates in registers: lane l of warp
// w owns a contiguous run of at most kO (odd) candidates of the warp's segment, so
// (warp, lane, run index) is position order.  Digit 2 and digit 3 are counted
// with per-lane shared atomics over the owned keys only; the kept rows' output
// slots come from one block scan of (rows > T, rows == T) per thread.  Returns
// false, having written nothing, when a segment holds more than 32 * kO
// candidates (the caller then uses seg_refine + seg_write).  Output slots are
// bounds-checked against k (they stay below k whenever the histogram the
// threshold digit came from describes these scores).
constexpr int kOwn = 9;         // row schedule: within its 64-register budget
// The split schedule's finish: up to 7,680 candidates, without spills at one CTA
// per SM (1M-context decode queries' candidate sets reach 5-7K when the k-th
// score falls in a dense bin; past 32 * kO per warp the slower two-pass refine
// and write take over).
constexpr int kOwnStaged = 15;
static_assert(kMaxTopk <= kBins, "seg_finish stages the output in the histogram");
// hist2_ready: `hist` already holds the second-digit histogram of the
// candidates in bin d1 (built by the chunk CTAs), so it is not rebuilt here.
template <int kO, class Segs>
__device__ __forceinline__ bool seg_finish(const Segs &sg, uint32_t d1, uint32_t r2, uint32_t k, uint32_t *hist,
                                           uint64_t *scan, uint32_t *sel, int32_t *out, bool hist2_ready = false) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint2 *p = sg.ptr(w, 0);
    const uint32_t c = sg.count(w, 0);
    const uint32_t m = ((c + 31) / 32) | 1u;  // odd run length: the lanes' loads fall in distinct banks
    if (!hist2_ready) zero_hist(hist, kBins);
    if (__syncthreads_or(m > static_cast<uint32_t>(kO) || sg.pieces(w) != 1)) return false;
    const uint32_t b0 = min(c, lane * m), b1 = min(c, b0 + m);
    uint32_t key[kO];
#pragma unroll
    for (int j = 0; j < kO; ++j) key[j] = b0 + j < b1 ? p[b0 + j].x : 0u;
    if (!hist2_ready) {
#pragma unroll
        for (int j = 0; j < kO; ++j)
            if (b0 + j < b1 && first_digit(key[j]) == d1) atomicAdd(&hist[(key[j] >> 8) & 0xFFFu], 1u);
        __syncthreads();
    }
    find_digit(hist, kBins, r2, scan, sel);
    const uint32_t d2 = sel[0];
    const uint32_t r3 = r2 - sel[1];
    const uint32_t p24 = (d1 << 12) | d2;
    __syncthreads();  // every thread has read sel and hist
    if (threadIdx.x < kBins3) hist[threadIdx.x] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kO; ++j)
        if (b0 + j < b1 && (key[j] >> 8) == p24) atomicAdd(&hist[key[j] & 0xFFu], 1u);
    __syncthreads();
    find_digit(hist, kBins3, r3, scan, sel);
    const uint32_t T = (p24 << 8) | sel[0];
    const uint32_t need_eq = r3 - sel[1];
    uint32_t tg = 0, te = 0;
#pragma unroll
    for (int j = 0; j < kO; ++j) {
        tg += (b0 + j < b1 && key[j] > T) ? 1u : 0u;
        te += (b0 + j < b1 && key[j] == T) ? 1u : 0u;
    }
    uint64_t tot;
    const uint64_t ex = block_scan((static_cast<uint64_t>(te) << 32) | tg, scan, tot);
    uint32_t g = static_cast<uint32_t>(ex & 0xFFFFFFFFu), q = static_cast<uint32_t>(ex >> 32);
    // The kept rows land in shared memory first (each lane's run is scattered
    // over the output, which as global stores costs one sector per row), then
    // the k slots go out coalesced.  The histogram is free again here: every
    // thread has read the digits it held (find_digit ends with a barrier).
    int32_t *stage = reinterpret_cast<int32_t *>(hist);  // k <= kMaxTopk = kBins slots
#pragma unroll
    for (int j = 0; j < kO; ++j) {
        if (b0 + j >= b1) continue;
        if (key[j] > T) {
            const uint32_t slot = g + min(q, need_eq);
            if (slot < k) stage[slot] = static_cast<int32_t>(p[b0 + j].y);
            ++g;
        } else if (key[j] == T) {
            if (q < need_eq && g + q < k) stage[g + q] = static_cast<int32_t>(p[b0 + j].y);
            ++q;
        }
    }
    __syncthreads();
    if (out != nullptr)  // null: a run that only brings this code into the caches
        for (uint32_t x = threadIdx.x; x < k; x += kT) out[x] = stage[x];
    return true;
}

// reporter: the one CTA of query i that reports a position outside the cache
__device__ __forceinline__ int visible_rows(const TopkArgs &a, int i, bool reporter) {
    const int pos = a.q_pos[i];
    if (pos < 0 || pos >= a.L) {
        if (reporter && threadIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
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
    __align__(16) uint32_t hist[kBins];
    uint2 wbuf[kWarps * kWCap];
    uint32_t wcnt[kWarps], wg[kWarps], we[kWarps];
    uint64_t scan[kWarps];
    uint32_t sel[4];
    int flag;
};

// Load kU float4 groups of a warp slice: element e = base + (j * 32 + lane) * 4 + x
// (elements at or past `hi` read as 0 and are masked by the caller).
__device__ __forceinline__ void load_warp_batch(const float *row, int base, int hi, float (&v)[kU][4]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < kU; ++j) {
        const int e0 = base + (j * 32 + lane) * 4;
        if (e0 + 4 <= hi) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
            v[j][0] = f.x, v[j][1] = f.y, v[j][2] = f.z, v[j][3] = f.w;
        } else {
#pragma unroll
            for (int x = 0; x < 4; ++x) v[j][x] = e0 + x < hi ? __ldg(row + e0 + x) : 0.f;
        }
    }
}

// Append, in position order, the rows of a loaded batch whose first digit is at
// least d_lo to a warp's (key, position) buffer of capacity cap; cnt counts every
// such row, also past the capacity.  Groups of 128 rows without a candidate cost
// one ballot.  kPos (d_lo above 0x800, the digit of +0.0): only positive scores
// qualify, and a row's first digit is at least d_lo exactly when its bits, read
// as a signed integer, are at least tbits = the bits of the bin's smallest
// value -- negative scores, -0.0, +0.0 and the zeros loaded past `hi` all read
// below it -- so a row costs one integer compare and only kept rows form a key.
template <bool kPos>
__device__ __forceinline__ void compact_batch_t(const float (&v)[kU][4], int base, int hi, uint32_t d_lo, uint2 *buf,
                                                uint32_t cap, uint32_t &cnt) {
    const int lane = threadIdx.x & 31;
    const int32_t tbits = static_cast<int32_t>((d_lo << 20) & 0x7FFFFFFFu);
#pragma unroll
    for (int j = 0; j < kU; ++j) {
        const int e0 = base + (j * 32 + lane) * 4;
        uint32_t u[4], pick = 0;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if constexpr (kPos) {
                if (__float_as_int(v[j][x]) >= tbits) pick |= 1u << x;
            } else {
                u[x] = order_key(v[j][x]);
                if (e0 + x < hi && first_digit(u[x]) >= d_lo) pick |= 1u << x;
            }
        }
        if (__ballot_sync(0xffffffffu, pick != 0u) == 0u) continue;
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
                if (slot < cap) buf[slot] = make_uint2(kPos ? order_key(v[j][x]) : u[x], static_cast<uint32_t>(e0 + x));
                ++slot;
            }
        }
        cnt += __shfl_sync(0xffffffffu, incl, 31);
    }
}

__device__ __forceinline__ void compact_batch(const float (&v)[kU][4], int base, int hi, uint32_t d_lo, uint2 *buf,
                                              uint32_t cap, uint32_t &cnt) {
    if (d_lo > 0x800u)
        compact_batch_t<true>(v, base, hi, d_lo, buf, cap, cnt);
    else
        compact_batch_t<false>(v, base, hi, d_lo, buf, cap, cnt);
}

__global__ void __launch_bounds__(kT, 2) topk_row_kernel(const TopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowSmem &sm = *reinterpret_cast<RowSmem *>(smem_raw);
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();
    const bool exact = a.hist_ready != 0;
    // the histogram does not depend on the position: its loads go out first
    uint32_t hv[kBins / kT];
    if (exact) {
        const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
#pragma unroll
        for (int j = 0; j < kBins / kT; ++j) hv[j] = __ldg(g + threadIdx.x + j * kT);
    }
    const int n = visible_rows(a, i, true);
    if (exact) {  // leave the histogram zero for the next indexer launch
        uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
#pragma unroll
        for (int j = 0; j < kBins / kT; ++j) g[threadIdx.x + j * kT] = 0u;
    }
    if (n <= a.topk) {
        write_all(a, i, n);
        return;
    }
    const uint32_t k = static_cast<uint32_t>(a.topk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    // each warp streams a contiguous slice of the row; its first batch is in
    // flight while the threshold digit is found
    const int sub = ((n + kWarps - 1) / kWarps + 127) / 128 * 128;
    const int wlo = min(n, warp * sub), whi = min(n, wlo + sub);
    float v[kU][4];
    if (exact) load_warp_batch(row, wlo, whi, v);

    // ---- 1. a threshold digit d_lo: rows with first digit >= d_lo are candidates
    uint32_t d_lo, above_exact = 0;
    if (exact) {
#pragma unroll
        for (int j = 0; j < kBins / kT; ++j) sm.hist[threadIdx.x + j * kT] = hv[j];
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
            float sv[4];
            if (e0 + 4 <= n) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(row + e0));
                sv[0] = f.x, sv[1] = f.y, sv[2] = f.z, sv[3] = f.w;
            } else {
#pragma unroll
                for (int x = 0; x < 4; ++x) sv[x] = e0 + x < n ? __ldg(row + e0 + x) : 0.f;
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
                hist_add(sm.hist, e0 + x < n ? first_digit(order_key(sv[x])) : 0xFFFFFFFFu);
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

    // ---- 2. candidates
    {
        uint2 *mine = sm.wbuf + warp * kWCap;
        uint32_t cnt = 0;
        for (int base = wlo; base < whi; base += 32 * 4 * kU) {
            if (!exact || base != wlo) load_warp_batch(row, base, whi, v);
            compact_batch(v, base, whi, d_lo, mine, kWCap, cnt);
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
        if (!seg_finish<kOwn>(sg, d1, k - above1, k, sm.hist, sm.scan, sm.sel, out)) {
            uint32_t T, need_eq;
            seg_refine(sg, d1, k - above1, sm.hist, sm.scan, sm.sel, T, need_eq);
            seg_write(sg, T, need_eq, k, out, sm.wg, sm.we);
        }
    }
    if (threadIdx.x == 0) a.cnt[i] = a.topk;
}

// ---------------------------------------------------------------- split schedule
// (1) first-digit histogram of a chunk, added into the query's global histogram.
__global__ void __launch_bounds__(kT, 2) topk_hist_kernel(const TopkArgs a, int chunk) {
    __shared__ uint32_t hist[kBins];
    const int i = blockIdx.y, p = blockIdx.x;
    griddep_wait();
    const int n = visible_rows(a, i, p == 0);
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

// (2) one launch per query set: every CTA collects its chunk's candidates (first
// digit >= the threshold digit) in position order -- each warp compacts a
// contiguous slice into a private buffer, the 16 warp counts place the slices --
// and the last CTA of a query to finish (a ticket in global memory) walks all the
// chunks' candidates in position order and writes the query's result.
struct CollectSmem {
    __align__(16) uint32_t hist[kBins];
    uint64_t scan[kWarps];
    uint32_t sel[4];
    uint2 wbuf[kWarps][kWarpCap];
    uint32_t wcount[kWarps], woff[kWarps + 1];
};

// The finishing CTA: candidates staged in shared memory as warp segments (warp
// w's chunks, in order, at a running offset).
struct MergeSmem {
    __align__(16) uint32_t hist[kBins];
    uint2 cand[kWarps * kWCap];
    uint32_t coff[kSplitMax + 1];
    uint32_t wcnt[kWarps], wg[kWarps], we[kWarps];
    uint64_t scan[kWarps];
    uint32_t sel[4];
};

struct SplitSmem {
    union {
        CollectSmem c;
        MergeSmem m;
    } u;
    int last;  // 1: this CTA finishes the query; 2: the first to finish its chunk
};

// The finishing CTA's refine and write, as a function that is not inlined, so
// that a run of it on an empty candidate set executes the very instructions the
// finish executes later.  The first chunk CTA of each query to take its ticket
// makes that run before it exits: the finish is the only code of the path that
// no other CTA runs first, and with its instructions fetched from DRAM (the
// step's streams evict them from L2) it ran 2-9 us slower than with them cached.
struct StagedSegs;
__device__ __noinline__ bool seg_finish_staged(const StagedSegs sg, uint32_t d1, uint32_t r2, uint32_t k,
                                               uint32_t *hist, uint64_t *scan, uint32_t *sel, int32_t *out);

// The staged candidates are one array in position order, so warp w may take
// an equal share of it regardless of chunk boundaries: [w*M/16, (w+1)*M/16).
struct StagedSegs {
    const uint2 *cand;
    const uint32_t total;  // M
    __device__ int pieces(int) const { return 1; }
    __device__ uint32_t begin(int w) const {
        return static_cast<uint32_t>((static_cast<uint64_t>(total) * w) / kWarps);
    }
    __device__ const uint2 *ptr(int w, int) const { return cand + begin(w); }
    __device__ uint32_t count(int w, int) const { return begin(w + 1) - begin(w); }
};

__device__ __noinline__ bool seg_finish_staged(const StagedSegs sg, uint32_t d1, uint32_t r2, uint32_t k,
                                               uint32_t *hist, uint64_t *scan, uint32_t *sel, int32_t *out) {
    return seg_finish<kOwnStaged>(sg, d1, r2, k, hist, scan, sel, out, true);
}

// Finish query i from the chunks' candidates (written by other CTAs of this
// launch: read through L2).
__device__ __forceinline__ void merge_query(const TopkArgs &a, int i, int n, int n_chunks, uint32_t d1,
                                            uint32_t above1, MergeSmem &sm) {
    const uint32_t k = static_cast<uint32_t>(a.topk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    int32_t *out = a.idx + static_cast<int64_t>(i) * a.topk;
    const uint32_t *counts = a.gcount + static_cast<int64_t>(i) * kSplitMax;
    // chunk counts -> offsets (a block scan; count > cap marks an overflow)
    {
        const uint32_t c = threadIdx.x < n_chunks ? __ldcg(counts + threadIdx.x) : 0u;
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
    uint32_t *g2 = a.ghist2 + static_cast<int64_t>(i) * kBins;
    if (overflow) {
        for (int b = threadIdx.x; b < kBins; b += kT) g2[b] = 0u;  // zero for the next launch
        finish_stream(row, n, k, d1, above1, sm.hist, sm.scan, sm.sel, out);
    } else {
        // the second-digit histogram the chunk CTAs built (16-byte pieces, L2)
        for (int e = threadIdx.x; e < kBins / 4; e += kT)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&sm.hist[4 * e])), "l"(g2 + 4 * e)
                         : "memory");
        // stage: warp w copies chunks w, w + 16, ... with asynchronous copies
        // (all in flight at once).  The L1-allocating form is safe here: this
        // CTA is the only reader of these lines in this launch, after every
        // writer's fence, so no earlier copy of them can sit in this SM's L1.
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
        for (int b = threadIdx.x; b < kBins; b += kT) g2[b] = 0u;  // read above; zero for the next launch
        const StagedSegs sg{sm.cand, sm.coff[n_chunks]};
        if (!seg_finish_staged(sg, d1, k - above1, k, sm.hist, sm.scan, sm.sel, out)) {
            uint32_t T, need_eq;
            seg_refine(sg, d1, k - above1, sm.hist, sm.scan, sm.sel, T, need_eq);
            seg_write(sg, T, need_eq, k, out, sm.wg, sm.we);
        }
    }
    if (threadIdx.x == 0) a.cnt[i] = a.topk;
}

// kPerSm CTAs per SM.  One, where the plan gives each query enough chunks with
// one CTA per SM: the finishing CTA's digit search and output then run in
// registers (at two CTAs per SM the 64-register cap spills them, which costs
// the finish about a microsecond per phase).  Two for many queries, which need
// more chunks per query than one CTA per SM allows (a chunk's candidates must
// fit its buffers).
template <int kPerSm>
__global__ void __launch_bounds__(kT, kPerSm) topk_split_kernel(const TopkArgs a, int chunk, int n_chunks) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SplitSmem &ss = *reinterpret_cast<SplitSmem *>(smem_raw);
    CollectSmem &cs = ss.u.c;
    const int i = blockIdx.y, p = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // positions that are inputs of the call are read before the wait, so the
    // chunk's score loads go out together with the histogram's
    const int n_early = a.pos_early ? visible_rows(a, i, p == 0) : 0;
    griddep_wait();
    uint32_t hv[kBins / kT];
    {
        const uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
#pragma unroll
        for (int j = 0; j < kBins / kT; ++j) hv[j] = __ldg(g + threadIdx.x + j * kT);
    }
    const int n = a.pos_early ? n_early : visible_rows(a, i, p == 0);
    if (n <= a.topk) {  // every chunk of the query sees the same n
        if (p == 0) {
            write_all(a, i, n);
            uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;  // zero for the next launch
            for (int b = threadIdx.x; b < kBins; b += kT) g[b] = 0u;
        }
        return;
    }
    const int lo = min(n, p * chunk), hi = min(n, lo + chunk);
    const float *row = a.scores + static_cast<int64_t>(i) * a.ld;
    const int sub = ((hi - lo + kWarps - 1) / kWarps + 127) / 128 * 128;
    const int wlo = min(hi, lo + warp * sub), whi = min(hi, wlo + sub);
    float v[kU][4];
    load_warp_batch(row, wlo, whi, v);  // in flight while the threshold digit is found
#pragma unroll
    for (int j = 0; j < kBins / kT; ++j) cs.hist[threadIdx.x + j * kT] = hv[j];
    __syncthreads();
    find_digit(cs.hist, kBins, static_cast<uint32_t>(a.topk), cs.scan, cs.sel);
    const uint32_t d1 = cs.sel[0], above1 = cs.sel[1];
    uint32_t cnt = 0;
    for (int base0 = wlo; base0 < whi; base0 += 128 * kU) {
        if (base0 != wlo) load_warp_batch(row, base0, whi, v);
        compact_batch(v, base0, whi, d1, cs.wbuf[warp], kWarpCap, cnt);
    }
    if (lane == 0) cs.wcount[warp] = cnt;
    {
        // second digit of this warp's candidates in the threshold bin, into the
        // query's histogram (the finishing CTA reads it instead of building it)
        __syncwarp();
        uint32_t *g2 = a.ghist2 + static_cast<int64_t>(i) * kBins;
        const uint32_t c = min(cnt, static_cast<uint32_t>(kWarpCap));
        for (uint32_t j = lane; j < c; j += 32) {
            const uint32_t u = cs.wbuf[warp][j].x;
            if (first_digit(u) == d1) atomicAdd(&g2[(u >> 8) & 0xFFFu], 1u);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t o = 0;
        bool over = false;
        for (int w = 0; w < kWarps; ++w) {
            cs.woff[w] = o;
            o += cs.wcount[w];
            over |= cs.wcount[w] > static_cast<uint32_t>(kWarpCap);
        }
        // a warp buffer that overflowed makes the chunk report more than the
        // per-chunk capacity, which sends the query down the streaming path
        cs.woff[kWarps] = over ? static_cast<uint32_t>(kSplitCap) + 1u : o;
    }
    __syncthreads();
    const uint32_t total = cs.woff[kWarps];
    uint2 *dst = a.gcand + (static_cast<int64_t>(i) * kSplitMax + p) * kSplitCap;
    if (total <= static_cast<uint32_t>(kSplitCap)) {
        const uint32_t c = cs.wcount[warp];
        for (uint32_t j = lane; j < c; j += 32) dst[cs.woff[warp] + j] = cs.wbuf[warp][j];
    }
    if (threadIdx.x == 0) a.gcount[static_cast<int64_t>(i) * kSplitMax + p] = total;
    // The next kernel (the attention) may start its prologue on the SMs the chunk
    // CTAs leave; it still waits for this whole grid before reading the selection.
    griddep_launch_dependents();

    // ---- publish; the last CTA of the query finishes it.  The barrier orders every
    // thread's candidate, count and histogram writes before thread 0's fence, which
    // is cumulative: one device-scope fence releases them all with the ticket, and
    // one more, in the last CTA, acquires the other chunks' writes for all its
    // threads (their reads follow the second barrier).
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(a.gticket + i, 1u);
        ss.last = prev == static_cast<uint32_t>(n_chunks - 1) ? 1 : (prev == 0 ? 2 : 0);
        if (ss.last == 1) __threadfence();
    }
    __syncthreads();
    if (ss.last == 2) {
        // the query's first chunk to finish runs the finish on no candidates: no
        // global writes; the shared memory it reads and writes is its own
        MergeSmem &wm = ss.u.m;
        const StagedSegs none{wm.cand, 0u};
        seg_finish_staged(none, 0u, 1u, 1u, wm.hist, wm.scan, wm.sel, nullptr);
        return;
    }
    if (ss.last != 1) return;
    // every chunk has read the histogram and taken its ticket: leave both zero
    // for the next launch
    {
        uint32_t *g = a.ghist + static_cast<int64_t>(i) * kBins;
        for (int b = threadIdx.x; b < kBins; b += kT) g[b] = 0u;
        if (threadIdx.x == 0) a.gticket[i] = 0;
    }
    merge_query(a, i, n, n_chunks, d1, above1, ss.u.m);
}

// P chunks per query, chunks multiples of 2048 rows: at most one CTA per SM when
// that still gives every query kSplitMinChunks chunks (per_sm = 1), else at most
// two (per_sm = 2).  The grid stays within one wave of resident CTAs: a CTA left
// for a second wave would start only when a first-wave CTA exits, and every
// query's finish waits for its last chunk.
constexpr int kSplitMinChunks = 8;  // a query's ~2-4K candidates stay within a chunk's buffers
void split_plan(const TopkArgs &a, int num_sms, int &P, int &chunk, int &per_sm) {
    per_sm = num_sms / a.n_q >= kSplitMinChunks ? 1 : 2;
    P = per_sm * num_sms / a.n_q;
    P = P < 1 ? 1 : (P > kSplitMax ? kSplitMax : P);
    chunk = (a.L + P - 1) / P;
    chunk = (chunk + 2047) / 2048 * 2048;
    P = (a.L + chunk - 1) / chunk;
}

}  // namespace

bool topk_uses_split(int n_q, int max_ctx) { return max_ctx > kTopkSplitMinCtx && n_q <= kTopkSplitMaxQueries; }

cudaError_t launch_topk_hist(const TopkArgs &a, int num_sms, cudaStream_t st) {
    int P, chunk, per_sm;
    split_plan(a, num_sms, P, chunk, per_sm);
    return launch_pdl(topk_hist_kernel, dim3(P, a.n_q), dim3(kT), 0, st, a, chunk);
}

cudaError_t launch_topk(const TopkArgs &a, int num_sms, cudaStream_t st) {
    cudaError_t e;
    if (!topk_uses_split(a.n_q, a.L)) {
        const size_t smem = sizeof(RowSmem);
        if ((e = set_max_dynamic_smem(topk_row_kernel, static_cast<int>(smem))) != cudaSuccess)
            return e;
        return launch_pdl(topk_row_kernel, dim3(a.n_q), dim3(kT), smem, st, a);
    }
    int P, chunk, per_sm;
    split_plan(a, num_sms, P, chunk, per_sm);
    if (!a.hist_ready) {
        if ((e = cudaMemsetAsync(a.ghist, 0, topk_zeroed_bytes(a.n_q), st)) != cudaSuccess) return e;
        if ((e = launch_pdl(topk_hist_kernel, dim3(P, a.n_q), dim3(kT), 0, st, a, chunk)) != cudaSuccess) return e;
    }
    if (per_sm == 1) {
        if ((e = set_max_dynamic_smem(topk_split_kernel<1>, static_cast<int>(sizeof(SplitSmem)))) != cudaSuccess)
            return e;
        return launch_pdl(topk_split_kernel<1>, dim3(P, a.n_q), dim3(kT), sizeof(SplitSmem), st, a, chunk, P);
    }
    if ((e = set_max_dynamic_smem(topk_split_kernel<2>, static_cast<int>(sizeof(SplitSmem)))) != cudaSuccess) return e;
    return launch_pdl(topk_split_kernel<2>, dim3(P, a.n_q), dim3(kT), sizeof(SplitSmem), st, a, chunk, P);
}

static_assert(kWaitLimitNs == kDeviceWaitLimitNs, "one device wait limit");

namespace {
// The bounded-wait probe: the barrier expects one arrival that never comes.
__global__ void bounded_wait_probe_kernel(uint32_t *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait(&bar, 0, status, nullptr, limit_ns);
}
}  // namespace

cudaError_t launch_bounded_wait_probe(uint32_t *status, uint64_t limit_ns, cudaStream_t st) {
    bounded_wait_probe_kernel<<<1, 1, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

// The tickets are padded to a multiple of 4 words so that the second-digit
// histograms after them start on a 16-byte boundary (they are copied with
// 16-byte cp.async).
static size_t ticket_words(int n_q) { return (static_cast<size_t>(n_q) + 3) & ~static_cast<size_t>(3); }
size_t topk_zeroed_bytes(int n_q) {
    return sizeof(uint32_t) * (2 * static_cast<size_t>(kBins) * n_q + ticket_words(n_q));
}

// Scratch: [n_q][4096] first-digit histograms, [n_q] tickets, then [n_q][4096]
// second-digit histograms (split schedule).  All are zero between calls: dsa_workspace_init zeroes them, a top-k launch zeroes
// each query's histogram and ticket once it has used them, and the one launch
// that builds histograms without an indexer (hist_ready == 0) zeroes them first.
// The split schedule adds [n_q][kSplitMax] candidate counts and the candidates.
size_t topk_scratch_bytes(int n_q, int max_ctx) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t hist = al(topk_zeroed_bytes(n_q));
    if (!topk_uses_split(n_q, max_ctx)) return hist;
    const size_t counts = sizeof(uint32_t) * kSplitMax * n_q;
    const size_t cand = sizeof(uint2) * static_cast<size_t>(kSplitCap) * kSplitMax * n_q;
    return hist + al(counts) + al(cand);
}

void topk_bind_scratch(TopkArgs &a, void *scratch) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    uint8_t *p = static_cast<uint8_t *>(scratch);
    a.ghist = reinterpret_cast<uint32_t *>(p);
    a.gticket = a.ghist + static_cast<size_t>(kBins) * a.n_q;
    a.ghist2 = a.gticket + ticket_words(a.n_q);
    if (!topk_uses_split(a.n_q, a.L)) return;
    p += al(topk_zeroed_bytes(a.n_q));
    a.gcount = reinterpret_cast<uint32_t *>(p);
    p += al(sizeof(uint32_t) * kSplitMax * a.n_q);
    a.gcand = reinterpret_cast<uint2 *>(p);
}

}  // namespace dsa
