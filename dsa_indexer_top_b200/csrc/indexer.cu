// indexer.cu -- lightning-indexer scores.
//
// score(t,s) = sum_h w[t,h] * max(0, q_idx[t,h] . k_idx[s]) for s <= t
// ("GLM-5.2 -- Model techniques map", "Checked in its code", Indexer-selected
// sparse attention: the indexer scores past tokens per head, index_n_heads = 32,
// index_head_dim = 128; row "QK normalization": one key per token, [B,S,1,D]).
//
// Tensor-core path (bf16, 32 x 128): a persistent, warp-specialised kernel.
//   warp 0      TMA producer: 128-key x 128-dim tiles (32 KB, two 64-dim boxes,
//               128-byte swizzle) into a ring of shared-memory stages; the
//               query tile (G queries x 32 heads x 128 dims) once per group.
//   warp 1      tcgen05.mma issuer: D[128 keys][32G] = K_tile (M=128, K-major)
//               x Q^T (N = 32G, K-major), K = 128 in eight K=16 steps, fp32
//               accumulators in TMEM, double-buffered.
//   warps 2..   epilogue (4, 8 or 16 warps for 1, 2-4 or 8 queries per tile;
//               warp w reads TMEM lane quadrant w % 4 and its share of the
//               queries): tcgen05.ld of its 32 lanes (one key per lane), ReLU,
//               multiply by w and sum the 32 heads inside the thread, causal mask,
//               coalesced fp32 store of one score per key per query.
// Work items are (query group, key tile) pairs over a grid of at most two CTAs
// per SM (one query per tile; three for FP8) or one (several): contiguous
// ranges per CTA, or, for long bf16 contexts, claimed two at a time from a
// counter in the workspace so that the CTAs of faster SMs take more of them and
// all finish together.  The producer hands each item to the MMA issuer and the
// epilogue through a small ring in shared memory.  Tiles past the group's last
// visible key are skipped.
//
// FP8 variant (E4M3 queries and keys, each row scaled by a positive float): the
// same kernel with 16 KB tiles (one 128-byte box of E4M3 bytes per tile), four
// K = 32 tcgen05.mma.kind::f8f6f4 steps per tile, the query scale folded into w
// and the key scale applied to the finished score -- both factor out of the
// ReLU because they are positive.
#include <algorithm>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kTileKeys = 128;
constexpr int kClaim = 2;  // work items per claim
constexpr int kRing = 8;   // items in flight between the producer and the epilogue (> stages + 2)

// F8: queries and keys are E4M3 bytes (the FP8 variant) instead of bf16.
template <int G, bool F8>
struct IdxCfg {
    static constexpr int N = 32 * G;
    static constexpr int kElem = F8 ? 1 : 2;                     // bytes per value
    static constexpr int kTileBytes = kTileKeys * kIdxDim * kElem;  // 32 KB bf16, 16 KB FP8
    static constexpr int kBoxes = kElem;                          // 128-byte-wide boxes per row
    static constexpr int kKSteps = F8 ? kIdxDim / 32 : kIdxDim / 16;  // MMA K = 32 (8-bit) or 16
    // One query per tile: several independent load -> MMA -> epilogue pipelines
    // per SM keep the key stream at the rate of a plain TMA read stream, where one
    // CTA with deeper buffering loses about 6% to the MMA turnaround of each
    // stage, and more than about 128 KB in flight per SM lowers the stream rate
    // again.  bf16: two CTAs x two 32 KB stages; FP8 (half the bytes per key, the
    // same epilogue work): three CTAs x three 16 KB stages (measured best).
    static constexpr int kCtasPerSm = G == 1 ? (F8 ? 3 : 2) : 1;
    static constexpr int kStages = G == 1 ? (F8 ? 3 : 2) : 4;
    static constexpr int kBBytes = N * kIdxDim * kElem;
    static constexpr int kTmemCols = (2 * N < 32) ? 32 : 2 * N;
    static constexpr int kSmem = kStages * kTileBytes + kBBytes + 1024;
    static constexpr uint32_t kIdesc = F8 ? idesc_e4m3(128, N) : idesc_bf16(128, N, false, false);
    // epilogue warps: one per TMEM lane quadrant for one query per tile, two
    // (each half of the queries) for 2 or 4, four (each a quarter) for 8 -- with
    // 8 queries per tile the ReLU-weighted head sums outweigh the MMA, so the
    // epilogue gets four warps per scheduler
    static constexpr int kEpiWarps = G >= 8 ? 16 : (G >= 2 ? 8 : 4);
    static constexpr int kThreads = (2 + kEpiWarps) * 32;
};

// Sequence and last visible position of a query group; every role calls this
// with the same arguments and so skips the same tiles.
template <int G>
__device__ __forceinline__ void group_info(const IdxTcArgs &a, int g, int &seq, int &max_pos) {
    int q0 = g * G;
    int nq = min(G, a.n_q - q0);
    seq = a.k_shared ? 0 : __ldg(a.q_seq + q0);
    max_pos = -1;
    if (seq < 0 || seq >= a.n_seq) {
        seq = -1;
        return;
    }
    for (int i = 0; i < nq; ++i) {
        int p = __ldg(a.q_pos + q0 + i);
        if (p >= 0 && p < a.L) max_pos = max(max_pos, p);
    }
}

// A run of consecutive work items, as (query group, key tile), stepped without
// a division per item: `left` items from tile j of group g.
struct ItemRun {
    long long left = 0;
    int g = 0, j = 0;
    __device__ __forceinline__ void start(long long first, long long count, int tpg) {
        left = count;
        g = static_cast<int>(first / tpg);
        j = static_cast<int>(first - static_cast<long long>(g) * tpg);
    }
    __device__ __forceinline__ void take(int tpg, int &og, int &oj) {
        og = g;
        oj = j;
        --left;
        if (++j == tpg) {
            j = 0;
            ++g;
        }
    }
    // the rest of the group just taken is skipped too (its tiles lie further
    // past the last visible key, or the group has no valid query)
    __device__ __forceinline__ void skip_group(int tpg) {
        if (j != 0) {
            left -= min(left, static_cast<long long>(tpg - j));
            j = 0;
            ++g;
        }
    }
};

// The work items a consumer role (MMA issuer, epilogue warp) walks, in the
// producer's order: with claimed work the ring the producer fills (group -1
// ends it); otherwise the CTA's contiguous range, skipping what the producer
// skips.
template <int G>
struct ItemWalk {
    ItemRun run;
    int sg = -1, seq = -1, max_pos = -1;
    __device__ __forceinline__ ItemWalk(long long begin, long long end, int tpg) { run.start(begin, end - begin, tpg); }
    __device__ __forceinline__ bool next(const IdxTcArgs &a, int tpg, long long k, const int2 *ring,
                                         uint64_t *ring_bar, int *abort_flag, int &g, int &j) {
        if (!a.work) {
            while (run.left > 0) {
                run.take(tpg, g, j);
                if (g != sg) {
                    group_info<G>(a, g, seq, max_pos);
                    sg = g;
                }
                if (seq < 0 || j * kTileKeys > max_pos) {
                    run.skip_group(tpg);
                    continue;
                }
                return true;
            }
            return false;
        }
        const int r = static_cast<int>(k % kRing);
        if (!mbar_wait(&ring_bar[r], static_cast<uint32_t>((k / kRing) & 1), a.status, abort_flag)) return false;
        const volatile int *v = reinterpret_cast<const volatile int *>(&ring[r]);
        g = v[0];
        j = v[1];
        return g >= 0;
    }
};

template <int G, bool F8>
__global__ void __launch_bounds__(IdxCfg<G, F8>::kThreads, IdxCfg<G, F8>::kCtasPerSm)
    idx_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_q, const IdxTcArgs a) {
    using Cfg = IdxCfg<G, F8>;
    constexpr int kATileBytes = Cfg::kTileBytes;
    constexpr int N = Cfg::N;
    constexpr int S = Cfg::kStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *a_tiles = smem;                      // S x 32 KB
    uint8_t *b_tile = smem + S * kATileBytes;     // N rows x 128 dims

    __shared__ uint64_t full_bar[S], empty_bar[S];
    __shared__ uint64_t tmem_full[2], tmem_empty[2];
    __shared__ uint64_t b_full, b_empty, mma_done;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    constexpr int E = Cfg::kEpiWarps;
    __shared__ __align__(16) float w_sh[E][N];  // one private copy per epilogue warp
    // Fused top-k first-digit histogram of the current query (one query per
    // tile only), flushed into a.ghist when the epilogue moves to another query.
    __shared__ uint32_t ehist[G == 1 ? kTopkBins : 1];
    __shared__ uint64_t epi_bar;
    __shared__ int2 item_q[kRing];          // claimed (group, tile) in issue order; group -1 ends the work
    __shared__ uint64_t item_bar[kRing];    // item_q[r] written (one arrival per use)
    static_assert(kRing >= S + 3, "the ring outlasts the producer's lead over the epilogue");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tmem_full[s], 1);
            mbar_init(&tmem_empty[s], E);
        }
        mbar_init(&b_full, 1);
        mbar_init(&b_empty, 1);
        mbar_init(&mma_done, 1);
        mbar_init(&epi_bar, 4);
        for (int r = 0; r < kRing; ++r) mbar_init(&item_bar[r], 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, Cfg::kTmemCols);
        tmem_relinquish();
    }
    const bool fuse_hist = (G == 1) && a.ghist != nullptr;
    if (fuse_hist)
        for (int b = threadIdx.x; b < kTopkBins; b += Cfg::kThreads) ehist[b] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    griddep_wait();

    const long long total = a.total_items;
    const int tpg = a.tiles_per_group;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // one query per tile (decode): keys are read once, evict them first; several
            // (prefill): every query group re-reads the chunk's keys, keep them in L2
            const uint64_t stream_policy = G == 1 ? l2_evict_first_policy() : l2_evict_last_policy();
            int cur_g = -1, seq = -1, max_pos = -1;
            bool group_loaded = false;
            int b_uses = 0;
            long long k_tiles = 0;
            int last_use[S];
            for (int s = 0; s < S; ++s) last_use[s] = -1;
            // Claimed work: the claim after the current one is requested as soon as
            // the current one starts, so its latency hides behind the current items.
            // Otherwise one contiguous range per CTA.
            // The last two rounds of claims take one item each, so the CTAs finish
            // within about one item of each other.
            ItemRun run;
            long long next = total;
            int next_sz = kClaim;  // items in the claim at `next`
            const long long tail = 2LL * kClaim * gridDim.x;
            if (a.work) {
                next = static_cast<long long>(atomicAdd(a.work, static_cast<unsigned long long>(kClaim)));
            } else {
                const long long begin = total * blockIdx.x / gridDim.x;
                run.start(begin, total * (blockIdx.x + 1) / gridDim.x - begin, tpg);
            }
            for (;;) {
                if (run.left == 0) {
                    if (next >= total) break;
                    run.start(next, min(static_cast<long long>(next_sz), total - next), tpg);
                    next_sz = next + tail < total ? kClaim : 1;
                    next = static_cast<long long>(atomicAdd(a.work, static_cast<unsigned long long>(next_sz)));
                }
                int g, j;
                run.take(tpg, g, j);
                if (g != cur_g) {
                    group_info<G>(a, g, seq, max_pos);
                    cur_g = g;
                    group_loaded = false;
                    // a group without one valid query is skipped whole, so the epilogue
                    // never checks it: report it here
                    if (seq < 0 || max_pos < 0) report_status(a.status, DSA_ERR_INVALID);
                }
                if (seq < 0 || j * kTileKeys > max_pos) {
                    run.skip_group(tpg);
                    continue;
                }
                if (a.work) {  // claimed work: the consumers learn the item from the ring
                    const int r = static_cast<int>(k_tiles % kRing);
                    item_q[r] = make_int2(g, j);
                    mbar_arrive(&item_bar[r]);
                }
                if (!group_loaded) {
                    if (b_uses > 0 &&
                        !mbar_wait(&b_empty, (b_uses - 1) & 1, a.status, &abort_flag))
                        break;
                    mbar_arrive_expect_tx(&b_full, Cfg::kBBytes);
                    // box x = 64 bf16 or 128 FP8 values: 128 bytes
#pragma unroll
                    for (int bx = 0; bx < Cfg::kBoxes; ++bx)
                        tma_load_2d(b_tile + bx * N * 128, &tmap_q, &b_full, bx * 64, g * N);
                    ++b_uses;
                    group_loaded = true;
                }
                const int stage = static_cast<int>(k_tiles % S);
                const int use = static_cast<int>(k_tiles / S);
                if (!mbar_wait(&empty_bar[stage], (use & 1) ^ 1, a.status, &abort_flag)) break;
                uint8_t *dst = a_tiles + stage * kATileBytes;
                mbar_arrive_expect_tx(&full_bar[stage], kATileBytes);
#pragma unroll
                for (int bx = 0; bx < Cfg::kBoxes; ++bx)
                    tma_load_3d_hint(dst + bx * (kTileKeys * 128), &tmap_k, &full_bar[stage], bx * 64, j * kTileKeys,
                                     seq, stream_policy);
                last_use[stage] = use;
                ++k_tiles;
            }
            if (a.work) {
                item_q[k_tiles % kRing] = make_int2(-1, 0);  // the end (also after an abort: the consumers stop)
                mbar_arrive(&item_bar[k_tiles % kRing]);
                // this CTA claims nothing more; the last CTA to get here leaves the
                // counters zero for the next launch (while its pipeline drains)
                if (atomicAdd(a.work + 1, 1ull) == gridDim.x - 1) {
                    atomicExch(a.work, 0ull);
                    atomicExch(a.work + 1, 0ull);
                }
            }
            // Drain: every copy this thread issued has landed before the CTA exits.
            for (int s = 0; s < S; ++s)
                if (last_use[s] >= 0) mbar_wait(&full_bar[s], last_use[s] & 1, a.status, nullptr);
            if (b_uses > 0) mbar_wait(&b_full, (b_uses - 1) & 1, a.status, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int cur_g = -1;
            bool group_ready = false;
            int b_uses = 0;
            long long k_tiles = 0;
            ItemWalk<G> walk(total * blockIdx.x / gridDim.x, total * (blockIdx.x + 1) / gridDim.x, tpg);
            int g, j;
            while (walk.next(a, tpg, k_tiles, item_q, item_bar, &abort_flag, g, j)) {
                if (g != cur_g) {
                    cur_g = g;
                    group_ready = false;
                }
                if (!group_ready) {
                    if (b_uses > 0) umma_commit(&b_empty);  // previous group's MMAs release B
                    if (!mbar_wait(&b_full, b_uses & 1, a.status, &abort_flag)) break;
                    tc_fence_after();
                    ++b_uses;
                    group_ready = true;
                }
                const int stage = static_cast<int>(k_tiles % S);
                const int use = static_cast<int>(k_tiles / S);
                const int acc = static_cast<int>(k_tiles & 1);
                const int acc_use = static_cast<int>(k_tiles >> 1);
                if (!mbar_wait(&tmem_empty[acc], (acc_use & 1) ^ 1, a.status, &abort_flag)) break;
                tc_fence_after();
                if (!mbar_wait(&full_bar[stage], use & 1, a.status, &abort_flag)) break;
                tc_fence_after();
                const uint64_t adesc = sdesc_sw128(smem_u32(a_tiles + stage * kATileBytes), 16, 1024);
                const uint64_t bdesc = sdesc_sw128(smem_u32(b_tile), 16, 1024);
                const uint32_t d_tmem = tmem_base + acc * N;
#pragma unroll
                for (int kk = 0; kk < Cfg::kKSteps; ++kk) {
                    // offsets in 16-byte units added to the descriptors' start-address field:
                    // each K step covers 32 bytes of a 128-byte row; bf16 rows span two boxes
                    const uint64_t aoff = static_cast<uint64_t>(((kk >> 2) * (kTileKeys * 128) + (kk & 3) * 32) >> 4);
                    const uint64_t boff = static_cast<uint64_t>(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4);
                    if constexpr (F8)
                        umma_e4m3(d_tmem, adesc + aoff, bdesc + boff, Cfg::kIdesc, kk > 0 ? 1u : 0u);
                    else
                        umma_bf16(d_tmem, adesc + aoff, bdesc + boff, Cfg::kIdesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty_bar[stage]);
                umma_commit(&tmem_full[acc]);
                ++k_tiles;
            }
            umma_commit(&mma_done);
            mbar_wait(&mma_done, 0, a.status, nullptr);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        // queries of the tile this warp handles
        constexpr int kQPerWarp = G / (E / 4);
        const int qlo = ((warp - 2) >> 2) * kQPerWarp;
        float *w_mine = w_sh[warp - 2];
        const int etid = threadIdx.x - 64;
        int cur_g = -1, seq = -1, max_pos = -1;
        int qpos[kQPerWarp];   // this warp's queries of the current group
        bool qok[kQPerWarp];
        // Several queries per tile (prefill): the head weights of the warp's first
        // query stay in registers for the whole group, the second query's are read
        // from shared memory per tile (both do not fit in the 96 registers a thread
        // has at this block size: measured slower with the spills).
        float w0[G == 1 ? 1 : 32];
        long long k_tiles = 0;
        uint32_t epi_phase = 0;
        bool hist_dirty = false;
        // all four epilogue warps meet (bounded wait on an mbarrier)
        auto epi_sync = [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive(&epi_bar);
            mbar_wait(&epi_bar, epi_phase, a.status, &abort_flag);
            epi_phase ^= 1;
        };
        auto flush_hist = [&](int g) {
            epi_sync();
            uint32_t *dst = a.ghist + static_cast<int64_t>(g) * kTopkBins;
            for (int b = etid; b < kTopkBins; b += 128) {
                const uint32_t v = ehist[b];
                if (v) {
                    atomicAdd(dst + b, v);
                    ehist[b] = 0;
                }
            }
            epi_sync();
        };
        ItemWalk<G> walk(total * blockIdx.x / gridDim.x, total * (blockIdx.x + 1) / gridDim.x, tpg);
        int g, j;
        while (walk.next(a, tpg, k_tiles, item_q, item_bar, &abort_flag, g, j)) {
            if (g != cur_g) {
                if (fuse_hist && hist_dirty) {
                    flush_hist(cur_g);
                    hist_dirty = false;
                }
                group_info<G>(a, g, seq, max_pos);
                cur_g = g;
                const int q0 = g * G;
                __syncwarp();  // this warp no longer reads the previous group's w
                for (int e = lane; e < N; e += 32) {
                    const int qi = q0 + e / 32;
                    float wv = qi < a.n_q ? __ldg(a.w + static_cast<int64_t>(qi) * kIdxHeads + (e & 31)) : 0.f;
                    // FP8: a positive per-(query, head) scale factors out of the ReLU onto w
                    if (F8 && a.q_scale && qi < a.n_q) wv *= __ldg(a.q_scale + static_cast<int64_t>(qi) * kIdxHeads + (e & 31));
                    w_mine[e] = wv;
                }
                __syncwarp();
                if constexpr (G > 1) {
#pragma unroll
                    for (int h = 0; h < 32; ++h) w0[h] = w_mine[qlo * 32 + h];
                }
#pragma unroll
                for (int ii = 0; ii < kQPerWarp; ++ii) {
                    const int qi = q0 + qlo + ii;
                    qpos[ii] = -1;
                    qok[ii] = false;
                    if (qi < a.n_q) {
                        const int p = __ldg(a.q_pos + qi);
                        const int sq = __ldg(a.q_seq + qi);
                        const bool seq_ok = a.k_shared ? (sq >= 0 && sq < a.n_seq) : (sq == seq);
                        qok[ii] = p >= 0 && p < a.L && seq_ok && seq >= 0;
                        qpos[ii] = p;
                        if (!qok[ii] && lane == 0) report_status(a.status, DSA_ERR_INVALID);
                    }
                }
            }
            const int acc = static_cast<int>(k_tiles & 1);
            const int acc_use = static_cast<int>(k_tiles >> 1);
            const int s = j * kTileKeys + quad * 32 + lane;
            // FP8: the key's positive scale factors out of every head's ReLU (loaded
            // before the wait for the accumulator, so its latency is hidden)
            const float ks = (F8 && a.k_scale && s < a.L) ? __ldg(a.k_scale + static_cast<int64_t>(seq) * a.ks_seq_stride + s)
                                                         : 1.f;
            if (!mbar_wait(&tmem_full[acc], acc_use & 1, a.status, &abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * N;
#pragma unroll
            for (int ii = 0; ii < kQPerWarp; ++ii) {
                const int i = qlo + ii;
                float score = 0.f;
                if constexpr (G == 1) {
                    uint32_t r[32];
                    tmem_ld32(taddr + i * 32, r);
                    tmem_ld_wait();
                    const float4 *w4 = reinterpret_cast<const float4 *>(w_mine + i * 32);
#pragma unroll
                    for (int h4 = 0; h4 < 8; ++h4) {
                        const float4 wv = w4[h4];
                        score = fmaf(wv.x, fmaxf(u2f(r[4 * h4]), 0.f), score);
                        score = fmaf(wv.y, fmaxf(u2f(r[4 * h4 + 1]), 0.f), score);
                        score = fmaf(wv.z, fmaxf(u2f(r[4 * h4 + 2]), 0.f), score);
                        score = fmaf(wv.w, fmaxf(u2f(r[4 * h4 + 3]), 0.f), score);
                    }
                } else {
                    // 16 heads per TMEM load (room for the weights in registers);
                    // the same head order as above, so the same sums
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t r[16];
                        tmem_ld16(taddr + i * 32 + 16 * hh, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 16; ++h) {
                            const float wv = ii == 0 ? w0[16 * hh + h] : w_mine[i * 32 + 16 * hh + h];
                            score = fmaf(wv, fmaxf(u2f(r[h]), 0.f), score);
                        }
                    }
                }
                if (F8) score *= ks;
                const bool vis = qok[ii] && s <= qpos[ii];
                if (vis) a.scores[static_cast<int64_t>(g * G + i) * a.ld + s] = score;
                if (fuse_hist) hist_add(ehist, vis ? first_digit(order_key(score)) : 0xFFFFFFFFu);
            }
            hist_dirty = true;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[acc]);
            ++k_tiles;
        }
        if (fuse_hist && hist_dirty && !abort_flag) flush_hist(cur_g);
    }

    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ---------------------------------------------------------------- generic path
// One thread per (query, key); the query's heads x dims and weights sit in
// shared memory.  Any head count / dim, bf16 or fp32 inputs.
template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__global__ void __launch_bounds__(256) idx_score_generic_kernel(const IdxGenericArgs a) {
    extern __shared__ float sq[];  // heads*dim query values, then heads weights
    const int i = blockIdx.y;
    const T *q = static_cast<const T *>(a.q) + static_cast<int64_t>(i) * a.heads * a.dim;
    for (int e = threadIdx.x; e < a.heads * a.dim; e += blockDim.x) sq[e] = to_f<T>(q[e]);
    for (int e = threadIdx.x; e < a.heads; e += blockDim.x)
        sq[a.heads * a.dim + e] = a.w[static_cast<int64_t>(i) * a.heads + e];
    __syncthreads();
    const int pos = a.q_pos[i];
    const int seq = a.q_seq[i];
    const bool ok = pos >= 0 && pos < a.L && seq >= 0 && seq < a.n_seq;
    if (!ok) {
        if (blockIdx.x == 0 && threadIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
        return;
    }
    const T *kb = static_cast<const T *>(a.k) + (a.k_seq_stride ? static_cast<int64_t>(seq) * a.k_seq_stride : 0);
    const float *wv = sq + a.heads * a.dim;
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s <= pos; s += gridDim.x * blockDim.x) {
        const T *kr = kb + static_cast<int64_t>(s) * a.k_row_stride;
        float score = 0.f;
        for (int h = 0; h < a.heads; ++h) {
            const float *qh = sq + h * a.dim;
            float dot = 0.f;
            for (int d = 0; d < a.dim; ++d) dot = fmaf(qh[d], to_f<T>(kr[d]), dot);
            score = fmaf(wv[h], fmaxf(dot, 0.f), score);
        }
        a.scores[static_cast<int64_t>(i) * a.ld + s] = score;
    }
}

template <int G, bool F8>
cudaError_t launch_tc(const CUtensorMap &tk, const CUtensorMap &tq, const IdxTcArgs &a, int num_sms,
                      cudaStream_t st) {
    using Cfg = IdxCfg<G, F8>;
    const long long slots = static_cast<long long>(num_sms) * Cfg::kCtasPerSm;
    const int grid = static_cast<int>(a.total_items < slots ? a.total_items : slots);
    cudaError_t e = set_max_dynamic_smem(idx_score_tc_kernel<G, F8>, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(idx_score_tc_kernel<G, F8>, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmem, st, tk, tq, a);
}

template <bool F8>
cudaError_t launch_tc_g(int G, const CUtensorMap &tmap_k, const CUtensorMap &tmap_q, const IdxTcArgs &a,
                        int num_sms, cudaStream_t st) {
    switch (G) {
        case 1: return launch_tc<1, F8>(tmap_k, tmap_q, a, num_sms, st);
        case 2: return launch_tc<2, F8>(tmap_k, tmap_q, a, num_sms, st);
        case 4: return launch_tc<4, F8>(tmap_k, tmap_q, a, num_sms, st);
        case 8: return launch_tc<8, F8>(tmap_k, tmap_q, a, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_idx_score_tc(int G, bool fp8, const CUtensorMap &tmap_k, const CUtensorMap &tmap_q,
                                const IdxTcArgs &a, int num_sms, cudaStream_t st) {
    return fp8 ? launch_tc_g<true>(G, tmap_k, tmap_q, a, num_sms, st)
               : launch_tc_g<false>(G, tmap_k, tmap_q, a, num_sms, st);
}

cudaError_t launch_idx_score_generic(const IdxGenericArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * (static_cast<size_t>(a.heads) * a.dim + a.heads);
    const int bx = std::min((a.L + 255) / 256, 1024);
    dim3 grid(bx, a.n_q);
    if (a.is_bf16) {
        cudaError_t e = set_max_dynamic_smem(idx_score_generic_kernel<__nv_bfloat16>, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        idx_score_generic_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
    } else {
        cudaError_t e = set_max_dynamic_smem(idx_score_generic_kernel<float>, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        idx_score_generic_kernel<float><<<grid, 256, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace dsa
