// mla.cu -- sparse absorbed MLA attention over the selected cache rows.
//
// For query i, head h and selected rows s_j (j < cnt[i]):
//   l_j = scale * (q_lat[i,h] . c_{s_j} + q_rope[i,h] . r_{s_j})
//   out[i,h] = sum_j softmax(l)_j c_{s_j},  lse[i,h] = log sum_j exp(l_j)
// ("GLM-5.2 -- Model techniques map", "Checked in its code": Indexer-selected
// sparse attention -- attention only over the index_topk selected tokens;
// Multi-head latent attention -- 512-dim latent + 64-dim RoPE key per token;
// Learnable attention sink -- plain float32 softmax, no sink.)
//
// Tensor-core path (bf16, 64 heads, 512 + 64): one CTA per (query, split,
// layer) walks its share of the selected rows in chunks of 64, software-pipelined
// across warp roles with mbarriers (every wait bounded):
//   producers (warps 4-7)  gather chunk c+1 -- 64 rows x 1152 B into nine
//            64-column blocks of 128-byte-swizzled shared memory -- into one of
//            two 72 KB slots while chunk c is computed: bf16 caches by TMA row
//            gathers (four rows per op, issued by the lanes), packed FP8 caches
//            by per-lane loads widened to fp16; the 64 x 576 query tile once per
//            CTA (TMA boxes for bf16).
//   MMA issuer (warp 8)   S = Q . C^T (M = 64 heads, N = 64 rows, K = 576, both
//            operands K-major): 36 tcgen05.mma into TMEM columns 64*slot; then
//            O^T += C_lat^T . P^T (the row tile read MN-major: M = 4 x 128 latent
//            dims, N = 64 heads, K = 64 rows) into columns 128..383.
//   softmax (warps 0-3)   the M = 64 accumulator keeps heads 16w..16w+15 in
//            lanes 32w..32w+15; lanes l and l + 16 of warp w share head 16w + l
//            (rows 0..31 and 32..63 of the chunk, one 16x32bx2 TMEM load):
//            running max, exponentials and sum in registers, combined with one
//            shuffle; P (bf16) as one 128-byte line per head in the slot's freed
//            RoPE block; the accumulated O is rescaled only when a head's maximum
//            grows by more than 2^8.
//   epilogue (warps 0-7)  reads O^T from TMEM: the final bf16 output (one CTA
//            per query) or fp32 partials + (max, sum) per head for a split-K
//            merge (decode with few queries).
#include <climits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "tma_encode.cuh"

namespace dsa {
namespace {

constexpr int kChunk = 64;                          // selected rows per pipeline chunk
constexpr int kMlaThreads = 288;                    // 4 softmax + 4 producer + 1 MMA warp
constexpr int kBlockBytes = kChunk * 128;           // 64 rows (or heads) x 64 dims bf16 = 8 KB
constexpr int kBlocks = kRow / 64;                  // 9 column blocks (8 latent + rope)
constexpr int kSlotBytes = kBlocks * kBlockBytes;   // 72 KB: one chunk of rows
constexpr int kQBytes = kBlocks * kBlockBytes;      // 72 KB: 64 heads x 576
constexpr int kMlaSmem = kQBytes + 2 * kSlotBytes + 1024;
constexpr int kTmemCols = 512;                      // S slots: 0..127, O^T: 128..383
constexpr int kOCol = 128;
constexpr uint32_t kIdescS = idesc_bf16(64, 64, false, false);
constexpr uint32_t kIdescO = idesc_bf16(128, 64, true, false);
// Packed FP8 caches run the MMAs in fp16 (E4M3 codes, the queries and the RoPE
// keys are exact in fp16): S has a latent half (codes, the row scale applied in
// the softmax) in columns 64*slot and a RoPE half in columns kSRopeCol + 64*slot.
constexpr uint32_t kIdescS16 = idesc_f16(64, 64, false, false);
constexpr uint32_t kIdescO16 = idesc_f16(128, 64, true, false);
constexpr int kSRopeCol = 384;
// A running maximum is kept until a head's chunk maximum exceeds it by more than
// this many powers of two (probabilities stay below 2^8); only then is the
// accumulated O rescaled.
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Two E4M3 codes (low byte first) as two fp16 (low half first): exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
    return static_cast<uint32_t>(hr.x) | (static_cast<uint32_t>(hr.y) << 16);
}

// Eight bf16 values (one 16-byte piece) as eight fp16, rounded to nearest (exact
// for bf16 values of magnitude within fp16's normal range).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
        const __half2 h = __floats2half2_rn(f.x, f.y);
        w[k] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// kFp8: the caches are packed FP8 rows [512 E4M3 codes | 64 bf16 RoPE | float32
// scale | padding].  The producers widen the codes (exactly) and the RoPE keys and
// queries to fp16 into the same swizzled tiles; the MMAs run kind::f16 on fp16;
// the softmax scales each row's latent logit by its sigma and folds sigma into
// the fp16 P, so O = sum_j p_j sigma_j code_j.
// One CTA per SM (217 KB of shared memory).  Nine warps spread over the SM's
// four sub-partitions (three on one of them, whose 16K-register file they
// share) allow at most 168 registers per thread.
template <bool kFp8>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_tc_kernel(const MlaArgs a, const __grid_constant__ MlaMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *q_sm = smem;
    uint8_t *slot_sm = smem + kQBytes;  // slot s at slot_sm + s * kSlotBytes

    // o_done[s]: the O-MMA of the chunk in slot s completed (the slot may be refilled)
    __shared__ uint64_t q_full, slot_full[2], s_full[2], p_full[2], o_done[2], fin, sm_bar;
    __shared__ uint64_t raw_full[2];  // FP8: a chunk's gathered bytes (before widening) are in the slot
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int row_idx[2][kChunk];  // [slot][chunk row]: cache row, or -1 (padding)
    __shared__ float row_sigma[kFp8 ? 2 : 1][kChunk];  // FP8 caches: [slot][chunk row] row scale
    __shared__ float alpha_sm[kMlaHeads], m_fin[kMlaHeads], l_fin[kMlaHeads], inv_l[kMlaHeads];
    __shared__ int rescale_w[4];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, i = blockIdx.y, layer = blockIdx.z;
    const MlaLayerPtrs lp = a.layer[layer];
    const float c2 = a.scale * kLog2e;

    if (tid == 0) {
        mbar_init(&q_full, kFp8 ? 4 : 1);  // bf16: one arrival with the TMA byte count
        for (int s = 0; s < 2; ++s) {
            mbar_init(&slot_full[s], 4);    // one per producer warp (+ the TMA bytes for bf16)
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&o_done[s], 1);
            mbar_init(&raw_full[s], 4);  // one per producer warp, with its bytes
        }
        mbar_init(&fin, 1);
        mbar_init(&sm_bar, 4);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base_sh;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(lp.q) + static_cast<int64_t>(i) * kMlaHeads * kRow;
    const uint32_t q_addr = smem_u32(q_sm);
    if (!kFp8 && tid == 4 * 32) {
        // The query tile is an input of the step, not written by the kernel this
        // launch depends on: nine 64-head x 64-dim TMA boxes, issued before the
        // dependency wait.
        tma_prefetch_desc(&maps.q[layer]);
        tma_prefetch_desc(&maps.kv[layer]);
        mbar_arrive_expect_tx(&q_full, kQBytes);
#pragma unroll 1
        for (int b = 0; b < kBlocks; ++b) tma_load_2d(q_sm + b * kBlockBytes, &maps.q[layer], &q_full, 64 * b, i * kMlaHeads);
    }
    if (kFp8 && warp >= 4 && warp < 8) {
        // The query tile is an input of the step, not written by the kernel this
        // launch depends on: its copy (heads 16*pw .. 16*pw+15 per producer warp)
        // is issued before the dependency wait.
        const int pw = warp - 4;
        for (int hh = 0; hh < 16; ++hh) {
            const int h = 16 * pw + hh;
#pragma unroll
            for (int tt = 0; tt < 3; ++tt) {
                const int ch = lane + 32 * tt;
                if (ch < kRow / 8)
                    cp_async_16(q_addr + (ch >> 3) * kBlockBytes + sw128_offset(h, ch & 7), q + h * kRow + ch * 8);
            }
        }
        cp_async_commit();
        if constexpr (kFp8) {
            // fp16 queries for the fp16 MMAs: each thread converts the pieces it
            // copied, in place, while the previous kernel may still be running
            cp_async_wait_all();
            for (int hh = 0; hh < 16; ++hh) {
                const int h = 16 * pw + hh;
#pragma unroll
                for (int tt = 0; tt < 3; ++tt) {
                    const int ch = lane + 32 * tt;
                    if (ch < kRow / 8) {
                        const uint32_t adr = q_addr + (ch >> 3) * kBlockBytes + sw128_offset(h, ch & 7);
                        uint4 v;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                     : "r"(adr)
                                     : "memory");
                        v = bf16x8_to_f16x8(v);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(v.x), "r"(v.y), "r"(v.z),
                                     "r"(v.w)
                                     : "memory");
                    }
                }
            }
            // this warp's share of the fp16 query tile is in (for the MMAs' async reads)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_full);
        }
    }
    int seq = a.q_seq[i];  // an input of the step, like the query tile
    griddep_wait();

    const int si = i / a.sel_group;  // the selection row this query reads
    const int32_t *sel = a.idx + static_cast<int64_t>(si) * a.topk;
    const int c_begin = split * a.chunks_per_cta;
    // producers: the first two chunks' indices (this lane's row, and the chunk's
    // first row) are requested with the count, not after it; later chunks' two
    // chunks ahead of their turn
    int r_first = -1, f_first = -1, r_second = -1, f_second = -1;
    if (warp >= 4 && warp < 8) {
        const int j0 = c_begin * kChunk + 16 * (warp - 4) + (lane & 15);
        if (j0 < a.topk) r_first = __ldg(sel + j0);
        if (c_begin * kChunk < a.topk) f_first = __ldg(sel + c_begin * kChunk);
        if (j0 + kChunk < a.topk) r_second = __ldg(sel + j0 + kChunk);
        if ((c_begin + 1) * kChunk < a.topk) f_second = __ldg(sel + (c_begin + 1) * kChunk);
    }
    int cnt = a.cnt[si];
    if (!(seq >= 0 && seq < a.n_seq && cnt >= 0 && cnt <= a.topk)) {
        if (tid == 0) report_status(a.status, DSA_ERR_INVALID);
        cnt = 0;
        seq = 0;
    }
    const int nch = (cnt + kChunk - 1) / kChunk;
    const int nloc = max(0, min(c_begin + a.chunks_per_cta, nch) - c_begin);
    const uint8_t *kv8 = static_cast<const uint8_t *>(lp.kv) + static_cast<int64_t>(seq) * a.kv_seq_stride;

    if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ producers
        const int pw = warp - 4;  // rows (and the query tile's heads) 16*pw .. 16*pw+15
        // the rows of all sequences form one 2-D tensor (rows of kv_row_stride)
        const int seq_row0 = a.kv_row_stride > 0 ? static_cast<int>(static_cast<int64_t>(seq) * (a.kv_seq_stride / a.kv_row_stride)) : 0;
        const int rl = 16 * pw + (lane & 15);
        if constexpr (!kFp8) {
            int issued = 0;                        // chunks whose row gathers this warp has issued
            int r_cur = r_first, f_cur = f_first;    // chunk t's index (this lane's row) and first row
            int r_nx = r_second, f_nx = f_second;    // chunk t + 1's
            for (int t = 0; t < nloc; ++t) {
                const int c = c_begin + t, s = t & 1, u = t >> 1;
                // chunk t + 2's indices are requested now: they land while this chunk
                // and the next wait for their slots and are issued
                int r_n2 = -1, f_n2 = -1;
                if (t + 2 < nloc) {
                    const int j2 = (c + 2) * kChunk + rl;
                    if (j2 < a.topk) r_n2 = __ldg(sel + j2);
                    f_n2 = __ldg(sel + (c + 2) * kChunk);
                }
                if (t >= 2 && !mbar_wait(&o_done[s], (u - 1) & 1, a.status, &abort_flag)) break;
                const int j = c * kChunk + rl;
                int r = -1;
                if (j < cnt) {
                    r = r_cur;
                    if (r < 0 || r >= a.L) {
                        report_status(a.status, DSA_ERR_INVALID);
                        r = -1;
                    }
                }
                if (lane < 16) row_idx[s][rl] = r;
                const uint32_t sb = smem_u32(slot_sm + s * kSlotBytes);
                // The warp's 16 rows as 4 row gathers per 64-dim block (36 TMA ops,
                // lanes 0-31 then 0-3): padding rows and rejected indices fetch the
                // chunk's first row instead (in range; masked in the softmax), so
                // every op moves whole rows and the byte count is fixed.
                int f = f_cur;
                if (f < 0 || f >= a.L) f = 0;
                const int gr = seq_row0 + (r >= 0 ? r : f);
                const int g0 = lane / 9, b0 = lane - 9 * g0;
                int y0[4], y1[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    y0[qq] = __shfl_sync(0xffffffffu, gr, 4 * g0 + qq);
                    y1[qq] = __shfl_sync(0xffffffffu, gr, 12 + qq);
                }
                __syncwarp();  // row_idx written before the arrival releases it
                if (lane == 0) mbar_arrive_expect_tx(&slot_full[s], 16 * kRow * 2);
                const uint32_t wb = sb + (16 * pw) * 128;
                tma_gather4(wb + b0 * kBlockBytes + g0 * 512, &maps.kv[layer], &slot_full[s], 64 * b0, y0[0], y0[1],
                            y0[2], y0[3]);
                if (lane < 4)
                    tma_gather4(wb + (5 + lane) * kBlockBytes + 3 * 512, &maps.kv[layer], &slot_full[s],
                                64 * (5 + lane), y1[0], y1[1], y1[2], y1[3]);
                issued = t + 1;
                r_cur = r_nx;
                f_cur = f_nx;
                r_nx = r_n2;
                f_nx = f_n2;
            }
            if (lane == 0) {
                // every TMA copy this warp requested has landed before the CTA may exit
                // (the consumers may have stopped early on an abort): the last phase of
                // each slot it filled, and the query tile
                for (int t = max(0, issued - 2); t < issued; ++t)
                    mbar_wait(&slot_full[t & 1], (t >> 1) & 1, a.status, nullptr);
                if (pw == 0) mbar_wait(&q_full, 0, a.status, nullptr);
            }
        } else {
            // Packed FP8 rows.  Each chunk's bytes for this warp's 16 rows arrive by TMA
            // row gathers on raw_full[slot]: the codes (four 128-byte boxes per row,
            // unswizzled) into the slot's blocks 4..7 as staging, the RoPE key (one
            // 64 x bf16 box, swizzled) into block 8.  The warp then widens them in the
            // slot: codes to the fp16 tiles (exact), the RoPE key to fp16 in place, and
            // marks the slot full.  Issuing a chunk (when its slot is free) and widening
            // one (when its bytes are in) are polled, not waited for in turn, so the next
            // chunk's gathers are in flight while this one is widened and computed.
            // Padding rows fetch the chunk's first row (masked in the softmax, scale 0).
            int n_iss = 0, n_conv = 0;             // chunks issued / widened by this warp
            int r_iss = r_first, f_iss = f_first;    // chunk n_iss's index (this lane's row) and first row
            int r_iss2 = r_second, f_iss2 = f_second;  // chunk n_iss + 1's
            float sig0 = 0.f, sig1 = 0.f;          // lanes < 16: the scale of this lane's row, per slot
            uint64_t t_idle = 0;
            while (n_conv < nloc) {
                bool did = false;
                if (n_iss < nloc && n_iss < n_conv + 2) {
                    const int s = n_iss & 1;
                    bool free = n_iss < 2;
                    if (!free) {
                        uint32_t ok = 0;
                        if (lane == 0) ok = mbar_test_wait(&o_done[s], ((n_iss >> 1) - 1) & 1) ? 1u : 0u;
                        free = __shfl_sync(0xffffffffu, ok, 0) != 0u;
                    }
                    if (free) {
                        const int c = c_begin + n_iss;
                        const int j = c * kChunk + rl;
                        int r = -1;
                        if (j < cnt) {
                            r = r_iss;
                            if (r < 0 || r >= a.L) {
                                report_status(a.status, DSA_ERR_INVALID);
                                r = -1;
                            }
                        }
                        int f = f_iss;
                        if (f < 0 || f >= a.L) f = 0;
                        // the indices of the chunk after next are requested now
                        r_iss = r_iss2;
                        f_iss = f_iss2;
                        r_iss2 = -1;
                        f_iss2 = -1;
                        if (n_iss + 2 < nloc) {
                            const int j2 = (c + 2) * kChunk + rl;
                            if (j2 < a.topk) r_iss2 = __ldg(sel + j2);
                            f_iss2 = __ldg(sel + (c + 2) * kChunk);
                        }
                        if (lane < 16) row_idx[s][rl] = r;
                        const int gr = seq_row0 + (r >= 0 ? r : f);
                        // lanes 0..15: codes of row group lane / 4, box lane % 4;
                        // lanes 16..19: RoPE keys of row group lane - 16
                        const int g = lane < 16 ? (lane >> 2) : (lane - 16) & 3;
                        int y[4];
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) y[qq] = __shfl_sync(0xffffffffu, gr, 4 * g + qq);
                        if (lane == 0) mbar_arrive_expect_tx(&raw_full[s], 16 * (kLatent + 2 * kRope));
                        __syncwarp();
                        const uint32_t sb = smem_u32(slot_sm + s * kSlotBytes);
                        const uint32_t rows_off = (16 * pw + 4 * g) * 128;
                        if (lane < 16)
                            tma_gather4(sb + (4 + (lane & 3)) * kBlockBytes + rows_off, &maps.kv[layer], &raw_full[s],
                                        128 * (lane & 3), y[0], y[1], y[2], y[3]);
                        else if (lane < 20)
                            tma_gather4(sb + 8 * kBlockBytes + rows_off, &maps.kvr[layer], &raw_full[s], kFp8RopeOff / 2,
                                        y[0], y[1], y[2], y[3]);
                        // the scale of the row this lane's row fetched (a padding row's P is 0),
                        // loaded straight into the slot's register: it is read only when the
                        // chunk is widened, so nothing here waits for it
                        if (lane < 16) {
                            const float *sp = reinterpret_cast<const float *>(
                                kv8 + static_cast<int64_t>(r >= 0 ? r : f) * a.kv_row_stride + kFp8ScaleOff);
                            if (s == 0)
                                sig0 = __ldg(sp);
                            else
                                sig1 = __ldg(sp);
                        }
                        ++n_iss;
                        did = true;
                    }
                }
                if (n_conv < n_iss) {
                    const int s = n_conv & 1;
                    uint32_t ok = 0;
                    if (lane == 0) ok = mbar_test_wait(&raw_full[s], (n_conv >> 1) & 1) ? 1u : 0u;
                    if (__shfl_sync(0xffffffffu, ok, 0) != 0u) {
                        const uint32_t sb = smem_u32(slot_sm + s * kSlotBytes);
                        // codes: 4 lanes per row (a 128-code quarter each), 8 rows per pass;
                        // every read of a pass before any write (blocks 4..7 hold both the
                        // staged codes and the widened tiles; a row only touches its own lines)
#pragma unroll
                        for (int pass = 0; pass < 2; ++pass) {
                            const int row = 16 * pw + 8 * pass + (lane >> 2);
                            const int q = lane & 3;
                            const uint32_t src = sb + (4 + q) * kBlockBytes + row * 128;
                            uint4 raw[8];
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const int kk = (k + lane) & 7;
                                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(raw[k].x), "=r"(raw[k].y), "=r"(raw[k].z), "=r"(raw[k].w)
                                             : "r"(src + 16 * kk)
                                             : "memory");
                            }
                            __syncwarp();
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const int kk = (k + lane) & 7;  // codes 128q + 16kk .. +15: block 2q + kk/4
                                const uint32_t dst = sb + (2 * q + (kk >> 2)) * kBlockBytes;
                                const int c0 = 2 * (kk & 3);
                                const uint32_t w0 = raw[k].x, w1 = raw[k].y, w2 = raw[k].z, w3 = raw[k].w;
                                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128_offset(row, c0)),
                                             "r"(e4m3x2_to_f16x2(w0 & 0xffffu)), "r"(e4m3x2_to_f16x2(w0 >> 16)),
                                             "r"(e4m3x2_to_f16x2(w1 & 0xffffu)), "r"(e4m3x2_to_f16x2(w1 >> 16))
                                             : "memory");
                                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128_offset(row, c0 + 1)),
                                             "r"(e4m3x2_to_f16x2(w2 & 0xffffu)), "r"(e4m3x2_to_f16x2(w2 >> 16)),
                                             "r"(e4m3x2_to_f16x2(w3 & 0xffffu)), "r"(e4m3x2_to_f16x2(w3 >> 16))
                                             : "memory");
                            }
                            __syncwarp();
                        }
                        // RoPE keys (bf16, swizzled by the TMA) to fp16 in place: 16 rows x 8 pieces
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int idx = lane + 32 * e;
                            const uint32_t adr = sb + 8 * kBlockBytes + sw128_offset(16 * pw + (idx >> 3), idx & 7);
                            uint4 v;
                            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                         : "r"(adr)
                                         : "memory");
                            v = bf16x8_to_f16x8(v);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(v.x), "r"(v.y),
                                         "r"(v.z), "r"(v.w)
                                         : "memory");
                        }
                        if (lane < 16) row_sigma[s][rl] = s == 0 ? sig0 : sig1;
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&slot_full[s]);
                        ++n_conv;
                        did = true;
                    }
                }
                if (did) {
                    t_idle = 0;
                } else {
                    // nothing ready: bounded, like every wait, and stopped by an abort
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0) t_idle = now;
                    uint32_t stop = 0;
                    if (lane == 0) {
                        if (*reinterpret_cast<volatile int *>(&abort_flag)) stop = 1;
                        else if (now - t_idle > kWaitLimitNs) {
                            report_status(a.status, DSA_ERR_TIMEOUT);
                            abort_flag = 1;
                            stop = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, stop, 0) != 0u) break;
                    __nanosleep(64);  // leave the issue slots to the softmax warp on this SM sub-partition
                }
            }
            if (lane == 0) {
                // every gather this warp issued has landed before the CTA may exit
                for (int n = n_conv; n < n_iss; ++n) mbar_wait(&raw_full[n & 1], (n >> 1) & 1, a.status, nullptr);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        // Issues S of chunk ts as soon as its rows are in, and O of chunk to as
        // soon as its P is written, whichever comes first (ts <= to + 1: S of a
        // slot is rewritten only after that slot's O was issued).  Bounded.
        if (lane == 0 && nloc > 0) {
            // base descriptors; each MMA adds its (16-byte unit) offset to the
            // start-address field, which never carries out of it
            const uint32_t sb0 = smem_u32(slot_sm), sb1 = smem_u32(slot_sm + kSlotBytes);
            const uint64_t qdesc = sdesc_sw128(q_addr, 16, 1024);
            const uint64_t cdesc0 = sdesc_sw128(sb0, 16, 1024), cdesc1 = sdesc_sw128(sb1, 16, 1024);
            const uint64_t odesc0 = sdesc_sw128(sb0, kBlockBytes, 1024), odesc1 = sdesc_sw128(sb1, kBlockBytes, 1024);
            const uint64_t pdesc0 = sdesc_sw128(sb0 + 8 * kBlockBytes, 16, 1024);
            const uint64_t pdesc1 = sdesc_sw128(sb1 + 8 * kBlockBytes, 16, 1024);
            bool ok = mbar_wait(&q_full, 0, a.status, &abort_flag);
            int ts = 0, to = 0;
            uint64_t t0 = global_timer_ns();
            uint32_t spin = 0;
            while (ok && to < nloc) {
                bool progressed = false;
                if (ts < nloc && ts <= to + 1 && mbar_test_wait(&slot_full[ts & 1], (ts >> 1) & 1)) {
                    tc_fence_after();
                    const int s = ts & 1;
                    const uint64_t cdesc = s ? cdesc1 : cdesc0;
                    if constexpr (!kFp8) {
#pragma unroll
                        for (int kk = 0; kk < kRow / 16; ++kk) {
                            const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                            umma_bf16(tbase + 64 * s, qdesc + koff, cdesc + koff, kIdescS, kk > 0 ? 1u : 0u);
                        }
                    } else {
                        // latent half (codes) and RoPE half into separate accumulators
#pragma unroll
                        for (int kk = 0; kk < kRow / 16; ++kk) {
                            const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4);
                            const bool rope = kk >= kLatent / 16;
                            umma_bf16(tbase + (rope ? kSRopeCol : 0) + 64 * s, qdesc + koff, cdesc + koff, kIdescS16,
                                      (kk > 0 && kk != kLatent / 16) ? 1u : 0u);
                        }
                    }
                    umma_commit(&s_full[s]);
                    ++ts;
                    progressed = true;
                }
                if (to < ts && mbar_test_wait(&p_full[to & 1], (to >> 1) & 1)) {
                    tc_fence_after();
                    const int sp = to & 1;
                    const uint64_t adesc = sp ? odesc1 : odesc0;  // latent blocks, MN-major
                    const uint64_t bdesc = sp ? pdesc1 : pdesc0;  // P in the RoPE block
#pragma unroll
                    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                        for (int kk = 0; kk < kChunk / 16; ++kk) {
                            umma_bf16(tbase + kOCol + 64 * mt,
                                      adesc + static_cast<uint64_t>((2 * mt * kBlockBytes + kk * 2048) >> 4),
                                      bdesc + static_cast<uint64_t>((kk * 32) >> 4), kFp8 ? kIdescO16 : kIdescO,
                                      (to > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(&o_done[sp]);
                    ++to;
                    progressed = true;
                }
                if (progressed) {
                    t0 = global_timer_ns();
                    spin = 0;
                } else if ((++spin & 63u) == 0) {
                    if (abort_flag) break;
                    if (global_timer_ns() - t0 > kWaitLimitNs) {
                        report_status(a.status, DSA_ERR_TIMEOUT);
                        abort_flag = 1;
                        break;
                    }
                }
            }
            umma_commit(&fin);
            mbar_wait(&fin, 0, a.status, nullptr);  // every MMA of this CTA has completed
        }
    } else {
        // ------------------------------------------------------------ softmax
        // Head 16w + (lane & 15) is held by two lanes: lane < 16 takes the chunk's
        // rows 0..31, lane + 16 rows 32..63 (one tcgen05.ld of shape 16x32bx2);
        // the two combine their maximum and their sum with one shuffle each and
        // keep identical running (m, l).
        const int h = 16 * warp + (lane & 15);
        const int rbase = 32 * (lane >> 4);  // first chunk row of this lane
        const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
        float m = -INFINITY, l = 0.f;
        uint32_t sm_phase = 0;
        for (int t = 0; t < nloc; ++t) {
            const int s = t & 1, u = t >> 1;
            if (!mbar_wait(&slot_full[s], u & 1, a.status, &abort_flag)) break;  // row_idx of the chunk
            if (!mbar_wait(&s_full[s], u & 1, a.status, &abort_flag)) break;
            tc_fence_after();
            float mc = -INFINITY;
            {
                uint32_t r[32];
                tmem_ld16x2_32<32>(lane_base + 64 * s, r);
                if constexpr (kFp8) {
                    // logit = sigma_j * (q_lat . code_j) + q_rope . r_j
                    uint32_t rr[32];
                    tmem_ld16x2_32<32>(lane_base + kSRopeCol + 64 * s, rr);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(fmaf(row_sigma[s][rbase + x], u2f(r[x]), u2f(rr[x])));
                } else {
                    tmem_ld_wait();
                }
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    if (row_idx[s][rbase + x] >= 0) mc = fmaxf(mc, u2f(r[x]));
            }
            mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, 16));
            float al = 1.f;
            if (mc != -INFINITY && (m == -INFINITY || (mc - m) * c2 > kRescaleLog2)) {
                al = (m == -INFINITY) ? 0.f : exp2f((m - mc) * c2);
                m = mc;
            }
            if (lane < 16) alpha_sm[h] = al;
            const bool need = __any_sync(0xffffffffu, al != 1.f && t > 0);
            if (lane == 0) rescale_w[warp] = need ? 1 : 0;
            // the four softmax warps meet: every head's alpha is needed below
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm_bar);
            if (!mbar_wait(&sm_bar, sm_phase, a.status, &abort_flag)) break;
            sm_phase ^= 1;
            const bool any_need = (rescale_w[0] | rescale_w[1] | rescale_w[2] | rescale_w[3]) != 0;
            if (any_need) {
                // O is rescaled only after the previous chunk's O-MMA completed.  The
                // parity wait is exact although most chunks skip it: the producers
                // observed this barrier's previous phase (chunk t-3) before gathering
                // chunk t-1 into the same slot, and its next phase needs chunk t+1.
                const int tp = t - 1;
                if (!mbar_wait(&o_done[tp & 1], (tp >> 1) & 1, a.status, &abort_flag)) break;
                tc_fence_after();
#pragma unroll 1
                for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t ta = lane_base + kOCol + 64 * mt + 32 * half;
                        uint32_t r[32];
                        tmem_ld32(ta, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(u2f(r[x]) * alpha_sm[half * 32 + x]);
                        tmem_st32(ta, r);
                    }
                }
                tmem_st_wait();
            }
            uint32_t r[32];  // the chunk's logits again (cheaper than keeping them live)
            tmem_ld16x2_32<32>(lane_base + 64 * s, r);
            if constexpr (kFp8) {
                uint32_t rr[32];
                tmem_ld16x2_32<32>(lane_base + kSRopeCol + 64 * s, rr);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(fmaf(row_sigma[s][rbase + x], u2f(r[x]), u2f(rr[x])));
            } else {
                tmem_ld_wait();
            }
            {
                uint8_t *pl = slot_sm + s * kSlotBytes + 8 * kBlockBytes;  // head h's P line
                float sum = 0.f;
#pragma unroll
                for (int jc = 0; jc < 4; ++jc) {
                    if constexpr (!kFp8) {
                        __align__(16) __nv_bfloat16 pb[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const int xr = 8 * jc + x;
                            const float pf = (row_idx[s][rbase + xr] >= 0) ? exp2f((u2f(r[xr]) - m) * c2) : 0.f;
                            pb[x] = __float2bfloat16_rn(pf);
                            sum += __bfloat162float(pb[x]);  // the sum uses the value the MMA sees
                        }
                        *reinterpret_cast<uint4 *>(pl + sw128_offset(h, (rbase >> 3) + jc)) =
                            *reinterpret_cast<const uint4 *>(pb);
                    } else {
                        // P' = p * sigma in fp16 (the MMA multiplies it by the exact codes)
                        __align__(16) __half pb[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const int xr = 8 * jc + x;
                            const float pf = (row_idx[s][rbase + xr] >= 0) ? exp2f((u2f(r[xr]) - m) * c2) : 0.f;
                            pb[x] = __float2half_rn(pf * row_sigma[s][rbase + xr]);
                            sum += pf;
                        }
                        *reinterpret_cast<uint4 *>(pl + sw128_offset(h, (rbase >> 3) + jc)) =
                            *reinterpret_cast<const uint4 *>(pb);
                    }
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 16);
                l = l * al + sum;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[s]);
        }
        if (lane < 16) {
            m_fin[h] = m;
            l_fin[h] = l;
        }
    }

    griddep_launch_dependents();
    __syncthreads();  // every role has left its loop: `go` is uniform
    const bool go = nloc > 0 && !abort_flag;
    if (go) {
        mbar_wait(&fin, 0, a.status, &abort_flag);
        tc_fence_after();
        if (tid < kMlaHeads) inv_l[tid] = 1.f / l_fin[tid];
        __syncthreads();
        if (warp < 8) {
            const int quad = warp & 3;
            const int mt0 = (warp < 4) ? 0 : 2;
            const bool final_out = (a.n_splits == 1);
            for (int mt = mt0; mt < mt0 + 2; ++mt) {
                const int d = mt * 128 + quad * 32 + lane;
                // both 32-head halves of this lane's latent dim in flight before one wait
                uint32_t r0[32], r1[32];
                const uint32_t ta = tbase + (static_cast<uint32_t>(quad * 32) << 16) + kOCol + mt * 64;
                tmem_ld32(ta, r0);
                tmem_ld32(ta + 32, r1);
                tmem_ld_wait();
                if (final_out) {
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(lp.out) + static_cast<int64_t>(i) * kMlaHeads * kLatent;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        o[x * kLatent + d] = __float2bfloat16_rn(u2f(r0[x]) * inv_l[x]);
                        o[(32 + x) * kLatent + d] = __float2bfloat16_rn(u2f(r1[x]) * inv_l[32 + x]);
                    }
                } else {
                    float *po = a.part_o + ((static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits + split) * kMlaHeads * kLatent;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        po[x * kLatent + d] = u2f(r0[x]);
                        po[(32 + x) * kLatent + d] = u2f(r1[x]);
                    }
                }
            }
        }
        if (tid < kMlaHeads) {
            if (a.n_splits == 1) {
                if (lp.lse) lp.lse[static_cast<int64_t>(i) * kMlaHeads + tid] = m_fin[tid] * a.scale + logf(l_fin[tid]);
            } else {
                float *ml = a.part_ml + (((static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits + split) * kMlaHeads + tid) * 2;
                ml[0] = m_fin[tid] * c2;  // log2 units
                ml[1] = l_fin[tid];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// Merge split-K partials: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// One CTA per (2 heads, query, layer), 256 threads: thread t owns 4 dims of
// head 2 * blockIdx.x + t / 128.  The partials of the first 16 splits are loaded
// (16-byte loads, all in flight) before the split weights are known: the merge
// is one round trip to L2 plus the weight shuffles.
constexpr int kCombineHeads = 2;
constexpr int kCombineBatch = 16;  // splits whose partials are held in registers at once

__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaArgs a) {
    const int hp = blockIdx.x, i = blockIdx.y, layer = blockIdx.z;
    const MlaLayerPtrs lp = a.layer[layer];
    __shared__ float wgt[kCombineHeads][32];
    griddep_wait();  // splits per query: at most 32 by the planner
    int cnt = a.cnt[i / a.sel_group];
    if (cnt < 0 || cnt > a.topk) cnt = 0;
    const int nch = (cnt + kChunk - 1) / kChunk;
    const int ns = min(32, (nch + a.chunks_per_cta - 1) / a.chunks_per_cta);
    const int64_t base = (static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits;
    const int hl = threadIdx.x >> 7;
    const int h = hp * kCombineHeads + hl;
    const int d = (threadIdx.x & 127) * 4;
    const float *po = a.part_o + (base * kMlaHeads + h) * kLatent + d;  // split s at + s * kMlaHeads * kLatent
    float4 x[kCombineBatch];
#pragma unroll
    for (int s = 0; s < kCombineBatch; ++s)
        x[s] = s < ns ? *reinterpret_cast<const float4 *>(po + static_cast<int64_t>(s) * kMlaHeads * kLatent)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    // (max, sum) of every split: warp w < 2 handles head 2 * hp + w, lane = split
    {
        const int wl = threadIdx.x >> 5, s = threadIdx.x & 31;
        if (wl < kCombineHeads) {
            const int hh = hp * kCombineHeads + wl;
            float m = -INFINITY, l = 0.f;
            if (s < ns) {
                const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + ((base + s) * kMlaHeads + hh) * 2);
                m = ml.x;
                l = ml.y;
            }
            float M = m;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            const float wv = (m == -INFINITY) ? 0.f : exp2f(m - M);
            float L = wv * l;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            wgt[wl][s] = s < ns ? wv / L : 0.f;
            if (s == 0 && lp.lse) lp.lse[static_cast<int64_t>(i) * kMlaHeads + hh] = (M + log2f(L)) * kLn2;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kCombineBatch; ++s) {
        const float wv = wgt[hl][s];
        acc.x += wv * x[s].x, acc.y += wv * x[s].y, acc.z += wv * x[s].z, acc.w += wv * x[s].w;
    }
    for (int s = kCombineBatch; s < ns; ++s) {  // more than 16 splits (long contexts, few queries)
        const float4 y = *reinterpret_cast<const float4 *>(po + static_cast<int64_t>(s) * kMlaHeads * kLatent);
        const float wv = wgt[hl][s];
        acc.x += wv * y.x, acc.y += wv * y.y, acc.z += wv * y.z, acc.w += wv * y.w;
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(lp.out) + (static_cast<int64_t>(i) * kMlaHeads + h) * kLatent + d;
    __align__(8) __nv_bfloat16 ob[4] = {__float2bfloat16_rn(acc.x), __float2bfloat16_rn(acc.y),
                                        __float2bfloat16_rn(acc.z), __float2bfloat16_rn(acc.w)};
    *reinterpret_cast<uint2 *>(o) = *reinterpret_cast<const uint2 *>(ob);
}

// ---------------------------------------------------------------- generic path
// One CTA per (query, head, layer): logits of the selected rows into shared
// memory, block max / sum, then each thread accumulates a few output dims.
template <typename T>
__device__ __forceinline__ float ld_f(const T *p);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st_f(T *p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float *p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float block_reduce(float v, float *buf, bool is_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, y) : v + y;
    }
    if (lane == 0) buf[warp] = v;
    __syncthreads();
    float r = buf[0];
    for (int w = 1; w < nw; ++w) r = is_max ? fmaxf(r, buf[w]) : r + buf[w];
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(128) mla_generic_kernel(const MlaArgs a) {
    extern __shared__ float sh[];  // q (dk) then logits (topk)
    __shared__ float buf[32];
    __shared__ int bad;
    const int i = blockIdx.x, h = blockIdx.y, layer = blockIdx.z;
    const MlaLayerPtrs lp = a.layer[layer];
    const int dk = a.d_lat + a.d_rope;
    float *qs = sh;
    float *lg = sh + dk;
    const T *q = static_cast<const T *>(lp.q) + (static_cast<int64_t>(i) * a.heads + h) * dk;
    for (int d = threadIdx.x; d < dk; d += blockDim.x) qs[d] = ld_f<T>(q + d);
    if (threadIdx.x == 0) bad = 0;
    int seq = a.q_seq[i];
    int cnt = a.cnt[i / a.sel_group];
    if (seq < 0 || seq >= a.n_seq || cnt < 0 || cnt > a.topk) {
        if (threadIdx.x == 0 && h == 0) report_status(a.status, DSA_ERR_INVALID);
        seq = 0;
        cnt = 0;
    }
    __syncthreads();
    const T *kv = static_cast<const T *>(lp.kv) + static_cast<int64_t>(seq) * a.kv_seq_stride;
    const int32_t *sel = a.idx + static_cast<int64_t>(i / a.sel_group) * a.topk;
    float m = -INFINITY;
    for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
        const int r = sel[j];
        float l = -INFINITY;
        if (r >= 0 && r < a.L) {
            const T *row = kv + static_cast<int64_t>(r) * a.kv_row_stride;
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot = fmaf(qs[d], ld_f<T>(row + d), dot);
            l = dot * a.scale;
        } else {
            bad = 1;
        }
        lg[j] = l;
        m = fmaxf(m, l);
    }
    m = block_reduce(m, buf, true);
    float s = 0.f;
    for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
        const float p = (lg[j] == -INFINITY) ? 0.f : __expf(lg[j] - m);
        lg[j] = p;
        s += p;
    }
    s = block_reduce(s, buf, false);  // also orders the lg writes before the reads below
    if (bad && threadIdx.x == 0) report_status(a.status, DSA_ERR_INVALID);
    T *o = static_cast<T *>(lp.out) + (static_cast<int64_t>(i) * a.heads + h) * a.d_lat;
    for (int d = threadIdx.x; d < a.d_lat; d += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < cnt; ++j) {
            const int r = sel[j];
            if (lg[j] != 0.f) acc = fmaf(lg[j], ld_f<T>(kv + static_cast<int64_t>(r) * a.kv_row_stride + d), acc);
        }
        st_f<T>(o + d, cnt > 0 ? acc / s : 0.f);
    }
    if (threadIdx.x == 0 && lp.lse) lp.lse[static_cast<int64_t>(i) * a.heads + h] = cnt > 0 ? m + logf(s) : -INFINITY;
}

template <bool kFp8>
cudaError_t launch_mla_tc_t(const MlaArgs &a, const MlaMaps &maps, cudaStream_t st) {
    cudaError_t e = set_max_dynamic_smem(mla_tc_kernel<kFp8>, kMlaSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_splits, a.n_q, a.n_layers);
    return launch_pdl(mla_tc_kernel<kFp8>, grid, dim3(kMlaThreads), kMlaSmem, st, a, maps);
}

}  // namespace

int64_t mla_gather_rows(int64_t kv_seq_stride, int64_t kv_row_stride, int n_seq, int max_ctx) {
    if (kv_row_stride <= 0 || kv_seq_stride % kv_row_stride != 0) return -1;
    return static_cast<int64_t>(n_seq - 1) * (kv_seq_stride / kv_row_stride) + max_ctx;
}

bool encode_mla_maps(const MlaArgs &a, MlaMaps &maps) {
    EncodeTiledFn enc = tma_encode_fn();
    if (!enc) return false;
    const int64_t rows = mla_gather_rows(a.kv_seq_stride, a.kv_row_stride, a.n_seq, a.L);
    if (rows < 1 || rows > INT32_MAX || static_cast<int64_t>(a.n_q) * kMlaHeads > INT32_MAX) return false;
    const cuuint32_t es[2] = {1, 1};
    if (a.kv_fp8) {
        for (int l = 0; l < a.n_layers; ++l) {
            // packed rows as bytes {656, rows}: one-row boxes of 128 codes, unswizzled
            const cuuint64_t kd[2] = {static_cast<cuuint64_t>(kFp8Row), static_cast<cuuint64_t>(rows)};
            const cuuint64_t ks[1] = {static_cast<cuuint64_t>(a.kv_row_stride)};
            const cuuint32_t kb[2] = {128, 1};
            if (enc(&maps.kv[l], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(a.layer[l].kv), kd, ks, kb, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return false;
            // the same rows as bf16 {328, rows}: one-row boxes of the 64-value RoPE key
            const cuuint64_t rd[2] = {static_cast<cuuint64_t>(kFp8Row / 2), static_cast<cuuint64_t>(rows)};
            const cuuint32_t rb[2] = {64, 1};
            if (enc(&maps.kvr[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.layer[l].kv), rd, ks, rb,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return false;
        }
        return true;
    }
    for (int l = 0; l < a.n_layers; ++l) {
        // cache rows: {576 dims, rows}, one-row boxes of 64 dims (the gathers' unit)
        const cuuint64_t kd[2] = {static_cast<cuuint64_t>(kRow), static_cast<cuuint64_t>(rows)};
        const cuuint64_t ks[1] = {static_cast<cuuint64_t>(a.kv_row_stride) * 2};
        const cuuint32_t kb[2] = {64, 1};
        if (enc(&maps.kv[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.layer[l].kv), kd, ks, kb, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
        // queries: {576 dims, n_q * 64 heads}, boxes of 64 dims x 64 heads
        const cuuint64_t qd[2] = {static_cast<cuuint64_t>(kRow), static_cast<cuuint64_t>(a.n_q) * kMlaHeads};
        const cuuint64_t qs[1] = {static_cast<cuuint64_t>(kRow) * 2};
        const cuuint32_t qb[2] = {64, static_cast<cuuint32_t>(kMlaHeads)};
        if (enc(&maps.q[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.layer[l].q), qd, qs, qb, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

cudaError_t launch_mla_tc(const MlaArgs &a, const MlaMaps &maps, cudaStream_t st) {
    return a.kv_fp8 ? launch_mla_tc_t<true>(a, maps, st) : launch_mla_tc_t<false>(a, maps, st);
}

cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t st) {
    dim3 grid(kMlaHeads / kCombineHeads, a.n_q, a.n_layers);
    return launch_pdl(mla_combine_kernel, grid, dim3(256), 0, st, a);
}

cudaError_t launch_mla_generic(const MlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * (static_cast<size_t>(a.d_lat + a.d_rope) + a.topk);
    dim3 grid(a.n_q, a.heads, a.n_layers);
    if (a.is_bf16) {
        cudaError_t e = set_max_dynamic_smem(mla_generic_kernel<__nv_bfloat16>, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mla_generic_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(a);
    } else {
        cudaError_t e = set_max_dynamic_smem(mla_generic_kernel<float>, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mla_generic_kernel<float><<<grid, 128, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace dsa
