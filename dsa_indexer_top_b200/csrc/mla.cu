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
// Tensor-core path (bf16, 64 heads, 512 + 64), one CTA of 8 warps per (query,
// split, layer), 128 selected rows per chunk:
//   gather   the chunk's 128 rows (1152 B each) are copied with 16-byte cp.async
//            into nine 64-column blocks of 128-byte-swizzled shared memory; the
//            query's 64 x 576 tile likewise, once per CTA.
//   S-MMA    S^T[128 rows][64 heads] = C (M = 128, K-major) x Q^T (N = 64,
//            K-major), K = 576: 36 tcgen05.mma, fp32 in TMEM columns 0..63.
//   softmax  warps 0-3 read one row each from TMEM; per-head maxima and sums
//            across the 128 rows by a shuffle transpose-reduction and a 4-warp
//            combine; P (bf16) is written into the freed RoPE block.
//   O-MMA    O^T[512 dims][64 heads] += C_lat^T (M = 4 x 128, MN-major view of
//            the same tile) x P^T (N = 64, K-major), K = 128 rows: 32 MMAs into
//            TMEM columns 64..319.  Several chunks per CTA use an online softmax
//            (O rescaled in TMEM when a head's maximum grows).
//   epilogue all 8 warps read O^T from TMEM; either the final bf16 output
//            (one CTA per query) or fp32 partials + (max, sum) for a split-K
//            merge (decode: several CTAs per query).
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kMlaThreads = 256;
constexpr int kQBlockBytes = kMlaHeads * 128;          // 64 heads x 64 dims bf16 = 8 KB
constexpr int kCBlockBytes = kRowsPerChunk * 128;      // 128 rows x 64 dims bf16 = 16 KB
constexpr int kBlocks = kRow / 64;                     // 9 column blocks (8 latent + rope)
constexpr int kQBytes = kBlocks * kQBlockBytes;        // 72 KB
constexpr int kCBytes = kBlocks * kCBlockBytes;        // 144 KB
constexpr int kMlaSmem = kQBytes + kCBytes + 1024;
constexpr int kTmemCols = 512;                          // S: 0..63, O: 64..319
constexpr uint32_t kIdescS = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescO = idesc_bf16(128, 64, true, true);
// A running maximum is kept until a head's chunk maximum exceeds it by more than
// this many powers of two (probabilities stay below 2^8, exact in bf16 range);
// only then is the accumulated O rescaled.
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Transpose-reduction inside a warp: on entry lane L holds v[0..63] (one value
// per head for its row); on exit v[0], v[1] hold the reduction over the warp's
// 32 rows for heads 2L and 2L+1.
template <bool kMax>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[64], int lane) {
#pragma unroll
    for (int o = 16, half = 32; o >= 1; o >>= 1, half >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float send = upper ? v[j] : v[j + half];
            const float keep = upper ? v[j + half] : v[j];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[j] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
}

__global__ void __launch_bounds__(kMlaThreads, 1) mla_tc_kernel(const MlaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *q_sm = smem;
    uint8_t *c_sm = smem + kQBytes;
    uint8_t *p_sm = c_sm + 8 * kCBlockBytes;  // P reuses the RoPE block after the S-MMA

    __shared__ uint64_t bar_s, bar_o;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int need_rescale;
    __shared__ int row_idx[kRowsPerChunk];
    __shared__ float red[4][kMlaHeads];
    __shared__ float m_run[kMlaHeads], l_run[kMlaHeads], alpha[kMlaHeads], inv_l[kMlaHeads];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, i = blockIdx.y, layer = blockIdx.z;
    const MlaLayerPtrs lp = a.layer[layer];
    const float c2 = a.scale * kLog2e;

    if (tid == 0) {
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        abort_flag = 0;
        need_rescale = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    if (tid < kMlaHeads) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.f;
        alpha[tid] = 1.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base_sh;

    int seq = a.q_seq[i];
    int cnt = a.cnt[i];
    bool ok = seq >= 0 && seq < a.n_seq && cnt >= 0 && cnt <= a.topk;
    if (!ok) {
        if (tid == 0) report_status(a.status, DSA_ERR_INVALID);
        cnt = 0;
        seq = 0;
    }
    const int nch = (cnt + kRowsPerChunk - 1) / kRowsPerChunk;
    const int c_begin = split * a.chunks_per_cta;
    const int c_end = min(c_begin + a.chunks_per_cta, nch);
    const __nv_bfloat16 *kv = static_cast<const __nv_bfloat16 *>(lp.kv) + static_cast<int64_t>(seq) * a.kv_seq_stride;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(lp.q) + static_cast<int64_t>(i) * kMlaHeads * kRow;
    const uint32_t q_addr = smem_u32(q_sm), c_addr = smem_u32(c_sm), p_addr = smem_u32(p_sm);

    // the query tile does not depend on the selection: start its copy first
    if (c_begin < c_end) {
        for (int f = tid; f < kMlaHeads * (kRow / 8); f += kMlaThreads) {
            const int h = f / (kRow / 8), ch = f % (kRow / 8);
            cp_async_16(q_addr + (ch >> 3) * kQBlockBytes + sw128_offset(h, ch & 7), q + h * kRow + ch * 8);
        }
        cp_async_commit();
    }
    // row index of selected slot j of this query (-1: none or out of range)
    auto load_idx = [&](int c) -> int {
        const int j = c * kRowsPerChunk + tid;
        int r = -1;
        if (j < cnt) {
            r = a.idx[static_cast<int64_t>(i) * a.topk + j];
            if (r < 0 || r >= a.L) {
                report_status(a.status, DSA_ERR_INVALID);
                r = -1;
            }
        }
        return r;
    };
    int pending = (tid < kRowsPerChunk && c_begin < c_end) ? load_idx(c_begin) : -1;

    int done = 0;  // chunks whose O-MMA was issued
    for (int c = c_begin; c < c_end; ++c, ++done) {
        const bool first = (c == c_begin);
        // ---- 1. row indices of this chunk (previous O-MMA must be done with C)
        if (!first && !mbar_wait(&bar_o, (done - 1) & 1, a.status, &abort_flag)) break;
        if (tid < kRowsPerChunk) row_idx[tid] = pending;
        __syncthreads();
        // the next chunk's indices load while this chunk is gathered and computed
        if (tid < kRowsPerChunk && c + 1 < c_end) pending = load_idx(c + 1);
        // ---- 2. gather the chunk's rows
        for (int f = tid; f < kRowsPerChunk * (kRow / 8); f += kMlaThreads) {
            const int r = f / (kRow / 8), ch = f % (kRow / 8);
            const uint32_t dst = c_addr + (ch >> 3) * kCBlockBytes + sw128_offset(r, ch & 7);
            const int src_row = row_idx[r];
            if (src_row >= 0) {
                cp_async_16(dst, kv + static_cast<int64_t>(src_row) * a.kv_row_stride + ch * 8);
            } else {
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
            }
        }
        cp_async_commit();
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncthreads();
        // ---- 3. S^T = C . Q^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kRow / 16; ++kk) {
                const uint32_t koff = (kk & 3) * 32;
                const uint64_t ad = sdesc_sw128(c_addr + (kk >> 2) * kCBlockBytes + koff, 16, 1024);
                const uint64_t bd = sdesc_sw128(q_addr + (kk >> 2) * kQBlockBytes + koff, 16, 1024);
                umma_bf16(tbase, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
            }
            umma_commit(&bar_s);
        }
        // ---- 4. softmax over the chunk's rows, per head
        const int row = warp * 32 + lane;  // warps 0-3: one selected row per thread
        const uint32_t s_taddr = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        if (warp < 4) {
            mbar_wait(&bar_s, done & 1, a.status, &abort_flag);  // on timeout the CTA aborts below
            tc_fence_after();
            float v[64];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(s_taddr, r0);
                tmem_ld32(s_taddr + 32, r1);
                tmem_ld_wait();
                const bool valid = row_idx[row] >= 0;
#pragma unroll
                for (int h = 0; h < 32; ++h) {
                    v[h] = valid ? u2f(r0[h]) : -INFINITY;
                    v[h + 32] = valid ? u2f(r1[h]) : -INFINITY;
                }
            }
            warp_transpose_reduce<true>(v, lane);
            red[warp][2 * lane] = v[0];
            red[warp][2 * lane + 1] = v[1];
        }
        __syncthreads();
        if (abort_flag) break;
        if (tid < kMlaHeads) {
            const float mc = fmaxf(fmaxf(red[0][tid], red[1][tid]), fmaxf(red[2][tid], red[3][tid]));
            const float m_old = m_run[tid];
            float al = 1.f;
            if (mc != -INFINITY && (m_old == -INFINITY || (mc - m_old) * c2 > kRescaleLog2)) {
                al = (m_old == -INFINITY) ? 0.f : exp2f((m_old - mc) * c2);
                m_run[tid] = mc;
                if (!first) need_rescale = 1;
            }
            alpha[tid] = al;
        }
        __syncthreads();
        if (warp < 4) {
            // P[row][head] (bf16, 128-byte swizzled rows: the MN-major B operand)
            uint32_t r0[32], r1[32];
            tmem_ld32(s_taddr, r0);
            tmem_ld32(s_taddr + 32, r1);
            tmem_ld_wait();
            const bool valid = row_idx[row] >= 0;
            float v[64];
#pragma unroll
            for (int h = 0; h < 64; ++h) {
                const float sv = u2f(h < 32 ? r0[h] : r1[h - 32]);
                const float m = m_run[h];
                const float pf = (!valid || m == -INFINITY) ? 0.f : exp2f((sv - m) * c2);
                v[h] = pf;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                __align__(16) __nv_bfloat16 pb[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    pb[x] = __float2bfloat16_rn(v[8 * j + x]);
                    v[8 * j + x] = __bfloat162float(pb[x]);  // the sum uses the value the MMA sees
                }
                *reinterpret_cast<uint4 *>(p_sm + sw128_offset(row, j)) = *reinterpret_cast<const uint4 *>(pb);
            }
            warp_transpose_reduce<false>(v, lane);
            red[warp][2 * lane] = v[0];
            red[warp][2 * lane + 1] = v[1];
            fence_proxy_async_smem();
        }
        __syncthreads();
        if (tid < kMlaHeads)
            l_run[tid] = l_run[tid] * alpha[tid] + (red[0][tid] + red[1][tid]) + (red[2][tid] + red[3][tid]);
        // ---- rescale the running O when a head's maximum grew
        if (need_rescale) {
            const int quad = warp & 3;
            const int mt0 = (warp < 4) ? 0 : 2;
            for (int mt = mt0; mt < mt0 + 2; ++mt) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t ta = tbase + (static_cast<uint32_t>(quad * 32) << 16) + 64 + mt * 64 + half * 32;
                    uint32_t r[32];
                    tmem_ld32(ta, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(u2f(r[x]) * alpha[half * 32 + x]);
                    tmem_st32(ta, r);
                }
            }
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) need_rescale = 0;
        // ---- 5. O^T += C_lat^T . P^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                for (int kk = 0; kk < kRowsPerChunk / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(c_addr + 2 * mt * kCBlockBytes + kk * 2048, kCBlockBytes, 1024);
                    const uint64_t bd = sdesc_sw128(p_addr + kk * 2048, kCBlockBytes, 1024);
                    umma_bf16(tbase + 64 + mt * 64, ad, bd, kIdescO, (!first || kk > 0) ? 1u : 0u);
                }
            }
            umma_commit(&bar_o);
        }
    }

    __syncthreads();  // every thread has left the loop: `go` is uniform
    const bool go = done > 0 && !abort_flag;
    if (go) {
        if (tid < kMlaHeads) inv_l[tid] = 1.f / l_run[tid];
        mbar_wait(&bar_o, (done - 1) & 1, a.status, &abort_flag);
        tc_fence_after();
        __syncthreads();
        const int quad = warp & 3;
        const int mt0 = (warp < 4) ? 0 : 2;
        const bool final_out = (a.n_splits == 1);
        for (int mt = mt0; mt < mt0 + 2; ++mt) {
            const int d = mt * 128 + quad * 32 + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tbase + (static_cast<uint32_t>(quad * 32) << 16) + 64 + mt * 64 + half * 32, r);
                tmem_ld_wait();
                if (final_out) {
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(lp.out) + static_cast<int64_t>(i) * kMlaHeads * kLatent;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int h = half * 32 + x;
                        o[h * kLatent + d] = __float2bfloat16_rn(u2f(r[x]) * inv_l[h]);
                    }
                } else {
                    float *po = a.part_o + ((static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits + split) * kMlaHeads * kLatent;
#pragma unroll
                    for (int x = 0; x < 32; ++x) po[(half * 32 + x) * kLatent + d] = u2f(r[x]);
                }
            }
        }
        if (tid < kMlaHeads) {
            if (final_out) {
                if (lp.lse) lp.lse[static_cast<int64_t>(i) * kMlaHeads + tid] = m_run[tid] * a.scale + logf(l_run[tid]);
            } else {
                float *ml = a.part_ml + (((static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits + split) * kMlaHeads + tid) * 2;
                ml[0] = m_run[tid] * c2;  // log2 units
                ml[1] = l_run[tid];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// Merge split-K partials: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// One CTA per (4 heads, query, layer).
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaArgs a) {
    const int hg = blockIdx.x, i = blockIdx.y, layer = blockIdx.z;
    const MlaLayerPtrs lp = a.layer[layer];
    __shared__ float wgt[4][kMaxTopk / kRowsPerChunk];
    int cnt = a.cnt[i];
    if (cnt < 0 || cnt > a.topk) cnt = 0;
    const int nch = (cnt + kRowsPerChunk - 1) / kRowsPerChunk;
    const int ns = (nch + a.chunks_per_cta - 1) / a.chunks_per_cta;
    const int64_t base = (static_cast<int64_t>(layer) * a.n_q + i) * a.n_splits;
    // (max, sum) of every split for the 4 heads: one thread per (head, split)
    {
        const int hl = threadIdx.x >> 5, s = threadIdx.x & 31;  // warps 0-3: one head each
        if (hl < 4) {
            const int h = hg * 4 + hl;
            float m = -INFINITY, l = 0.f;
            if (s < ns) {
                const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + ((base + s) * kMlaHeads + h) * 2);
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
            if (s < ns) wgt[hl][s] = wv / L;
            if (s == 0 && lp.lse) lp.lse[static_cast<int64_t>(i) * kMlaHeads + h] = (M + log2f(L)) * kLn2;
        }
    }
    __syncthreads();
    // 4 heads x 512 dims = 2048 outputs, 8 per thread
    const int e = threadIdx.x * 8;
    const int hl = e / kLatent, d = e % kLatent;
    const int h = hg * 4 + hl;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 8
    for (int s = 0; s < ns; ++s) {
        const float *po = a.part_o + ((base + s) * kMlaHeads + h) * kLatent + d;
        const float4 x0 = *reinterpret_cast<const float4 *>(po);
        const float4 x1 = *reinterpret_cast<const float4 *>(po + 4);
        const float wv = wgt[hl][s];
        acc[0] += wv * x0.x; acc[1] += wv * x0.y; acc[2] += wv * x0.z; acc[3] += wv * x0.w;
        acc[4] += wv * x1.x; acc[5] += wv * x1.y; acc[6] += wv * x1.z; acc[7] += wv * x1.w;
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(lp.out) + (static_cast<int64_t>(i) * kMlaHeads + h) * kLatent + d;
    __align__(16) __nv_bfloat16 ob[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) ob[x] = __float2bfloat16_rn(acc[x]);
    *reinterpret_cast<uint4 *>(o) = *reinterpret_cast<const uint4 *>(ob);
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
    int cnt = a.cnt[i];
    if (seq < 0 || seq >= a.n_seq || cnt < 0 || cnt > a.topk) {
        if (threadIdx.x == 0 && h == 0) report_status(a.status, DSA_ERR_INVALID);
        seq = 0;
        cnt = 0;
    }
    __syncthreads();
    const T *kv = static_cast<const T *>(lp.kv) + static_cast<int64_t>(seq) * a.kv_seq_stride;
    const int32_t *sel = a.idx + static_cast<int64_t>(i) * a.topk;
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

}  // namespace

cudaError_t launch_mla_tc(const MlaArgs &a, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMlaSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_splits, a.n_q, a.n_layers);
    mla_tc_kernel<<<grid, kMlaThreads, kMlaSmem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t st) {
    dim3 grid(kMlaHeads / 4, a.n_q, a.n_layers);
    mla_combine_kernel<<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_mla_generic(const MlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * (static_cast<size_t>(a.d_lat + a.d_rope) + a.topk);
    dim3 grid(a.n_q, a.heads, a.n_layers);
    if (a.is_bf16) {
        cudaError_t e = cudaFuncSetAttribute(mla_generic_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mla_generic_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(mla_generic_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mla_generic_kernel<float><<<grid, 128, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace dsa
