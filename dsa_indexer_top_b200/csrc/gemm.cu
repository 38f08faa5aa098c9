// gemm.cu -- the dense contractions upstream and downstream of the attention
// path ("GLM-5.2 -- Model techniques map", "Checked in its code": Multi-head
// latent attention -- kv_a_proj_with_mqa, the per-head kv_b_proj halves W_UK /
// W_UV of the absorbed form; QK normalization -- the indexer key projection wk):
//   C[b][m][n] = sum_k A[b][m][k] * B[b][n][k]      (bf16 operands, fp32 sums)
// with both operands K-major, i.e. B in the [out][in] layout of a linear layer's
// weight.  A tcgen05 kernel: one CTA per (128 x BN output tile, K split, batch);
//   warp 0      TMA producer: 128 x 64 tiles of A and BN x 64 tiles of B
//               (128-byte swizzle) into a ring of shared-memory stages;
//   warp 1      MMA issuer: tcgen05.mma kind::f16, M = 128, N = BN, K = 16 steps,
//               fp32 accumulator in TMEM;
//   warps 2-5   epilogue: tcgen05.ld of one TMEM lane quadrant each (one output
//               row per thread), fp32 or bf16 rows stored as 16-byte pieces
//               (output rows and batch strides are multiples of 16 bytes).
// Split-K (grid y) writes fp32 partials that a consumer sums in a fixed order.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 192;

template <int BN>
struct GemmCfg {
    static constexpr int kATile = kGemmBM * kGemmBK * 2;  // 16 KB
    static constexpr int kBTile = BN * kGemmBK * 2;
    static constexpr int kStage = kATile + kBTile;
    static constexpr int kSmem = kGemmStages * kStage + 1024;
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    static constexpr uint32_t kIdesc = idesc_bf16(kGemmBM, BN, false, false);
};

template <int BN>
__global__ void __launch_bounds__(kGemmThreads) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a,
                                                               const __grid_constant__ CUtensorMap tmap_b,
                                                               const GemmArgs g) {
    using Cfg = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full_bar[kGemmStages], empty_bar[kGemmStages], acc_full;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = blockIdx.x, mt = blockIdx.y % g.m_tiles, split = blockIdx.y / g.m_tiles, b = blockIdx.z;
    const int kb_total = (g.K + kGemmBK - 1) / kGemmBK;
    const int kb0 = split * g.kb_per_split;
    const int nkb = max(0, min(kb0 + g.kb_per_split, kb_total) - kb0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_full, 1);
        abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base_sh;
    griddep_wait();

    if (warp == 0) {
        if (lane == 0) {
            int last_use[kGemmStages];
            for (int s = 0; s < kGemmStages; ++s) last_use[s] = -1;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kGemmStages, use = kb / kGemmStages;
                if (!mbar_wait(&empty_bar[s], (use & 1) ^ 1, g.status, &abort_flag)) break;
                uint8_t *dst = smem + s * Cfg::kStage;
                mbar_arrive_expect_tx(&full_bar[s], Cfg::kStage);
                const int kx = (kb0 + kb) * kGemmBK;
                if (g.a_batch_inner)
                    tma_load_3d(dst, &tmap_a, &full_bar[s], kx, b, mt * kGemmBM);
                else
                    tma_load_3d(dst, &tmap_a, &full_bar[s], kx, mt * kGemmBM, b);
                if (g.b_batch_inner)
                    tma_load_3d(dst + Cfg::kATile, &tmap_b, &full_bar[s], kx, b, nt * BN);
                else
                    tma_load_3d(dst + Cfg::kATile, &tmap_b, &full_bar[s], kx, nt * BN, b);
                last_use[s] = use;
            }
            // every copy this thread issued has landed before the CTA moves on
            for (int s = 0; s < kGemmStages; ++s)
                if (last_use[s] >= 0) mbar_wait(&full_bar[s], last_use[s] & 1, g.status, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kGemmStages, use = kb / kGemmStages;
                if (!mbar_wait(&full_bar[s], use & 1, g.status, &abort_flag)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * Cfg::kStage);
                const uint64_t adesc = sdesc_sw128(a_addr, 16, 1024);
                const uint64_t bdesc = sdesc_sw128(a_addr + Cfg::kATile, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 16; ++kk)  // 32 bytes of each 128-byte row per step
                    umma_bf16(tbase, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2),
                              Cfg::kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&empty_bar[s]);
            }
            umma_commit(&acc_full);  // also when no MMA ran (nkb == 0): the epilogue writes zeros
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31, one output row each
        const int quad = warp & 3;
        const int m = mt * kGemmBM + quad * 32 + lane;
        const bool have = nkb > 0;
        if (mbar_wait(&acc_full, 0, g.status, &abort_flag)) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tbase + (static_cast<uint32_t>(quad * 32) << 16) + c0, r);
                tmem_ld_wait();
                const int n0 = nt * BN + c0;
                if (m >= g.M || n0 >= g.N) continue;
                if (!have) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = 0u;
                }
                const bool full = n0 + 32 <= g.N;  // the row's 32 columns as 16-byte stores
                if (g.out_f32) {
                    float *o = g.out_f32 + split * g.s_split + b * g.s_batch + static_cast<int64_t>(m) * g.ldc + n0;
                    if (full) {
#pragma unroll
                        for (int x = 0; x < 32; x += 4)
                            *reinterpret_cast<uint4 *>(o + x) = make_uint4(r[x], r[x + 1], r[x + 2], r[x + 3]);
                    } else {
                        for (int x = 0; x < 32; ++x)
                            if (n0 + x < g.N) o[x] = u2f(r[x]);
                    }
                } else {
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(g.out_bf16) + b * g.s_batch +
                                       static_cast<int64_t>(m) * g.ldc + n0;
                    if (full) {
#pragma unroll
                        for (int x = 0; x < 32; x += 8) {
                            uint32_t pk[4];
#pragma unroll
                            for (int y = 0; y < 4; ++y) {
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(u2f(r[x + 2 * y]), u2f(r[x + 2 * y + 1]));
                                pk[y] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                            *reinterpret_cast<uint4 *>(o + x) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    } else {
                        for (int x = 0; x < 32; ++x)
                            if (n0 + x < g.N) o[x] = __float2bfloat16_rn(u2f(r[x]));
                    }
                }
            }
        }
    }
    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, Cfg::kTmemCols);
    }
}

// ---------------------------------------------------------------- few rows of A
// The same contraction when A has at most kSkinnyM rows (decode-sized batches):
// B (the weights) is streamed once with 16-byte loads, A's rows sit in shared
// memory.  Each warp takes WR rows of B and keeps two 16-byte loads of each in
// flight, its lanes splitting K in 8-element pieces; a row's M partial sums are
// reduced across the warp and written like the tensor-core kernel's output
// (fp32 split-K partials or bf16).  One CTA per (8 * WR rows of B, K split,
// batch).  HBM-bound on B.  Two shapes, both 4 rows of B per warp: up to 4 rows
// of A in at most 85 registers, so three CTAs share an SM and more loads are in
// flight per SM; up to 16 rows of A at one CTA per SM.
constexpr int kSkinnyM = 16;
constexpr int kSkinnyThreads = 256;
template <int MM, int WR>
struct SkinnyCfg {
    static constexpr int kRows = WR * (kSkinnyThreads / 32);  // rows of B per CTA
};

template <int MM, int WR>
__global__ void __launch_bounds__(kSkinnyThreads, MM <= 4 ? 3 : 1) gemm_skinny_kernel(const GemmSkinnyArgs g) {
    extern __shared__ __align__(16) uint8_t sm_raw[];
    __nv_bfloat16 *a_sm = reinterpret_cast<__nv_bfloat16 *>(sm_raw);  // [M][kc]
    const int nb = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = split * g.k_per_split;
    const int kc = min(g.k_per_split, g.K - k0);  // a multiple of 8
    griddep_wait();
    // A rows [M][k0, k0 + kc) into shared memory, 16 bytes at a time
    const int pieces = kc / 8;
    for (int e = threadIdx.x; e < g.M * pieces; e += kSkinnyThreads) {
        const int m = e / pieces, pc = e % pieces;
        const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(g.a) + b * g.a_batch + static_cast<int64_t>(m) * g.a_row +
                                   k0 + pc * 8;
        *reinterpret_cast<uint4 *>(a_sm + m * kc + pc * 8) = __ldg(reinterpret_cast<const uint4 *>(src));
    }
    __syncthreads();
    const int n0 = nb * SkinnyCfg<MM, WR>::kRows + warp * WR;
    if (n0 < g.N) {
        const int nr = min(WR, g.N - n0);
        const __nv_bfloat16 *bbase = static_cast<const __nv_bfloat16 *>(g.b) + b * g.b_batch + static_cast<int64_t>(n0) * g.b_row + k0;
        float acc[WR][MM];
#pragma unroll
        for (int r = 0; r < WR; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[r][m] = 0.f;
#pragma unroll 2
        for (int pc = lane; pc < pieces; pc += 32) {
            uint4 wv[WR];
#pragma unroll
            for (int r = 0; r < WR; ++r)
                wv[r] = r < nr ? __ldg(reinterpret_cast<const uint4 *>(bbase + r * g.b_row + pc * 8)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                if (m >= g.M) break;
                const uint4 av = *reinterpret_cast<const uint4 *>(a_sm + m * kc + pc * 8);
                const uint32_t a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a4[y]));
#pragma unroll
                    for (int r = 0; r < WR; ++r) {
                        const uint32_t w4[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
                        const float2 wf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[y]));
                        acc[r][m] = fmaf(wf.x, af.x, acc[r][m]);
                        acc[r][m] = fmaf(wf.y, af.y, acc[r][m]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < WR; ++r) {
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                if (m >= g.M) break;
                float v = acc[r][m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && r < nr) {
                    const int n = n0 + r;
                    if (g.out_f32)
                        g.out_f32[split * g.s_split + b * g.s_batch + static_cast<int64_t>(m) * g.ldc + n] = v;
                    else
                        static_cast<__nv_bfloat16 *>(g.out_bf16)[b * g.s_batch + static_cast<int64_t>(m) * g.ldc + n] =
                            __float2bfloat16_rn(v);
                }
            }
        }
    }
    griddep_launch_dependents();
}

template <int BN>
cudaError_t launch_gemm_bn(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &g, cudaStream_t st) {
    using Cfg = GemmCfg<BN>;
    cudaError_t e = set_max_dynamic_smem(gemm_tc_kernel<BN>, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    const int n_tiles = (g.N + BN - 1) / BN;
    dim3 grid(n_tiles, g.m_tiles * g.k_splits, g.batch);
    return launch_pdl(gemm_tc_kernel<BN>, grid, dim3(kGemmThreads), Cfg::kSmem, st, ta, tb, g);
}


template <int MM, int WR>
cudaError_t launch_skinny_cfg(const GemmSkinnyArgs &g, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(g.M) * g.k_per_split * 2;
    cudaError_t e = set_max_dynamic_smem(gemm_skinny_kernel<MM, WR>, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int k_splits = (g.K + g.k_per_split - 1) / g.k_per_split;
    constexpr int rows = SkinnyCfg<MM, WR>::kRows;
    dim3 grid((g.N + rows - 1) / rows, k_splits, g.batch);
    return launch_pdl(gemm_skinny_kernel<MM, WR>, grid, dim3(kSkinnyThreads), smem, st, g);
}

}  // namespace

cudaError_t launch_gemm_skinny(const GemmSkinnyArgs &g, cudaStream_t st) {
    if (g.M < 1 || g.M > kSkinnyM) return cudaErrorInvalidValue;
    return g.M <= 4 ? launch_skinny_cfg<4, 4>(g, st) : launch_skinny_cfg<16, 4>(g, st);
}

int skinny_rows_per_cta(int M) { return M <= 4 ? SkinnyCfg<4, 4>::kRows : SkinnyCfg<16, 4>::kRows; }

cudaError_t launch_gemm_tc(int bn, const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &g, cudaStream_t st) {
    switch (bn) {
        case 64: return launch_gemm_bn<64>(ta, tb, g, st);
        case 128: return launch_gemm_bn<128>(ta, tb, g, st);
        case 256: return launch_gemm_bn<256>(ta, tb, g, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dsa
