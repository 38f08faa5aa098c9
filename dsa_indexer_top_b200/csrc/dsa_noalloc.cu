// dsa_noalloc.cu -- dsa_sparse_mla_decode_noalloc: the split-K sparse MLA decode
// with its scratch in a fixed, file-scope device array instead of a
// caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// attention step: code running inside a captured or pre-planned execution whose
// memory was fixed up front, plugins and runtimes that hand a kernel only its
// input/output tensors, or hosts where cudaMalloc is not allowed on the serving
// path.  For them this entry point needs no workspace: its split-K partials
// live in g_mla_decode_scratch below, which every GPU that loads the library
// keeps until the process exits.
#include <mutex>

#include "dsa.h"
#include "kernels.cuh"

using namespace dsa;

namespace {

constexpr size_t kStatusBytes = 256;
// Size of the static scratch: status word + split-K partials.  32 MiB holds
// the partials of up to 15 queries at topk = 2048 (2,105,344 bytes per query).
constexpr size_t kNoallocScratchBytes = static_cast<size_t>(32) << 20;

__device__ __align__(256) uint8_t g_mla_decode_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  The host-side
// symbol is only a stand-in; the real address comes from cudaGetSymbolAddress,
// looked up once per device (with that device current) and cached.
dsa_status scratch_for_current_device(uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mla_decode_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<uint8_t *>(g_scratch_ptr[dev]);
    return DSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" dsa_status dsa_sparse_mla_decode_noalloc(const dsa_queries *queries, const dsa_mla *mla,
                                                    const int32_t *idx, const int32_t *cnt, int32_t topk,
                                                    void *stream) {
    if (!queries || queries->n_q < 0 || queries->n_seq < 1 || queries->max_ctx < 1) return DSA_ERR_INVALID;
    if (queries->n_q > 0 && (!queries->q_seq || !queries->q_pos)) return DSA_ERR_INVALID;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt || !mla) return DSA_ERR_INVALID;
    const dsa_mla &m = *mla;
    if (m.kv_dtype != 0 && m.kv_dtype != m.dtype && m.kv_dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID;
    const bool fp8 = m.kv_dtype == DSA_FP8_E4M3;  // packed rows, strides in bytes
    const int64_t min_row = fp8 ? int64_t(m.d_latent) + 2 * int64_t(m.d_rope) + 4 : int64_t(m.d_latent) + m.d_rope;
    if (!m.q || !m.kv || !m.out || m.kv_seq_stride < 0 || m.kv_row_stride < min_row) return DSA_ERR_INVALID;
    // Only the tensor-core shape uses scratch: bf16 queries, 64 heads, 512 + 64.
    const int64_t al = fp8 ? 16 : 8;
    if (m.dtype != DSA_BF16 || m.heads != kMlaHeads || m.d_latent != kLatent || m.d_rope != kRope ||
        !aligned16(m.q) || !aligned16(m.kv) || !aligned16(m.out) || m.kv_row_stride % al != 0 ||
        m.kv_seq_stride % al != 0 || (fp8 && m.kv_row_stride < kFp8Row))
        return DSA_ERR_UNSUPPORTED;
    const int n_splits = (topk + kRowsPerChunk - 1) / kRowsPerChunk;
    const size_t need = kStatusBytes + (n_splits > 1 ? mla_partial_bytes(1, queries->n_q, n_splits) : 0);
    if (need > kNoallocScratchBytes) return DSA_ERR_WORKSPACE;  // beyond the static scratch
    uint8_t *scratch = nullptr;
    dsa_status s = scratch_for_current_device(&scratch);
    if (s != DSA_OK) return s;
    if (queries->n_q == 0) return DSA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The status word must start at zero; the partials are fully rewritten.
    if (cudaMemsetAsync(scratch, 0, kStatusBytes, st) != cudaSuccess) return DSA_ERR_CUDA;

    MlaArgs a = {};
    a.layer[0].q = m.q;
    a.layer[0].kv = m.kv;
    a.layer[0].out = m.out;
    a.layer[0].lse = m.lse;
    a.n_layers = 1;
    a.kv_seq_stride = m.kv_seq_stride;
    a.kv_row_stride = m.kv_row_stride;
    a.q_seq = queries->q_seq;
    a.idx = idx;
    a.cnt = cnt;
    a.topk = topk;
    a.n_q = queries->n_q;
    a.n_seq = queries->n_seq;
    a.L = queries->max_ctx;
    a.heads = m.heads;
    a.d_lat = m.d_latent;
    a.d_rope = m.d_rope;
    a.scale = m.scale;
    a.is_bf16 = 1;
    a.kv_fp8 = fp8 ? 1 : 0;
    a.status = reinterpret_cast<uint32_t *>(scratch);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    int plan_splits, cpc;
    mla_plan(queries->n_q, 1, topk, true, sms, n_splits, plan_splits, cpc);  // at most the bound above
    a.n_splits = plan_splits;
    a.chunks_per_cta = cpc;
    if (plan_splits > 1) {
        a.part_o = reinterpret_cast<float *>(scratch + kStatusBytes);
        const size_t rows = static_cast<size_t>(queries->n_q) * plan_splits * kMlaHeads;
        a.part_ml = reinterpret_cast<float *>(scratch + kStatusBytes + rows * kLatent * sizeof(float));
        if (launch_mla_tc(a, st) != cudaSuccess) return DSA_ERR_CUDA;
        return launch_mla_combine(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
    }
    return launch_mla_tc(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
