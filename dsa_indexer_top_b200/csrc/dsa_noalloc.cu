// dsa_noalloc.cu -- dsa_sparse_mla_decode_noalloc: the split-K sparse MLA decode
// with its scratch in a fixed, file-scope device array instead of a
// caller-provided workspace, and dsa_noalloc_check_status, which reads that
// array's status word.
//
// Some callers cannot allocate device memory at the point where they run the
// attention step: code running inside a captured or pre-planned execution whose
// memory was fixed up front, plugins and runtimes that hand a kernel only its
// input/output tensors, or hosts where cudaMalloc is not allowed on the serving
// path.  For them this entry point needs no workspace: its status word and
// split-K partials live in g_mla_decode_scratch below, which every GPU that
// loads the library keeps until the process exits.
#include <cstring>
#include <mutex>

#include "abi_checks.cuh"
#include "dsa.h"
#include "kernels.cuh"

using namespace dsa;

namespace {

constexpr size_t kStatusBytes = 256;
// Size of the static scratch: status word + split-K partials.  The decode plan
// gives a query at most (SMs / queries) splits, so its partials stay below
// SMs x 131,584 bytes (about 19.5 MB on a 148-SM B200) whatever the batch.
constexpr size_t kNoallocScratchBytes = static_cast<size_t>(32) << 20;

__device__ __align__(256) uint8_t g_mla_decode_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device.  The host-side
// symbol is only a stand-in; the real address comes from cudaGetSymbolAddress
// with the device current.  It is looked up again on every call made outside
// stream capture (so a context re-created after a device reset gets its own
// address) and cached per device for calls made while `st` is capturing.
dsa_status scratch_for_current_device(cudaStream_t st, uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cap == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mla_decode_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<uint8_t *>(g_scratch_ptr[dev]);
    return DSA_OK;
}

int num_sms(int dev) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    return sms;
}

}  // namespace

extern "C" dsa_status dsa_sparse_mla_decode_noalloc(const dsa_queries *queries, const dsa_mla *mla,
                                                    const int32_t *idx, const int32_t *cnt, int32_t topk,
                                                    void *stream) {
    // the same checks as dsa_sparse_mla_decode (shared validators)
    if (!valid_queries(queries)) return DSA_ERR_INVALID;
    if (topk < 1 || topk > kMaxTopk || !idx || !cnt) return DSA_ERR_INVALID;
    const dsa_status chk = check_mla_layers(mla, 1);
    if (chk != DSA_OK) return chk;
    // Only the tensor-core shape uses scratch: bf16 queries, 64 heads, 512 + 64.
    if (!mla_tc_ok(mla) || !mla_tc_rows_ok(mla, queries->n_seq, queries->max_ctx)) return DSA_ERR_UNSUPPORTED;
    const dsa_mla &m = *mla;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
    // the split plan of this call (the one the launch uses) sizes the scratch
    int n_splits, cpc;
    mla_plan(queries->n_q, 1, topk, true, num_sms(dev), kMlaMaxSplits, n_splits, cpc);
    const size_t need = kStatusBytes + (n_splits > 1 ? mla_partial_bytes(1, queries->n_q, n_splits) : 0);
    if (need > kNoallocScratchBytes) return DSA_ERR_WORKSPACE;  // beyond the static scratch
    uint8_t *scratch = nullptr;
    dsa_status s = scratch_for_current_device(st, &scratch);
    if (s != DSA_OK) return s;
    if (queries->n_q == 0) return DSA_OK;
    // The status word starts at zero when the library loads and is cleared by
    // dsa_noalloc_check_status; the partials are fully rewritten by each call.

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
    a.kv_fp8 = mla_kv_fp8(&m) ? 1 : 0;
    a.sel_group = 1;
    a.status = reinterpret_cast<uint32_t *>(scratch);
    a.n_splits = n_splits;
    a.chunks_per_cta = cpc;
    MlaMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_mla_maps(a, maps)) return DSA_ERR_CUDA;
    if (n_splits > 1) {
        a.part_o = reinterpret_cast<float *>(scratch + kStatusBytes);
        const size_t rows = static_cast<size_t>(queries->n_q) * n_splits * kMlaHeads;
        a.part_ml = reinterpret_cast<float *>(scratch + kStatusBytes + rows * kLatent * sizeof(float));
        if (launch_mla_tc(a, maps, st) != cudaSuccess) return DSA_ERR_CUDA;
        return launch_mla_combine(a, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
    }
    return launch_mla_tc(a, maps, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

extern "C" dsa_status dsa_noalloc_check_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *scratch = nullptr;
    dsa_status s = scratch_for_current_device(st, &scratch);
    if (s != DSA_OK) return s;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (v != 0 && cudaMemsetAsync(scratch, 0, sizeof(v), st) != cudaSuccess) return DSA_ERR_CUDA;
    return static_cast<dsa_status>(v);
}
