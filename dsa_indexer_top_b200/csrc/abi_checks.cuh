// abi_checks.cuh -- host-side argument checks shared by the entry points of the
// C ABI (dsa_abi.cu, dsa_noalloc.cu), so that every entry point accepts exactly
// the same inputs.  Internal; not part of the public header.
#pragma once

#include <climits>
#include <cstdint>

#include "dsa.h"
#include "kernels.cuh"

namespace dsa {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_queries(const dsa_queries *qs) {
    if (!qs) return false;
    if (qs->n_q < 0 || qs->n_seq < 1 || qs->max_ctx < 1 || qs->seq_run < 1) return false;
    if (qs->n_q > 0 && (!qs->q_seq || !qs->q_pos)) return false;
    return true;
}

inline bool mla_kv_fp8(const dsa_mla *m) { return m->kv_dtype == DSA_FP8_E4M3; }

// The tensor-core MLA shape: bf16 queries/outputs, 64 heads, 512 + 64, aligned
// bases and strides (bf16 cache: strides in elements, multiples of 8; packed FP8
// rows: strides in bytes, multiples of 16).
inline bool mla_tc_ok(const dsa_mla *m) {
    const bool shape = m->dtype == DSA_BF16 && m->heads == kMlaHeads && m->d_latent == kLatent &&
                       m->d_rope == kRope && aligned16(m->q) && aligned16(m->kv) && aligned16(m->out);
    if (mla_kv_fp8(m))
        return shape && m->kv_row_stride % 16 == 0 && m->kv_seq_stride % 16 == 0 && m->kv_row_stride >= kFp8Row;
    return shape && m->kv_row_stride % 8 == 0 && m->kv_seq_stride % 8 == 0 && m->kv_row_stride >= kRow;
}

// Caches on the tensor-core path are read by TMA row gathers over one 2-D tensor
// of every sequence's rows: the sequence stride a whole number of rows (or 0)
// and at most INT32_MAX rows in all.
inline bool mla_tc_rows_ok(const dsa_mla *m, int n_seq, int max_ctx) {
    const int64_t rows = mla_gather_rows(m->kv_seq_stride, m->kv_row_stride, n_seq, max_ctx);
    return rows >= 1 && rows <= INT32_MAX;
}

// Every layer described and consistent with layer 0 (one shape, dtype, scale,
// stride and cache format for the whole call).
inline dsa_status check_mla_layers(const dsa_mla *layers, int n_layers) {
    if (!layers || n_layers < 1 || n_layers > kMaxLayers) return DSA_ERR_INVALID;
    const dsa_mla &m0 = layers[0];
    for (int l = 0; l < n_layers; ++l) {
        const dsa_mla &m = layers[l];
        if (!m.q || !m.kv || !m.out) return DSA_ERR_INVALID;
        if (m.heads < 1 || m.d_latent < 1 || m.d_rope < 0 || (m.dtype != DSA_BF16 && m.dtype != DSA_F32))
            return DSA_ERR_INVALID;
        if (m.kv_dtype != 0 && m.kv_dtype != m.dtype && m.kv_dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID;
        // a packed FP8 row holds d_latent codes, d_rope bf16 values and a float32 scale
        const int64_t min_row = mla_kv_fp8(&m) ? int64_t(m.d_latent) + 2 * int64_t(m.d_rope) + 4
                                               : int64_t(m.d_latent) + m.d_rope;
        if (m.kv_row_stride < min_row || m.kv_seq_stride < 0) return DSA_ERR_INVALID;
        if (m.heads != m0.heads || m.d_latent != m0.d_latent || m.d_rope != m0.d_rope || m.dtype != m0.dtype ||
            m.scale != m0.scale || m.kv_row_stride != m0.kv_row_stride || m.kv_seq_stride != m0.kv_seq_stride ||
            mla_kv_fp8(&m) != mla_kv_fp8(&m0))
            return DSA_ERR_INVALID;
    }
    return DSA_OK;
}

}  // namespace dsa
