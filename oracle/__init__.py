"""fp64 CPU oracle for the GLM-5.2 DeepSeek-Sparse-Attention hot path.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's
CPU-baseline / reference leg are the only callers.  The product library never
imports this package, and this package imports nothing from the product.

The arithmetic lives in ``dsa_oracle.c`` (plain C, double precision); this module
only compiles it with gcc and marshals numpy arrays in and out.  Inputs are passed
as float32 (bf16 values widen to float32 exactly); outputs are float64.

Functions and the passages they follow (page title, section):
  index_scores     -- "GLM-5.2 -- Model techniques map", "Checked in its code",
                      Indexer-selected sparse attention; one key per token.
  topk             -- same row: min(index_topk, n) largest scores, int32 indices.
  sparse_mla       -- same page, rows Multi-head latent attention / Learnable
                      attention sink / Partial RoPE (absorbed form, plain softmax).
  sparse_mla_fp8   -- sparse_mla over a cache with 8-bit (E4M3) latents and one
                      float32 scale per row ("GLM-5.2 -- Model techniques map",
                      inference quantization: FP8 inference; row format read
                      here, the pages give none).
  dense_mla        -- textbook causal attention (the topk >= n special case).
  indexshare_group -- "GLM 5.2 -- Hermosa AI", "MLA + DSA with IndexShare".
  sparse_mla_mtp   -- "GLM-5.2 -- LLM atlas", raw config.json fields
                      (index_share_for_mtp_iteration): the queries of one MTP
                      iteration share one selection.
Every function is pinned by tests in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    i64 = ctypes.c_int64
    ci = ctypes.c_int
    lib.oracle_max_threads.restype = ci
    lib.oracle_index_scores.argtypes = [ci, ci, ci, _f32p, _f32p, _f32p, i64, i64, _i32p, _i32p, ci, _f64p]
    lib.oracle_topk.argtypes = [ci, ci, _f64p, _i32p, ci, _i32p, _i32p]
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_index_scores_e4m3.argtypes = [ci, ci, ci, _u8p, ctypes.c_void_p, _f32p, _u8p, ctypes.c_void_p, i64,
                                             i64, i64, _i32p, _i32p, ci, _f64p]
    lib.oracle_sparse_mla.argtypes = [ci, ci, ci, ci, ctypes.c_double, _f32p, _f32p, i64, i64,
                                      _i32p, _i32p, _i32p, ci, _f64p, ctypes.c_void_p]
    lib.oracle_dense_mla.argtypes = [ci, ci, ci, ci, ctypes.c_double, _f32p, _f32p, i64, i64,
                                     _i32p, _i32p, _f64p, ctypes.c_void_p]
    lib.oracle_sparse_mla_fp8.argtypes = [ci, ci, ci, ci, ctypes.c_double, _f32p, _u8p, i64, i64,
                                          _i32p, _i32p, _i32p, ci, _f64p, ctypes.c_void_p]
    _lib = lib
    return lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def index_scores(q, w, k, q_seq, q_pos):
    """q [n_q,H,D], w [n_q,H], k [n_seq,L,D] -> scores [n_q,L] (NaN where s > q_pos)."""
    q, w, k = _f32(q), _f32(w), _f32(k)
    q_seq, q_pos = _i32(q_seq), _i32(q_pos)
    n_q, heads, dim = q.shape
    n_seq, L, kd = k.shape
    assert kd == dim and w.shape == (n_q, heads)
    assert np.all((q_pos >= 0) & (q_pos < L)) and np.all((q_seq >= 0) & (q_seq < n_seq))
    out = np.empty((n_q, L), dtype=np.float64)
    _load().oracle_index_scores(n_q, heads, dim, q, w, k, L * dim, dim, q_seq, q_pos, L, out)
    return out


def e4m3_to_double(code: int) -> float:
    """Value of one E4M3 code (0..255), decoded from the format definition."""
    return float(_load().oracle_e4m3_to_double(int(code) & 0xFF))


def index_scores_e4m3(q8, q_scale, w, k8, k_scale, q_seq, q_pos):
    """FP8 variant: q8 [n_q,H,D] and k8 [n_seq,L,D] uint8 E4M3 codes, q_scale [n_q,H]
    and k_scale [n_seq,L] float32 (or None = 1), w [n_q,H] -> scores [n_q,L] (NaN where
    s > q_pos), on the exact operands e4m3(code) * scale."""
    q8 = np.ascontiguousarray(np.asarray(q8, dtype=np.uint8))
    k8 = np.ascontiguousarray(np.asarray(k8, dtype=np.uint8))
    w = _f32(w)
    q_seq, q_pos = _i32(q_seq), _i32(q_pos)
    n_q, heads, dim = q8.shape
    n_seq, L, kd = k8.shape
    assert kd == dim and w.shape == (n_q, heads)
    assert np.all((q_pos >= 0) & (q_pos < L)) and np.all((q_seq >= 0) & (q_seq < n_seq))
    qs = None if q_scale is None else _f32(q_scale)
    ks = None if k_scale is None else _f32(k_scale)
    if qs is not None:
        assert qs.shape == (n_q, heads)
    if ks is not None:
        assert ks.shape == (n_seq, L)
    out = np.empty((n_q, L), dtype=np.float64)
    _load().oracle_index_scores_e4m3(n_q, heads, dim, q8, None if qs is None else qs.ctypes.data, w, k8,
                                     None if ks is None else ks.ctypes.data, L * dim, dim, L, q_seq, q_pos, L, out)
    return out


def topk(scores, q_pos, k):
    """scores [n_q,L] -> (idx [n_q,k] int32 ascending, -1 padded; cnt [n_q] int32)."""
    scores = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    q_pos = _i32(q_pos)
    n_q, L = scores.shape
    assert np.all((q_pos >= 0) & (q_pos < L))
    idx = np.empty((n_q, k), dtype=np.int32)
    cnt = np.empty((n_q,), dtype=np.int32)
    _load().oracle_topk(n_q, L, scores, q_pos, int(k), idx, cnt)
    return idx, cnt


def sparse_mla(q, kv, q_seq, idx, cnt, d_lat, scale):
    """q [n_q,H,d_lat+d_rope], kv [n_seq,L,d_lat+d_rope], idx [n_q,topk], cnt [n_q]
    -> (out [n_q,H,d_lat] float64, lse [n_q,H] float64)."""
    q, kv = _f32(q), _f32(kv)
    q_seq, idx, cnt = _i32(q_seq), _i32(idx), _i32(cnt)
    n_q, heads, dk = q.shape
    n_seq, L, kvd = kv.shape
    assert kvd == dk and 0 < d_lat <= dk
    topk_ = idx.shape[1]
    for i in range(n_q):
        sel = idx[i, : cnt[i]]
        assert np.all((sel >= 0) & (sel < L)), "selected index out of range"
    out = np.empty((n_q, heads, d_lat), dtype=np.float64)
    lse = np.empty((n_q, heads), dtype=np.float64)
    _load().oracle_sparse_mla(n_q, heads, d_lat, dk - d_lat, float(scale), q, kv, L * dk, dk,
                              q_seq, idx, cnt, topk_, out, lse.ctypes.data)
    return out, lse


def sparse_mla_fp8(q, kv8, q_seq, idx, cnt, d_lat, d_rope, scale):
    """FP8 latent cache: q [n_q,H,d_lat+d_rope] float, kv8 [n_seq,L,row_bytes] uint8
    rows [E4M3 latent codes (d_lat) | bf16 RoPE key (2*d_rope bytes) | float32 scale |
    padding], idx [n_q,topk], cnt [n_q] -> (out [n_q,H,d_lat], lse [n_q,H]) float64,
    attending over c = scale_row * e4m3(code)."""
    q = _f32(q)
    kv8 = np.ascontiguousarray(np.asarray(kv8, dtype=np.uint8))
    q_seq, idx, cnt = _i32(q_seq), _i32(idx), _i32(cnt)
    n_q, heads, dk = q.shape
    n_seq, L, row_bytes = kv8.shape
    assert dk == d_lat + d_rope and row_bytes >= d_lat + 2 * d_rope + 4 and d_lat % 4 == 0
    topk_ = idx.shape[1]
    for i in range(n_q):
        sel = idx[i, : cnt[i]]
        assert np.all((sel >= 0) & (sel < L)), "selected index out of range"
    out = np.empty((n_q, heads, d_lat), dtype=np.float64)
    lse = np.empty((n_q, heads), dtype=np.float64)
    _load().oracle_sparse_mla_fp8(n_q, heads, d_lat, d_rope, float(scale), q, kv8, L * row_bytes, row_bytes,
                                  q_seq, idx, cnt, topk_, out, lse.ctypes.data)
    return out, lse


def dense_mla(q, kv, q_seq, q_pos, d_lat, scale):
    """Causal attention over every s <= q_pos -> (out [n_q,H,d_lat], lse [n_q,H])."""
    q, kv = _f32(q), _f32(kv)
    q_seq, q_pos = _i32(q_seq), _i32(q_pos)
    n_q, heads, dk = q.shape
    n_seq, L, kvd = kv.shape
    assert kvd == dk and np.all(q_pos < L)
    out = np.empty((n_q, heads, d_lat), dtype=np.float64)
    lse = np.empty((n_q, heads), dtype=np.float64)
    _load().oracle_dense_mla(n_q, heads, d_lat, dk - d_lat, float(scale), q, kv, L * dk, dk,
                             q_seq, q_pos, out, lse.ctypes.data)
    return out, lse


def indexshare_group(q_idx, w, k_idx, q_seq, q_pos, topk_, q_mla_layers, kv_layers, d_lat, scale):
    """Layer 0 selects (scores -> top-k); every layer attends with that selection.

    Returns (idx, cnt, [out_l], [lse_l]).  Composed from the functions above in
    the order the IndexShare passage gives: select once, reuse for later layers.
    """
    scores = index_scores(q_idx, w, k_idx, q_seq, q_pos)
    idx, cnt = topk(scores, q_pos, topk_)
    outs, lses = [], []
    for q_l, kv_l in zip(q_mla_layers, kv_layers):
        o, l = sparse_mla(q_l, kv_l, q_seq, idx, cnt, d_lat, scale)
        outs.append(o)
        lses.append(l)
    return idx, cnt, outs, lses


def sparse_mla_mtp(q, kv, q_seq, idx_g, cnt_g, draft_tokens, d_lat, scale):
    """Queries in groups of `draft_tokens` consecutive queries; every query of
    group g attends over selection row g (idx_g [n_q / D, topk], cnt_g [n_q / D]).
    Composed from sparse_mla with the group's selection repeated per query
    ("GLM-5.2 -- LLM atlas", raw config.json fields: index_share_for_mtp_iteration
    -- the tokens of an MTP iteration share the index selection)."""
    idx_g, cnt_g = _i32(idx_g), _i32(cnt_g)
    assert np.asarray(q).shape[0] == idx_g.shape[0] * draft_tokens
    return sparse_mla(q, kv, q_seq, np.repeat(idx_g, draft_tokens, axis=0), np.repeat(cnt_g, draft_tokens),
                      d_lat, scale)
