"""ctypes binding of libdsa.so (include/dsa.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing
but turn torch tensors into plain pointers and sizes, call the library on the
current CUDA stream, and raise DsaError on a non-OK status.  All arithmetic runs
in the library's CUDA kernels; there is no other code path.  If libdsa.so is
missing the first call raises (build it with `python -m dsa_indexer_top_b200.build`).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT = range(6)
DSA_BF16, DSA_F32, DSA_FP8_E4M3 = 0, 1, 2
DSA_OP_INDEX_SCORES, DSA_OP_TOPK, DSA_OP_MLA_DECODE, DSA_OP_MLA_PREFILL, DSA_OP_INDEXSHARE_GROUP, DSA_OP_SHARD_MERGE = range(6)
DSA_INDEXER_TOPK_HIST = 1
DSA_MLA_FP8_ROW_BYTES = 656
DSA_TOPK_HIST_FROM_INDEXER = 1


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} ({status})")


class _Queries(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int32), ("n_seq", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("seq_run", ctypes.c_int32), ("q_seq", ctypes.c_void_p), ("q_pos", ctypes.c_void_p)]


class _Indexer(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("q", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("k_seq_stride", ctypes.c_int64), ("k_row_stride", ctypes.c_int64),
                ("q_scale", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("ks_seq_stride", ctypes.c_int64)]


class _CacheWriter(ctypes.Structure):
    _fields_ = [("n_tok", ctypes.c_int32), ("hidden", ctypes.c_int32), ("h", ctypes.c_void_p),
                ("h_row_stride", ctypes.c_int64), ("w", ctypes.c_void_p), ("rms_weight", ctypes.c_void_p),
                ("ln_weight", ctypes.c_void_p), ("ln_bias", ctypes.c_void_p), ("tok_seq", ctypes.c_void_p),
                ("tok_pos", ctypes.c_void_p), ("n_seq", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("kv", ctypes.c_void_p), ("kv_seq_stride", ctypes.c_int64), ("kv_row_stride", ctypes.c_int64),
                ("k_idx", ctypes.c_void_p), ("k_seq_stride", ctypes.c_int64), ("k_row_stride", ctypes.c_int64),
                ("eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


class _Mla(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("scale", ctypes.c_float), ("kv_dtype", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p), ("kv_seq_stride", ctypes.c_int64),
                ("kv_row_stride", ctypes.c_int64), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


_lib_handle = None


def lib():
    """Load libdsa.so once (raises OSError when it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with `python -m dsa_indexer_top_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        st = ctypes.c_int
        h.dsa_index_scores.argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Indexer), P, I64, P, SZ, P]
        h.dsa_topk.argtypes = [ctypes.POINTER(_Queries), P, I64, I32, I32, P, P, P, SZ, P]
        for name in ("dsa_sparse_mla_decode", "dsa_sparse_mla_prefill"):
            getattr(h, name).argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Mla), P, P, I32, P, SZ, P]
        h.dsa_sparse_mla_mtp.argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Mla), P, P, I32, I32, P, SZ, P]
        h.dsa_sparse_mla_decode_noalloc.argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Mla), P, P, I32, P]
        h.dsa_noalloc_check_status.argtypes = [P]
        h.dsa_indexshare_group.argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Indexer),
                                           ctypes.POINTER(_Mla), I32, I32, P, P, P, SZ, P]
        h.dsa_indexshare_group_host.argtypes = [ctypes.POINTER(_Queries), ctypes.POINTER(_Indexer),
                                                ctypes.POINTER(_Mla), I32, I32, P, P, P, SZ, P, P, SZ, P, P, SZ, P]
        h.dsa_shard_candidates.argtypes = [ctypes.POINTER(_Queries), P, I64, P, P, I32, I32, P, P, P, SZ, P]
        h.dsa_shard_merge.argtypes = [ctypes.POINTER(_Queries), I32, P, P, I32, I32, I32, P, P, P, P, P, SZ, P]
        h.dsa_shard_combine.argtypes = [ctypes.POINTER(_Queries), I32, I32, I32, P, P, P, P, P, P]
        h.dsa_write_cache_rows.argtypes = [ctypes.POINTER(_CacheWriter), P, SZ, P]
        h.dsa_cache_writer_workspace_bytes.argtypes = [I32, I32]
        h.dsa_cache_writer_workspace_bytes.restype = SZ
        h.dsa_absorb_queries.argtypes = [I32, I32, P, P, P, P, ctypes.c_float, P, P, SZ, P]
        h.dsa_up_project.argtypes = [I32, I32, P, P, P, P, SZ, P]
        h.dsa_workspace_bytes.argtypes = [I32, ctypes.POINTER(_Queries), I32, I32, I32, I32]
        h.dsa_workspace_bytes.restype = SZ
        h.dsa_workspace_init.argtypes = [P, SZ, P]
        h.dsa_check_status.argtypes = [P, P]
        h.dsa_debug_bounded_wait.argtypes = [P, SZ, ctypes.c_uint64, P]
        h.dsa_debug_bounded_wait.restype = st
        h.dsa_status_str.argtypes = [st]
        h.dsa_status_str.restype = ctypes.c_char_p
        for name in ("dsa_index_scores", "dsa_topk", "dsa_sparse_mla_decode", "dsa_sparse_mla_prefill",
                     "dsa_sparse_mla_mtp", "dsa_sparse_mla_decode_noalloc", "dsa_noalloc_check_status",
                     "dsa_indexshare_group", "dsa_indexshare_group_host", "dsa_workspace_init", "dsa_check_status",
                     "dsa_shard_candidates", "dsa_shard_merge", "dsa_shard_combine",
                     "dsa_write_cache_rows", "dsa_absorb_queries", "dsa_up_project"):
            getattr(h, name).restype = st
        _lib_handle = h
    return _lib_handle


def status_str(status: int) -> str:
    return lib().dsa_status_str(int(status)).decode()


def _check(status: int, where: str):
    if status != DSA_OK:
        raise DsaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is None:
        if _raw_stream is not None:
            return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.float8_e4m3fn:
        return DSA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ descriptors
class _CStruct:
    """A descriptor whose C struct (pointers, strides, sizes) is built on first
    use and kept until a field is assigned: repeated calls skip the marshalling.
    The tensors are held, so their pointers stay valid; a tensor whose storage is
    replaced in place (Tensor.set_) needs its field assigned again."""

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        object.__setattr__(self, "_cs", None)

    def c(self):
        cs = self.__dict__.get("_cs")
        if cs is None:
            cs = self._make()
            object.__setattr__(self, "_cs", cs)
        return cs


@dataclass
class Queries(_CStruct):
    q_seq: torch.Tensor          # int32 [n_q]
    q_pos: torch.Tensor          # int32 [n_q]
    n_seq: int
    max_ctx: int
    seq_run: int = 1

    def _make(self) -> _Queries:
        return _Queries(self.q_pos.numel(), self.n_seq, self.max_ctx, self.seq_run,
                        self.q_seq.data_ptr() if self.q_seq.numel() else None,
                        self.q_pos.data_ptr() if self.q_pos.numel() else None)


@dataclass
class Indexer(_CStruct):
    q: torch.Tensor              # [n_q, heads, dim] (bf16, fp32 or float8_e4m3fn)
    w: torch.Tensor              # float32 [n_q, heads]
    k: torch.Tensor              # [n_seq, L, dim] or [L, dim] (shared cache), q's dtype
    flags: int = 0               # DSA_INDEXER_TOPK_HIST or 0
    q_scale: Optional[torch.Tensor] = None   # FP8 only: float32 [n_q, heads], positive
    k_scale: Optional[torch.Tensor] = None   # FP8 only: float32 [n_seq, L] or [L] (shared), positive

    def _make(self) -> _Indexer:
        shared = self.k.dim() == 2
        seq_stride = 0 if shared else self.k.stride(0)
        ks = self.k_scale
        ks_stride = 0 if ks is None or ks.dim() == 1 else ks.stride(0)
        return _Indexer(self.q.shape[1], self.q.shape[2], _dtype_code(self.q), self.flags, self.q.data_ptr(),
                        self.w.data_ptr(), self.k.data_ptr(), seq_stride, self.k.stride(-2),
                        None if self.q_scale is None else self.q_scale.data_ptr(),
                        None if ks is None else ks.data_ptr(), ks_stride)


@dataclass
class Mla(_CStruct):
    q: torch.Tensor              # [n_q, heads, d_latent + d_rope]
    kv: torch.Tensor             # [n_seq, L, d_latent + d_rope] or [L, ...] (shared), q's dtype;
                                 # or uint8 [n_seq, L, >= DSA_MLA_FP8_ROW_BYTES]: packed FP8 rows
    out: torch.Tensor            # [n_q, heads, d_latent]
    d_latent: int
    scale: float
    lse: Optional[torch.Tensor] = None   # float32 [n_q, heads]

    def _make(self) -> _Mla:
        shared = self.kv.dim() == 2
        seq_stride = 0 if shared else self.kv.stride(0)
        heads, dk = self.q.shape[1], self.q.shape[2]
        kv_dtype = DSA_FP8_E4M3 if self.kv.dtype == torch.uint8 else 0
        return _Mla(heads, self.d_latent, dk - self.d_latent, _dtype_code(self.q), float(self.scale), kv_dtype,
                    self.q.data_ptr(), self.kv.data_ptr(), seq_stride, self.kv.stride(-2),
                    self.out.data_ptr(), self.lse.data_ptr() if self.lse is not None else None)


@dataclass
class CacheWriter(_CStruct):
    h: torch.Tensor              # bf16 [n_tok, hidden]
    w: torch.Tensor              # bf16 [704, hidden]: latent 512 | RoPE key 64 | indexer key 128
    rms_weight: torch.Tensor     # float32 [512]
    ln_weight: torch.Tensor      # float32 [128]
    ln_bias: torch.Tensor        # float32 [128]
    tok_seq: torch.Tensor        # int32 [n_tok]
    tok_pos: torch.Tensor        # int32 [n_tok]
    kv: Optional[torch.Tensor]   # bf16 [n_seq, L, 576] latent cache, or None
    k_idx: Optional[torch.Tensor]  # bf16 [n_seq, L, 128] indexer keys, or None
    eps: float = 1e-5
    rope_theta: float = 8.0e6

    def _make(self) -> _CacheWriter:
        ref = self.kv if self.kv is not None else self.k_idx
        return _CacheWriter(self.h.shape[0], self.h.shape[1], self.h.data_ptr(), self.h.stride(0), self.w.data_ptr(),
                            self.rms_weight.data_ptr(), self.ln_weight.data_ptr(), self.ln_bias.data_ptr(),
                            self.tok_seq.data_ptr(), self.tok_pos.data_ptr(), ref.shape[0], ref.shape[1],
                            None if self.kv is None else self.kv.data_ptr(),
                            0 if self.kv is None else self.kv.stride(0), 0 if self.kv is None else self.kv.stride(1),
                            None if self.k_idx is None else self.k_idx.data_ptr(),
                            0 if self.k_idx is None else self.k_idx.stride(0),
                            0 if self.k_idx is None else self.k_idx.stride(1), self.eps, self.rope_theta)


# ------------------------------------------------------------------ entry points
def dsa_workspace_bytes(op: int, queries: Queries, topk: int = 1, mla_heads: int = 64, d_latent: int = 512,
                        n_layers: int = 1) -> int:
    return int(lib().dsa_workspace_bytes(op, ctypes.byref(queries.c()), topk, mla_heads, d_latent, n_layers))


def dsa_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().dsa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_workspace_init")


def dsa_check_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the workspace status word (returns the code)."""
    return int(lib().dsa_check_status(_ptr(ws), _stream(stream)))


def dsa_debug_bounded_wait(ws: torch.Tensor, limit_ns: int, stream=None):
    _check(lib().dsa_debug_bounded_wait(_ptr(ws), ws.numel() * ws.element_size(), int(limit_ns), _stream(stream)),
           "dsa_debug_bounded_wait")


def dsa_index_scores(queries: Queries, indexer: Indexer, scores: torch.Tensor, ws: torch.Tensor, stream=None):
    qc, ic = queries.c(), indexer.c()
    _check(lib().dsa_index_scores(ctypes.byref(qc), ctypes.byref(ic), _ptr(scores), scores.stride(0), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "dsa_index_scores")


def dsa_topk(queries: Queries, scores: torch.Tensor, topk: int, idx: torch.Tensor, cnt: torch.Tensor,
             ws: torch.Tensor, stream=None, flags: int = 0):
    qc = queries.c()
    _check(lib().dsa_topk(ctypes.byref(qc), _ptr(scores), scores.stride(0), topk, flags, _ptr(idx), _ptr(cnt), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "dsa_topk")


def dsa_sparse_mla_decode(queries: Queries, mla: Mla, idx: torch.Tensor, cnt: torch.Tensor, topk: int,
                          ws: torch.Tensor, stream=None):
    qc, mc = queries.c(), mla.c()
    _check(lib().dsa_sparse_mla_decode(ctypes.byref(qc), ctypes.byref(mc), _ptr(idx), _ptr(cnt), topk, _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "dsa_sparse_mla_decode")


def dsa_sparse_mla_prefill(queries: Queries, mla: Mla, idx: torch.Tensor, cnt: torch.Tensor, topk: int,
                           ws: torch.Tensor, stream=None):
    qc, mc = queries.c(), mla.c()
    _check(lib().dsa_sparse_mla_prefill(ctypes.byref(qc), ctypes.byref(mc), _ptr(idx), _ptr(cnt), topk, _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)), "dsa_sparse_mla_prefill")


def dsa_sparse_mla_mtp(queries: Queries, mla: Mla, idx: torch.Tensor, cnt: torch.Tensor, topk: int,
                       draft_tokens: int, ws: torch.Tensor, stream=None):
    qc, mc = queries.c(), mla.c()
    _check(lib().dsa_sparse_mla_mtp(ctypes.byref(qc), ctypes.byref(mc), _ptr(idx), _ptr(cnt), topk, draft_tokens,
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "dsa_sparse_mla_mtp")


def dsa_sparse_mla_decode_noalloc(queries: Queries, mla: Mla, idx: torch.Tensor, cnt: torch.Tensor, topk: int,
                                  stream=None):
    qc, mc = queries.c(), mla.c()
    _check(lib().dsa_sparse_mla_decode_noalloc(ctypes.byref(qc), ctypes.byref(mc), _ptr(idx), _ptr(cnt), topk,
                                               _stream(stream)), "dsa_sparse_mla_decode_noalloc")


def dsa_noalloc_check_status(stream=None) -> int:
    """Synchronise, read and clear the no-workspace calls' status word (returns the code)."""
    return int(lib().dsa_noalloc_check_status(_stream(stream)))


def dsa_indexshare_group(queries: Queries, indexer: Indexer, layers: Sequence[Mla], topk: int, idx: torch.Tensor,
                         cnt: torch.Tensor, ws: torch.Tensor, stream=None):
    qc, ic = queries.c(), indexer.c()
    arr = (_Mla * len(layers))(*[m.c() for m in layers])
    _check(lib().dsa_indexshare_group(ctypes.byref(qc), ctypes.byref(ic), arr, len(layers), topk, _ptr(idx),
                                      _ptr(cnt), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_indexshare_group")


class GroupHostCall:
    """dsa_indexshare_group_host with its arguments converted once: a decode loop
    whose buffers stay put (the descriptors, pinned host blocks and device blocks
    of every step are the same) calls this each step.  h_in -> d_in is copied
    before the group call and d_out -> h_out after it, on `stream` (default: the
    stream current when this is made); each host buffer has its device buffer's
    byte size and the descriptors point into the device buffers."""

    def __init__(self, queries: Queries, indexer: Indexer, layers: Sequence[Mla], topk: int, idx: torch.Tensor,
                 cnt: torch.Tensor, ws: torch.Tensor, h_in: torch.Tensor, d_in: torch.Tensor, h_out: torch.Tensor,
                 d_out: torch.Tensor, stream=None):
        def nbytes(t):
            return t.numel() * t.element_size()
        if nbytes(h_in) != nbytes(d_in) or nbytes(h_out) != nbytes(d_out):
            raise ValueError("host and device buffers differ in size")
        self._keep = (queries, indexer, list(layers), idx, cnt, ws, h_in, d_in, h_out, d_out)
        self._qc, self._ic = queries.c(), indexer.c()
        self._arr = (_Mla * len(layers))(*[m.c() for m in layers])
        self._args = (ctypes.byref(self._qc), ctypes.byref(self._ic), self._arr, len(layers), topk, _ptr(idx),
                      _ptr(cnt), _ptr(ws), nbytes(ws), _ptr(h_in), _ptr(d_in), nbytes(h_in), _ptr(h_out),
                      _ptr(d_out), nbytes(h_out), _stream(stream))
        self._fn = lib().dsa_indexshare_group_host

    def __call__(self):
        _check(self._fn(*self._args), "dsa_indexshare_group_host")


def dsa_indexshare_group_host(queries: Queries, indexer: Indexer, layers: Sequence[Mla], topk: int,
                              idx: torch.Tensor, cnt: torch.Tensor, ws: torch.Tensor, h_in: torch.Tensor,
                              d_in: torch.Tensor, h_out: torch.Tensor, d_out: torch.Tensor, stream=None):
    """The group call with its inputs copied from h_in (pinned host) to d_in before it
    and its outputs from d_out to h_out (pinned host) after it, all enqueued on the
    stream; the descriptors point into the device buffers."""
    GroupHostCall(queries, indexer, layers, topk, idx, cnt, ws, h_in, d_in, h_out, d_out, stream)()


def dsa_shard_candidates(queries: Queries, scores: torch.Tensor, idx: torch.Tensor, cnt: torch.Tensor, topk: int,
                         row_offset: int, cand_score: torch.Tensor, cand_pos: torch.Tensor, ws: torch.Tensor,
                         stream=None):
    qc = queries.c()
    _check(lib().dsa_shard_candidates(ctypes.byref(qc), _ptr(scores), scores.stride(0), _ptr(idx), _ptr(cnt), topk,
                                      row_offset, _ptr(cand_score), _ptr(cand_pos), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)), "dsa_shard_candidates")


def dsa_shard_merge(queries: Queries, n_shards: int, cand_score: torch.Tensor, cand_pos: torch.Tensor, topk: int,
                    row_begin: int, row_end: int, idx: torch.Tensor, cnt: torch.Tensor, local_idx: torch.Tensor,
                    local_cnt: torch.Tensor, ws: torch.Tensor, stream=None):
    qc = queries.c()
    _check(lib().dsa_shard_merge(ctypes.byref(qc), n_shards, _ptr(cand_score), _ptr(cand_pos), topk, row_begin,
                                 row_end, _ptr(idx), _ptr(cnt), _ptr(local_idx), _ptr(local_cnt), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "dsa_shard_merge")


def dsa_shard_combine(queries: Queries, part_out: torch.Tensor, part_lse: torch.Tensor, part_cnt: torch.Tensor,
                      out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    """part_out [n_parts, n_q, heads, d_latent] bf16, part_lse [n_parts, n_q, heads], part_cnt [n_parts, n_q]."""
    qc = queries.c()
    n_parts, _, heads, d_lat = part_out.shape
    _check(lib().dsa_shard_combine(ctypes.byref(qc), n_parts, heads, d_lat, _ptr(part_out), _ptr(part_lse),
                                   _ptr(part_cnt), _ptr(out), _ptr(lse), _stream(stream)), "dsa_shard_combine")


def dsa_cache_writer_workspace_bytes(n_tok: int, hidden: int) -> int:
    return int(lib().dsa_cache_writer_workspace_bytes(n_tok, hidden))


def dsa_write_cache_rows(writer: CacheWriter, ws: torch.Tensor, stream=None):
    wc = writer.c()
    _check(lib().dsa_write_cache_rows(ctypes.byref(wc), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_write_cache_rows")


def dsa_absorb_queries(q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk_t: torch.Tensor, pos: torch.Tensor,
                       rope_theta: float, q_out: torch.Tensor, ws: torch.Tensor, stream=None):
    """q_nope [n, H, 192], q_rope [n, H, 64], w_uk_t [H, 512, 192], pos int32 [n] -> q_out [n, H, 576]."""
    n, heads = q_nope.shape[0], q_nope.shape[1]
    _check(lib().dsa_absorb_queries(n, heads, _ptr(q_nope), _ptr(q_rope), _ptr(w_uk_t), _ptr(pos), rope_theta,
                                    _ptr(q_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_absorb_queries")


def dsa_up_project(o_lat: torch.Tensor, w_uv: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, stream=None):
    """o_lat [n, H, 512], w_uv [H, 256, 512] -> out [n, H, 256]."""
    n, heads = o_lat.shape[0], o_lat.shape[1]
    _check(lib().dsa_up_project(n, heads, _ptr(o_lat), _ptr(w_uv), _ptr(out), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "dsa_up_project")


# ------------------------------------------------------------------ conveniences
def workspace(op: int, queries: Queries, topk: int = 1, n_layers: int = 1, device="cuda", stream=None):
    """Allocate (torch) and zero-initialise a workspace for `op`."""
    n = dsa_workspace_bytes(op, queries, topk, 64, 512, n_layers)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    dsa_workspace_init(ws, stream)
    return ws


def scores_buffer(n_q: int, max_ctx: int, device="cuda") -> torch.Tensor:
    """float32 [n_q, ld] with ld = max_ctx rounded up to a multiple of 4."""
    ld = (max_ctx + 3) // 4 * 4
    return torch.empty((n_q, ld), dtype=torch.float32, device=device)


def default_scale(d_nope: int = 192, d_rope: int = 64) -> float:
    return 1.0 / math.sqrt(d_nope + d_rope)
