"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/dsa.h declares, rejects bad arguments synchronously
before any launch, and sizes workspaces as documented."""
import ctypes
import os
import re

import pytest

from dsa_indexer_top_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    syms = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            syms |= set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text))
    return syms


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    syms = declared_symbols()
    assert {"dsa_index_scores", "dsa_topk", "dsa_sparse_mla_decode", "dsa_sparse_mla_prefill",
            "dsa_indexshare_group", "dsa_workspace_bytes"} <= syms
    for s in sorted(syms):
        assert hasattr(lib, s), f"{s} not exported"


def test_status_strings():
    assert B.status_str(B.DSA_OK) == "DSA_OK"
    assert B.status_str(B.DSA_ERR_TIMEOUT) == "DSA_ERR_TIMEOUT"
    assert B.status_str(99) == "DSA_ERR_UNKNOWN"


def _q(n_q=4, n_seq=4, L=1000, seq_run=1):
    return B._Queries(n_q, n_seq, L, seq_run, 0x1000, 0x2000)


def test_workspace_bytes():
    lib = B.lib()
    q = _q(n_q=8, L=32768)
    assert lib.dsa_workspace_bytes(B.DSA_OP_INDEX_SCORES, ctypes.byref(q), 2048, 64, 512, 1) == 256
    # top-k: status + first-digit histograms, one ticket per query and the
    # second-digit histograms (256-aligned) + (split schedule: 8 queries,
    # ctx > 8192) per-chunk counts and candidates
    hist = ((8 * 4096 * 4 + 8 * 4 + 8 * 4096 * 4 + 255) // 256) * 256  # tickets padded to 4 words
    split = hist + 8 * 64 * 4 + 8 * 64 * 1024 * 8
    assert lib.dsa_workspace_bytes(B.DSA_OP_TOPK, ctypes.byref(q), 2048, 64, 512, 1) == 256 + split
    q2 = _q(n_q=8, L=8192)
    assert lib.dsa_workspace_bytes(B.DSA_OP_TOPK, ctypes.byref(q2), 2048, 64, 512, 1) == 256 + hist
    dec = lib.dsa_workspace_bytes(B.DSA_OP_MLA_DECODE, ctypes.byref(q), 2048, 64, 512, 1)
    # status + the region the indexer / top-k keep zero (left alone, so the calls of
    # a step can share one workspace) + up to 32 splits (64-row chunks) x 8 queries
    # x 64 heads x (512 + 2) floats, 256-aligned
    assert dec == 256 + hist + ((8 * 32 * 64 * 514 * 4 + 255) // 256) * 256
    assert lib.dsa_workspace_bytes(B.DSA_OP_MLA_DECODE, ctypes.byref(q), 64, 64, 512, 1) == 256
    grp = lib.dsa_workspace_bytes(B.DSA_OP_INDEXSHARE_GROUP, ctypes.byref(q), 2048, 64, 512, 4)
    scores = 8 * 32768 * 4
    assert grp == 256 + scores + split + ((4 * 8 * 32 * 64 * 514 * 4 + 255) // 256) * 256
    assert lib.dsa_workspace_bytes(77, ctypes.byref(q), 2048, 64, 512, 1) == 0


class _FakeWs:
    """An aligned host address standing in for a workspace: validation runs
    before any use of it, so nothing dereferences it."""
    ptr = 0x10000
    size = 1 << 30


def _idx(heads=32, dim=128, dtype=0, q=0x3000, w=0x4000, k=0x5000, kss=1000 * 128, krs=128):
    return B._Indexer(heads, dim, dtype, 0, q, w, k, kss, krs)


def _mla(heads=64, dl=512, dr=64, dtype=0, q=0x6000, kv=0x7000, out=0x8000, kss=1000 * 576, krs=576):
    return B._Mla(heads, dl, dr, dtype, 0.0625, 0, q, kv, kss, krs, out, None)


@pytest.mark.parametrize("case", [
    "null_queries", "neg_nq", "zero_ctx", "bad_seq_run", "null_pos", "bad_dim", "bad_dtype", "row_stride",
    "seq_stride", "ld_small", "ld_unaligned", "scores_null"])
def test_index_scores_rejects(case):
    lib = B.lib()
    q = _q()
    ix = _idx()
    ld = 1000
    scores = 0x9000
    if case == "neg_nq": q.n_q = -1
    if case == "zero_ctx": q.max_ctx = 0
    if case == "bad_seq_run": q.seq_run = 0
    if case == "null_pos": q.q_pos = None
    if case == "bad_dim": ix.dim = 0
    if case == "bad_dtype": ix.dtype = 5
    if case == "row_stride": ix.k_row_stride = 64
    if case == "seq_stride": ix.k_seq_stride = 999 * 128
    if case == "ld_small": ld = 996
    if case == "ld_unaligned": ld = 1002
    if case == "scores_null": scores = 0
    qp = None if case == "null_queries" else ctypes.byref(q)
    st = lib.dsa_index_scores(qp, ctypes.byref(ix), scores, ld, _FakeWs.ptr, _FakeWs.size, None)
    assert st == B.DSA_ERR_INVALID


@pytest.mark.parametrize("case,expect", [
    ("heads16", "unsupported"), ("row_stride_136", "unsupported"), ("seq_stride_not16", "unsupported"),
    ("ks_stride_short", "invalid"), ("ks_stride_negative", "invalid"),
])
def test_index_scores_fp8_validation(case, expect):
    """FP8 (E4M3) indexers run on the tensor-core path only (32 x 128, 16-element
    TMA strides); a per-key scale array must cover max_ctx rows per sequence."""
    lib = B.lib()
    q = _q()
    ix = _idx(dtype=B.DSA_FP8_E4M3)
    if case == "heads16": ix.heads = 16
    if case == "row_stride_136": ix.k_row_stride = 136
    if case == "seq_stride_not16": ix.k_seq_stride = 1000 * 128 + 8
    if case == "ks_stride_short": ix.k_scale, ix.ks_seq_stride = 0xA000, 500
    if case == "ks_stride_negative": ix.ks_seq_stride = -1
    st = lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, _FakeWs.ptr, _FakeWs.size, None)
    assert st == (B.DSA_ERR_UNSUPPORTED if expect == "unsupported" else B.DSA_ERR_INVALID)


def test_debug_bounded_wait_validation():
    lib = B.lib()
    lib.dsa_debug_bounded_wait.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_void_p]
    assert lib.dsa_debug_bounded_wait(None, 0, 1000, None) == B.DSA_ERR_INVALID
    assert lib.dsa_debug_bounded_wait(_FakeWs.ptr, _FakeWs.size, 3_000_000_000, None) == B.DSA_ERR_INVALID


def test_workspace_checks():
    lib = B.lib()
    q, ix = _q(), _idx()
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, 0, 1 << 20, None) == B.DSA_ERR_WORKSPACE
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, 0x10010, 1 << 20, None) == B.DSA_ERR_WORKSPACE
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, 0x10000, 128, None) == B.DSA_ERR_WORKSPACE
    m = _mla()
    need = lib.dsa_workspace_bytes(B.DSA_OP_MLA_DECODE, ctypes.byref(q), 2048, 64, 512, 1)
    assert lib.dsa_sparse_mla_decode(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, 0x10000, need - 1,
                                     None) == B.DSA_ERR_WORKSPACE


@pytest.mark.parametrize("topk", [0, -3, 4097])
def test_topk_rejects_bad_k(topk):
    lib = B.lib()
    q = _q()
    assert lib.dsa_topk(ctypes.byref(q), 0x9000, 1000, topk, 0, 0xA000, 0xB000, _FakeWs.ptr, _FakeWs.size,
                        None) == B.DSA_ERR_INVALID


def test_flags_validated():
    lib = B.lib()
    q = _q()
    assert lib.dsa_topk(ctypes.byref(q), 0x9000, 1000, 64, 6, 0xA000, 0xB000, _FakeWs.ptr, _FakeWs.size,
                        None) == B.DSA_ERR_INVALID
    ix = _idx()
    ix.flags = 2
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, _FakeWs.ptr, _FakeWs.size,
                                None) == B.DSA_ERR_INVALID
    ix.flags = B.DSA_INDEXER_TOPK_HIST   # needs a top-k sized workspace
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(ix), 0x9000, 1000, 0x10000, 256,
                                None) == B.DSA_ERR_WORKSPACE


def test_mla_rejects():
    lib = B.lib()
    q = _q()
    for kw in [dict(q=0), dict(kv=0), dict(out=0), dict(heads=0), dict(dtype=3), dict(krs=500),
               dict(dl=0)]:
        m = _mla(**kw)
        st = lib.dsa_sparse_mla_prefill(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, _FakeWs.ptr,
                                        _FakeWs.size, None)
        assert st == B.DSA_ERR_INVALID, kw
    m = _mla()
    assert lib.dsa_sparse_mla_prefill(ctypes.byref(q), ctypes.byref(m), 0, 0xB000, 2048, _FakeWs.ptr,
                                      _FakeWs.size, None) == B.DSA_ERR_INVALID


def test_group_rejects_layer_mismatch_and_count():
    lib = B.lib()
    q, ix = _q(), _idx()
    arr = (B._Mla * 2)(_mla(), _mla(dl=256, krs=576))
    assert lib.dsa_indexshare_group(ctypes.byref(q), ctypes.byref(ix), arr, 2, 2048, 0xA000, 0xB000, _FakeWs.ptr,
                                    _FakeWs.size, None) == B.DSA_ERR_INVALID
    arr5 = (B._Mla * 5)(*[_mla() for _ in range(5)])
    assert lib.dsa_indexshare_group(ctypes.byref(q), ctypes.byref(ix), arr5, 5, 2048, 0xA000, 0xB000, _FakeWs.ptr,
                                    _FakeWs.size, None) == B.DSA_ERR_INVALID


def test_group_host_rejects_before_any_copy():
    """The host-buffer group call checks everything before it enqueues a copy: the
    group call's own argument errors, and a null host or device buffer with a
    non-zero size (all pointers here are fake, so any copy or launch would fail)."""
    lib = B.lib()
    q, ix = _q(), _idx()

    def call(arr, n, ws_size=_FakeWs.size, bufs=(0x20000, 0x30000, 0x40000, 0x50000)):
        h_in, d_in, h_out, d_out = bufs
        return lib.dsa_indexshare_group_host(ctypes.byref(q), ctypes.byref(ix), arr, n, 2048, 0xA000, 0xB000,
                                             _FakeWs.ptr, ws_size, h_in, d_in, 4096, h_out, d_out, 4096, None)

    assert call((B._Mla * 2)(_mla(), _mla(dl=256, krs=576)), 2) == B.DSA_ERR_INVALID
    one = (B._Mla * 1)(_mla())
    good = [0x20000, 0x30000, 0x40000, 0x50000]
    for k in range(4):
        bufs = list(good)
        bufs[k] = None
        assert call(one, 1, bufs=tuple(bufs)) == B.DSA_ERR_INVALID, k
    assert call(one, 1, ws_size=16) == B.DSA_ERR_WORKSPACE


def test_zero_queries_is_a_noop():
    lib = B.lib()
    q = _q(n_q=0)
    assert lib.dsa_index_scores(ctypes.byref(q), ctypes.byref(_idx()), 0x9000, 1000, _FakeWs.ptr, _FakeWs.size,
                                None) == B.DSA_OK


@pytest.mark.parametrize("case,expect", [
    ("kv_dtype_unknown", "invalid"), ("row_too_short", "invalid"), ("row_not16", "unsupported"),
    ("row_below_packed", "unsupported"), ("seq_not16", "unsupported"), ("f32_queries", "unsupported"),
    ("heads32", "unsupported"), ("kv_unaligned", "unsupported"),
])
def test_mla_fp8_cache_validation(case, expect):
    """Packed FP8 latent caches (kv_dtype = DSA_FP8_E4M3): byte strides, multiples
    of 16, rows of at least 656 bytes, tensor-core shape only; a row shorter than
    codes + RoPE + scale is invalid for any shape."""
    lib = B.lib()
    q = _q()
    m = _mla(kss=1000 * 656, krs=656)
    m.kv_dtype = B.DSA_FP8_E4M3
    if case == "kv_dtype_unknown": m.kv_dtype = 7
    if case == "row_too_short": m.kv_row_stride = 640
    if case == "row_not16": m.kv_row_stride = 664
    if case == "row_below_packed": m.kv_row_stride = 648
    if case == "seq_not16": m.kv_seq_stride = 1000 * 656 + 8
    if case == "f32_queries": m.dtype = B.DSA_F32
    if case == "heads32": m.heads = 32
    if case == "kv_unaligned": m.kv = 0x7008
    want = B.DSA_ERR_INVALID if expect == "invalid" else B.DSA_ERR_UNSUPPORTED
    for fn in (lib.dsa_sparse_mla_prefill, lib.dsa_sparse_mla_decode):
        assert fn(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, _FakeWs.ptr, _FakeWs.size, None) == want
    assert lib.dsa_sparse_mla_decode_noalloc(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, None) == want


def test_group_rejects_mixed_cache_types():
    lib = B.lib()
    q, ix = _q(), _idx()
    m8 = _mla(kss=1000 * 656, krs=656)
    m8.kv_dtype = B.DSA_FP8_E4M3
    m16 = _mla(kss=1000 * 656, krs=656)
    arr = (B._Mla * 2)(m8, m16)
    assert lib.dsa_indexshare_group(ctypes.byref(q), ctypes.byref(ix), arr, 2, 2048, 0xA000, 0xB000, _FakeWs.ptr,
                                    _FakeWs.size, None) == B.DSA_ERR_INVALID


def test_mla_kv_dtype_same_as_dtype_is_accepted_by_validation():
    """kv_dtype equal to dtype means the plain cache: validation passes through to
    the workspace check (a too-small workspace is then the first error)."""
    lib = B.lib()
    q = _q()
    m = _mla()
    m.kv_dtype = B.DSA_BF16
    assert lib.dsa_sparse_mla_prefill(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, _FakeWs.ptr, 128,
                                      None) == B.DSA_ERR_WORKSPACE
    m.dtype = m.kv_dtype = B.DSA_F32
    assert lib.dsa_sparse_mla_prefill(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, _FakeWs.ptr, 128,
                                      None) == B.DSA_ERR_WORKSPACE


def test_mtp_rejects_bad_group_size():
    lib = B.lib()
    q = _q(n_q=6)
    m = _mla()
    for d in (0, -1, 4):  # 4 does not divide 6
        assert lib.dsa_sparse_mla_mtp(ctypes.byref(q), ctypes.byref(m), 0xA000, 0xB000, 2048, d, _FakeWs.ptr,
                                      _FakeWs.size, None) == B.DSA_ERR_INVALID


def test_shard_calls_validate():
    lib = B.lib()
    q = _q(n_q=2, L=5000)
    P = 0xC000
    # merge: shard count, ranges, workspace
    assert lib.dsa_shard_merge(ctypes.byref(q), 0, P, P, 2048, 0, 10, P, P, P, P, _FakeWs.ptr, _FakeWs.size,
                               None) == B.DSA_ERR_INVALID
    assert lib.dsa_shard_merge(ctypes.byref(q), 65, P, P, 2048, 0, 10, P, P, P, P, _FakeWs.ptr, _FakeWs.size,
                               None) == B.DSA_ERR_INVALID
    assert lib.dsa_shard_merge(ctypes.byref(q), 2, P, P, 2048, 10, 5, P, P, P, P, _FakeWs.ptr, _FakeWs.size,
                               None) == B.DSA_ERR_INVALID
    need = lib.dsa_workspace_bytes(B.DSA_OP_SHARD_MERGE, ctypes.byref(q), 2048, 0, 0, 4)
    # status + merged scores and positions (4 shards x 2048 per query) + counts + the
    # merged top-k (indices, counts) + the top-k scratch of 8192-wide rows
    assert need > 256 + 2 * (2 * 4 * 2048 * 4) + 2 * 2048 * 4
    assert lib.dsa_shard_merge(ctypes.byref(q), 4, P, P, 2048, 0, 10, P, P, P, P, _FakeWs.ptr, need - 1,
                               None) == B.DSA_ERR_WORKSPACE
    # candidates: null outputs; combine: shapes the kernel does not cover
    assert lib.dsa_shard_candidates(ctypes.byref(q), P, 5000, P, P, 2048, 0, None, P, _FakeWs.ptr, _FakeWs.size,
                                    None) == B.DSA_ERR_INVALID
    assert lib.dsa_shard_combine(ctypes.byref(q), 2, 63, 512, P, P, P, P, None, None) == B.DSA_ERR_UNSUPPORTED
    assert lib.dsa_shard_combine(ctypes.byref(q), 2, 64, 1024, P, P, P, P, None, None) == B.DSA_ERR_UNSUPPORTED
    assert lib.dsa_shard_combine(ctypes.byref(q), 0, 64, 512, P, P, P, P, None, None) == B.DSA_ERR_INVALID


def test_producer_calls_validate():
    lib = B.lib()
    P = 0xD000
    w = B._CacheWriter(4, 6144, P, 6144, P, P, P, P, P, P, 2, 1000, P, 1000 * 576, 576, P, 1000 * 128, 128,
                       1e-5, 8e6)
    need = lib.dsa_cache_writer_workspace_bytes(4, 6144)
    # 4 tokens: one M tile x 6 N tiles, split 24 ways along K (4 blocks of 64 each)
    assert need == 256 + ((24 * 4 * 704 * 4 + 255) // 256) * 256
    assert lib.dsa_write_cache_rows(ctypes.byref(w), _FakeWs.ptr, need - 1, None) == B.DSA_ERR_WORKSPACE
    bad = B._CacheWriter(4, 6144, P, 6144, None, P, P, P, P, P, 2, 1000, P, 1000 * 576, 576, P, 1000 * 128, 128,
                         1e-5, 8e6)
    assert lib.dsa_write_cache_rows(ctypes.byref(bad), _FakeWs.ptr, need, None) == B.DSA_ERR_INVALID
    odd = B._CacheWriter(4, 6100, P, 6100, P, P, P, P, P, P, 2, 1000, P, 1000 * 576, 576, P, 1000 * 128, 128,
                         1e-5, 8e6)
    assert lib.dsa_write_cache_rows(ctypes.byref(odd), _FakeWs.ptr, need, None) == B.DSA_ERR_INVALID
    assert lib.dsa_absorb_queries(4, 64, P, P, None, P, 8e6, P, _FakeWs.ptr, 256, None) == B.DSA_ERR_INVALID
    assert lib.dsa_absorb_queries(4, 64, P, P, P, P, 8e6, P, _FakeWs.ptr, 128, None) == B.DSA_ERR_WORKSPACE
    assert lib.dsa_up_project(4, 64, P, P, None, _FakeWs.ptr, 256, None) == B.DSA_ERR_INVALID
    assert lib.dsa_up_project(0, 64, P, P, P, _FakeWs.ptr, 256, None) == B.DSA_OK


def test_descriptor_struct_follows_field_assignments():
    """The binding's descriptors build their C struct once and rebuild it when a
    field is assigned (so repeated calls skip the marshalling but never pass a
    stale pointer, flag or size)."""
    import torch

    q = torch.zeros(4, 32, 128, dtype=torch.bfloat16)
    w = torch.zeros(4, 32)
    k = torch.zeros(4, 64, 128, dtype=torch.bfloat16)
    ix = B.Indexer(q, w, k)
    c0 = ix.c()
    assert ix.c() is c0 and c0.flags == 0
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    c1 = ix.c()
    assert c1 is not c0 and c1.flags == B.DSA_INDEXER_TOPK_HIST
    k2 = torch.zeros(4, 64, 128, dtype=torch.bfloat16)
    ix.k = k2
    assert ix.c().k == k2.data_ptr()
    qs = B.Queries(torch.zeros(3, dtype=torch.int32), torch.zeros(3, dtype=torch.int32), n_seq=2, max_ctx=10)
    assert qs.c().n_q == 3
    qs.q_pos = torch.zeros(5, dtype=torch.int32)
    qs.q_seq = torch.zeros(5, dtype=torch.int32)
    assert qs.c().n_q == 5
