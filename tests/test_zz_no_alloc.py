"""dsa_sparse_mla_decode_noalloc -- the decode attention call for callers that
cannot allocate device memory (no workspace; scratch lives in a fixed array in
the library).  Checked through the C ABI against dsa_sparse_mla_decode, which
uses a caller workspace, on two calls in a row (the shared scratch keeps the
previous call's contents, which must not leak into the next result).

Collected last on purpose (file name) so a failure here stops a -x run only
after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu


def _noalloc(q, mla, idx, cnt, topk):
    fn = B.lib().dsa_sparse_mla_decode_noalloc
    fn.argtypes = [ctypes.POINTER(B._Queries), ctypes.POINTER(B._Mla), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    qc, mc = q.c(), mla.c()
    return fn(ctypes.byref(qc), ctypes.byref(mc), idx.data_ptr(), cnt.data_ptr(), topk,
              torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_decode_twice(cuda_ok):
    dev = torch.device("cuda")
    base = wl.NAMED["decode_32k"]
    for call, (seed, L, topk) in enumerate([(21, 5000, 2048), (22, 3300, 1024)]):
        w = wl.scaled(base, n_seq=3, L=L, q_pos=(L - 1, L // 2, 700), q_seq=(1, 2, 0), topk=topk, seed=seed)
        x = C.to_device(wl.make_inputs(w))
        q, _, mlas = C.descriptors(w, x)
        idx, cnt = C.random_selection(w, seed=seed)
        idx, cnt = idx.to(dev), cnt.to(dev)
        ref = mlas[0]
        ws = B.workspace(B.DSA_OP_MLA_DECODE, q, topk, device=dev)
        B.dsa_sparse_mla_decode(q, ref, idx, cnt, topk, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK
        out = torch.full_like(ref.out, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        got = B.Mla(ref.q, ref.kv, out, w.d_lat, w.scale, lse)
        st = _noalloc(q, got, idx, cnt, topk)
        assert st == B.DSA_OK, B.status_str(st)
        torch.cuda.synchronize()
        C.assert_attention_close(out, ref.out.float().cpu().numpy().astype(np.float64), "bf16", f"call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref.lse.cpu().numpy(), atol=1e-3, rtol=0)


def test_noalloc_rejects_oversize(cuda_ok):
    dev = torch.device("cuda")
    n_q = 16  # 16 queries x 16 splits x 131,584 B > 32 MiB
    q = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev), torch.zeros(n_q, dtype=torch.int32, device=dev),
                  n_seq=1, max_ctx=4096)
    qm = torch.zeros((n_q, 64, 576), dtype=torch.bfloat16, device=dev)
    kv = torch.zeros((1, 4096, 576), dtype=torch.bfloat16, device=dev)
    out = torch.zeros((n_q, 64, 512), dtype=torch.bfloat16, device=dev)
    idx = torch.zeros((n_q, 2048), dtype=torch.int32, device=dev)
    cnt = torch.ones(n_q, dtype=torch.int32, device=dev)
    assert _noalloc(q, B.Mla(qm, kv, out, 512, 0.0625), idx, cnt, 2048) == B.DSA_ERR_WORKSPACE
