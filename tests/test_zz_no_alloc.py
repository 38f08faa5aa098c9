"""dsa_sparse_mla_decode_noalloc -- the decode attention call for callers that
cannot allocate device memory (a runtime or plugin that only hands over its
input/output tensors, or memory planned up front): no workspace, the scratch
lives in a fixed array inside the library.  Checked through the C ABI against
the oracle and against dsa_sparse_mla_decode (which uses a caller workspace),
on two calls in a row (the shared scratch keeps the previous call's contents,
which must not leak into the next result), on a bf16 and a packed FP8 cache, on
a multi-split and a single-split plan, and with the status word read back.

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


def _noalloc_status():
    fn = B.lib().dsa_noalloc_check_status
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(torch.cuda.current_stream().cuda_stream)


def _case(n_q, L, topk, seed):
    base = wl.NAMED["decode_32k"]
    pos = tuple(int(L - 1 - (i * 997) % (L // 2)) for i in range(n_q))
    return wl.scaled(base, n_seq=n_q, L=L, q_pos=pos, q_seq=tuple((i + 1) % n_q for i in range(n_q)), topk=topk,
                     seed=seed)


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16_cache", "fp8_cache"])
@pytest.mark.parametrize("plan", ["multi_split", "single_split"])
def test_noalloc_matches_oracle_and_workspace_decode_twice(cuda_ok, fp8, plan):
    """Two calls in a row: a multi-split plan (3 queries, topk 2048 then 1024)
    or a single-split one (topk 128: one CTA per query, no partials; then 96
    queries, which the plan gives one split each)."""
    dev = torch.device("cuda")
    cases = [(3, 5000, 2048, 21), (3, 3300, 1024, 22)] if plan == "multi_split" else \
            [(3, 3000, 128, 23), (96, 2500, 2048, 24)]
    assert _noalloc_status() == B.DSA_OK  # nothing left over from earlier calls
    for call, (n_q, L, topk, seed) in enumerate(cases):
        w = _case(n_q, L, topk, seed)
        xh = wl.make_inputs(w, layers=[0])
        x = C.to_device(xh)
        q, _, mlas = C.descriptors(w, x)
        ref = mlas[0]
        kv8h = None
        if fp8:
            kv8h = wl.fp8_latent_inputs(w, xh)
            ref = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])[0]
        idx, cnt = C.random_selection(w, seed=seed)
        idx_d, cnt_d = idx.to(dev), cnt.to(dev)
        ws = B.workspace(B.DSA_OP_MLA_DECODE, q, topk, device=dev)
        B.dsa_sparse_mla_decode(q, ref, idx_d, cnt_d, topk, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK
        out = torch.full_like(ref.out, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        got = B.Mla(ref.q, ref.kv, out, w.d_lat, w.scale, lse)
        st = _noalloc(q, got, idx_d, cnt_d, topk)
        assert st == B.DSA_OK, B.status_str(st)
        assert _noalloc_status() == B.DSA_OK
        # against the oracle (fp64), within the attention tolerance
        if fp8:
            o_ref, l_ref = C.oracle_mla_fp8(w, xh, kv8h, 0, idx.numpy(), cnt.numpy())
        else:
            o_ref, l_ref = C.oracle_mla(w, xh, 0, idx.numpy(), cnt.numpy())
        C.assert_attention_close(out, o_ref, "bf16", f"call {call}")
        C.assert_lse_close(lse, l_ref, "bf16")
        # and against the workspace entry point, which runs the same plan
        C.assert_attention_close(out, ref.out.float().cpu().numpy().astype(np.float64), "bf16",
                                 f"call {call} vs workspace decode")
        np.testing.assert_allclose(lse.cpu().numpy(), ref.lse.cpu().numpy(), atol=1e-3, rtol=0)


def test_noalloc_accepts_batches_whose_plan_fits(cuda_ok):
    """16 queries at topk 2048: the decode plan gives each query SMs / 16 splits,
    whose partials fit the fixed array (a bound by the worst-case split count
    would have rejected this call)."""
    dev = torch.device("cuda")
    w = _case(16, 2600, 2048, 25)
    xh = wl.make_inputs(w, layers=[0])
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    idx, cnt = C.random_selection(w, seed=25)
    st = _noalloc(q, mlas[0], idx.to(dev), cnt.to(dev), w.topk)
    assert st == B.DSA_OK, B.status_str(st)
    assert _noalloc_status() == B.DSA_OK
    o_ref, _ = C.oracle_mla(w, xh, 0, idx.numpy(), cnt.numpy())
    C.assert_attention_close(mlas[0].out, o_ref, "bf16")


def test_noalloc_reports_device_errors_through_its_status(cuda_ok):
    """A selected index past the cache end is skipped on the device and reported
    in the fixed array's status word; reading it back clears it."""
    dev = torch.device("cuda")
    w = _case(2, 1500, 256, 26)
    x = C.to_device(wl.make_inputs(w, layers=[0]))
    q, _, mlas = C.descriptors(w, x)
    idx, cnt = C.random_selection(w, seed=26)
    idx[1, 5] = w.L + 7  # in the selection (cnt = 256), out of the cache's range
    assert _noalloc(q, mlas[0], idx.to(dev), cnt.to(dev), w.topk) == B.DSA_OK
    assert _noalloc_status() == B.DSA_ERR_INVALID
    assert _noalloc_status() == B.DSA_OK
