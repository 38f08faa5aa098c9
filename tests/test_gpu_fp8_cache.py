"""GPU parity of sparse MLA over packed FP8 latent caches (kv_dtype =
DSA_FP8_E4M3): 512 E4M3 codes, the bf16 RoPE key and a float32 scale per row.

Outputs are compared with the oracle's attention over the exact values
sigma * e4m3(code) (fp64) within the bf16 tolerances; selections come from the
indexer and stay bit-exact.  A second check compares the two cache formats: with
power-of-two scales every sigma * e4m3(code) is exact in bf16, so the bf16 path
reads the same values from an equivalent bf16 cache; the FP8 path (fp16 tiles,
sigma folded into an fp16 P) must be at least as close to the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu

D32 = wl.NAMED["decode_32k"]

GROUP_CASES = {
    # n > topk, n < topk, n == topk, n == topk + 1 in one batch
    "decode_edges": wl.scaled(D32, n_seq=4, L=3000, q_pos=(2999, 1500, 2047, 2048), q_seq=(0, 1, 2, 3)),
    # IndexShare group of 4 layers, each with its own FP8 cache
    "indexshare_small": wl.scaled(D32, n_seq=2, L=3000, q_pos=(2999, 2500), q_seq=(0, 1), n_layers=4, seed=12),
    # 40 queries of one sequence: the prefill schedule (one CTA per query)
    "prefill_small": wl.scaled(D32, n_seq=1, L=4173, q_pos=tuple(range(3000, 3040)), q_seq=(0,) * 40, seed=8),
    # every sequence reads one shared cache (sequence stride 0)
    "shared_cache": wl.scaled(D32, n_seq=3, L=2600, q_pos=(2599, 2400, 2100), q_seq=(0, 1, 2),
                              shared_cache=True, seed=10),
}


@pytest.fixture(scope="module")
def dev(cuda_ok):
    B.lib()
    return torch.device("cuda")


@pytest.mark.parametrize("decode", [True, False])
@pytest.mark.parametrize("topk,L", [(2048, 3000), (300, 1000), (100, 500), (4096, 5000)])
def test_fp8_cache_mla_alone(dev, decode, topk, L):
    """Random selections (ragged counts, chunks cut short) on both schedules."""
    w = wl.scaled(D32, n_seq=3, L=L, q_pos=(L - 1, L // 3, 5), q_seq=(2, 0, 1), topk=topk, seed=topk + 1)
    xh = wl.make_inputs(w, layers=[0])
    kv8h = wl.fp8_latent_inputs(w, xh)
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    mlas = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])
    idx, cnt = C.random_selection(w, seed=L + 1)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, topk, device=dev)
    (B.dsa_sparse_mla_decode if decode else B.dsa_sparse_mla_prefill)(q, mlas[0], idx.to(dev), cnt.to(dev), topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    out, lse = C.oracle_mla_fp8(w, xh, kv8h, 0, idx.numpy(), cnt.numpy())
    C.assert_attention_close(mlas[0].out, out, "bf16")
    C.assert_lse_close(mlas[0].lse, lse, "bf16")


@pytest.mark.parametrize("name", list(GROUP_CASES))
def test_fp8_cache_indexshare_group(dev, name):
    """dsa_indexshare_group with FP8 caches on every layer: the bf16 indexer's
    selection bit-exact, every layer's attention within tolerance."""
    w = GROUP_CASES[name]
    xh = wl.make_inputs(w)
    kv8h = wl.fp8_latent_inputs(w, xh)
    x = C.to_device(xh)
    seq_run = w.n_q if len(set(w.q_seq)) == 1 else 1
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run)
    mlas = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_indexshare_group(q, ix, mlas, w.topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    _, ridx, rcnt = C.oracle_selection(w, xh)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    for layer, m in enumerate(mlas):
        out, lse = C.oracle_mla_fp8(w, xh, kv8h, layer, ridx, rcnt)
        C.assert_attention_close(m.out, out, "bf16", f"layer {layer}")
        C.assert_lse_close(m.lse, lse, "bf16")


def test_fp8_indexer_and_fp8_cache_chain(dev):
    """Both FP8 variants in the three-call chain (scores with the fused histogram
    -> top-k -> decode attention), twice on one workspace."""
    w = GROUP_CASES["decode_edges"]
    xh = wl.make_inputs(w)
    f8h = wl.fp8_indexer_inputs(w, xh)
    kv8h = wl.fp8_latent_inputs(w, xh)
    x, f8 = C.to_device(xh), C.to_device(f8h)
    q, _, mlas = C.descriptors(w, x)
    mlas = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])
    ix = C.fp8_indexer(w, f8, x, flags=B.DSA_INDEXER_TOPK_HIST)
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    _, ridx, rcnt = C.oracle_selection_fp8(w, f8h, xh)
    out, lse = C.oracle_mla_fp8(w, xh, kv8h, 0, ridx, rcnt)
    for step in range(2):
        idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
        mlas[0].out.fill_(float("nan"))
        B.dsa_index_scores(q, ix, scores, ws)
        B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        B.dsa_sparse_mla_decode(q, mlas[0], idx, cnt, w.topk, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
        C.assert_attention_close(mlas[0].out, out, "bf16", f"step {step}")
        C.assert_lse_close(mlas[0].lse, lse, "bf16")


@pytest.mark.parametrize("decode", [True, False])
def test_fp8_cache_at_least_as_precise_as_bf16_cache(dev, decode):
    """Power-of-two row scales: sigma * e4m3(code) is exact in bf16, so the bf16
    path attends over exactly the FP8 cache's values.  Against the oracle, the FP8
    path (exact fp16 codes, sigma applied to the logits and folded into an fp16 P)
    is no less precise than the bf16 path (bf16 P), and both are within tolerance."""
    w = wl.scaled(D32, n_seq=2, L=2500, q_pos=(2499, 1000), q_seq=(0, 1), topk=2048, seed=31)
    xh = wl.make_inputs(w, layers=[0])
    kv8 = wl.fp8_latent_inputs(w, xh)[0]
    # 2^-8 .. 2^-7: about the recipe's amax / 448, so the latents keep their N(0, 1) size
    e = torch.randint(-8, -6, (w.n_seq, w.L, 1), generator=torch.Generator().manual_seed(32)).float()
    kv8[..., 640:644] = torch.pow(2.0, e).contiguous().view(torch.uint8)
    c = kv8[..., :512].contiguous().view(torch.float8_e4m3fn).float() * torch.pow(2.0, e)
    kv16 = torch.cat([c.to(torch.bfloat16), kv8[..., 512:640].contiguous().view(torch.bfloat16)], dim=-1)
    assert torch.equal(kv16[..., :512].float(), c)  # exact in bf16
    x = C.to_device(xh)
    x["kv"] = [kv16.to(dev)]
    q, _, mlas = C.descriptors(w, x)
    ref = mlas[0]
    idx, cnt = C.random_selection(w, seed=33, device=dev)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, w.topk, device=dev)
    call = B.dsa_sparse_mla_decode if decode else B.dsa_sparse_mla_prefill
    call(q, ref, idx, cnt, w.topk, ws)
    out = torch.full_like(ref.out, float("nan"))
    lse = torch.full_like(ref.lse, float("nan"))
    got = B.Mla(ref.q, kv8.to(dev), out, w.d_lat, w.scale, lse)
    call(q, got, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    o_ref, l_ref = C.oracle_mla_fp8(w, xh, [kv8], 0, idx.cpu().numpy(), cnt.cpu().numpy())
    C.assert_attention_close(out, o_ref, "bf16", "fp8 cache")
    C.assert_attention_close(ref.out, o_ref, "bf16", "bf16 cache")
    e8 = np.abs(out.float().cpu().numpy() - o_ref)
    e16 = np.abs(ref.out.float().cpu().numpy() - o_ref)
    assert e8.max() <= e16.max() * 1.05 and e8.mean() <= e16.mean() * 1.05, (e8.max(), e16.max(), e8.mean(), e16.mean())
    C.assert_lse_close(lse, l_ref, "bf16")


def test_fp8_cache_precision_margin(dev):
    """The FP8 cache's worst error on a decode batch at GLM-5.2 shapes, with the
    workload recipe's scales (amax / 448, not powers of two): well inside the
    bf16 tolerance (measured max-abs is stated in the design notes)."""
    w = wl.scaled(D32, n_seq=4, L=8000, q_pos=(7999, 7000, 5000, 3000), q_seq=(0, 1, 2, 3), topk=2048, seed=34)
    xh = wl.make_inputs(w, layers=[0])
    kv8h = wl.fp8_latent_inputs(w, xh)
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    m = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])[0]
    idx, cnt = C.random_selection(w, seed=35, device=dev)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, w.topk, device=dev)
    B.dsa_sparse_mla_decode(q, m, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    o_ref, _ = C.oracle_mla_fp8(w, xh, kv8h, 0, idx.cpu().numpy(), cnt.cpu().numpy())
    err = np.abs(m.out.float().cpu().numpy() - o_ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())


def test_fp8_cache_noalloc(dev):
    """The no-workspace decode entry point reads packed FP8 caches too."""
    w = wl.scaled(D32, n_seq=3, L=4000, q_pos=(3999, 2000, 700), q_seq=(1, 2, 0), topk=2048, seed=41)
    xh = wl.make_inputs(w, layers=[0])
    kv8h = wl.fp8_latent_inputs(w, xh)
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    m = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])[0]
    idx, cnt = C.random_selection(w, seed=42)
    idx_d, cnt_d = idx.to(dev), cnt.to(dev)
    fn = B.lib().dsa_sparse_mla_decode_noalloc
    fn.argtypes = [ctypes.POINTER(B._Queries), ctypes.POINTER(B._Mla), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    qc, mc = q.c(), m.c()
    st = fn(ctypes.byref(qc), ctypes.byref(mc), idx_d.data_ptr(), cnt_d.data_ptr(), w.topk,
            torch.cuda.current_stream().cuda_stream)
    assert st == B.DSA_OK, B.status_str(st)
    torch.cuda.synchronize()
    out, lse = C.oracle_mla_fp8(w, xh, kv8h, 0, idx.numpy(), cnt.numpy())
    C.assert_attention_close(m.out, out, "bf16")
    C.assert_lse_close(m.lse, lse, "bf16")


def test_fp8_cache_unsupported_shapes(dev):
    """Packed FP8 caches run on the tensor-core shape only: fp32 queries are
    rejected before any launch."""
    w = wl.scaled(D32, n_seq=1, L=300, q_pos=(299,), q_seq=(0,), topk=64, seed=51)
    xh = wl.make_inputs(w, layers=[0])
    kv8 = wl.fp8_latent_inputs(w, xh)[0].to(dev)
    x = C.to_device(xh)
    q, _, _ = C.descriptors(w, x)
    qf = x["q_mla"][0].float()
    out = torch.empty((1, 64, 512), dtype=torch.float32, device=dev)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, w.topk, device=dev)
    idx = torch.arange(64, dtype=torch.int32, device=dev)[None]
    cnt = torch.full((1,), 64, dtype=torch.int32, device=dev)
    with pytest.raises(B.DsaError) as e:
        B.dsa_sparse_mla_prefill(q, B.Mla(qf, kv8, out, 512, w.scale), idx, cnt, w.topk, ws)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
