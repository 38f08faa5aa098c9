"""Property tests on random small shapes (Hypothesis, derandomized so every run
draws the same cases).

CPU: the oracle's top-k against numpy's stable argsort, its indexer against
the ReLU identity (a plain matmul), and its FP8-latent attention against plain
softmax attention on the exact latents, on random shapes and values.
GPU: the whole chain (indexer -> top-k -> sparse MLA, decode and prefill
schedules, with and without the fused histogram) on random contexts, positions,
batch sizes and top-k sizes; indices bit-exact and outputs within tolerance of
the oracle."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

CPU_SETTINGS = settings(max_examples=40, derandomize=True, deadline=None,
                        suppress_health_check=[HealthCheck.too_slow])
GPU_SETTINGS = settings(max_examples=16, derandomize=True, deadline=None,
                        suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


@CPU_SETTINGS
@given(n_q=st.integers(1, 4), L=st.integers(1, 300), k=st.integers(1, 64), seed=st.integers(0, 2**31 - 1),
       ties=st.booleans())
def test_oracle_topk_is_stable_argsort(n_q, L, k, seed, ties):
    g = np.random.default_rng(seed)
    scores = (g.integers(-3, 4, (n_q, L)) if ties else g.standard_normal((n_q, L))).astype(np.float64)
    q_pos = g.integers(0, L, n_q).astype(np.int32)
    idx, cnt = oracle.topk(scores, q_pos, k)
    for i in range(n_q):
        n = q_pos[i] + 1
        kk = min(k, n)
        order = np.argsort(-scores[i, :n], kind="stable")[:kk]
        assert cnt[i] == kk
        np.testing.assert_array_equal(idx[i, :kk], np.sort(order))
        assert np.all(idx[i, kk:] == -1)


@CPU_SETTINGS
@given(heads=st.integers(1, 6), dim=st.integers(1, 20), L=st.integers(1, 40), seed=st.integers(0, 2**31 - 1))
def test_oracle_indexer_is_relu_of_a_matmul(heads, dim, L, seed):
    g = np.random.default_rng(seed)
    q = g.integers(-4, 5, (2, heads, dim)).astype(np.float32)
    w = np.exp2(g.integers(-3, 2, (2, heads))).astype(np.float32)
    k = g.integers(-4, 5, (1, L, dim)).astype(np.float32)
    q_pos = np.array([L - 1, (L - 1) // 2], dtype=np.int32)
    got = oracle.index_scores(q, w, k, [0, 0], q_pos)
    for i in range(2):
        dots = q[i].astype(np.float64) @ k[0].astype(np.float64).T          # [heads, L]
        ref = (w[i][:, None] * (dots + np.abs(dots)) / 2).sum(0)
        t = q_pos[i]
        np.testing.assert_array_equal(got[i, : t + 1], ref[: t + 1])


@CPU_SETTINGS
@given(heads=st.integers(1, 4), d_lat=st.sampled_from([4, 8, 16, 32]), d_rope=st.integers(0, 8),
       L=st.integers(1, 30), k=st.integers(1, 12), seed=st.integers(0, 2**31 - 1))
def test_oracle_fp8_latent_attention_is_softmax_attention(heads, d_lat, d_rope, L, k, seed):
    """The FP8-cache oracle on random packed rows (any codes but NaN, any positive
    scale) equals a plain float64 softmax attention over the exact latents, which
    torch's own float8 / bf16 decoding gives."""
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 256, (1, L, d_lat), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                      # no NaN codes (0x38 is 1.0)
    sigma = torch.exp2(torch.rand((1, L), generator=g) * 12 - 10)
    rope = torch.randn((1, L, d_rope), generator=g).to(torch.bfloat16)
    rb = wl.fp8_row_bytes(d_lat, d_rope)
    rows = torch.zeros((1, L, rb), dtype=torch.uint8)
    rows[..., :d_lat] = codes
    rows[..., d_lat: d_lat + 2 * d_rope] = rope.view(torch.uint8)
    rows[..., d_lat + 2 * d_rope: d_lat + 2 * d_rope + 4] = sigma.contiguous().unsqueeze(-1).view(torch.uint8)
    c = codes.view(torch.float8_e4m3fn).double() * sigma.double()[..., None]
    kv = torch.cat([c, rope.double()], -1)[0].numpy()
    q = torch.randn((1, heads, d_lat + d_rope), generator=g).numpy().astype(np.float32) * 0.05
    n = L
    kk = min(k, n)
    sel = np.sort(np.random.default_rng(seed).choice(n, size=kk, replace=False)).astype(np.int32)
    idx = np.full((1, k), -1, np.int32)
    idx[0, :kk] = sel
    scale = 0.3
    out, lse = oracle.sparse_mla_fp8(q, rows.numpy(), [0], idx, [kk], d_lat, d_rope, scale)
    logits = scale * (q[0].astype(np.float64) @ kv[sel].T)               # [heads, kk]
    m = logits.max(1, keepdims=True)
    p = np.exp(logits - m)
    ref = (p / p.sum(1, keepdims=True)) @ kv[sel, :d_lat]
    scale_out = max(1.0, float(np.abs(kv[sel, :d_lat]).max()))
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12 * scale_out)
    np.testing.assert_allclose(lse[0], m[:, 0] + np.log(p.sum(1)), rtol=0, atol=1e-11 * max(1.0, float(np.abs(m).max())))


@pytest.mark.gpu
@GPU_SETTINGS
@given(n_seq=st.integers(1, 4), L=st.integers(1, 3000), topk=st.sampled_from([1, 7, 64, 500, 2048]),
       frac=st.lists(st.floats(0.0, 1.0), min_size=4, max_size=4), seed=st.integers(1, 10**6),
       fused=st.booleans(), decode=st.booleans())
def test_chain_random_shapes(cuda_ok, n_seq, L, topk, frac, seed, fused, decode):
    q_pos = tuple(int(round(f * (L - 1))) for f in frac[:n_seq])
    w = wl.scaled(wl.NAMED["decode_32k"], n_seq=n_seq, L=L, q_pos=q_pos, q_seq=tuple(range(n_seq)), topk=topk,
                  seed=seed)
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    q, ix, mlas = C.descriptors(w, x, seq_run=1)
    if fused:
        ix.flags = B.DSA_INDEXER_TOPK_HIST
    dev = x["q_pos"].device
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
    B.dsa_index_scores(q, ix, scores, ws)
    B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER if fused else 0)
    for m in mlas:
        (B.dsa_sparse_mla_decode if decode else B.dsa_sparse_mla_prefill)(q, m, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    _, ridx, rcnt = C.oracle_selection(w, xh)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    out, lse = C.oracle_mla(w, xh, 0, ridx, rcnt)
    C.assert_attention_close(mlas[0].out, out, w.dtype, "out")
    C.assert_lse_close(mlas[0].lse, lse, w.dtype)
