"""Parity at the five named workloads' full sizes, in the call sequence the
benchmark times (dsa_index_scores -> dsa_topk -> sparse MLA per layer, decode
schedule up to 256 queries, prefill schedule above).  The GPU runs the whole
batch; the oracle recomputes sampled queries one by one (scores bit-exact over
every visible key, indices bit-exact, attention within tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu

SAMPLES = {
    "tiny": None,                       # every query
    "decode_32k": None,
    "prefill_64k": [0, 1, 2047, 4095],
    "indexshare_128k": [0, 31],
    "decode_1m": [2],
}


@pytest.mark.parametrize("name", wl.NAMED_ORDER)
def test_named_workload_full_size(cuda_ok, name):
    w = wl.NAMED[name]
    dev = torch.device("cuda")
    x = wl.make_inputs(w, device=dev)
    seq_run = w.n_q if len(set(w.q_seq)) == 1 else 1
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run)
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_index_scores(q, ix, scores, ws)
    B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
    mla = B.dsa_sparse_mla_decode if w.n_q <= 256 else B.dsa_sparse_mla_prefill
    for m in mlas:
        mla(q, m, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK

    rows = list(range(w.n_q)) if SAMPLES[name] is None else SAMPLES[name]
    for i in rows:
        b = 0 if w.shared_cache else w.q_seq[i]
        t = w.q_pos[i]
        k_h = x["k_idx"][b].cpu().float().numpy()[None]
        sc = oracle.index_scores(C.host_f32(x["q_idx"][i:i + 1]), C.host_f32(x["w"][i:i + 1]), k_h, [0], [t])
        got_sc = scores[i, : t + 1].cpu().double().numpy()
        np.testing.assert_array_equal(got_sc, sc[0, : t + 1], err_msg=f"scores of query {i}")
        ridx, rcnt = oracle.topk(sc, [t], w.topk)
        np.testing.assert_array_equal(idx[i].cpu().numpy(), ridx[0], err_msg=f"indices of query {i}")
        assert int(cnt[i]) == int(rcnt[0])
        sel = ridx[0, : rcnt[0]]
        for layer, m in enumerate(mlas):
            kv_rows = x["kv"][layer][b].cpu()[torch.from_numpy(sel.astype(np.int64))].float().numpy()[None]
            out, lse = oracle.sparse_mla(C.host_f32(x["q_mla"][layer][i:i + 1]), kv_rows, [0],
                                         np.arange(len(sel), dtype=np.int32)[None], rcnt, w.d_lat, w.scale)
            C.assert_attention_close(m.out[i:i + 1], out, w.dtype, f"query {i} layer {layer}")
            C.assert_lse_close(m.lse[i:i + 1], lse, w.dtype)


@pytest.mark.parametrize("name", ["decode_32k", "decode_1m"])
def test_fp8_indexer_full_size(cuda_ok, name):
    """FP8 (E4M3) indexer variant at full size with the fused histogram and the
    top-k, as the benchmark's --indexer-fp8 option runs it: scores bit-exact over
    every visible key and indices bit-exact for a sampled query."""
    w = wl.NAMED[name]
    dev = torch.device("cuda")
    x = wl.make_inputs(w, device=dev, layers=[])
    f8 = wl.fp8_indexer_inputs(w, x, device=dev)
    q, _, _ = C.descriptors(w, x, seq_run=1)
    ix = C.fp8_indexer(w, f8, x, flags=B.DSA_INDEXER_TOPK_HIST)
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_index_scores(q, ix, scores, ws)
    B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
    assert B.dsa_check_status(ws) == B.DSA_OK
    i = w.n_q - 1
    b, t = w.q_seq[i], w.q_pos[i]
    sc = oracle.index_scores_e4m3(f8["q8"][i:i + 1].view(torch.uint8).cpu().numpy(),
                                  f8["q_scale"][i:i + 1].cpu().numpy(), C.host_f32(x["w"][i:i + 1]),
                                  f8["k8"][b:b + 1].view(torch.uint8).cpu().numpy(),
                                  f8["k_scale"][b:b + 1].cpu().numpy(), [0], [t])
    np.testing.assert_array_equal(scores[i, : t + 1].cpu().double().numpy(), sc[0, : t + 1])
    ridx, rcnt = oracle.topk(sc, [t], w.topk)
    np.testing.assert_array_equal(idx[i].cpu().numpy(), ridx[0])
    assert int(cnt[i]) == int(rcnt[0])


@pytest.mark.parametrize("name", ["indexshare_128k", "decode_1m"])
def test_fp8_latent_cache_full_size(cuda_ok, name):
    """FP8 latent caches at full size, as the benchmark's --mla-fp8 option runs them
    (bf16 indexer with the fused histogram, top-k, decode attention on every layer's
    packed FP8 cache): indices bit-exact and every layer's attention within tolerance
    of the oracle for sampled queries."""
    w = wl.NAMED[name]
    dev = torch.device("cuda")
    x = wl.make_inputs(w, device=dev)
    kv8 = wl.fp8_latent_inputs(w, x, device=dev)
    q, ix, mlas = C.descriptors(w, x, seq_run=1)
    mlas = C.with_fp8_caches(w, mlas, kv8)
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_index_scores(q, ix, scores, ws)
    B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
    for m in mlas:
        B.dsa_sparse_mla_decode(q, m, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    for i in SAMPLES[name]:
        b, t = w.q_seq[i], w.q_pos[i]
        k_h = x["k_idx"][b].cpu().float().numpy()[None]
        sc = oracle.index_scores(C.host_f32(x["q_idx"][i:i + 1]), C.host_f32(x["w"][i:i + 1]), k_h, [0], [t])
        ridx, rcnt = oracle.topk(sc, [t], w.topk)
        np.testing.assert_array_equal(idx[i].cpu().numpy(), ridx[0], err_msg=f"indices of query {i}")
        sel = torch.from_numpy(ridx[0, : rcnt[0]].astype(np.int64))
        for layer, m in enumerate(mlas):
            rows = kv8[layer][b].cpu()[sel].numpy()[None]            # the selected packed rows only
            out, lse = oracle.sparse_mla_fp8(C.host_f32(x["q_mla"][layer][i:i + 1]), rows, [0],
                                             np.arange(len(sel), dtype=np.int32)[None], rcnt, w.d_lat, w.d_rope,
                                             w.scale)
            C.assert_attention_close(m.out[i:i + 1], out, "bf16", f"query {i} layer {layer}")
            C.assert_lse_close(m.lse[i:i + 1], lse, "bf16")
