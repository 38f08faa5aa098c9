"""Parity at the five named workloads' full sizes, in the call sequence the
benchmark times (dsa_index_scores -> dsa_topk -> sparse MLA per layer, decode
schedule up to 256 queries, prefill schedule above).  The GPU runs the whole
batch; the oracle recomputes every query of the decode workloads and, for the
prefill chunk, every 16th query plus the first and the last 64 (scores
bit-exact over every visible key, indices bit-exact, attention within
tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu

def _prefill_sample(n_q):
    """Every 16th query plus the first and the last 64."""
    return sorted(set(range(0, n_q, 16)) | set(range(64)) | set(range(n_q - 64, n_q)))


SAMPLES = {
    "tiny": None,                       # every query
    "decode_32k": None,
    "prefill_64k": _prefill_sample(4096),
    "indexshare_128k": None,            # all 32 queries, every layer
    "decode_1m": None,                  # all 4 queries
}


def check_rows(w, x, rows, scores, idx, cnt, mlas, kv8=None):
    """Oracle checks of the queries in `rows`, batched per sequence (the oracle
    spreads (query, key) pairs and (query, head) pairs over the host's cores):
    scores bit-exact over every visible key, indices and counts bit-exact, and
    every layer's attention (over the oracle's own selection) within tolerance."""
    rows = np.asarray(rows)
    q_seq = np.asarray(w.q_seq)[rows]
    q_pos = np.asarray(w.q_pos)[rows]
    seqs = [0] if w.shared_cache else sorted(set(q_seq.tolist()))
    got_idx = idx.cpu().numpy()
    got_cnt = cnt.cpu().numpy()
    batches = []
    for b in seqs:
        in_seq = rows if w.shared_cache else rows[q_seq == b]
        batches += [(b, in_seq[j: j + 64]) for j in range(0, len(in_seq), 64)]  # bounded host memory
    for b, sel_rows in batches:
        pos = np.asarray(w.q_pos)[sel_rows]
        k_h = x["k_idx"][b].cpu().float().numpy()[None]
        sc = oracle.index_scores(C.host_f32(x["q_idx"][sel_rows]), C.host_f32(x["w"][sel_rows]), k_h,
                                 np.zeros(len(sel_rows), np.int32), pos)
        del k_h
        if scores is not None:
            got_sc = scores[torch.from_numpy(sel_rows)].cpu().double().numpy()
            for j, i in enumerate(sel_rows):
                t = pos[j]
                np.testing.assert_array_equal(got_sc[j, : t + 1], sc[j, : t + 1], err_msg=f"scores of query {i}")
        ridx, rcnt = oracle.topk(sc, pos, w.topk)
        del sc
        np.testing.assert_array_equal(got_idx[sel_rows], ridx, err_msg=f"indices of sequence {b}")
        np.testing.assert_array_equal(got_cnt[sel_rows], rcnt)
        # attention over the selected rows only: [n, topk, row] gathered per query
        gidx = torch.from_numpy(np.where(ridx >= 0, ridx, 0).astype(np.int64))
        local = np.where(np.arange(w.topk)[None, :] < rcnt[:, None], np.arange(w.topk)[None, :], -1).astype(np.int32)
        for layer, m in enumerate(mlas):
            qm = C.host_f32(x["q_mla"][layer][sel_rows])
            if kv8 is None:
                cache = x["kv"][layer][b]
                rows_h = cache[gidx.to(cache.device)].cpu().float().numpy()
                out, lse = oracle.sparse_mla(qm, rows_h, np.arange(len(sel_rows), dtype=np.int32), local, rcnt,
                                             w.d_lat, w.scale)
            else:
                cache = kv8[layer][b]
                rows_h = cache[gidx.to(cache.device)].cpu().numpy()
                out, lse = oracle.sparse_mla_fp8(qm, rows_h, np.arange(len(sel_rows), dtype=np.int32), local, rcnt,
                                                 w.d_lat, w.d_rope, w.scale)
            sr = torch.from_numpy(sel_rows)
            C.assert_attention_close(m.out[sr], out, "bf16" if kv8 is not None else w.dtype,
                                     f"sequence {b} layer {layer}")
            C.assert_lse_close(m.lse[sr], lse, "bf16" if kv8 is not None else w.dtype)


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
    check_rows(w, x, rows, scores, idx, cnt, mlas)


@pytest.mark.parametrize("name", wl.NAMED_ORDER)
def test_named_workload_group_call_full_size(cuda_ok, name):
    """The same workloads through the one-call entry point the benchmark times
    (dsa_indexshare_group: scores in the workspace, decode schedule up to 256
    queries, prefill above): indices and attention against the oracle."""
    w = wl.NAMED[name]
    dev = torch.device("cuda")
    x = wl.make_inputs(w, device=dev)
    seq_run = w.n_q if len(set(w.q_seq)) == 1 else 1
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run)
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_indexshare_group(q, ix, mlas, w.topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    rows = list(range(w.n_q)) if SAMPLES[name] is None else SAMPLES[name][::4]
    check_rows(w, x, rows, None, idx, cnt, mlas)


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
    check_rows(w, x, list(range(w.n_q)), scores, idx, cnt, mlas, kv8=kv8)
