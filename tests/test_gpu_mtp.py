"""dsa_sparse_mla_mtp -- multi-token-prediction iterations share one selection
("GLM-5.2 -- LLM atlas", raw config.json fields: index_share_for_mtp_iteration):
the D queries of a group (a sequence's base token and its draft tokens) attend
over the selection made for the base token.  Through the C ABI against the
oracle's sparse_mla_mtp, on bf16 and packed FP8 caches, on the decode (split-K)
and prefill schedules, and as a chain: the indexer and top-k select for the
base tokens, then every token of the group attends."""
import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu
D32 = wl.NAMED["decode_32k"]


def _mtp_workload(n_g, D, L, topk, seed):
    """Group g: base position t_g, queries at t_g .. t_g + D - 1 of sequence g."""
    base = [L - D - (g * 613) % (L // 3) for g in range(n_g)]
    pos = tuple(b + d for b in base for d in range(D))
    seq = tuple(g for g in range(n_g) for _ in range(D))
    return wl.scaled(D32, n_seq=n_g, L=L, q_pos=pos, q_seq=seq, topk=topk, seed=seed), base


def _group_selection(base, L, topk, seed):
    rng = np.random.default_rng(seed)
    idx = np.full((len(base), topk), -1, dtype=np.int32)
    cnt = np.zeros(len(base), dtype=np.int32)
    for g, t in enumerate(base):
        k = min(topk, t + 1)
        idx[g, :k] = np.sort(rng.choice(t + 1, size=k, replace=False)) if t + 1 > k else np.arange(k)
        cnt[g] = k
    return idx, cnt


@pytest.mark.parametrize("n_g,D,L,topk,fp8", [
    (4, 2, 5000, 2048, False),     # decode plan, 8 queries, two per selection
    (3, 3, 2700, 1024, False),     # ragged tails, odd group size
    (2, 4, 9000, 2048, True),      # packed FP8 cache
    (66, 4, 1200, 256, False),     # 264 queries: the prefill schedule
])
def test_mtp_attention_matches_oracle(cuda_ok, n_g, D, L, topk, fp8):
    dev = torch.device("cuda")
    w, base = _mtp_workload(n_g, D, L, topk, seed=70 + D)
    xh = wl.make_inputs(w, layers=[0])
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    m = mlas[0]
    kv8h = None
    if fp8:
        kv8h = wl.fp8_latent_inputs(w, xh)
        m = C.with_fp8_caches(w, mlas, [t.to(dev) for t in kv8h])[0]
    idx, cnt = _group_selection(base, L, topk, seed=80 + D)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, topk, device=dev)
    B.dsa_sparse_mla_mtp(q, m, torch.from_numpy(idx).to(dev), torch.from_numpy(cnt).to(dev), topk, D, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    q_seq = xh["q_seq"].numpy()
    if fp8:
        rep_idx, rep_cnt = np.repeat(idx, D, axis=0), np.repeat(cnt, D)
        out, lse = oracle.sparse_mla_fp8(C.host_f32(xh["q_mla"][0]), kv8h[0].numpy(), q_seq, rep_idx, rep_cnt,
                                         w.d_lat, w.d_rope, w.scale)
    else:
        out, lse = oracle.sparse_mla_mtp(C.host_f32(xh["q_mla"][0]), C.host_f32(xh["kv"][0]), q_seq, idx, cnt, D,
                                         w.d_lat, w.scale)
    C.assert_attention_close(m.out, out, "bf16")
    C.assert_lse_close(m.lse, lse, "bf16")


def test_mtp_chain_selects_once_per_group(cuda_ok):
    """Indexer and top-k on the base tokens only, then all D tokens of each group
    attend over that selection; indices bit-exact, attention within tolerance."""
    dev = torch.device("cuda")
    n_g, D, L, topk = 4, 3, 6000, 2048
    w, base = _mtp_workload(n_g, D, L, topk, seed=91)
    xh = wl.make_inputs(w, layers=[0])
    x = C.to_device(xh)
    q_all, _, mlas = C.descriptors(w, x)
    rows = torch.arange(0, n_g * D, D)
    wb = wl.scaled(w, q_pos=tuple(base), q_seq=tuple(range(n_g)))
    qb = B.Queries(x["q_seq"][rows.to(dev)].contiguous(), x["q_pos"][rows.to(dev)].contiguous(), n_seq=n_g,
                   max_ctx=L)
    ix = B.Indexer(x["q_idx"][rows.to(dev)].contiguous(), x["w"][rows.to(dev)].contiguous(), x["k_idx"],
                   flags=B.DSA_INDEXER_TOPK_HIST)
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q_all, topk, 1, dev)
    scores = B.scores_buffer(n_g, L, dev)
    idx = torch.empty((n_g, topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((n_g,), dtype=torch.int32, device=dev)
    B.dsa_index_scores(qb, ix, scores, ws)
    B.dsa_topk(qb, scores, topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
    B.dsa_sparse_mla_mtp(q_all, mlas[0], idx, cnt, topk, D, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    xb = {"q_idx": xh["q_idx"][rows], "w": xh["w"][rows], "k_idx": xh["k_idx"],
          "q_seq": torch.arange(n_g, dtype=torch.int32), "q_pos": torch.tensor(base, dtype=torch.int32)}
    _, ridx, rcnt = C.oracle_selection(wb, xb)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    out, lse = oracle.sparse_mla_mtp(C.host_f32(xh["q_mla"][0]), C.host_f32(xh["kv"][0]), xh["q_seq"].numpy(), ridx,
                                     rcnt, D, w.d_lat, w.scale)
    C.assert_attention_close(mlas[0].out, out, "bf16")
    C.assert_lse_close(mlas[0].lse, lse, "bf16")


def test_mtp_rejects_group_size_not_dividing_queries(cuda_ok):
    dev = torch.device("cuda")
    w, base = _mtp_workload(2, 2, 800, 64, seed=99)
    x = C.to_device(wl.make_inputs(w, layers=[0]))
    q, _, mlas = C.descriptors(w, x)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, 64, device=dev)
    idx = torch.zeros((2, 64), dtype=torch.int32, device=dev)
    cnt = torch.ones(2, dtype=torch.int32, device=dev)
    for bad in (0, 3):
        with pytest.raises(B.DsaError) as e:
            B.dsa_sparse_mla_mtp(q, mlas[0], idx, cnt, 64, bad, ws)
        assert e.value.status == B.DSA_ERR_INVALID
