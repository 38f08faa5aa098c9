"""Key-range sharding of one long sequence, G ranks emulated in one process on
one GPU: every rank's phases run through the C ABI in turn (select, merge +
attend, combine) and the all-gathers become concatenations.  The global
selection must be bit-identical to the oracle's top-k over the whole sequence
on every rank, and the combined attention within tolerance of the oracle's
attention over it."""
import numpy as np
import pytest
import torch

from dsa_indexer_top_b200 import sharded as S
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu
D32 = wl.NAMED["decode_32k"]


@pytest.mark.parametrize("L,G,topk", [
    (20000, 2, 2048),
    (20001, 3, 2048),     # uneven shards
    (5000, 4, 2048),      # shards shorter than topk: each keeps all its visible rows
    (40000, 8, 1024),
])
def test_sharded_decode_matches_oracle(cuda_ok, L, G, topk):
    dev = torch.device("cuda")
    pos = (L - 1, L - 3, L - 1 - (L // G) // 2)      # every query sees the last shard
    w = wl.scaled(D32, n_seq=1, L=L, q_pos=pos, q_seq=(0, 0, 0), topk=topk, seed=L % 97 + G)
    xh = wl.make_inputs(w, layers=[0])
    x = C.to_device(xh)
    n_q = w.n_q
    ranks = [S.ShardRank(g, G, L, n_q, topk, 64, 512, dev) for g in range(G)]
    ins = [S.ShardInputs(x["q_pos"], x["q_idx"], x["w"], x["k_idx"][0, r.begin:r.end], x["q_mla"][0],
                         x["kv"][0][0, r.begin:r.end], w.d_lat, w.scale) for r in ranks]
    cands = [r.select(xi) for r, xi in zip(ranks, ins)]
    all_s = torch.stack([c[0].clone() for c in cands])
    all_p = torch.stack([c[1].clone() for c in cands])
    parts = [r.merge_attend(xi, all_s, all_p) for r, xi in zip(ranks, ins)]
    po = torch.stack([p[0].clone() for p in parts])
    pl = torch.stack([p[1].clone() for p in parts])
    pc = torch.stack([p[2].clone() for p in parts])
    out = torch.empty((n_q, 64, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((n_q, 64), dtype=torch.float32, device=dev)
    ranks[0].combine(ins[0], po, pl, pc, out, lse)
    for r in ranks:
        r.check_status()

    _, ridx, rcnt = C.oracle_selection(w, xh)
    for r in ranks:  # every rank holds the same global selection
        np.testing.assert_array_equal(r.idx.cpu().numpy(), ridx, err_msg=f"rank {r.rank}")
        np.testing.assert_array_equal(r.cnt.cpu().numpy(), rcnt)
    assert int(pc.sum()) == int(rcnt.sum())  # the ranks' parts cover the selection once
    o_ref, l_ref = C.oracle_mla(w, xh, 0, ridx, rcnt)
    C.assert_attention_close(out, o_ref, "bf16")
    C.assert_lse_close(lse, l_ref, "bf16")
