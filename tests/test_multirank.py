"""The benchmark's multi-process logic on CPU: two gloo ranks, each with its own
timing, agree on the max over ranks and on the whole-job (weak-scaling) value."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is slower
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        v = bench.weak_scaling_value(world, n_q=8, n_layers=1, steps=100, tot_ms_max=m)
        bench.barrier(world)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_value():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1]
    m, v = out[0]
    assert m == 15.0
    # 2 ranks x 8 queries x 1 layer x 100 steps in 15 ms
    assert v == pytest.approx(2 * 8 * 100 / 0.015)


def test_single_rank_value_and_max_are_local():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_value(1, 4, 4, 10, 2.0) == pytest.approx(4 * 4 * 10 / 0.002)


# ------------------------------------------------------------------ key-range shards
class _OracleShardRank:
    """The per-rank phases of dsa_indexer_top_b200.sharded.ShardRank written with
    the oracle on the CPU (the same contracts: local top-k candidates with
    sequence positions; the merge = top-k of the rank-ordered candidate list,
    ties to the lower position; the local part of the selection; attention over
    it; the log-sum-exp combine), so that the collective orchestration in
    sharded.step can run on gloo ranks without a GPU."""

    def __init__(self, rank, n_shards, L, topk):
        from dsa_indexer_top_b200 import sharded as S
        self.rank, self.n_shards, self.topk = rank, n_shards, topk
        self.begin, self.end = S.shard_ranges(L, n_shards)[rank]

    def select(self, x):
        import numpy as np
        import oracle
        pos_l = np.minimum(x["q_pos"], self.end - 1) - self.begin
        k = x["k"][self.begin:self.end][None]
        sc = oracle.index_scores(x["q_idx"], x["w"], k, np.zeros(len(pos_l), np.int32), pos_l)
        idx, cnt = oracle.topk(sc, pos_l, self.topk)
        cs = np.zeros(idx.shape, np.float32)
        cp = np.full(idx.shape, -1, np.int32)
        for i in range(len(cnt)):
            sel = idx[i, : cnt[i]]
            cs[i, : cnt[i]] = sc[i, sel]
            cp[i, : cnt[i]] = sel + self.begin
        return torch.from_numpy(cs), torch.from_numpy(cp)

    def merge_attend(self, x, all_s, all_p):
        import numpy as np
        import oracle
        all_s, all_p = all_s.numpy(), all_p.numpy()
        n_q = all_s.shape[1]
        width = self.n_shards * self.topk
        ms = np.zeros((n_q, width))
        mp = np.full((n_q, width), -1, np.int64)
        last = np.zeros(n_q, np.int32)
        for i in range(n_q):
            keep = all_p[:, i, :].reshape(-1) >= 0           # rank order = position order
            n = int(keep.sum())
            ms[i, :n] = all_s[:, i, :].reshape(-1)[keep]
            mp[i, :n] = all_p[:, i, :].reshape(-1)[keep]
            last[i] = n - 1
        sel, cnt = oracle.topk(ms, last, self.topk)
        self.idx = np.full((n_q, self.topk), -1, np.int32)
        loc = np.full((n_q, self.topk), -1, np.int32)
        lcnt = np.zeros(n_q, np.int32)
        for i in range(n_q):
            g = mp[i, sel[i, : cnt[i]]]
            self.idx[i, : cnt[i]] = g
            mine = g[(g >= self.begin) & (g < self.end)] - self.begin
            loc[i, : len(mine)] = mine
            lcnt[i] = len(mine)
        self.cnt = cnt
        kv = x["kv"][self.begin:self.end][None]
        o, l = oracle.sparse_mla(x["q_mla"], kv, np.zeros(n_q, np.int32), loc, lcnt, x["d_lat"], x["scale"])
        return torch.from_numpy(o), torch.from_numpy(l), torch.from_numpy(lcnt)

    def combine(self, x, po, pl, pc, out, lse=None):
        import numpy as np
        po, pl, pc = po.numpy(), pl.numpy(), pc.numpy()
        lw = np.where(pc[:, :, None] > 0, pl, -np.inf)                       # [parts, n_q, heads]
        m = lw.max(0)
        wts = np.exp(lw - m)
        s = wts.sum(0)
        out.copy_(torch.from_numpy((wts[..., None] * po).sum(0) / s[..., None]))
        if lse is not None:
            lse.copy_(torch.from_numpy(m + np.log(s)))


def _shard_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        from dsa_indexer_top_b200 import sharded as S
        rng = np.random.default_rng(5)            # the same inputs on every rank
        L, n_q, topk, H, d_lat, d_rope = 700, 3, 64, 4, 16, 8
        x = {"q_pos": np.array([699, 690, 650], np.int32),
             "q_idx": rng.integers(-3, 4, (n_q, 4, 8)).astype(np.float32),
             "w": (2.0 ** rng.integers(-2, 2, (n_q, 4))).astype(np.float32),
             "k": rng.integers(-3, 4, (L, 8)).astype(np.float32),
             "q_mla": rng.standard_normal((n_q, H, d_lat + d_rope)).astype(np.float32),
             "kv": rng.standard_normal((L, d_lat + d_rope)).astype(np.float32), "d_lat": d_lat, "scale": 0.2}
        r = _OracleShardRank(rank, world, L, topk)
        o = torch.empty((n_q, H, d_lat), dtype=torch.float64)
        lse = torch.empty((n_q, H), dtype=torch.float64)
        idx, cnt = S.step(r, x, o, lse)
        out[rank] = (idx, cnt, o.numpy(), lse.numpy(), x)
    finally:
        dist.destroy_process_group()


def test_sharded_decode_two_gloo_ranks_equals_unsharded():
    """Two gloo ranks, each holding half of a 700-row sequence, run the sharded
    step (candidates all-gathered, merged with the tie rule, partial attention
    all-gathered and combined): both end with the unsharded top-k and attention."""
    import numpy as np
    import oracle
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_shard_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    x = out[0][4]
    n_q = len(x["q_pos"])
    sc = oracle.index_scores(x["q_idx"], x["w"], x["k"][None], np.zeros(n_q, np.int32), x["q_pos"])
    ridx, rcnt = oracle.topk(sc, x["q_pos"], 64)
    o_ref, l_ref = oracle.sparse_mla(x["q_mla"], x["kv"][None], np.zeros(n_q, np.int32), ridx, rcnt, x["d_lat"],
                                     x["scale"])
    for rank in range(world):
        idx, cnt, o, lse, _ = out[rank]
        np.testing.assert_array_equal(idx, ridx)
        np.testing.assert_array_equal(cnt, rcnt)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_shard_ranges_cover_the_sequence_in_order():
    from dsa_indexer_top_b200 import sharded as S
    for L, G in [(10, 3), (1 << 20, 8), (7, 7), (100, 1)]:
        r = S.shard_ranges(L, G)
        assert r[0][0] == 0 and r[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        sizes = [e - b for b, e in r]
        assert max(sizes) - min(sizes) <= 1
