"""Key-range sharding of one long sequence's decode over several GPUs.

Rank g of G holds the contiguous rows [row_begin_g, row_end_g) of one
sequence's indexer keys and latent cache.  One decode step for queries near
the end of the sequence:

  select   (per rank)  dsa_index_scores + dsa_topk on the shard, then
                       dsa_shard_candidates: <= topk (score, position) pairs
  exchange             all-gather of the candidates (16 KB per query per rank)
  merge    (per rank)  dsa_shard_merge: the global top-k of all candidates (ties
                       to the lower position) and this rank's part of it
  attend   (per rank)  dsa_sparse_mla_decode over that part of the shard
  exchange             all-gather of the partial outputs, lse and part counts
  combine  (per rank)  dsa_shard_combine: the log-sum-exp merge

Every step of the path runs in the library's kernels; this module only slices
the shards, calls the C ABI and moves the candidates and partial outputs with
torch.distributed collectives (NCCL on GPUs).  The phases are separate methods
so that one process can also run every rank's phases in turn on one GPU (the
exchange is then a concatenation); with a process group, `step` runs them with
all-gathers.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from dsa_indexer_top_b200 import binding as B


def shard_ranges(L: int, n_shards: int):
    """Contiguous, near-equal row ranges [begin, end) of an L-row sequence, in
    rank order (row counts differ by at most one; the first L % n ranks get the
    extra row)."""
    assert 1 <= n_shards <= L
    base, extra = divmod(L, n_shards)
    out, b = [], 0
    for g in range(n_shards):
        n = base + (1 if g < extra else 0)
        out.append((b, b + n))
        b += n
    return out


def local_positions(q_pos: torch.Tensor, begin: int, end: int) -> torch.Tensor:
    """Shard-relative positions of the queries: the last shard row each query
    sees.  Every query must see the shard (q_pos >= begin)."""
    if int(q_pos.min()) < begin:
        raise ValueError("sharded decode: every query must see every shard (q_pos >= the last shard's first row)")
    return (torch.clamp(q_pos, max=end - 1) - begin).to(torch.int32)


@dataclass
class ShardInputs:
    """One rank's inputs: the queries (replicated on every rank) and its shard."""
    q_pos: torch.Tensor          # int32 [n_q] sequence positions (device)
    q_idx: torch.Tensor          # [n_q, 32, 128] indexer queries
    w: torch.Tensor              # float32 [n_q, 32]
    k: torch.Tensor              # [rows, 128] this shard's indexer keys
    q_mla: torch.Tensor          # [n_q, 64, 576]
    kv: torch.Tensor             # [rows, 576] this shard's latent rows (or packed FP8 rows)
    d_lat: int
    scale: float


class ShardRank:
    """Buffers and the per-rank phases of one sharded decode step."""

    def __init__(self, rank: int, n_shards: int, L: int, n_q: int, topk: int, heads: int, d_lat: int, device):
        self.rank, self.n_shards, self.L, self.n_q, self.topk = rank, n_shards, L, n_q, topk
        self.begin, self.end = shard_ranges(L, n_shards)[rank]
        self.rows = self.end - self.begin
        dev = torch.device(device)
        self.dev = dev
        self.q_seq = torch.zeros(n_q, dtype=torch.int32, device=dev)
        qd = B.Queries(self.q_seq, self.q_seq, n_seq=1, max_ctx=self.rows)
        self.ws_sel = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, qd, topk, 1, dev)
        self.ws_merge = B.workspace(B.DSA_OP_SHARD_MERGE, qd, topk, n_shards, dev)
        self.scores = B.scores_buffer(n_q, self.rows, dev)
        self.idx_l = torch.empty((n_q, topk), dtype=torch.int32, device=dev)
        self.cnt_l = torch.empty((n_q,), dtype=torch.int32, device=dev)
        self.cand_score = torch.empty((n_q, topk), dtype=torch.float32, device=dev)
        self.cand_pos = torch.empty((n_q, topk), dtype=torch.int32, device=dev)
        self.idx = torch.empty((n_q, topk), dtype=torch.int32, device=dev)        # global selection
        self.cnt = torch.empty((n_q,), dtype=torch.int32, device=dev)
        self.local_idx = torch.empty((n_q, topk), dtype=torch.int32, device=dev)
        self.local_cnt = torch.empty((n_q,), dtype=torch.int32, device=dev)
        self.out_part = torch.empty((n_q, heads, d_lat), dtype=torch.bfloat16, device=dev)
        self.lse_part = torch.empty((n_q, heads), dtype=torch.float32, device=dev)

    def queries(self, q_pos: torch.Tensor) -> B.Queries:
        return B.Queries(self.q_seq, local_positions(q_pos, self.begin, self.end), n_seq=1, max_ctx=self.rows)

    def select(self, x: ShardInputs):
        """Local scores and top-k; returns this rank's candidates."""
        q = self.queries(x.q_pos)
        ix = B.Indexer(x.q_idx, x.w, x.k, flags=B.DSA_INDEXER_TOPK_HIST)
        B.dsa_index_scores(q, ix, self.scores, self.ws_sel)
        B.dsa_topk(q, self.scores, self.topk, self.idx_l, self.cnt_l, self.ws_sel,
                   flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        B.dsa_shard_candidates(q, self.scores, self.idx_l, self.cnt_l, self.topk, self.begin, self.cand_score,
                               self.cand_pos, self.ws_sel)
        return self.cand_score, self.cand_pos

    def merge_attend(self, x: ShardInputs, all_score: torch.Tensor, all_pos: torch.Tensor):
        """Global selection from the gathered candidates, then attention over this
        rank's part of it; returns the partial (out, lse, count)."""
        q = self.queries(x.q_pos)
        B.dsa_shard_merge(q, self.n_shards, all_score, all_pos, self.topk, self.begin, self.end, self.idx, self.cnt,
                          self.local_idx, self.local_cnt, self.ws_merge)
        m = B.Mla(x.q_mla, x.kv, self.out_part, x.d_lat, x.scale, self.lse_part)
        B.dsa_sparse_mla_decode(q, m, self.local_idx, self.local_cnt, self.topk, self.ws_sel)
        return self.out_part, self.lse_part, self.local_cnt

    def combine(self, x: ShardInputs, parts_out, parts_lse, parts_cnt, out: torch.Tensor,
                lse: Optional[torch.Tensor] = None):
        q = self.queries(x.q_pos)
        B.dsa_shard_combine(q, parts_out, parts_lse, parts_cnt, out, lse)

    def check_status(self):
        for ws in (self.ws_sel, self.ws_merge):
            st = B.dsa_check_status(ws)
            if st != B.DSA_OK:
                raise B.DsaError(st, f"sharded decode, rank {self.rank}")


def _all_gather(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    import torch.distributed as dist
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


def step(rank_state: ShardRank, x: ShardInputs, out: torch.Tensor, lse: Optional[torch.Tensor] = None, group=None):
    """One sharded decode step on this rank (every rank calls it, in the same
    order): select, all-gather candidates, merge + attend, all-gather partials,
    combine.  `out` receives the full attention output on every rank."""
    world = rank_state.n_shards
    cs, cp = rank_state.select(x)
    all_s, all_p = _all_gather(cs, world, group), _all_gather(cp, world, group)
    o, l, c = rank_state.merge_attend(x, all_s, all_p)
    all_o, all_l, all_c = _all_gather(o, world, group), _all_gather(l, world, group), _all_gather(c, world, group)
    rank_state.combine(x, all_o, all_l, all_c, out, lse)
    return rank_state.idx, rank_state.cnt
