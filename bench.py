"""Benchmark of the DSA hot path: query-tokens/s per layer and % of HBM roofline.

One step = one pass of the whole path over one batch of synthetic inputs already
resident in HBM, made by ONE call of the public C ABI: dsa_indexshare_group
(indexer -> top-k -> sparse MLA of every layer of the workload; with one layer it
is the plain full-layer step).  The step is captured once in a CUDA graph with
CUDA events at its two ends; L2 is flushed before every timed step (a 256 MB
write, then a 256 MB read, so that no dirty line is written back inside the
timed region).  A second graph made of the separate calls (dsa_index_scores, dsa_topk,
dsa_sparse_mla_*) with events between them gives the per-stage breakdown and the
per-kernel rooflines.  After timing, the results of the timed graph are compared
bitwise with one eager step on a freshly initialised workspace and with the
separate calls' results (`self_check`).

The headline line is the 4 x 1,048,576 decode (the configuration the HBM
roofline target is set on).  The same JSON line carries, under `per_config`,
the other named workloads (tiny, decode 8 x 32K, prefill 4096 x 64K, IndexShare
4 x 32 x 128K) and the FP8 variants of the two long-context decodes, each with
its own value, step time, breakdown, rooflines and self-check.

`e2e` times the same step end to end through the public API with host buffers,
eagerly, every step: one dsa_indexshare_group_host call copies the step's query
inputs from pinned host memory, runs the group call (argument checks, tensor-map
encoding, launches) and copies the outputs and indices back to pinned host memory.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode_1m]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

With N > 1 (torchrun, one process per GPU) every rank runs its own batch of each
workload (independent sequences, no collective on the data path: weak scaling);
times are the max over ranks and `value` counts every rank's queries.
"""
from __future__ import annotations

import argparse
import gc
import json
import os
import statistics
import subprocess
import threading
import time

import numpy as np
import torch

from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl

METRIC = "query-tokens/s per layer (indexer+top-k+sparse MLA); % of HBM roofline"
UNIT = "qtok/s/layer"
ROOT = os.path.dirname(os.path.abspath(__file__))
DECODE_MAX_QUERIES = 256    # the group call's MLA uses the decode (split-K) schedule up to this many queries
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Before every timed step: write a 256 MB buffer (evicts everything the
    previous step left in the 126 MB L2), then read a second 256 MB buffer, so the
    dirty lines of the write are written back here, outside the timed region, and
    the step starts with an L2 of clean lines that hold none of its data."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def fill_(self, v):
        self.w.fill_(v)
        self.r.amax()
REFERENCE_BUDGET_S = 120.0  # timed oracle work of one --impl reference run
HEADLINE = "decode_1m"
# the other workloads reported inside the headline line, with the FP8 variants
# (indexer keys and latent cache both in E4M3) of the two long-context decodes
PER_CONFIG = [("decode_32k", False), ("prefill_64k", False), ("indexshare_128k", False), ("tiny", False),
              ("decode_1m", True), ("indexshare_128k", True)]
PER_CONFIG_MAX_STEPS = 50

# dram__bytes_read.sum + dram__bytes_write.sum of one launch of a stage's kernels
# (workload, stage, fp8) -> bytes, from one-kernel ncu captures of the current
# kernels on the one-query case of the workload (`--n-seq 1`), times its 4
# queries: every term of a decode stage's traffic grows with the queries (keys and
# scores per sequence, selected rows, split-K partials).  The captures are cold
# (ncu flushes the caches), so the attention's entry includes re-reading its
# split-K partials, which stay in L2 inside a step.  Entries are removed when a
# kernel changes; missing entries report null.
NCU_TRAFFIC: dict = {
    ("decode_1m", "index_scores", False): 4 * (268_491_008 + 5_246_720),
    ("decode_1m", "index_scores", True): 4 * (138_483_712 + 4_256_768),
    ("decode_1m", "topk", False): 4 * 4_322_816,
    ("decode_1m", "sparse_mla", False): 4 * (2_502_400 + 2_118_400),   # mla_tc + mla_combine
    ("decode_1m", "sparse_mla", True): 4 * (1_728_768 + 2_118_400),
}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------ algorithmic bytes / flops
def path_bytes(w: wl.Workload, indexer_fp8: bool = False, mla_fp8: bool = False):
    """Algorithmic HBM bytes of one step (each input byte once, outputs once).
    indexer_fp8: E4M3 indexer keys and queries (1 byte per value) plus a float32
    scale per key and per (query, head).  mla_fp8: each selected cache row is one
    packed 656-byte FP8 row (codes, bf16 RoPE key, scale, padding)."""
    vis = np.array(w.q_pos, dtype=np.int64) + 1
    seqs = {}
    for s, t in zip(w.q_seq, w.q_pos):
        key = 0 if w.shared_cache else s
        seqs[key] = max(seqs.get(key, 0), t + 1)
    key_rows = sum(seqs.values())
    eb = w.elem_bytes
    key_b = w.idx_dim + 4 if indexer_fp8 else w.idx_dim * eb             # per key row
    qry_b = w.idx_dim + 8 if indexer_fp8 else w.idx_dim * eb + 4         # per (query, head): q, w (+ scale)
    idx_in = key_rows * key_b + w.n_q * w.idx_heads * qry_b
    idx_out = int(vis.sum()) * 4
    cnt = np.minimum(vis, w.topk)
    row_b = wl.fp8_row_bytes(w.d_lat, w.d_rope) if mla_fp8 else (w.d_lat + w.d_rope) * eb
    rows = int(cnt.sum()) * row_b
    q_out = w.n_q * w.mla_heads * ((w.d_lat + w.d_rope) * eb + w.d_lat * eb + 4)
    return {
        "indexer": idx_in + idx_out,
        "topk": idx_out + w.n_q * (w.topk + 1) * 4,
        "mla": w.n_layers * (rows + q_out),
        # the path's roofline bytes: indexer keys + gathered rows + q/out
        "path": key_rows * key_b + w.n_layers * (rows + q_out) + w.n_q * w.idx_heads * qry_b,
    }


def path_flops(w: wl.Workload):
    """Tensor-core FLOPs of a step: the indexer's q.k products over every visible
    key, and the MLA's S (576-deep) and O (512-deep) products over the selection."""
    vis = np.array(w.q_pos, dtype=np.int64) + 1
    cnt = np.minimum(vis, w.topk)
    idx = 2 * w.idx_heads * w.idx_dim * int(vis.sum())
    mla = 2 * w.mla_heads * (2 * w.d_lat + w.d_rope) * int(cnt.sum()) * w.n_layers
    return {"indexer": idx, "mla": mla}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.windows = []
        sel = str(device_index)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            pass
        self.cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                    "-i", sel]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.samples.append((time.time(), parts))

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        wins = [(t0, t1)] if t0 is not None else self.windows
        inside = [p for t, p in self.samples if any(a - 0.06 <= t <= b + 0.06 for a, b in wins)]
        inside = inside or [p for _, p in self.samples]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for p in inside for j in range(4) if p[3 + j].lower() == "active"})
        sm = [float(p[0]) for p in inside if p[0].replace(".", "").isdigit()]
        mx = [float(p[1]) for p in inside if p[1].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside)}


def count_kernel_nodes(fn) -> int | None:
    """Kernels one call of fn() launches: fn is captured into a throw-away CUDA
    graph whose kernel nodes are counted (events and memsets are not kernels)."""
    try:
        from cuda.bindings import runtime as rt
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        err, _, n = rt.cudaGraphGetNodes(g.raw_cuda_graph(), 0)
        err, nodes, n = rt.cudaGraphGetNodes(g.raw_cuda_graph(), n)
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        cnt = sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
        del g
        return cnt
    except Exception:
        return None


# ------------------------------------------------------------------ the step
class Step:
    """Device buffers and descriptors of one workload; the timed step is one
    dsa_indexshare_group call, the breakdown step the separate calls."""

    def __init__(self, w: wl.Workload, dev, seed_offset: int = 0, fp8: bool = False):
        self.w = w
        self.dev = dev
        self.fp8 = fp8
        w = wl.scaled(w, seed=w.seed + seed_offset) if seed_offset else w
        self.x = wl.make_inputs(w, device=dev)
        self.seq_run = w.n_q if len(set(w.q_seq)) == 1 else 1
        x = self.x
        self.q = B.Queries(x["q_seq"], x["q_pos"], n_seq=w.n_seq, max_ctx=w.L, seq_run=self.seq_run)
        self.f8 = None
        if fp8:  # E4M3 indexer queries and keys with per-row scales
            self.f8 = wl.fp8_indexer_inputs(w, x, device=dev)
            f8 = self.f8
            self.ix = B.Indexer(f8["q8"], x["w"], f8["k8"][0] if w.shared_cache else f8["k8"],
                                q_scale=f8["q_scale"], k_scale=f8["k_scale"][0] if w.shared_cache else f8["k_scale"])
            x["k_idx"] = None  # the bf16 keys are not read
        else:
            self.ix = B.Indexer(x["q_idx"], x["w"], x["k_idx"][0] if w.shared_cache else x["k_idx"])
        # the separate calls: the indexer leaves the top-k's first-digit histograms
        self.ix_sep = B.Indexer(self.ix.q, self.ix.w, self.ix.k, flags=B.DSA_INDEXER_TOPK_HIST,
                                q_scale=self.ix.q_scale, k_scale=self.ix.k_scale)
        if fp8:  # packed E4M3 latent rows with a per-row scale
            caches = wl.fp8_latent_inputs(w, x, device=dev)
            x["kv"] = None  # the bf16 caches are not read
        else:
            caches = x["kv"]
        self.mlas, self.mlas_sep = [], []
        for layer in range(w.n_layers):
            kv = caches[layer][0] if w.shared_cache else caches[layer]
            for lst in (self.mlas, self.mlas_sep):
                out = torch.empty((w.n_q, w.mla_heads, w.d_lat), dtype=w.torch_dtype, device=dev)
                lse = torch.empty((w.n_q, w.mla_heads), dtype=torch.float32, device=dev)
                lst.append(B.Mla(x["q_mla"][layer], kv, out, w.d_lat, w.scale, lse))
        self.ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, self.q, w.topk, w.n_layers, dev)
        self.ws_sep = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, self.q, w.topk, w.n_layers, dev)
        self.scores = B.scores_buffer(w.n_q, w.L, dev)
        self.idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
        self.idx_sep = torch.empty_like(self.idx)
        self.cnt_sep = torch.empty_like(self.cnt)
        self.decode = w.n_q <= DECODE_MAX_QUERIES
        self.mla_fn = B.dsa_sparse_mla_decode if self.decode else B.dsa_sparse_mla_prefill
        self.ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
        self.graph = None      # the timed step: events at its two ends only
        self.graph_bd = None   # the separate calls with events between the stages (breakdown)

    def run(self, events: bool = False):
        if events:
            self.ev[0].record()
        B.dsa_indexshare_group(self.q, self.ix, self.mlas, self.w.topk, self.idx, self.cnt, self.ws)
        if events:
            self.ev[1].record()

    def run_separate(self, events: bool = False):
        if events:
            self.ev[2].record()
        B.dsa_index_scores(self.q, self.ix_sep, self.scores, self.ws_sep)
        if events:
            self.ev[3].record()
        B.dsa_topk(self.q, self.scores, self.w.topk, self.idx_sep, self.cnt_sep, self.ws_sep,
                   flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        if events:
            self.ev[4].record()
        for m in self.mlas_sep:
            self.mla_fn(self.q, m, self.idx_sep, self.cnt_sep, self.w.topk, self.ws_sep)
        if events:
            self.ev[5].record()

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run()              # one eager pass each: one-time kernel attribute setup
            self.run_separate()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.launches = count_kernel_nodes(self.run)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            self.run(events=True)
        torch.cuda.synchronize()
        self.graph_bd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_bd, capture_error_mode="thread_local"):
            self.run_separate(events=True)
        torch.cuda.synchronize()

    def step_ms(self):
        return self.ev[0].elapsed_time(self.ev[1])

    def breakdown_ms(self):
        e = self.ev
        return (e[2].elapsed_time(e[3]), e[3].elapsed_time(e[4]), e[4].elapsed_time(e[5]))

    def release(self):
        self.graph = None
        self.graph_bd = None


class E2EStep:
    """The step end to end through the public API with host buffers, eager: one
    dsa_indexshare_group_host call copies the step's query inputs (indexer queries
    and weights, positions, every layer's MLA queries) from pinned host memory
    into one device buffer, runs the group call on them, and copies every layer's
    output plus the selected indices and counts back into pinned host memory.  The
    caches stay resident (model state)."""

    def __init__(self, step: Step):
        self.s = step
        w, x = step.w, step.x
        dev = step.dev
        ins = [("q_idx", step.ix.q), ("w", x["w"]), ("q_seq", x["q_seq"]), ("q_pos", x["q_pos"])]
        if step.ix.q_scale is not None:
            ins.append(("q_scale", step.ix.q_scale))
        ins += [(f"q_mla{l}", t) for l, t in enumerate(x["q_mla"])]
        self.d_in, self.h_in, vin = self._pack(ins, dev, fill=True)
        outs = [(f"out{l}", m.out) for l, m in enumerate(step.mlas)] + [("idx", step.idx), ("cnt", step.cnt)]
        self.d_out, self.h_out, vout = self._pack(outs, dev, fill=False)
        self.h2d = self.h_in.numel()
        self.d2h = self.h_out.numel()
        self.q = B.Queries(vin["q_seq"], vin["q_pos"], n_seq=w.n_seq, max_ctx=w.L, seq_run=step.seq_run)
        self.ix = B.Indexer(vin["q_idx"], vin["w"], step.ix.k, q_scale=vin.get("q_scale"), k_scale=step.ix.k_scale)
        self.mlas = [B.Mla(vin[f"q_mla{l}"], m.kv, vout[f"out{l}"], m.d_latent, m.scale, m.lse)
                     for l, m in enumerate(step.mlas)]
        self.idx, self.cnt = vout["idx"], vout["cnt"]
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        self.call = B.GroupHostCall(self.q, self.ix, self.mlas, step.w.topk, self.idx, self.cnt, step.ws,
                                    self.h_in, self.d_in, self.h_out, self.d_out)

    @staticmethod
    def _pack(items, dev, fill):
        offs, tot = [], 0
        for _, t in items:
            offs.append(tot)
            tot += (t.numel() * t.element_size() + 255) // 256 * 256
        d = torch.empty(tot, dtype=torch.uint8, device=dev)
        h = torch.zeros(tot, dtype=torch.uint8).pin_memory()
        views = {}
        for (name, t), o in zip(items, offs):
            nb = t.numel() * t.element_size()
            v = d[o:o + nb].view(t.dtype).view(t.shape)
            if fill:
                v.copy_(t)
                h[o:o + nb].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
            views[name] = v
        return d, h, views

    def run(self):
        s = self.s
        self.ev[0].record()
        t0 = time.perf_counter()
        self.call()
        self.call_s = time.perf_counter() - t0
        self.ev[1].record()

    def ms(self):
        return self.ev[0].elapsed_time(self.ev[1])


def self_check(step: Step) -> str:
    """The results the timed graph left (indices, counts, every layer's output)
    against one eager group call on a freshly initialised workspace, and against
    the separate calls' results: the path is deterministic (exact histogram
    counts, a fixed merge order), so all three must be bitwise equal.  A step
    whose calls corrupt each other's scratch across replays fails this.
    Reports; never raises."""
    try:
        w = step.w
        idx0, cnt0 = step.idx.clone(), step.cnt.clone()
        outs0 = [m.out.clone() for m in step.mlas]
        saved = step.ws
        step.ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, step.q, w.topk, w.n_layers, step.dev)
        try:
            step.run()
            torch.cuda.synchronize()
            st = B.dsa_check_status(step.ws)
        finally:
            step.ws = saved
        if st != B.DSA_OK:
            return f"fresh step status {B.status_str(st)}"
        same = torch.equal(idx0, step.idx) and torch.equal(cnt0, step.cnt)
        same = same and all(torch.equal(o0, m.out) for o0, m in zip(outs0, step.mlas))
        if not same:
            return "MISMATCH with a fresh-workspace step"
        if not (torch.equal(idx0, step.idx_sep) and torch.equal(cnt0, step.cnt_sep)):
            return "MISMATCH between the group call's and the separate calls' indices"
        # the group call plans its attention over all layers at once, the separate
        # calls per layer: with different split counts the partial sums are added
        # in another order, so outputs agree to rounding, not bit for bit
        diff = max(float((o0.float() - m.out.float()).abs().max()) for o0, m in zip(outs0, step.mlas_sep))
        if diff == 0.0:
            return "bitwise equal to a fresh-workspace step and to the separate calls"
        if diff <= 2e-2:
            return (f"bitwise equal to a fresh-workspace step; indices equal to the separate calls', "
                    f"outputs within {diff:.1e} (different split plans)")
        return f"MISMATCH between the group call and the separate calls: max-abs {diff:.3e}"
    except Exception as e:  # the check reports; the measurement stands on its own
        return f"error: {type(e).__name__}: {e}"


# ------------------------------------------------------------------ CPU oracle timing
def host_copies(w: wl.Workload, dev_x: dict, queries) -> dict:
    """Host copies of what the sampled queries read (their sequences only)."""
    seqs = sorted({0 if w.shared_cache else w.q_seq[i] for i in queries})
    return {"q_idx": dev_x["q_idx"].cpu(), "w": dev_x["w"].cpu(), "q_mla": [t.cpu() for t in dev_x["q_mla"]],
            "k": {b: dev_x["k_idx"][b].cpu() for b in seqs},
            "kv": {b: [t[b].cpu() for t in dev_x["kv"]] for b in seqs}}


def oracle_sample_time(w: wl.Workload, h: dict, queries) -> float:
    """Seconds the fp64 oracle takes for the whole path (scores over every visible
    key -> top-k -> MLA of every layer) of the given queries."""
    import oracle
    t0 = time.perf_counter()
    for i in queries:
        b = 0 if w.shared_cache else w.q_seq[i]
        k = h["k"][b].float().numpy()[None]
        sc = oracle.index_scores(h["q_idx"][i:i + 1].float().numpy(), h["w"][i:i + 1].numpy(), k, [0],
                                 [w.q_pos[i]])
        idx, cnt = oracle.topk(sc, [w.q_pos[i]], w.topk)
        sel = idx[0, : cnt[0]]
        for layer in range(w.n_layers):
            rows = h["kv"][b][layer][torch.from_numpy(sel.astype(np.int64))].float().numpy()[None]
            oracle.sparse_mla(h["q_mla"][layer][i:i + 1].float().numpy(), rows, [0],
                              np.arange(len(sel), dtype=np.int32)[None], cnt, w.d_lat, w.scale)
    return time.perf_counter() - t0


def cpu_baseline(w: wl.Workload, dev_x: dict, budget_s: float = 12.0):
    import oracle
    oracle.build()
    order = list(range(w.n_q))
    h = host_copies(w, dev_x, order[:1])
    t1 = oracle_sample_time(w, h, order[:1])
    n = max(1, min(w.n_q, int(budget_s / max(t1, 1e-6))))
    if n > 1:
        h = host_copies(w, dev_x, order[:n])
        t = oracle_sample_time(w, h, order[:n])
    else:
        t = t1
    return {"value": n * w.n_layers / t, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} of {w.n_q} queries of {w.name}, all {w.n_layers} layer(s), full path "
                      f"(fp64 scores over all visible keys, full sort, sparse MLA)"}


# ------------------------------------------------------------------ main
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(value: float, world: int, dev) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, n_q: int, n_layers: int, steps: int, tot_ms_max: float) -> float:
    """Whole-job query-tokens/s per layer: every rank processed its own batch of
    n_q queries x n_layers layers per step; the time is the slowest rank's."""
    return world * n_q * n_layers * steps / (tot_ms_max * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def config_of(w: wl.Workload, world: int, fp8: bool = False) -> dict:
    c = {**w.describe(), "parallelism": f"dp{world} (independent batches per GPU)",
         "l2": "flushed before every timed step (256 MB write, then a 256 MB read so the step starts with clean lines)", "graph": "CUDA graph per step",
         "entry_point": "dsa_indexshare_group"}
    if fp8:
        c["indexer_dtype"] = "e4m3 + per-row fp32 scales (FP8 variant)"
        c["latent_cache"] = "e4m3 + per-row fp32 scale, bf16 RoPE key, 656-byte rows (FP8 variant)"
    return c


def stage_rooflines(w: wl.Workload, fp8: bool, t_us: dict, hbm_peak: float, tc_peak: float, peak_kind: str):
    """Per-stage achieved rates against their bound, and the dominant stage."""
    by = path_bytes(w, indexer_fp8=fp8, mla_fp8=fp8)
    fl = path_flops(w)
    prefill = w.n_q > DECODE_MAX_QUERIES
    st = {}
    for name, key in (("index_scores", "indexer"), ("topk", "topk"), ("sparse_mla", "mla")):
        us = t_us[name]
        gbs = by[key] / (us * 1e-6) / 1e9
        e = {"kernel": {"index_scores": "idx_score_tc", "topk": "topk", "sparse_mla": "mla_tc (+ mla_combine)"}[name],
             "us": us, "algorithmic_bytes": by[key], "achieved_gbs": gbs, "hbm_frac": gbs / hbm_peak}
        if key in fl:
            tf = fl[key] / (us * 1e-6) / 1e12
            e["flops"] = fl[key]
            e["achieved_tflops"] = tf
            e["tensor_frac"] = tf / tc_peak
        st[name] = e
    dom = max(st, key=lambda k: st[k]["us"])
    d = st[dom]
    tensor_bound = prefill and dom in ("index_scores", "sparse_mla")
    if tensor_bound:
        roof = {"bound": "tensor", "kernel": d["kernel"], "achieved": d["achieved_tflops"], "peak": tc_peak,
                "unit": "TFLOP/s", "frac": d["tensor_frac"], "peak_kind": f"{peak_kind} bf16_tflops (burst)",
                "algorithmic_flops": d["flops"]}
    else:
        roof = {"bound": "hbm", "kernel": d["kernel"], "achieved": d["achieved_gbs"], "peak": hbm_peak, "unit": "GB/s",
                "frac": d["hbm_frac"], "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes": d["algorithmic_bytes"]}
    roof["avg_launch_us"] = d["us"]
    roof["stage"] = dom
    roof["traffic"] = NCU_TRAFFIC.get((w.name, dom, fp8))
    return roof, st


def measure(w: wl.Workload, fp8: bool, args, world: int, rank: int, dev, flush, clocks, steps: int,
            headline: bool):
    """Time one workload; returns its result dict (and the step, for e2e / baseline)."""
    step = Step(w, dev, seed_offset=rank, fp8=fp8)
    step.capture()
    for _ in range(args.warmup):
        flush.fill_(1)
        step.graph.replay()
    torch.cuda.synchronize()
    st = B.dsa_check_status(step.ws)
    if st != B.DSA_OK:
        raise SystemExit(f"{w.name}: device status {B.status_str(st)}")
    barrier(world)
    torch.cuda.synchronize()
    t_on = time.time()
    tot = 0.0
    for _ in range(steps):
        flush.fill_(1)
        step.graph.replay()
        torch.cuda.synchronize()
        tot += step.step_ms()
    t_off = time.time()
    clocks.window(t_on, t_off)
    barrier(world)
    tot_max = max_over_ranks(tot, world, dev)
    # per-stage times (separate calls, events between the stages)
    idx_t = topk_t = mla_t = 0.0
    n_bd = max(5, min(steps, 50))
    for _ in range(n_bd):
        flush.fill_(1)
        step.graph_bd.replay()
        torch.cuda.synchronize()
        b, c, d = step.breakdown_ms()
        idx_t += b
        topk_t += c
        mla_t += d
    t_us = {"index_scores": idx_t / n_bd * 1e3, "topk": topk_t / n_bd * 1e3, "sparse_mla": mla_t / n_bd * 1e3}
    ms_per_step = tot_max / steps
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    by = path_bytes(w, indexer_fp8=fp8, mla_fp8=fp8)
    roof, stages = stage_rooflines(w, fp8, t_us, hbm_peak, tc_peak, peak_kind)
    t_roof_us = by["path"] / (hbm_peak * 1e9) * 1e6
    res = {
        "value": weak_scaling_value(world, w.n_q, w.n_layers, steps, tot_max), "unit": UNIT,
        "ms_per_step": ms_per_step, "steps": steps,
        "dtype": ("e4m3 indexer, e4m3 latent cache, " + w.dtype + " MLA") if fp8 else w.dtype,
        "config": config_of(w, world, fp8),
        "roofline": roof,
        "path_roofline": {"bytes": by["path"], "t_roof_us": t_roof_us, "frac": t_roof_us / (ms_per_step * 1e3),
                          "peak_kind": f"{peak_kind} hbm_gbs"},
        "breakdown_us": {**t_us, "note": "separate calls in a graph with events between the stages"},
        "stages": stages,
        "gpu_launches": None if step.launches is None else step.launches * steps,
        "launches_per_step": step.launches,
        "clocks": clocks.summary(t_on, t_off),
    }
    res["self_check"] = self_check(step)
    return res, step


def e2e_measure(step: Step, world: int, dev, flush, steps: int):
    e2e = E2EStep(step)
    for _ in range(3):
        e2e.run()
    torch.cuda.synchronize()
    barrier(world)
    te, wall, call = 0.0, 0.0, 0.0
    for _ in range(steps):
        flush.fill_(1)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e2e.run()
        torch.cuda.synchronize()
        wall += time.perf_counter() - t0
        call += e2e.call_s
        te += e2e.ms()
    te = max_over_ranks(te, world, dev)
    w = step.w
    return {"value": world * w.n_q * w.n_layers * steps / (te * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": e2e.h2d, "d2h_bytes_per_step": e2e.d2h, "steps": steps,
            "host_wall_ms_per_step": 1e3 * wall / steps,
            "host_call_us": 1e6 * call / steps,  # the call's own host time (checks, copies, maps, launches)
            "how": "eager each step: dsa_indexshare_group_host (pinned H2D of the query inputs, the group "
                   "call, D2H of outputs + indices, all in the one C-ABI call, its arguments converted once)"}


def producers_measure(dev, flush, steps: int, hbm_peak: float, tc_peak: float, peak_kind: str) -> dict:
    """The producers around the path at GLM-5.2 shapes (hidden 6144, 64 heads), decode-sized (4 tokens)
    and prefill-sized (4096 tokens) batches: cache-row writer, query absorption, value up-projection.
    Each timed with CUDA events (L2 flushed before every launch) against its bound: the weights' HBM
    bytes for decode sizes, the GEMM FLOPs at the bf16 tensor peak for prefill sizes."""
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    H, hidden = 64, 6144
    out = {}

    def timed(fn):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            flush.fill_(1)
            # ~100 us of device spin so the eager call's host-side marshalling is
            # enqueued before the start event fires: the kernels' time, not the host's
            torch.cuda._sleep(200_000)
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize()
            tot += ev[0].elapsed_time(ev[1])
        return tot / steps * 1e3  # us

    def entry(us, weight_bytes, io_bytes, flops, prefill):
        gbs = (weight_bytes + io_bytes) / (us * 1e-6) / 1e9
        tf = flops / (us * 1e-6) / 1e12
        e = {"us": us, "bytes": weight_bytes + io_bytes, "flops": flops, "achieved_gbs": gbs,
             "achieved_tflops": tf}
        if prefill:
            e.update({"bound": "tensor", "frac": tf / tc_peak, "peak_kind": f"{peak_kind} bf16_tflops (burst)"})
        else:
            e.update({"bound": "hbm", "frac": gbs / hbm_peak, "peak_kind": f"{peak_kind} hbm_gbs"})
        return e

    w_cache = (torch.randn((704, hidden), generator=g, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    rms = torch.ones(512, device=dev)
    lnw, lnb = torch.ones(128, device=dev), torch.zeros(128, device=dev)
    w_uk_t = (torch.randn((H, 512, 192), generator=g, device=dev) / 192 ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn((H, 256, 512), generator=g, device=dev) / 512 ** 0.5).to(torch.bfloat16)
    for n in (4, 4096):
        pre = n > 256
        h = torch.randn((n, hidden), generator=g, device=dev).to(torch.bfloat16)
        seq = torch.zeros(n, dtype=torch.int32, device=dev)
        pos = torch.arange(n, dtype=torch.int32, device=dev)
        kv = torch.empty((1, n, 576), dtype=torch.bfloat16, device=dev)
        kidx = torch.empty((1, n, 128), dtype=torch.bfloat16, device=dev)
        cw = B.CacheWriter(h, w_cache, rms, lnw, lnb, seq, pos, kv, kidx)
        ws = torch.zeros(max(256, B.dsa_cache_writer_workspace_bytes(n, hidden)), dtype=torch.uint8, device=dev)
        us = timed(lambda: B.dsa_write_cache_rows(cw, ws))
        out[f"write_cache_rows_{n}"] = entry(us, w_cache.numel() * 2, n * (hidden + 704) * 2,
                                             2 * n * hidden * 704, pre)
        q_nope = torch.randn((n, H, 192), generator=g, device=dev).to(torch.bfloat16)
        q_rope = torch.randn((n, H, 64), generator=g, device=dev).to(torch.bfloat16)
        q_out = torch.empty((n, H, 576), dtype=torch.bfloat16, device=dev)
        ws2 = torch.zeros(256, dtype=torch.uint8, device=dev)
        us = timed(lambda: B.dsa_absorb_queries(q_nope, q_rope, w_uk_t, pos, 8.0e6, q_out, ws2))
        out[f"absorb_queries_{n}"] = entry(us, w_uk_t.numel() * 2, n * H * (192 + 64 + 576) * 2,
                                           2 * n * H * 192 * 512, pre)
        o_lat = torch.randn((n, H, 512), generator=g, device=dev).to(torch.bfloat16)
        o_v = torch.empty((n, H, 256), dtype=torch.bfloat16, device=dev)
        us = timed(lambda: B.dsa_up_project(o_lat, w_uv, o_v, ws2))
        out[f"up_project_{n}"] = entry(us, w_uv.numel() * 2, n * H * (512 + 256) * 2, 2 * n * H * 512 * 256, pre)
        assert B.dsa_check_status(ws) == B.DSA_OK and B.dsa_check_status(ws2) == B.DSA_OK
    return out


def run_reference(args, w: wl.Workload, world: int, rank: int):
    """The oracle as it stands on host cores: each step one query's full path."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    x = wl.make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    order = list(range(w.n_q))
    h = host_copies(w, x, order)
    for s in range(min(args.warmup, 3)):
        oracle_sample_time(w, h, [order[s % w.n_q]])
    # bounded: stop after REFERENCE_BUDGET_S of timed oracle work (long contexts
    # take seconds per query) and report the steps actually timed
    t, done = 0.0, 0
    for s in range(args.steps):
        t += oracle_sample_time(w, h, [order[s % w.n_q]])
        done += 1
        if t > REFERENCE_BUDGET_S:
            break
    value = done * w.n_layers / t
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": done,
            "warmup": args.warmup, "ms_per_step": 1e3 * t / done, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": "each step: one query of the workload, full path, all layers"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=list(wl.NAMED))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--fp8", action="store_true",
                    help="the headline workload with the FP8 variants (E4M3 indexer keys/queries and latent cache)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="only the headline workload")
    ap.add_argument("--no-producers", action="store_true", help="skip the producer measurements")
    ap.add_argument("--n-seq", type=int, default=0,
                    help="decode workloads: override the batch (a smaller case for profiling; not a bench line)")
    ap.add_argument("--n-q", type=int, default=0,
                    help="prefill: keep the last N queries of the chunk (a smaller case for profiling; not a bench line)")
    args = ap.parse_args()
    w = wl.NAMED[args.workload]
    small = False
    if args.n_seq and len(set(w.q_seq)) == w.n_q:
        w = wl.scaled(w, n_seq=args.n_seq, q_pos=w.q_pos[:1] * args.n_seq, q_seq=tuple(range(args.n_seq)),
                      name=f"{w.name}_b{args.n_seq}")
        small = True
    if args.n_q and len(set(w.q_seq)) == 1 and args.n_q < w.n_q:
        w = wl.scaled(w, q_pos=w.q_pos[-args.n_q:], q_seq=w.q_seq[-args.n_q:], name=f"{w.name}_q{args.n_q}")
        small = True
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B.lib()
    flush = L2Flush(dev)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)

    res, step = measure(w, args.fp8, args, world, rank, dev, flush, clocks, args.steps, True)
    line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": res["dtype"], "data": "synthetic",
            "config": res["config"]}
    for k in ("roofline", "path_roofline", "breakdown_us", "stages", "gpu_launches", "launches_per_step",
              "clocks", "self_check"):
        line[k] = res[k]
    if not args.no_e2e:
        line["e2e"] = e2e_measure(step, world, dev, flush, max(10, min(args.steps, 200)))
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.fp8:
        line["cpu_baseline"] = cpu_baseline(w, step.x)
    step.release()
    del step
    gc.collect()
    torch.cuda.empty_cache()

    if not args.no_producers and not small:
        hbm_peak, tc_peak, peak_kind = measured_peaks()
        line["producers"] = producers_measure(dev, flush, min(args.steps, PER_CONFIG_MAX_STEPS), hbm_peak, tc_peak,
                                              peak_kind)
    if not args.no_per_config and not small:
        per = {}
        n = min(args.steps, PER_CONFIG_MAX_STEPS)
        for name, fp8 in PER_CONFIG:
            if name == args.workload and fp8 == args.fp8:
                continue
            r, s = measure(wl.NAMED[name], fp8, args, world, rank, dev, flush, clocks, n, False)
            s.release()
            del s
            gc.collect()
            torch.cuda.empty_cache()
            per[name + ("+fp8" if fp8 else "")] = r
        line["per_config"] = per
        line["gpu_launches"] = (line["gpu_launches"] or 0) + sum((r["gpu_launches"] or 0) for r in per.values())
    clocks.stop()
    time.sleep(0.05)
    line["clocks"] = clocks.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
