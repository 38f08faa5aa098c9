"""Shared helpers of the test-suite: run the CUDA library through its C ABI and
the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl

# Tolerances on attention outputs (bf16 outputs: max-abs 2e-2, mean-abs 2e-3;
# fp32 inputs and outputs on the generic path: fp32 accumulation only).
TOL = {"bf16": (2e-2, 2e-3, 2e-3), "f32": (2e-4, 2e-5, 1e-4)}   # (max-abs, mean-abs, lse max-abs)


def to_device(x: dict, device="cuda") -> dict:
    out = {}
    for k, v in x.items():
        out[k] = [t.to(device) for t in v] if isinstance(v, list) else v.to(device)
    return out


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).contiguous().numpy()


def descriptors(w: wl.Workload, x: dict, seq_run: int = 1):
    """Queries / Indexer / per-layer Mla descriptors (outputs allocated here)."""
    dev = x["q_pos"].device
    q = B.Queries(x["q_seq"], x["q_pos"], n_seq=w.n_seq, max_ctx=w.L, seq_run=seq_run)
    k = x["k_idx"][0] if w.shared_cache else x["k_idx"]
    ix = B.Indexer(x["q_idx"], x["w"], k)
    mlas = []
    for layer in range(len(x["q_mla"])):
        kv = x["kv"][layer][0] if w.shared_cache else x["kv"][layer]
        out = torch.full((w.n_q, w.mla_heads, w.d_lat), float("nan"), dtype=w.torch_dtype, device=dev)
        lse = torch.full((w.n_q, w.mla_heads), float("nan"), dtype=torch.float32, device=dev)
        mlas.append(B.Mla(x["q_mla"][layer], kv, out, w.d_lat, w.scale, lse))
    return q, ix, mlas


def oracle_selection(w: wl.Workload, xh: dict, rows=None):
    """Oracle scores + top-k for the queries in `rows` (default all)."""
    rows = np.arange(w.n_q) if rows is None else np.asarray(rows)
    q_seq = xh["q_seq"].numpy()[rows]
    q_pos = xh["q_pos"].numpy()[rows]
    k = host_f32(xh["k_idx"])
    if w.shared_cache:
        q_seq_o = np.zeros_like(q_seq)
    else:
        q_seq_o = q_seq
    sc = oracle.index_scores(host_f32(xh["q_idx"])[rows], host_f32(xh["w"])[rows], k, q_seq_o, q_pos)
    idx, cnt = oracle.topk(sc, q_pos, w.topk)
    return sc, idx, cnt


def fp8_indexer(w: wl.Workload, f8: dict, x: dict, flags: int = 0) -> B.Indexer:
    """Indexer descriptor of the FP8 (E4M3) variant from wl.fp8_indexer_inputs."""
    k8 = f8["k8"][0] if w.shared_cache else f8["k8"]
    ks = f8["k_scale"][0] if w.shared_cache else f8["k_scale"]
    return B.Indexer(f8["q8"], x["w"], k8, flags=flags, q_scale=f8["q_scale"], k_scale=ks)


def oracle_selection_fp8(w: wl.Workload, f8h: dict, xh: dict, rows=None):
    """Oracle scores (on the exact dequantised E4M3 operands) + top-k."""
    rows = np.arange(w.n_q) if rows is None else np.asarray(rows)
    q_seq = xh["q_seq"].numpy()[rows]
    q_pos = xh["q_pos"].numpy()[rows]
    q_seq_o = np.zeros_like(q_seq) if w.shared_cache else q_seq
    q8 = f8h["q8"].view(torch.uint8).numpy()[rows]
    k8 = f8h["k8"].view(torch.uint8).numpy()
    sc = oracle.index_scores_e4m3(q8, f8h["q_scale"].numpy()[rows], host_f32(xh["w"])[rows], k8,
                                  f8h["k_scale"].numpy(), q_seq_o, q_pos)
    idx, cnt = oracle.topk(sc, q_pos, w.topk)
    return sc, idx, cnt


def oracle_mla(w: wl.Workload, xh: dict, layer: int, idx, cnt, rows=None):
    rows = np.arange(w.n_q) if rows is None else np.asarray(rows)
    q_seq = xh["q_seq"].numpy()[rows]
    if w.shared_cache:
        q_seq = np.zeros_like(q_seq)
    return oracle.sparse_mla(host_f32(xh["q_mla"][layer])[rows], host_f32(xh["kv"][layer]), q_seq, idx, cnt,
                             w.d_lat, w.scale)


def with_fp8_caches(w: wl.Workload, mlas, kv8_layers):
    """The same Mla descriptors reading packed FP8 latent caches (uint8 rows from
    wl.fp8_latent_inputs) instead of the bf16 ones; outputs reset to NaN."""
    out = []
    for m, kv8 in zip(mlas, kv8_layers):
        m.out.fill_(float("nan"))
        if m.lse is not None:
            m.lse.fill_(float("nan"))
        out.append(B.Mla(m.q, kv8[0] if w.shared_cache else kv8, m.out, m.d_latent, m.scale, m.lse))
    return out


def oracle_mla_fp8(w: wl.Workload, xh: dict, kv8h, layer: int, idx, cnt, rows=None):
    """Oracle attention of one layer over its packed FP8 cache (host uint8 rows)."""
    rows = np.arange(w.n_q) if rows is None else np.asarray(rows)
    q_seq = xh["q_seq"].numpy()[rows]
    if w.shared_cache:
        q_seq = np.zeros_like(q_seq)
    return oracle.sparse_mla_fp8(host_f32(xh["q_mla"][layer])[rows], kv8h[layer].cpu().numpy(), q_seq, idx, cnt,
                                 w.d_lat, w.d_rope, w.scale)


def assert_attention_close(got: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "out"):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    max_abs, mean_abs, _ = TOL[dtype]
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - ref)
    assert err.max() <= max_abs, f"{what}: max-abs error {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"{what}: mean-abs error {err.mean():.3e} > {mean_abs}"


def assert_lse_close(got: torch.Tensor, ref: np.ndarray, dtype: str):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    tol = TOL[dtype][2]
    err = np.abs(g - ref)
    assert err.max() <= tol * max(1.0, np.abs(ref).max()), f"lse: max-abs error {err.max():.3e}"


def random_selection(w: wl.Workload, seed: int, device="cpu"):
    """Seeded valid selections (unique, ascending, <= q_pos, -1 padded) for
    testing attention on its own."""
    rng = np.random.default_rng(seed)
    idx = np.full((w.n_q, w.topk), -1, dtype=np.int32)
    cnt = np.zeros(w.n_q, dtype=np.int32)
    for i, t in enumerate(w.q_pos):
        n = t + 1
        kk = min(w.topk, n)
        sel = np.sort(rng.choice(n, size=kk, replace=False)) if n > kk else np.arange(n)
        idx[i, :kk] = sel
        cnt[i] = kk
    return torch.from_numpy(idx).to(device), torch.from_numpy(cnt).to(device)
