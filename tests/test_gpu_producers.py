"""The producers around the path through the C ABI against the fp64 numpy
oracle (oracle/producers.py): the cache-row writer (latent row + indexer key
from the hidden state), query absorption and the value up-projection, at
GLM-5.2 shapes (hidden 6144, 64 heads), decode- and prefill-sized batches, with
RoPE positions up to 2^20 - 1.  Outputs are bf16 of magnitude ~1: max-abs 2e-2,
mean-abs 2e-3 (the attention outputs' bound, set by the bf16 rounding)."""
import ctypes

import numpy as np
import pytest
import torch

from dsa_indexer_top_b200 import binding as B
from oracle import producers as P

pytestmark = pytest.mark.gpu

HIDDEN = 6144
THETA = 8.0e6
EPS = 1e-5


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _close(got: torch.Tensor, want: np.ndarray, what: str):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    err = np.abs(g - want)
    assert err.max() <= 2e-2, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= 2e-3, f"{what}: mean-abs {err.mean():.3e}"


@pytest.mark.parametrize("n_tok", [3, 130, 300])
def test_write_cache_rows_matches_oracle(cuda_ok, n_tok):
    dev = torch.device("cuda")
    g = np.random.default_rng(100 + n_tok)
    h = _bf16(g.standard_normal((n_tok, HIDDEN)))
    w = _bf16(g.standard_normal((704, HIDDEN)) / np.sqrt(HIDDEN))
    rms_w = (1 + 0.1 * g.standard_normal(512)).astype(np.float32)
    ln_w = (1 + 0.1 * g.standard_normal(128)).astype(np.float32)
    ln_b = (0.1 * g.standard_normal(128)).astype(np.float32)
    n_seq, L = 2, 1 << 20
    seq = g.integers(0, n_seq, n_tok).astype(np.int32)
    pos = g.choice(L, size=n_tok, replace=False).astype(np.int32)
    pos[0] = L - 1
    kv = torch.full((n_seq, L, 576), float("nan"), dtype=torch.bfloat16, device=dev)
    kidx = torch.full((n_seq, L, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    hd, wd = h.to(dev), w.to(dev)
    rmsd, lnwd, lnbd = (torch.from_numpy(a).to(dev) for a in (rms_w, ln_w, ln_b))
    seqd, posd = torch.from_numpy(seq).to(dev), torch.from_numpy(pos).to(dev)
    cw = B.CacheWriter(hd, wd, rmsd, lnwd, lnbd, seqd, posd, kv, kidx, eps=EPS, rope_theta=THETA)
    ws = torch.zeros(B.dsa_cache_writer_workspace_bytes(n_tok, HIDDEN), dtype=torch.uint8, device=dev)
    B.dsa_write_cache_rows(cw, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    hf, wf = h.float().numpy(), w.float().numpy()
    rows = P.latent_rows(hf, wf[:576].T, rms_w, pos, theta=THETA)
    keys = P.indexer_keys(hf, wf[576:].T, ln_w, ln_b, pos, theta=THETA)
    s_t, p_t = torch.from_numpy(seq.astype(np.int64)), torch.from_numpy(pos.astype(np.int64))
    _close(kv[s_t.to(dev), p_t.to(dev)], rows, "latent rows")
    _close(kidx[s_t.to(dev), p_t.to(dev)], keys, "indexer keys")
    # rows of other positions are untouched
    free = sorted(set(range(16)) - set(pos[seq == 0].tolist()))[0]
    assert torch.isnan(kv[0, free].float()).all() and torch.isnan(kidx[0, free].float()).all()


@pytest.mark.parametrize("n_q", [5, 300])
def test_absorb_queries_matches_oracle(cuda_ok, n_q):
    dev = torch.device("cuda")
    g = np.random.default_rng(200 + n_q)
    H = 64
    q_nope = _bf16(g.standard_normal((n_q, H, 192)))
    q_rope = _bf16(g.standard_normal((n_q, H, 64)))
    w_uk = _bf16(g.standard_normal((H, 192, 512)) / np.sqrt(192))       # [H, d_nope, d_lat]
    pos = g.integers(0, 1 << 20, n_q).astype(np.int32)
    out = torch.full((n_q, H, 576), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    B.dsa_absorb_queries(q_nope.to(dev), q_rope.to(dev), w_uk.transpose(1, 2).contiguous().to(dev),
                         torch.from_numpy(pos).to(dev), THETA, out, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    want = P.absorb_queries(q_nope.float().numpy(), q_rope.float().numpy(), w_uk.float().numpy(), pos, theta=THETA)
    _close(out, want, "absorbed queries")


@pytest.mark.parametrize("n_q", [5, 300])
def test_up_project_matches_oracle(cuda_ok, n_q):
    dev = torch.device("cuda")
    g = np.random.default_rng(300 + n_q)
    H = 64
    o_lat = _bf16(g.standard_normal((n_q, H, 512)))
    w_uv = _bf16(g.standard_normal((H, 256, 512)) / np.sqrt(512))
    out = torch.full((n_q, H, 256), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    B.dsa_up_project(o_lat.to(dev), w_uv.to(dev), out, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    _close(out, P.up_project(o_lat.float().numpy(), w_uv.float().numpy()), "up-projection")
