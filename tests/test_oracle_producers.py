"""Pins for oracle/producers.py (the cache-row writers, query absorption and
value up-projection around the attention path).  Each check rests on something
other than the oracle:
  * a hand-worked interleaved RoPE example with literal trigonometric values
    (it also tells interleaved pairs from half-split ones, and a wrong frequency
    exponent or sign from the right one);
  * RoPE as multiplication by e^(i angle) of complex pairs, and its invariants
    (position 0 is the identity, pair norms are kept, dot products depend only
    on the position difference);
  * torch's own layer_norm and rms_norm (float64);
  * the non-absorbed MLA form through torch's scaled_dot_product_attention: per
    head keys [W_UK c | RoPE(r)] and values W_UV c, against the absorbed queries
    attended by the oracle's sparse_mla and up-projected.
"""
import math

import numpy as np
import torch

import oracle
from oracle import producers as P


def test_rope_hand_example():
    # d = 4, theta = 100: pair 0 turns by pos * 100^0, pair 1 by pos * 100^(-1/2)
    # = 0.1 rad per position.  x = [1, 0, 0, 1] at position 1:
    #   pair 0: (cos 1, sin 1);  pair 1: (0, 1) turned by 0.1 -> (-sin 0.1, cos 0.1)
    got = P.rope_interleaved(np.array([1.0, 0.0, 0.0, 1.0]), 1, theta=100.0)
    want = [0.5403023058681398, 0.8414709848078965, -0.09983341664682815, 0.9950041652780258]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # position 3, pair 1 only: (2, 0) turned by 0.3 rad -> (2 cos 0.3, 2 sin 0.3)
    got = P.rope_interleaved(np.array([0.0, 0.0, 2.0, 0.0]), 3, theta=100.0)
    np.testing.assert_allclose(got, [0, 0, 2 * 0.955336489125606, 2 * 0.29552020666133955], rtol=0, atol=1e-15)


def test_rope_is_complex_rotation_and_keeps_invariants():
    g = np.random.default_rng(1)
    d = 64
    x = g.standard_normal((5, d))
    pos = np.array([0, 1, 17, 4096, 1048575])
    got = P.rope_interleaved(x, pos)
    z = x[:, 0::2] + 1j * x[:, 1::2]
    ang = pos[:, None] * np.power(8.0e6, -np.arange(d // 2) * 2.0 / d)
    zr = z * np.exp(1j * ang)
    np.testing.assert_allclose(got[:, 0::2], zr.real, atol=1e-12)
    np.testing.assert_allclose(got[:, 1::2], zr.imag, atol=1e-12)
    np.testing.assert_array_equal(got[0], x[0])                                  # position 0
    np.testing.assert_allclose(np.hypot(got[:, 0::2], got[:, 1::2]), np.abs(z), atol=1e-12)
    q, k = g.standard_normal(d), g.standard_normal(d)
    base = P.rope_interleaved(q, 1000) @ P.rope_interleaved(k, 990)
    for shift in (1, 77, 5000):
        np.testing.assert_allclose(P.rope_interleaved(q, 1000 + shift) @ P.rope_interleaved(k, 990 + shift), base,
                                   rtol=1e-9)


def test_norms_match_torch():
    g = np.random.default_rng(2)
    x = g.standard_normal((7, 128)) * 3 + 0.5
    w, b = g.standard_normal(128), g.standard_normal(128)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (128,), torch.from_numpy(w), torch.from_numpy(b),
                                         eps=1e-5).numpy()
    np.testing.assert_allclose(P.layer_norm(x, w, b), ref, atol=1e-12)
    x2 = g.standard_normal((7, 512)) * 2
    w2 = g.standard_normal(512)
    ref2 = torch.nn.functional.rms_norm(torch.from_numpy(x2), (512,), torch.from_numpy(w2), eps=1e-5).numpy()
    np.testing.assert_allclose(P.rms_norm(x2, w2), ref2, atol=1e-12)


def test_indexer_keys_and_latent_rows():
    g = np.random.default_rng(3)
    T, hidden = 6, 96
    h = g.standard_normal((T, hidden))
    pos = np.array([0, 1, 2, 500, 70000, 1048575])
    w_k = g.standard_normal((hidden, 128)) / math.sqrt(hidden)
    lw, lb = 1 + 0.1 * g.standard_normal(128), 0.1 * g.standard_normal(128)
    k = P.indexer_keys(h, w_k, lw, lb, pos)
    ln = torch.nn.functional.layer_norm(torch.from_numpy(h @ w_k), (128,), torch.from_numpy(lw),
                                        torch.from_numpy(lb), eps=1e-5).numpy()
    np.testing.assert_allclose(k[:, :64], ln[:, :64], atol=1e-12)               # no-RoPE part untouched
    np.testing.assert_allclose(k[0], ln[0], atol=1e-12)                         # position 0
    np.testing.assert_allclose(np.hypot(k[:, 64::2], k[:, 65::2]), np.hypot(ln[:, 64::2], ln[:, 65::2]), atol=1e-12)
    w_kva = g.standard_normal((hidden, 576)) / math.sqrt(hidden)
    nw = 1 + 0.1 * g.standard_normal(512)
    rows = P.latent_rows(h, w_kva, nw, pos)
    y = h @ w_kva
    ref_c = torch.nn.functional.rms_norm(torch.from_numpy(y[:, :512]), (512,), torch.from_numpy(nw), eps=1e-5).numpy()
    np.testing.assert_allclose(rows[:, :512], ref_c, atol=1e-12)
    np.testing.assert_allclose(rows[0, 512:], y[0, 512:], atol=1e-12)
    zr = (y[:, 512::2] + 1j * y[:, 513::2]) * np.exp(1j * pos[:, None] * np.power(8.0e6, -np.arange(32) / 32.0))
    np.testing.assert_allclose(rows[:, 512::2], zr.real, atol=1e-9)
    np.testing.assert_allclose(rows[:, 513::2], zr.imag, atol=1e-9)


def test_absorbed_attention_equals_the_up_projected_form():
    """Per head: keys [W_UK c_s | r_s], values W_UV c_s, queries [q_nope | RoPE(q_rope)],
    scale 1/sqrt(d_nope + d_rope), attended with torch SDPA over the selected rows, equal
    W_UV applied to the absorbed attention (oracle.sparse_mla on absorb_queries)."""
    g = np.random.default_rng(4)
    H, d_lat, d_nope, d_rope, d_v, L = 3, 16, 12, 4, 8, 21
    scale = 1 / math.sqrt(d_nope + d_rope)
    w_uk = g.standard_normal((H, d_nope, d_lat)) / 4
    w_uv = g.standard_normal((H, d_v, d_lat)) / 4
    kv = np.concatenate([g.standard_normal((L, d_lat)),
                         P.rope_interleaved(g.standard_normal((L, d_rope)), np.arange(L))], axis=-1)
    q_nope, q_rope = g.standard_normal((2, H, d_nope)), g.standard_normal((2, H, d_rope))
    pos = np.array([20, 9])
    idx = np.array([[0, 3, 4, 9, 15, 20], [1, 2, 5, 9, -1, -1]], dtype=np.int32)
    cnt = np.array([6, 4], dtype=np.int32)
    qa = P.absorb_queries(q_nope, q_rope, w_uk, pos)
    kv32, qa32 = kv.astype(np.float32), qa.astype(np.float32)
    o_lat, _ = oracle.sparse_mla(qa32, kv32[None], [0, 0], idx, cnt, d_lat, scale)
    got = P.up_project(o_lat, w_uv)
    c, r = kv32[:, :d_lat].astype(np.float64), kv32[:, d_lat:].astype(np.float64)
    for i in range(2):
        sel = idx[i, : cnt[i]]
        k_h = np.concatenate([np.einsum("hkl,sl->hsk", w_uk, c[sel]), np.broadcast_to(r[sel], (H, len(sel), d_rope))], -1)
        v_h = np.einsum("hvl,sl->hsv", w_uv, c[sel])
        q_h = np.concatenate([q_nope[i], P.rope_interleaved(q_rope[i], pos[i])], -1)[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q_h), torch.from_numpy(k_h), torch.from_numpy(v_h), scale=scale).numpy()[:, 0]
        np.testing.assert_allclose(got[i], ref, rtol=1e-5, atol=1e-5)
