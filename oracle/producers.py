"""fp64 oracle of the producers around the attention path: what writes a token's
cache rows from its hidden state, and the per-head query absorption and output
up-projection of the absorbed MLA form.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the test-suite is the
only caller.  Plain numpy in float64; a matrix product is the one library step.

Passages followed (page title, section):
  [TM]  "GLM-5.2 -- Model techniques map", "Checked in its code":
        Multi-head latent attention -- kv_a_proj_with_mqa maps the hidden state to
        the 512-dim latent plus the 64-dim RoPE key, kv_a_layernorm (an RMSNorm
        over the latent), kv_b_proj up-projects the latent per head into a
        192-dim no-RoPE key part and a 256-dim value;
        QK normalization -- the indexer key is k_norm(wk(h)), k_norm a LayerNorm;
        Partial RoPE -- heads split [no-RoPE 192 | RoPE 64].
  [HA]  "GLM 5.2 -- Hermosa AI", "MLA + DSA with IndexShare": RoPE theta 8e6.
  [LA]  "GLM-5.2 -- LLM atlas", raw config.json fields: rope_interleave and
        indexer_rope_interleave true, rms_norm_eps 1e-5, qk_rope_head_dim 64,
        v_head_dim 256.

Readings where the pages are silent (listed with the others in the design notes):
  - interleaved RoPE rotates adjacent pairs (x[2i], x[2i+1]) of the RoPE part by
    pos * theta^(-2i/d), d the RoPE part's size;
  - the indexer key's RoPE part is its last 64 dims (qk_rope_head_dim), the
    RoPE part coming last as in every split the pages print;
  - LayerNorm and RMSNorm use eps = 1e-5 and carry a per-channel weight
    (LayerNorm also a bias).
"""
from __future__ import annotations

import numpy as np

ROPE_THETA = 8.0e6
NORM_EPS = 1e-5


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def rope_interleaved(x, pos, theta: float = ROPE_THETA):
    """x [..., d] (d even), pos broadcastable to x.shape[:-1]: each adjacent pair
    (x[2i], x[2i+1]) rotated by the angle pos * theta^(-2i/d)."""
    x = _f64(x)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d)                            # [d/2]
    ang = _f64(pos)[..., None] * inv_freq                          # [..., d/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def layer_norm(x, weight, bias, eps: float = NORM_EPS):
    """(x - mean) / sqrt(var + eps) * weight + bias over the last axis (biased var)."""
    x = _f64(x)
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).mean(-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(weight) + _f64(bias)


def rms_norm(x, weight, eps: float = NORM_EPS):
    """x / sqrt(mean(x^2) + eps) * weight over the last axis."""
    x = _f64(x)
    return x / np.sqrt((x * x).mean(-1, keepdims=True) + eps) * _f64(weight)


def indexer_keys(h, w_k, ln_weight, ln_bias, pos, d_rope: int = 64, theta: float = ROPE_THETA):
    """Indexer keys of tokens at positions pos: k = LayerNorm(h @ w_k), then RoPE on
    the last d_rope dims.  h [T, hidden], w_k [hidden, dim] -> [T, dim]."""
    k = layer_norm(_f64(h) @ _f64(w_k), ln_weight, ln_bias)
    k[..., -d_rope:] = rope_interleaved(k[..., -d_rope:], pos, theta)
    return k


def latent_rows(h, w_kva, norm_weight, pos, d_lat: int = 512, theta: float = ROPE_THETA):
    """Cache rows [c | r] of tokens at positions pos: h @ w_kva = [c~ | r~],
    c = RMSNorm(c~), r = RoPE(r~).  h [T, hidden], w_kva [hidden, d_lat + d_rope]."""
    y = _f64(h) @ _f64(w_kva)
    c = rms_norm(y[..., :d_lat], norm_weight)
    r = rope_interleaved(y[..., d_lat:], pos, theta)
    return np.concatenate([c, r], axis=-1)


def absorb_queries(q_nope, q_rope, w_uk, pos, theta: float = ROPE_THETA):
    """Absorbed MLA queries: per head h, q_lat[h] = w_uk[h]^T q_nope[h] (the no-RoPE
    key up-projection folded into the query) and the RoPE part rotated.
    q_nope [n, H, d_nope], q_rope [n, H, d_rope] (before RoPE), w_uk [H, d_nope,
    d_lat], pos [n] -> [n, H, d_lat + d_rope]."""
    q_lat = np.einsum("nhk,hkl->nhl", _f64(q_nope), _f64(w_uk))
    q_r = rope_interleaved(q_rope, _f64(pos)[:, None], theta)
    return np.concatenate([q_lat, q_r], axis=-1)


def up_project(o_lat, w_uv):
    """Per-head value up-projection of the absorbed output: o[h] = w_uv[h] @ o_lat[h].
    o_lat [n, H, d_lat], w_uv [H, d_v, d_lat] -> [n, H, d_v]."""
    return np.einsum("hvl,nhl->nhv", _f64(w_uv), _f64(o_lat))
