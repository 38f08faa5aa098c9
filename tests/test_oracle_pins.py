"""Pins for the fp64 oracle: each check rests on something other than the oracle.

Pins used (a plausible slip -- a dropped term, a wrong sign or index, a
transposed operand -- breaks at least one):
  * hand-worked examples under tests/golden/ (scores, selections, MLA outputs);
  * the identities relu(x) - relu(-x) = x and relu(x) + relu(-x) = |x|, which
    reduce the indexer to a plain matrix product (numpy matmul);
  * numpy's stable argsort as the reference ordering for top-k;
  * a brute-force validity check of every selection;
  * torch's scaled_dot_product_attention (float64, CPU) for the dense and the
    masked-sparse attention;
  * the non-absorbed MLA form (per-head up-projections W_UK, W_UV) against the
    absorbed form the oracle computes;
  * closed forms: constant rows, a single row, q = 0 (uniform weights);
  * the E4M3 8-bit float format's defining values and torch's float8_e4m3fn
    decoding, for the FP8 indexer variant, and the positive homogeneity of ReLU
    (a per-row scale of the keys or of a head's query factors out);
  * for the FP8 latent cache: torch's float8 / bf16 decoding of the packed bytes,
    SDPA on the exact values, and sparse_mla itself where power-of-two scales keep
    every value exact in float32.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- indexer
def test_indexer_hand_example():
    g = _load("indexer_topk_hand.json")
    q = np.array([g["q"], g["q"]], dtype=np.float32)
    w = np.array([g["w"], g["w"]], dtype=np.float32)
    k = np.array([g["k"]], dtype=np.float32)
    pos = [qq["pos"] for qq in g["queries"]]
    sc = oracle.index_scores(q, w, k, [0, 0], pos)
    for i, qq in enumerate(g["queries"]):
        n = qq["pos"] + 1
        assert sc[i, :n].tolist() == qq["scores"]
        assert np.all(np.isnan(sc[i, n:]))


def _rand_indexer(rng, n_q=5, H=3, D=7, n_seq=2, L=40):
    q = rng.integers(-4, 5, (n_q, H, D)).astype(np.float32)
    w = (2.0 ** rng.integers(-3, 2, (n_q, H))).astype(np.float32)
    k = rng.integers(-4, 5, (n_seq, L, D)).astype(np.float32)
    q_seq = rng.integers(0, n_seq, n_q).astype(np.int32)
    q_pos = np.full(n_q, L - 1, dtype=np.int32)
    return q, w, k, q_seq, q_pos


def test_indexer_relu_identities_reduce_to_matmul():
    rng = np.random.default_rng(0)
    q, w, k, q_seq, q_pos = _rand_indexer(rng)
    a = oracle.index_scores(q, w, k, q_seq, q_pos)
    b = oracle.index_scores(-q, w, k, q_seq, q_pos)
    for i in range(q.shape[0]):
        dots = k[q_seq[i]].astype(np.float64) @ q[i].astype(np.float64).T   # [L, H]
        lin = dots @ w[i].astype(np.float64)
        absd = np.abs(dots) @ w[i].astype(np.float64)
        np.testing.assert_allclose(a[i] - b[i], lin, rtol=0, atol=1e-9)
        np.testing.assert_allclose(a[i] + b[i], absd, rtol=0, atol=1e-9)


def test_indexer_single_head_nonnegative_is_matmul():
    rng = np.random.default_rng(1)
    q = rng.integers(0, 4, (3, 1, 9)).astype(np.float32)
    k = rng.integers(0, 4, (1, 17, 9)).astype(np.float32)
    w = np.ones((3, 1), dtype=np.float32)
    sc = oracle.index_scores(q, w, k, [0, 0, 0], [16, 16, 16])
    np.testing.assert_array_equal(sc, (q[:, 0, :].astype(np.float64) @ k[0].T.astype(np.float64)))


def test_indexer_one_hot_weight_selects_head():
    rng = np.random.default_rng(2)
    q, w, k, q_seq, q_pos = _rand_indexer(rng, H=4)
    for h in range(4):
        w1 = np.zeros_like(w)
        w1[:, h] = 1.0
        sc = oracle.index_scores(q, w1, k, q_seq, q_pos)
        for i in range(q.shape[0]):
            ref = np.maximum(k[q_seq[i]].astype(np.float64) @ q[i, h].astype(np.float64), 0.0)
            np.testing.assert_array_equal(sc[i], ref)


def test_indexer_causal_and_sequence_routing():
    rng = np.random.default_rng(3)
    q, w, k, q_seq, _ = _rand_indexer(rng, n_q=4, n_seq=3, L=30)
    q_pos = np.array([0, 7, 29, 13], dtype=np.int32)
    sc = oracle.index_scores(q, w, k, q_seq, q_pos)
    k2 = k.copy()
    for i in range(4):      # rows beyond a query's position must not matter
        k2[q_seq[i], q_pos[i] + 1:] = 99.0
    k2 = np.where(np.arange(30)[None, :, None] > q_pos.max(), 5.0, k2).astype(np.float32)
    sc2 = oracle.index_scores(q, w, k2, q_seq, q_pos)
    for i in range(4):
        n = q_pos[i] + 1
        assert np.isfinite(sc[i, :n]).all() and np.isnan(sc[i, n:]).all()
        # only this query's own sequence rows 0..t matter
        if all(q_pos[j] >= q_pos[i] or q_seq[j] != q_seq[i] for j in range(4)):
            np.testing.assert_array_equal(sc[i, :n], sc2[i, :n])
    # swapping caches together with q_seq gives the same scores
    perm = np.array([2, 0, 1])
    inv = np.argsort(perm)
    sc3 = oracle.index_scores(q, w, k[perm], inv[q_seq].astype(np.int32), q_pos)
    np.testing.assert_array_equal(np.nan_to_num(sc, nan=-1), np.nan_to_num(sc3, nan=-1))


def test_indexer_weight_linearity():
    rng = np.random.default_rng(4)
    q, w, k, q_seq, q_pos = _rand_indexer(rng)
    a = oracle.index_scores(q, w, k, q_seq, q_pos)
    b = oracle.index_scores(q, 4 * w, k, q_seq, q_pos)
    np.testing.assert_array_equal(4 * a, b)


# --------------------------------------------------------------------------- top-k
def test_topk_hand_examples():
    g = _load("indexer_topk_hand.json")
    q = np.array([g["q"]], dtype=np.float32)
    w = np.array([g["w"]], dtype=np.float32)
    k = np.array([g["k"]], dtype=np.float32)
    for qq in g["queries"]:
        sc = oracle.index_scores(q, w, k, [0], [qq["pos"]])
        for kk, expect in qq["topk"].items():
            idx, cnt = oracle.topk(sc, [qq["pos"]], int(kk))
            assert idx[0].tolist() == expect
            assert cnt[0] == min(int(kk), qq["pos"] + 1)
    for case in g["tie_cases"]:
        s = np.array([case["scores"]], dtype=np.float64)
        idx, cnt = oracle.topk(s, [s.shape[1] - 1], case["k"])
        assert idx[0].tolist() == case["idx"], case["why"]


def _is_valid_selection(scores_row, n, k, idx_row, cnt):
    kk = min(k, n)
    if cnt != kk:
        return False
    sel = idx_row[:kk]
    if not np.all(idx_row[kk:] == -1):
        return False
    if not (np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < n):
        return False
    chosen = set(sel.tolist())
    s = np.where(scores_row == 0, 0.0, scores_row)
    for a in chosen:                              # brute force: every kept row beats every dropped row
        for b in range(n):
            if b in chosen:
                continue
            if not (s[a] > s[b] or (s[a] == s[b] and a < b)):
                return False
    return True


@pytest.mark.parametrize("mode", ["ties", "normal", "equal"])
def test_topk_against_stable_argsort_and_brute_force(mode):
    n_q, L = 6, 53
    s = wl.random_scores(n_q, L, seed=11, mode=mode).double().numpy()
    q_pos = np.array([0, 3, 9, 25, 40, 52], dtype=np.int32)
    for k in (1, 4, 10, 26, 64):
        idx, cnt = oracle.topk(s, q_pos, k)
        for i in range(n_q):
            n = q_pos[i] + 1
            row = np.where(s[i, :n] == 0, 0.0, s[i, :n])
            order = np.argsort(-row, kind="stable")          # ties keep lower position first
            ref = np.sort(order[: min(k, n)])
            assert idx[i, : min(k, n)].tolist() == ref.tolist()
            assert _is_valid_selection(s[i, :n], n, k, idx[i], cnt[i])


def test_topk_ignores_invisible_scores():
    s = np.array([[1.0, 2.0, 3.0, 100.0, 100.0]])
    idx, cnt = oracle.topk(s, [2], 2)
    assert idx[0].tolist() == [1, 2] and cnt[0] == 2


# --------------------------------------------------------------------------- MLA
def test_mla_hand_examples():
    g = _load("mla_hand.json")
    for c in g["cases"]:
        q = np.array([[c["q"]]], dtype=np.float32)
        kv = np.array([c["rows"]], dtype=np.float32)
        n = kv.shape[1]
        idx = np.arange(n, dtype=np.int32)[None]
        out, lse = oracle.sparse_mla(q, kv, [0], idx, [n], c["d_lat"], c["scale"])
        if "out" in c:
            np.testing.assert_allclose(out[0, 0], c["out"], rtol=0, atol=1e-15)
        if "lse_minus_log2" in c:
            assert abs(lse[0, 0] - math.log(2) - c["lse_minus_log2"]) < 1e-15
        if "lse_minus_log3" in c:
            assert abs(lse[0, 0] - math.log(3) - c["lse_minus_log3"]) < 1e-15
        if "out_formula" in c:
            e = math.e
            p1 = e / (1 + e)
            np.testing.assert_allclose(out[0, 0], [4 * (1 - p1) + 8 * p1, -4 * (1 - p1)], atol=1e-14)
            assert abs(lse[0, 0] - math.log(1 + e)) < 1e-14


def _sdpa(q, k, v, mask, scale):
    """torch scaled_dot_product_attention in float64 on the CPU."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double(), torch.from_numpy(k).double(), torch.from_numpy(v).double(),
        attn_mask=torch.from_numpy(mask), scale=scale).numpy()


def _rand_mla(rng, n_q=4, H=3, d_lat=10, d_rope=4, n_seq=2, L=23):
    q = rng.standard_normal((n_q, H, d_lat + d_rope)).astype(np.float32)
    kv = rng.standard_normal((n_seq, L, d_lat + d_rope)).astype(np.float32)
    q_seq = rng.integers(0, n_seq, n_q).astype(np.int32)
    return q, kv, q_seq


def test_dense_mla_equals_sdpa():
    rng = np.random.default_rng(5)
    q, kv, q_seq = _rand_mla(rng)
    q_pos = np.array([0, 5, 22, 11], dtype=np.int32)
    out, _ = oracle.dense_mla(q, kv, q_seq, q_pos, 10, 0.3)
    for i in range(4):
        mask = np.arange(23) <= q_pos[i]
        ref = _sdpa(q[i][None], kv[q_seq[i]][None, None], kv[q_seq[i], :, :10][None, None],
                    mask[None, None, None, :].repeat(3, axis=2), 0.3)
        np.testing.assert_allclose(out[i], ref[0, 0] if ref.ndim == 4 else ref[0], atol=1e-12)


def test_sparse_mla_equals_masked_sdpa_and_dense_when_topk_covers():
    rng = np.random.default_rng(6)
    q, kv, q_seq = _rand_mla(rng)
    q_pos = np.array([3, 22, 9, 15], dtype=np.int32)
    topk = 8
    idx = np.full((4, topk), -1, dtype=np.int32)
    cnt = np.zeros(4, dtype=np.int32)
    for i in range(4):
        n = q_pos[i] + 1
        sel = np.sort(rng.choice(n, size=min(topk, n), replace=False))
        idx[i, : len(sel)] = sel
        cnt[i] = len(sel)
    out, lse = oracle.sparse_mla(q, kv, q_seq, idx, cnt, 10, 0.25)
    for i in range(4):
        mask = np.zeros(23, dtype=bool)
        mask[idx[i, : cnt[i]]] = True
        ref = _sdpa(q[i][None], kv[q_seq[i]][None, None], kv[q_seq[i], :, :10][None, None],
                    np.broadcast_to(mask, (1, 1, 3, 23)).copy(), 0.25)
        np.testing.assert_allclose(out[i], ref.reshape(3, 10), atol=1e-12)
    # topk >= visible count: sparse == dense causal attention
    full_idx = np.full((4, 32), -1, dtype=np.int32)
    for i in range(4):
        full_idx[i, : q_pos[i] + 1] = np.arange(q_pos[i] + 1)
    out_s, lse_s = oracle.sparse_mla(q, kv, q_seq, full_idx, q_pos + 1, 10, 0.25)
    out_d, lse_d = oracle.dense_mla(q, kv, q_seq, q_pos, 10, 0.25)
    np.testing.assert_array_equal(out_s, out_d)
    np.testing.assert_array_equal(lse_s, lse_d)


def test_mla_closed_forms():
    rng = np.random.default_rng(7)
    q, kv, q_seq = _rand_mla(rng, n_q=1, n_seq=1)
    const = rng.standard_normal(10).astype(np.float32)
    kv_c = kv.copy()
    kv_c[0, :, :10] = const                                  # identical latents
    idx = np.arange(12, dtype=np.int32)[None]
    out, _ = oracle.sparse_mla(q, kv_c, [0], idx, [12], 10, 0.7)
    np.testing.assert_allclose(out[0], np.broadcast_to(const, (3, 10)), atol=1e-12)  # sum p = 1
    one = np.array([[17]], dtype=np.int32)
    out1, lse1 = oracle.sparse_mla(q, kv, [0], one, [1], 10, 0.7)
    np.testing.assert_array_equal(out1[0], np.broadcast_to(kv[0, 17, :10].astype(np.float64), (3, 10)))
    np.testing.assert_allclose(lse1[0], 0.7 * (q[0].astype(np.float64) @ kv[0, 17].astype(np.float64)), atol=1e-12)
    qz = np.zeros_like(q)
    outz, lsez = oracle.sparse_mla(qz, kv, [0], idx, [12], 10, 0.7)
    np.testing.assert_allclose(outz[0], np.broadcast_to(kv[0, :12, :10].astype(np.float64).mean(0), (3, 10)), atol=1e-12)
    np.testing.assert_allclose(lsez[0], math.log(12), atol=1e-13)


def test_sparse_mla_order_of_selection_is_irrelevant():
    rng = np.random.default_rng(8)
    q, kv, q_seq = _rand_mla(rng, n_q=2)
    idx = np.array([[1, 4, 9, 20], [0, 2, 3, 7]], dtype=np.int32)
    a, la = oracle.sparse_mla(q, kv, q_seq, idx, [4, 4], 10, 0.5)
    b, lb = oracle.sparse_mla(q, kv, q_seq, idx[:, ::-1].copy(), [4, 4], 10, 0.5)
    np.testing.assert_allclose(a, b, atol=1e-13)
    np.testing.assert_allclose(la, lb, atol=1e-13)


def test_absorbed_equals_non_absorbed_mla():
    """Non-absorbed MLA (per-head k_nope = W_UK c, v = W_UV c, 192 + 64 query dims,
    scale 1/sqrt(256)) equals the absorbed form with q_lat = W_UK^T q_nope,
    followed by W_UV on the absorbed output."""
    rng = np.random.default_rng(9)
    H, d_lat, d_rope, d_nope, d_v, L = 3, 16, 4, 12, 8, 19
    scale = 1.0 / math.sqrt(d_nope + d_rope)
    W_UK = rng.standard_normal((H, d_nope, d_lat))
    W_UV = rng.standard_normal((H, d_v, d_lat))
    c = rng.standard_normal((L, d_lat))
    r = rng.standard_normal((L, d_rope))
    q_nope = rng.standard_normal((H, d_nope))
    q_rope = rng.standard_normal((H, d_rope))
    # textbook multi-head attention over up-projected keys and values
    ref = np.zeros((H, d_v))
    for h in range(H):
        k_h = np.concatenate([c @ W_UK[h].T, r], axis=1)          # [L, d_nope + d_rope]
        v_h = c @ W_UV[h].T                                       # [L, d_v]
        logits = scale * (k_h @ np.concatenate([q_nope[h], q_rope[h]]))
        p = np.exp(logits - logits.max())
        ref[h] = (p / p.sum()) @ v_h
    q_lat = np.einsum("hnl,hn->hl", W_UK, q_nope)
    # float32 inputs: keep values exactly representable by rounding first
    q_abs = np.concatenate([q_lat, q_rope], axis=1).astype(np.float32)
    kv = np.concatenate([c, r], axis=1).astype(np.float32)[None]
    out, _ = oracle.sparse_mla(q_abs[None], kv, [0], np.arange(L, dtype=np.int32)[None], [L], d_lat, scale)
    got = np.einsum("hvl,hl->hv", W_UV, out[0])
    # the only difference is float32 rounding of the inputs
    np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-4)


# --------------------------------------------------------------------------- IndexShare
def test_indexshare_group_reuses_layer0_selection():
    w = wl.scaled(wl.NAMED["tiny"], n_layers=3, L=96, q_pos=(40, 95, 70), q_seq=(0, 0, 0), topk=16)
    x = wl.make_inputs(w)
    f = lambda t: t.float().numpy()
    idx, cnt, outs, lses = oracle.indexshare_group(
        f(x["q_idx"]), f(x["w"]), f(x["k_idx"]), x["q_seq"].numpy(), x["q_pos"].numpy(), w.topk,
        [f(t) for t in x["q_mla"]], [f(t) for t in x["kv"]], w.d_lat, w.scale)
    sc = oracle.index_scores(f(x["q_idx"]), f(x["w"]), f(x["k_idx"]), x["q_seq"].numpy(), x["q_pos"].numpy())
    idx0, cnt0 = oracle.topk(sc, x["q_pos"].numpy(), w.topk)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_array_equal(cnt, cnt0)
    for layer in range(3):
        o, l = oracle.sparse_mla(f(x["q_mla"][layer]), f(x["kv"][layer]), x["q_seq"].numpy(), idx0, cnt0,
                                 w.d_lat, w.scale)
        np.testing.assert_array_equal(outs[layer], o)
        np.testing.assert_array_equal(lses[layer], l)
    assert not np.array_equal(outs[0], outs[1])        # layers really differ


# --------------------------------------------------------------------------- input recipe
def test_integer_recipe_scores_exact_in_float32():
    """With the integer/power-of-two recipe every score is exactly representable
    in float32 (so top-k decisions do not depend on summation order)."""
    w = wl.scaled(wl.NAMED["decode_32k"], n_seq=2, L=300, q_pos=(299, 150), q_seq=(0, 1))
    x = wl.make_inputs(w, layers=[])
    sc = oracle.index_scores(x["q_idx"].float().numpy(), x["w"].numpy(), x["k_idx"].float().numpy(),
                             x["q_seq"].numpy(), x["q_pos"].numpy())
    vis = sc[np.isfinite(sc)]
    assert np.all(vis.astype(np.float32).astype(np.float64) == vis)
    assert np.all(vis * 8 == np.round(vis * 8)) and vis.max() < 2 ** 17


# --------------------------------------------------------------------------- FP8 (E4M3) indexer variant
@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x38, 1.0), (0x40, 2.0), (0x44, 3.0), (0x48, 4.0), (0x30, 0.5), (0x3C, 1.5),
    (0x7E, 448.0), (0xFE, -448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0xB8, -1.0),
])
def test_e4m3_defining_values(code, value):
    # sign | 4-bit exponent (bias 7) | 3-bit mantissa; exponent 0 is subnormal (m/8 * 2^-6)
    assert oracle.e4m3_to_double(code) == value


def test_e4m3_nan_and_signed_zero():
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))
    z = oracle.e4m3_to_double(0x80)
    assert z == 0.0 and math.copysign(1.0, z) == -1.0


def test_e4m3_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_double(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def _fp8_case(seed, n_q=3, n_seq=2, L=37, heads=4, dim=16):
    g = torch.Generator().manual_seed(seed)
    qv = torch.randint(-4, 5, (n_q, heads, dim), generator=g).float()
    kv = torch.randint(-4, 5, (n_seq, L, dim), generator=g).float()
    q8 = qv.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    k8 = kv.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    w = torch.pow(2.0, torch.randint(-3, 2, (n_q, heads), generator=g).float()).numpy()
    q_seq = np.array([0, 1, 1][:n_q], dtype=np.int32)
    q_pos = np.array([L - 1, L - 5, 11][:n_q], dtype=np.int32)
    return qv.numpy(), kv.numpy(), q8, k8, w, q_seq, q_pos


def test_fp8_scores_with_unit_scales_equal_the_float_definition():
    qv, kv, q8, k8, w, q_seq, q_pos = _fp8_case(1)
    got = oracle.index_scores_e4m3(q8, None, w, k8, None, q_seq, q_pos)
    # the same integers as float32 through relu(x) = (x + |x|) / 2 and a plain matmul
    for i in range(qv.shape[0]):
        dots = np.einsum("hd,sd->hs", qv[i].astype(np.float64), kv[q_seq[i]].astype(np.float64))
        ref = (w[i][:, None] * (dots + np.abs(dots)) / 2).sum(0)
        t = q_pos[i]
        np.testing.assert_array_equal(got[i, : t + 1], ref[: t + 1])
        assert np.all(np.isnan(got[i, t + 1:]))


def test_fp8_scales_factor_out_of_relu():
    qv, kv, q8, k8, w, q_seq, q_pos = _fp8_case(2)
    g = np.random.default_rng(3)
    n_q, heads, _ = q8.shape
    n_seq, L, _ = k8.shape
    q_scale = g.uniform(0.25, 3.0, size=(n_q, heads)).astype(np.float32)
    k_scale = g.uniform(0.25, 3.0, size=(n_seq, L)).astype(np.float32)
    base = oracle.index_scores_e4m3(q8, None, w, k8, None, q_seq, q_pos)
    # a positive per-key scale multiplies that key's score
    with_k = oracle.index_scores_e4m3(q8, None, w, k8, k_scale, q_seq, q_pos)
    # a positive per-(query, head) scale acts as a factor on that head's weight
    with_q = oracle.index_scores_e4m3(q8, q_scale, w, k8, None, q_seq, q_pos)
    for i in range(n_q):
        t = q_pos[i]
        np.testing.assert_allclose(with_k[i, : t + 1], base[i, : t + 1] * k_scale[q_seq[i], : t + 1], rtol=1e-12)
        dots = np.einsum("hd,sd->hs", qv[i].astype(np.float64), kv[q_seq[i], : t + 1].astype(np.float64))
        ref_q = ((w[i].astype(np.float64) * q_scale[i].astype(np.float64))[:, None] * np.maximum(dots, 0)).sum(0)
        np.testing.assert_allclose(with_q[i, : t + 1], ref_q, rtol=1e-12)


# --------------------------------------------------------------------------- FP8 latent cache
def _pack_fp8_rows(codes_u8, rope_bf16, sigma_f32, row_bytes):
    """Byte rows [codes | RoPE bf16 | float32 scale | zero padding] from torch tensors
    ([..., d_lat] uint8, [..., d_rope] bf16, [...] float32)."""
    d_lat, d_rope = codes_u8.shape[-1], rope_bf16.shape[-1]
    rows = torch.zeros(codes_u8.shape[:-1] + (row_bytes,), dtype=torch.uint8)
    rows[..., :d_lat] = codes_u8
    rows[..., d_lat: d_lat + 2 * d_rope] = rope_bf16.contiguous().view(torch.uint8)
    rows[..., d_lat + 2 * d_rope: d_lat + 2 * d_rope + 4] = sigma_f32.contiguous().unsqueeze(-1).view(torch.uint8)
    return rows


def _fp8_cache(seed, n_seq, L, d_lat, d_rope, pow2_scales=False):
    """A random packed cache plus its exact values: (rows uint8, c float64, r float64)."""
    g = torch.Generator().manual_seed(seed)
    code = (torch.randn((n_seq, L, d_lat), generator=g) * 64).clamp(-448, 448).to(torch.float8_e4m3fn)
    rope = torch.randn((n_seq, L, d_rope), generator=g).to(torch.bfloat16)
    if pow2_scales:
        sigma = torch.pow(2.0, torch.randint(-7, -4, (n_seq, L), generator=g).float())
    else:
        sigma = torch.rand((n_seq, L), generator=g) * 0.05 + 0.003
    rows = _pack_fp8_rows(code.view(torch.uint8), rope, sigma, wl.fp8_row_bytes(d_lat, d_rope))
    # exact values through torch's own float8 / bf16 decoding
    c = code.to(torch.float64) * sigma.to(torch.float64)[..., None]
    r = rope.to(torch.float64)
    return rows.numpy(), c.numpy(), r.numpy()


def test_fp8_latent_single_row_is_the_scaled_row():
    """One selected row: the softmax weight is 1, so the output is that row's latent
    sigma * e4m3(code) exactly, and lse is the row's scaled logit (which also reads
    the RoPE bytes)."""
    d_lat, d_rope, H = 512, 64, 4
    rows, c, r = _fp8_cache(11, 1, 40, d_lat, d_rope)
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1, H, d_lat + d_rope)).astype(np.float32)
    out, lse = oracle.sparse_mla_fp8(q, rows, [0], np.array([[29]], np.int32), [1], d_lat, d_rope, 0.0625)
    np.testing.assert_array_equal(out[0], np.broadcast_to(c[0, 29], (H, d_lat)))
    row = np.concatenate([c[0, 29], r[0, 29]])
    np.testing.assert_allclose(lse[0], 0.0625 * (q[0].astype(np.float64) @ row), rtol=1e-13, atol=1e-13)


def test_fp8_latent_equals_sdpa_on_the_exact_cache():
    """Random selections on small dims against torch SDPA (float64) over the exact
    values; with topk covering every visible row, against dense causal SDPA."""
    d_lat, d_rope, H, L, n_seq, n_q = 12, 4, 3, 23, 2, 4
    rows, c, r = _fp8_cache(13, n_seq, L, d_lat, d_rope)
    kv = np.concatenate([c, r], axis=-1)
    rng = np.random.default_rng(14)
    q = rng.standard_normal((n_q, H, d_lat + d_rope)).astype(np.float32)
    q_seq = np.array([0, 1, 1, 0], np.int32)
    q_pos = np.array([4, 22, 9, 17], np.int32)
    topk = 8
    idx = np.full((n_q, topk), -1, np.int32)
    cnt = np.zeros(n_q, np.int32)
    for i in range(n_q):
        sel = np.sort(rng.choice(q_pos[i] + 1, size=min(topk, q_pos[i] + 1), replace=False))
        idx[i, : len(sel)] = sel
        cnt[i] = len(sel)
    scale = 1 / math.sqrt(11.0)
    out, _ = oracle.sparse_mla_fp8(q, rows, q_seq, idx, cnt, d_lat, d_rope, scale)
    full = np.full((n_q, L), -1, np.int32)
    for i in range(n_q):
        full[i, : q_pos[i] + 1] = np.arange(q_pos[i] + 1)
    out_all, _ = oracle.sparse_mla_fp8(q, rows, q_seq, full, q_pos + 1, d_lat, d_rope, scale)
    for i in range(n_q):
        for sel, o in ((idx[i, : cnt[i]], out[i]), (np.arange(q_pos[i] + 1), out_all[i])):
            mask = np.zeros(L, dtype=bool)
            mask[sel] = True
            ref = _sdpa(q[i][None], kv[q_seq[i]][None, None], c[q_seq[i]][None, None],
                        np.broadcast_to(mask, (1, 1, H, L)).copy(), scale)
            np.testing.assert_allclose(o, ref.reshape(H, d_lat), atol=1e-12)


def test_fp8_latent_with_power_of_two_scales_equals_the_float_oracle():
    """With power-of-two scales every latent value is exact in float32, so the FP8
    form must agree with sparse_mla on the float cache (same arithmetic order:
    bit for bit), at the GLM-5.2 sizes."""
    d_lat, d_rope, H, L = 512, 64, 8, 300
    rows, c, r = _fp8_cache(15, 2, L, d_lat, d_rope, pow2_scales=True)
    kv = np.concatenate([c, r], axis=-1).astype(np.float32)
    assert np.array_equal(kv.astype(np.float64), np.concatenate([c, r], axis=-1))
    rng = np.random.default_rng(16)
    q = rng.standard_normal((3, H, d_lat + d_rope)).astype(np.float32)
    q_seq = np.array([1, 0, 1], np.int32)
    idx = np.full((3, 64), -1, np.int32)
    cnt = np.array([64, 17, 1], np.int32)
    for i in range(3):
        idx[i, : cnt[i]] = np.sort(rng.choice(L, size=cnt[i], replace=False))
    a, la = oracle.sparse_mla_fp8(q, rows, q_seq, idx, cnt, d_lat, d_rope, 0.0625)
    b, lb = oracle.sparse_mla(q, kv, q_seq, idx, cnt, d_lat, 0.0625)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)


def test_fp8_latent_padding_bytes_are_ignored():
    d_lat, d_rope = 512, 64
    rows, _, _ = _fp8_cache(17, 1, 50, d_lat, d_rope)
    noisy = rows.copy()
    noisy[..., d_lat + 2 * d_rope + 4:] = np.random.default_rng(18).integers(0, 256, size=noisy[..., 644:].shape)
    rng = np.random.default_rng(19)
    q = rng.standard_normal((2, 4, d_lat + d_rope)).astype(np.float32)
    idx = np.array([[0, 7, 33, 49], [2, 3, -1, -1]], np.int32)
    a, la = oracle.sparse_mla_fp8(q, rows, [0, 0], idx, [4, 2], d_lat, d_rope, 0.0625)
    b, lb = oracle.sparse_mla_fp8(q, noisy, [0, 0], idx, [4, 2], d_lat, d_rope, 0.0625)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)


def test_fp8_latent_generator_layout():
    """fp8_latent_inputs holds the layer's bf16 cache in 8 bits: the RoPE key
    copied, every row's largest code at E4M3's 448, latents within E4M3's
    rounding (3 mantissa bits: relative error <= 2^-4, absolute <= 2^-10 * scale
    in the subnormal range) of the bf16 ones, zero padding."""
    w = wl.scaled(wl.NAMED["decode_32k"], n_seq=2, L=64, q_pos=(63, 10), q_seq=(0, 1))
    x = wl.make_inputs(w)
    rows = wl.fp8_latent_inputs(w, x)[0]
    assert rows.shape == (2, 64, 656) and rows.dtype == torch.uint8
    assert torch.equal(rows[..., 512:640].contiguous().view(torch.bfloat16), x["kv"][0][..., 512:])
    sigma = rows[..., 640:644].contiguous().view(torch.float32)
    codes = rows[..., :512].contiguous().view(torch.float8_e4m3fn).float()
    assert not torch.isnan(codes).any()
    assert torch.all(codes.abs().amax(-1) == 448.0)
    c = x["kv"][0][..., :512].float()
    err = (codes * sigma - c).abs()
    assert torch.all(err <= torch.maximum(c.abs() * 2.0 ** -4, sigma * 2.0 ** -10) * (1 + 1e-6))
    assert int(rows[..., 644:].sum()) == 0


def test_mtp_shared_selection_equals_masked_sdpa_per_query():
    """sparse_mla_mtp: every query of a group attends over its group's one
    selection -- checked per query against float64 SDPA with that selection as
    the mask (no oracle call on the reference side), and with one draft token
    per group it is sparse_mla itself."""
    rng = np.random.default_rng(61)
    D, n_g, H, d_lat, d_rope, L = 3, 2, 3, 10, 4, 23
    q = rng.standard_normal((n_g * D, H, d_lat + d_rope)).astype(np.float32)
    kv = rng.standard_normal((n_g, L, d_lat + d_rope)).astype(np.float32)
    q_seq = np.repeat(np.arange(n_g, dtype=np.int32), D)
    topk = 6
    idx_g = np.full((n_g, topk), -1, dtype=np.int32)
    cnt_g = np.array([6, 4], dtype=np.int32)
    for g in range(n_g):
        idx_g[g, : cnt_g[g]] = np.sort(rng.choice(15, size=cnt_g[g], replace=False))
    out, lse = oracle.sparse_mla_mtp(q, kv, q_seq, idx_g, cnt_g, D, d_lat, 0.3)
    for i in range(n_g * D):
        g = i // D
        mask = np.zeros(L, dtype=bool)
        mask[idx_g[g, : cnt_g[g]]] = True
        ref = _sdpa(q[i][None], kv[q_seq[i]][None, None], kv[q_seq[i], :, :d_lat][None, None],
                    np.broadcast_to(mask, (1, 1, H, L)).copy(), 0.3)
        np.testing.assert_allclose(out[i], ref.reshape(H, d_lat), atol=1e-12)
    # queries of one group differ (their own q), so their outputs differ
    assert not np.allclose(out[0], out[1])
    o1, l1 = oracle.sparse_mla_mtp(q[:n_g], kv, np.arange(n_g, dtype=np.int32), idx_g, cnt_g, 1, d_lat, 0.3)
    o2, l2 = oracle.sparse_mla(q[:n_g], kv, np.arange(n_g, dtype=np.int32), idx_g, cnt_g, d_lat, 0.3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
