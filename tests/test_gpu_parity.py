"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs.  Indices are compared bit for bit (the input recipe
makes every score exact in float32); attention outputs within max-abs 2e-2 and
mean-abs 2e-3 on bf16 outputs (tighter on the fp32 path)."""
import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_top_b200 import binding as B
from dsa_indexer_top_b200 import workloads as wl
from tests import common as C

pytestmark = pytest.mark.gpu

D32 = wl.NAMED["decode_32k"]

SMALL = {
    "tiny": wl.NAMED["tiny"],
    # n > topk, n < topk, n == topk, n == topk + 1 in one batch
    "decode_edges": wl.scaled(D32, n_seq=4, L=3000, q_pos=(2999, 1500, 2047, 2048), q_seq=(0, 1, 2, 3)),
    # context not a multiple of the 128-key tile, queries on a ragged tail
    "decode_ragged": wl.scaled(D32, n_seq=2, L=5037, q_pos=(5036, 4100), q_seq=(0, 1), seed=7),
    # several queries of one sequence share a tensor-core tile (seq_run = 40 -> 8 per tile)
    "prefill_small": wl.scaled(D32, n_seq=1, L=4173, q_pos=tuple(range(3000, 3040)), q_seq=(0,) * 40, seed=8),
    # causal start: positions 0..63 (every query keeps all visible rows)
    "prefill_start": wl.scaled(D32, n_seq=1, L=4096, q_pos=tuple(range(64)), q_seq=(0,) * 64, seed=9),
    # every sequence reads one shared cache (sequence stride 0)
    "shared_cache": wl.scaled(D32, n_seq=3, L=2600, q_pos=(2599, 2400, 2100), q_seq=(0, 1, 2),
                              shared_cache=True, seed=10),
    # heavy ties: indexer values in {-1, 0, 1}
    "ties": wl.scaled(D32, n_seq=2, L=6000, q_pos=(5999, 4444), q_seq=(0, 1), int_range=1, seed=11),
    # IndexShare group of 4 layers
    "indexshare_small": wl.scaled(D32, n_seq=2, L=3000, q_pos=(2999, 2500), q_seq=(0, 1), n_layers=4, seed=12),
}


def seq_run_of(w):
    runs = [w.n_q] if len(set(w.q_seq)) == 1 else [1]
    return runs[0]


@pytest.fixture(scope="module")
def dev(cuda_ok):
    B.lib()
    return torch.device("cuda")


def _run_steps(w, x, decode=True, fused=True):
    """The three-call chain (as timed by the benchmark): scores -> top-k -> MLA;
    `fused`: the indexer leaves the top-k's first-digit histograms."""
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run_of(w))
    if fused:
        ix.flags = B.DSA_INDEXER_TOPK_HIST
    dev = x["q_pos"].device
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    B.dsa_index_scores(q, ix, scores, ws)
    idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
    B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER if fused else 0)
    for m in mlas:
        (B.dsa_sparse_mla_decode if decode else B.dsa_sparse_mla_prefill)(q, m, idx, cnt, w.topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    return scores, idx, cnt, mlas


@pytest.mark.parametrize("name", ["decode_edges", "decode_ragged", "ties"])
@pytest.mark.parametrize("L_long", [False, True])
def test_repeated_steps_one_workspace(dev, name, L_long):
    """Several fused indexer -> top-k steps on one workspace: the top-k leaves the
    histograms and tickets zero for the next indexer launch, so every step
    matches the oracle (L_long: a context above the split-schedule threshold)."""
    w = SMALL[name]
    if L_long:
        w = wl.scaled(w, L=20000, q_pos=tuple(min(19999, p + 15000) for p in w.q_pos))
    xh = wl.make_inputs(w, layers=[])
    x = C.to_device(xh)
    q, ix, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    _, ridx, rcnt = C.oracle_selection(w, xh)
    for step in range(3):
        idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
        B.dsa_index_scores(q, ix, scores, ws)
        B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        assert B.dsa_check_status(ws) == B.DSA_OK
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt, err_msg=f"step {step}")
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx, err_msg=f"step {step}")


@pytest.mark.parametrize("L_long", [False, True])
def test_repeated_full_steps_one_workspace(dev, L_long):
    """The benchmark's step -- fused indexer, top-k, decode attention as three
    calls on one workspace -- three times in a row: the attention's split-K
    partials must not land on the histograms and tickets the next step's indexer
    and top-k expect zero, so every step matches the oracle."""
    w = SMALL["decode_edges"]
    if L_long:
        w = wl.scaled(w, L=20000, q_pos=tuple(min(19999, p + 15000) for p in w.q_pos))
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    _, ridx, rcnt = C.oracle_selection(w, xh)
    ref, ref_lse = C.oracle_mla(w, xh, 0, ridx, rcnt)
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    for step in range(3):
        idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
        mlas[0].out.fill_(float("nan"))
        B.dsa_index_scores(q, ix, scores, ws)
        B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        B.dsa_sparse_mla_decode(q, mlas[0], idx, cnt, w.topk, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK, f"step {step}"
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt, err_msg=f"step {step}")
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx, err_msg=f"step {step}")
        C.assert_attention_close(mlas[0].out, ref, w.dtype, f"step {step}")
        C.assert_lse_close(mlas[0].lse, ref_lse, w.dtype)


def test_bounded_wait_times_out_and_context_stays_usable(dev):
    """A device wait on a barrier that nothing completes gives up after its limit,
    reports DSA_ERR_TIMEOUT through the workspace status word (no hang, no
    fault), and the next calls on the same context are correct."""
    w = SMALL["decode_edges"]
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    q, _, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    B.dsa_debug_bounded_wait(ws, 20_000_000)  # 20 ms
    assert B.dsa_check_status(ws) == B.DSA_ERR_TIMEOUT
    assert B.dsa_check_status(ws) == B.DSA_OK  # read-and-clear
    _, idx, cnt, mlas = _run_steps(w, x)
    _, ridx, rcnt = C.oracle_selection(w, xh)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)


FP8_CASES = ["decode_edges", "decode_ragged", "prefill_small", "shared_cache", "ties"]


@pytest.mark.parametrize("name", FP8_CASES)
def test_fp8_index_scores_bit_exact(dev, name):
    """FP8 (E4M3) indexer with per-(query, head) and per-key scales: every visible
    score equals the oracle's (exact on the recipe's values)."""
    w = SMALL[name]
    xh = wl.make_inputs(w, layers=[])
    f8h = wl.fp8_indexer_inputs(w, xh)
    x, f8 = C.to_device(xh), C.to_device(f8h)
    q, _, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix = C.fp8_indexer(w, f8, x)
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    scores.fill_(float("nan"))
    B.dsa_index_scores(q, ix, scores, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    ref, _, _ = C.oracle_selection_fp8(w, f8h, xh)
    got = scores[:, : w.L].cpu().double().numpy()
    for i, t in enumerate(w.q_pos):
        np.testing.assert_array_equal(got[i, : t + 1], ref[i, : t + 1], err_msg=f"query {i}")


@pytest.mark.parametrize("name", ["decode_edges", "decode_ragged", "ties"])
@pytest.mark.parametrize("L_long", [False, True])
def test_fp8_fused_topk_matches_oracle(dev, name, L_long):
    """FP8 indexer with the fused first-digit histogram, then the top-k (row and
    split schedules), twice on one workspace: indices bit-exact both times."""
    w = SMALL[name]
    if L_long:
        w = wl.scaled(w, L=20000, q_pos=tuple(min(19999, p + 15000) for p in w.q_pos))
    xh = wl.make_inputs(w, layers=[])
    f8h = wl.fp8_indexer_inputs(w, xh)
    x, f8 = C.to_device(xh), C.to_device(f8h)
    q, _, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix = C.fp8_indexer(w, f8, x, flags=B.DSA_INDEXER_TOPK_HIST)
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    _, ridx, rcnt = C.oracle_selection_fp8(w, f8h, xh)
    for step in range(2):
        idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
        B.dsa_index_scores(q, ix, scores, ws)
        B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        assert B.dsa_check_status(ws) == B.DSA_OK
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt, err_msg=f"step {step}")
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx, err_msg=f"step {step}")


@pytest.mark.parametrize("which", ["no_q_scale", "no_k_scale", "no_scales"])
def test_fp8_null_scales_mean_one(dev, which):
    """FP8 scale arrays may be NULL (all 1): scores equal the oracle's with unit
    scales for the missing side."""
    w = SMALL["decode_ragged"]
    xh = wl.make_inputs(w, layers=[])
    f8h = wl.fp8_indexer_inputs(w, xh)
    if which in ("no_q_scale", "no_scales"):
        f8h["q_scale"] = torch.ones_like(f8h["q_scale"])
    if which in ("no_k_scale", "no_scales"):
        f8h["k_scale"] = torch.ones_like(f8h["k_scale"])
    x, f8 = C.to_device(xh), C.to_device(f8h)
    q, _, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix = C.fp8_indexer(w, f8, x)
    if which in ("no_q_scale", "no_scales"):
        ix.q_scale = None
    if which in ("no_k_scale", "no_scales"):
        ix.k_scale = None
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    B.dsa_index_scores(q, ix, scores, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    ref, _, _ = C.oracle_selection_fp8(w, f8h, xh)
    got = scores[:, : w.L].cpu().double().numpy()
    for i, t in enumerate(w.q_pos):
        np.testing.assert_array_equal(got[i, : t + 1], ref[i, : t + 1], err_msg=f"query {i}")


def test_fp8_unsupported_shape_is_rejected(dev):
    """The tiny workload's 4 x 32 indexer has no FP8 path: rejected before launch."""
    w = SMALL["tiny"]
    xh = wl.make_inputs(w, layers=[])
    x = C.to_device(xh)
    q, _, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ix = B.Indexer(x["q_idx"].to(torch.float8_e4m3fn), x["w"], x["k_idx"].to(torch.float8_e4m3fn))
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    with pytest.raises(B.DsaError) as e:
        B.dsa_index_scores(q, ix, scores, ws)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", list(SMALL))
def test_index_scores_bit_exact(dev, name):
    w = SMALL[name]
    xh = wl.make_inputs(w, layers=[])
    x = C.to_device(xh)
    q, ix, _ = C.descriptors(w, x, seq_run=seq_run_of(w))
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    scores.fill_(float("nan"))
    B.dsa_index_scores(q, ix, scores, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    ref, _, _ = C.oracle_selection(w, xh)
    got = scores[:, : w.L].cpu().double().numpy()
    for i, t in enumerate(w.q_pos):
        np.testing.assert_array_equal(got[i, : t + 1], ref[i, : t + 1], err_msg=f"query {i}")


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "fp8"])
@pytest.mark.parametrize("seq_run", [2, 4, 6, 12])
def test_index_scores_query_tiles(dev, seq_run, fp8):
    """Runs of seq_run queries per sequence, so the indexer tiles gcd(seq_run, 8)
    = 2 or 4 queries together (the 8-query tile is covered by the prefill cases):
    three sequences, positions spread over a ragged tail, every visible score
    equal to the oracle's."""
    n_seq, L = 3, 3173
    q_seq = tuple(b for b in range(n_seq) for _ in range(seq_run))
    q_pos = tuple(L - 1 - 37 * j - 101 * b for b in range(n_seq) for j in range(seq_run))
    w = wl.scaled(D32, n_seq=n_seq, L=L, q_pos=q_pos, q_seq=q_seq, seed=40 + seq_run)
    xh = wl.make_inputs(w, layers=[])
    x = C.to_device(xh)
    q, ix, _ = C.descriptors(w, x, seq_run=seq_run)
    if fp8:
        f8h = wl.fp8_indexer_inputs(w, xh)
        ix = C.fp8_indexer(w, C.to_device(f8h), x)
        ref, _, _ = C.oracle_selection_fp8(w, f8h, xh)
    else:
        ref, _, _ = C.oracle_selection(w, xh)
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    scores.fill_(float("nan"))
    B.dsa_index_scores(q, ix, scores, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    got = scores[:, : w.L].cpu().double().numpy()
    for i, t in enumerate(w.q_pos):
        np.testing.assert_array_equal(got[i, : t + 1], ref[i, : t + 1], err_msg=f"query {i}")


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("decode,fused", [(True, True), (False, True), (True, False)])
def test_chain_matches_oracle(dev, name, decode, fused):
    w = SMALL[name]
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    _, idx, cnt, mlas = _run_steps(w, x, decode=decode, fused=fused)
    _, ridx, rcnt = C.oracle_selection(w, xh)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    for layer, m in enumerate(mlas):
        out, lse = C.oracle_mla(w, xh, layer, ridx, rcnt)
        C.assert_attention_close(m.out, out, w.dtype, f"layer {layer} out")
        C.assert_lse_close(m.lse, lse, w.dtype)


@pytest.mark.parametrize("name", ["tiny", "decode_edges", "indexshare_small", "prefill_small", "shared_cache"])
def test_indexshare_group_call(dev, name):
    w = SMALL[name]
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    q, ix, mlas = C.descriptors(w, x, seq_run=seq_run_of(w))
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    idx = torch.empty((w.n_q, w.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.n_q,), dtype=torch.int32, device=dev)
    B.dsa_indexshare_group(q, ix, mlas, w.topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    ridx, rcnt, outs, lses = oracle.indexshare_group(
        C.host_f32(xh["q_idx"]), C.host_f32(xh["w"]), C.host_f32(xh["k_idx"]),
        np.zeros(w.n_q, np.int32) if w.shared_cache else xh["q_seq"].numpy(), xh["q_pos"].numpy(), w.topk,
        [C.host_f32(t) for t in xh["q_mla"]], [C.host_f32(t) for t in xh["kv"]], w.d_lat, w.scale)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    for layer, m in enumerate(mlas):
        C.assert_attention_close(m.out, outs[layer], w.dtype, f"layer {layer}")
        C.assert_lse_close(m.lse, lses[layer], w.dtype)


def _packed(tensors, dev):
    """One device buffer holding the tensors' bytes (256-byte aligned pieces, left
    zero) with a view per tensor, and a pinned host buffer holding their values."""
    offs, tot = [], 0
    for t in tensors:
        offs.append(tot)
        tot += (t.numel() * t.element_size() + 255) // 256 * 256
    d = torch.zeros(tot, dtype=torch.uint8, device=dev)
    h = torch.zeros(tot, dtype=torch.uint8).pin_memory()
    views = []
    for t, o in zip(tensors, offs):
        nb = t.numel() * t.element_size()
        views.append(d[o:o + nb].view(t.dtype).view(t.shape))
        h[o:o + nb].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
    return d, h, views


@pytest.mark.parametrize("name", ["decode_edges", "indexshare_small"])
def test_indexshare_group_host_buffers(dev, name):
    """The group call with its per-step inputs in pinned host memory and its
    outputs copied back to pinned host memory inside the call: the device input
    buffer starts zero, so the results can only come from the copied inputs; the
    host results match the oracle (indices and counts bit for bit)."""
    w = SMALL[name]
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    d_in, h_in, vin = _packed([x["q_idx"], x["w"], x["q_seq"], x["q_pos"]] + list(x["q_mla"]), dev)
    nl = len(x["q_mla"])
    outs = [torch.empty((w.n_q, w.mla_heads, w.d_lat), dtype=w.torch_dtype) for _ in range(nl)]
    outs += [torch.empty((w.n_q, w.topk), dtype=torch.int32), torch.empty((w.n_q,), dtype=torch.int32)]
    d_out, h_out, vout = _packed(outs, dev)
    xv = dict(x, q_idx=vin[0], w=vin[1], q_seq=vin[2], q_pos=vin[3], q_mla=vin[4:])
    q, ix, mlas = C.descriptors(w, xv, seq_run=seq_run_of(w))
    for layer, m in enumerate(mlas):
        m.out = vout[layer]
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, w.n_layers, dev)
    call = B.GroupHostCall(q, ix, mlas, w.topk, vout[nl], vout[nl + 1], ws, h_in, d_in, h_out, d_out)
    for _ in range(2):  # the prepared call, twice on the same buffers
        h_out.fill_(0xFF)
        call()
        torch.cuda.current_stream().synchronize()
    assert B.dsa_check_status(ws) == B.DSA_OK
    # the host copy, read through views of h_out laid out like d_out
    base = d_out.data_ptr()
    hv = [h_out[v.data_ptr() - base:v.data_ptr() - base + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
          for v in vout]
    ridx, rcnt, oouts, lses = oracle.indexshare_group(
        C.host_f32(xh["q_idx"]), C.host_f32(xh["w"]), C.host_f32(xh["k_idx"]),
        np.zeros(w.n_q, np.int32) if w.shared_cache else xh["q_seq"].numpy(), xh["q_pos"].numpy(), w.topk,
        [C.host_f32(t) for t in xh["q_mla"]], [C.host_f32(t) for t in xh["kv"]], w.d_lat, w.scale)
    np.testing.assert_array_equal(hv[nl].numpy(), ridx)
    np.testing.assert_array_equal(hv[nl + 1].numpy(), rcnt)
    for layer in range(nl):
        C.assert_attention_close(hv[layer], oouts[layer], w.dtype, f"layer {layer}")
        C.assert_lse_close(mlas[layer].lse, lses[layer], w.dtype)


@pytest.mark.parametrize("mode", ["ties", "normal", "equal"])
@pytest.mark.parametrize("L,topk", [(300, 64), (5000, 2048), (70000, 2048), (200000, 512), (700001, 2048)])
def test_topk_alone(dev, mode, L, topk):
    n_q = 5
    s = wl.random_scores(n_q, L, seed=L + topk, mode=mode)
    q_pos = torch.tensor([L - 1, L // 2, min(topk, L) - 1, min(topk, L - 1), 0], dtype=torch.int32)
    q = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev), q_pos.to(dev), n_seq=1, max_ctx=L)
    scores = B.scores_buffer(n_q, L, dev)
    scores[:, :L] = s.to(dev)
    ws = B.workspace(B.DSA_OP_TOPK, q, topk, device=dev)
    idx = torch.full((n_q, topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((n_q,), -7, dtype=torch.int32, device=dev)
    B.dsa_topk(q, scores, topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    ridx, rcnt = oracle.topk(s.double().numpy(), q_pos.numpy(), topk)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


@pytest.mark.parametrize("n_bin", [1500, 4000, 5200, 7000])
def test_topk_split_finish_sizes(dev, n_bin):
    """The split schedule's finish over candidate sets of every size class: 2040
    rows far above the rest and n_bin rows inside one first-digit bin ([10, 11)),
    so the finishing CTA stages 2040 + n_bin candidates (fewer than 9 per lane,
    up to 15 per lane, and past that the two-pass refine and write)."""
    n_q, L, topk = 2, 300_000, 2048
    g = torch.Generator().manual_seed(n_bin)
    s = torch.randn((n_q, L), generator=g) * 0.1
    for i in range(n_q):
        pos = torch.randperm(L // 2, generator=g)[:2040 + n_bin]  # all visible for both queries
        s[i, pos[:2040]] = 100.0 + torch.rand(2040, generator=g)
        s[i, pos[2040:]] = 10.0 + torch.rand(n_bin, generator=g)
    q_pos = torch.tensor([L - 1, L // 2], dtype=torch.int32)
    q = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev), q_pos.to(dev), n_seq=1, max_ctx=L)
    scores = B.scores_buffer(n_q, L, dev)
    scores[:, :L] = s.to(dev)
    ws = B.workspace(B.DSA_OP_TOPK, q, topk, device=dev)
    idx = torch.full((n_q, topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((n_q,), -7, dtype=torch.int32, device=dev)
    for _ in range(2):  # the second call runs on the zeroed histograms and tickets the first left
        B.dsa_topk(q, scores, topk, idx, cnt, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK
        ridx, rcnt = oracle.topk(s.double().numpy(), q_pos.numpy(), topk)
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


@pytest.mark.parametrize("L", [5000, 70000], ids=["row", "split"])
@pytest.mark.parametrize("topk", [100, 500, 2048], ids=["bin_of_1", "bin_of_zero", "negative"])
def test_topk_threshold_bin_boundaries(dev, L, topk):
    """Rows at the edges of the threshold's first-digit bin: 60 rows at 3.0, 70 at
    exactly 1.0 (the smallest value of its bin), 300 at the float just below 1.0
    (the previous bin), 400 zeros (half -0.0, half +0.0) and negatives, shuffled.
    topk 100 puts the threshold in the bin of 1.0 (candidates tested as positive
    integers), 500 in the bin of zero (-0.0 and +0.0 tie; lower positions win),
    2048 among the negatives."""
    n_q = 3
    g = torch.Generator().manual_seed(L + topk)
    below_one = float(np.nextafter(np.float32(1.0), np.float32(0.0)))
    s = torch.empty((n_q, L))
    for i in range(n_q):
        vals = torch.cat([torch.full((60,), 3.0), torch.full((70,), 1.0), torch.full((300,), below_one),
                          torch.full((200,), -0.0), torch.zeros(200),
                          -1.0 - 4.0 * torch.rand(L - 830, generator=g)])
        s[i] = vals[torch.randperm(L, generator=g)]
    assert float(s[0][s[0] < 1.0].max()) == below_one
    q_pos = torch.tensor([L - 1, L - 1 - L // 7, L // 2], dtype=torch.int32)
    q = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev), q_pos.to(dev), n_seq=1, max_ctx=L)
    scores = B.scores_buffer(n_q, L, dev)
    scores[:, :L] = s.to(dev)
    ws = B.workspace(B.DSA_OP_TOPK, q, topk, device=dev)
    idx = torch.full((n_q, topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((n_q,), -7, dtype=torch.int32, device=dev)
    ridx, rcnt = oracle.topk(s.double().numpy(), q_pos.numpy(), topk)
    for _ in range(2):
        B.dsa_topk(q, scores, topk, idx, cnt, ws)
        assert B.dsa_check_status(ws) == B.DSA_OK
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


@pytest.mark.parametrize("decode", [True, False])
@pytest.mark.parametrize("topk,L", [(2048, 3000), (300, 1000), (100, 500), (4096, 5000)])
def test_sparse_mla_alone(dev, decode, topk, L):
    w = wl.scaled(D32, n_seq=3, L=L, q_pos=(L - 1, L // 3, 5), q_seq=(2, 0, 1), topk=topk, seed=topk)
    xh = wl.make_inputs(w)
    x = C.to_device(xh)
    q, _, mlas = C.descriptors(w, x)
    idx, cnt = C.random_selection(w, seed=L)
    ws = B.workspace(B.DSA_OP_MLA_DECODE, q, topk, device=dev)
    (B.dsa_sparse_mla_decode if decode else B.dsa_sparse_mla_prefill)(q, mlas[0], idx.to(dev), cnt.to(dev), topk, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
    out, lse = C.oracle_mla(w, xh, 0, idx.numpy(), cnt.numpy())
    C.assert_attention_close(mlas[0].out, out, "bf16")
    C.assert_lse_close(mlas[0].lse, lse, "bf16")


# 4096 key tiles per query: the tensor-core indexer's CTAs claim their work from
# a counter in the workspace instead of taking contiguous ranges
L_CLAIMED = 4096 * 128


def test_claimed_work_repeated_steps_one_workspace(dev):
    """Long-context indexer steps whose CTAs claim work from the workspace
    counter: the last CTA of each launch re-zeroes it, so three fused indexer ->
    top-k steps on one workspace all match the oracle."""
    w = wl.scaled(D32, n_seq=2, L=L_CLAIMED, q_pos=(L_CLAIMED - 1, 300001), q_seq=(0, 1))
    xh = wl.make_inputs(w, layers=[])
    x = C.to_device(xh)
    q, ix, _ = C.descriptors(w, x)
    ix.flags = B.DSA_INDEXER_TOPK_HIST
    ws = B.workspace(B.DSA_OP_INDEXSHARE_GROUP, q, w.topk, 1, dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    _, ridx, rcnt = C.oracle_selection(w, xh)
    for step in range(3):
        idx = torch.full((w.n_q, w.topk), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((w.n_q,), -7, dtype=torch.int32, device=dev)
        B.dsa_index_scores(q, ix, scores, ws)
        B.dsa_topk(q, scores, w.topk, idx, cnt, ws, flags=B.DSA_TOPK_HIST_FROM_INDEXER)
        assert B.dsa_check_status(ws) == B.DSA_OK
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt, err_msg=f"step {step}")
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx, err_msg=f"step {step}")


@pytest.mark.parametrize("L", [1000, L_CLAIMED])
def test_device_detects_bad_positions(dev, L):
    w = wl.scaled(D32, n_seq=2, L=L, q_pos=(L - 1, 500), q_seq=(0, 1))
    x = C.to_device(wl.make_inputs(w, layers=[]))
    x["q_pos"][1] = L + 4000  # beyond the cache
    q, ix, _ = C.descriptors(w, x)
    ws = B.workspace(B.DSA_OP_INDEX_SCORES, q, device=dev)
    scores = B.scores_buffer(w.n_q, w.L, dev)
    B.dsa_index_scores(q, ix, scores, ws)
    assert B.dsa_check_status(ws) == B.DSA_ERR_INVALID
    assert B.dsa_check_status(ws) == B.DSA_OK      # reading clears it


@pytest.mark.parametrize("L", [5000, 70000])
def test_topk_reports_bad_position_of_any_query(dev, L):
    """A position outside the cache, on a query other than the first, is reported by
    the top-k called on its own (one CTA per query for L = 5000, chunk CTAs for L =
    70000); every other query's selection is still the oracle's, and the bad query
    selects nothing."""
    n_q, topk = 4, 2048
    s = wl.random_scores(n_q, L, seed=L, mode="normal")
    q_pos = torch.tensor([L - 1, L // 2, L + 7, L - 3], dtype=torch.int32)
    q = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev), q_pos.to(dev), n_seq=1, max_ctx=L)
    scores = B.scores_buffer(n_q, L, dev)
    scores[:, :L] = s.to(dev)
    ws = B.workspace(B.DSA_OP_TOPK, q, topk, device=dev)
    idx = torch.full((n_q, topk), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((n_q,), -7, dtype=torch.int32, device=dev)
    B.dsa_topk(q, scores, topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_ERR_INVALID
    good = [0, 1, 3]
    ridx, rcnt = oracle.topk(s[good].double().numpy(), q_pos[good].numpy(), topk)
    np.testing.assert_array_equal(cnt.cpu().numpy()[good], rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy()[good], ridx)
    assert int(cnt[2]) == 0 and bool((idx[2] == -1).all())
    # the next call on the same workspace is clean again
    q_ok = B.Queries(torch.zeros(n_q, dtype=torch.int32, device=dev),
                     torch.tensor([L - 1] * n_q, dtype=torch.int32, device=dev), n_seq=1, max_ctx=L)
    B.dsa_topk(q_ok, scores, topk, idx, cnt, ws)
    assert B.dsa_check_status(ws) == B.DSA_OK
