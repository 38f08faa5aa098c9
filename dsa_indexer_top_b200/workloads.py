"""Seeded synthetic inputs for the DSA hot path (shapes, value ranges, seeds).

This module holds no step of the method: it only draws random tensors with the
shapes and distributions of the five named workloads and of smaller parity
cases.  Both the CUDA library's tests/benchmark and the CPU oracle consume the
tensors it returns; neither side computes anything here.

Value recipe (so that every indexer score is exact in float32 and the top-k
indices can be compared bit for bit):
  * indexer queries/keys: integers drawn uniformly from [-a, a] (a = 3 for the
    tiny fp32 case, 4 otherwise), stored as bf16 (or fp32) -- exact;
  * head weights w: powers of two 2^e, e uniform in [e_lo, e_hi] -- exact;
  * MLA queries and latent cache rows [c (512) | r (64)]: N(0, 1), rounded to
    bf16 (round-to-nearest-even by torch) or kept fp32 for the tiny case.
With |q.k| <= 128 * 16 and at most 32 heads, each score is a multiple of 2^-3
below 2^17, which float32 holds exactly whatever the summation order.

FP8 latent cache (fp8_latent_inputs): the layer's own bf16 latents (N(0, 1))
stored the way a cache writer would store them in 8 bits -- per row a float32
scale amax(|c|) / 448 and the E4M3 codes of c / scale -- next to the layer's
bf16 RoPE key, packed as one byte row.  (Writing the cache is upstream of the
attention path; the path only reads it.)

FP8 indexer variant (fp8_indexer_inputs): the same integer queries and keys
stored as E4M3 bytes (integers up to 16 are exact in E4M3), with per-(query,
head) scales 2^e, e in [-1, 1], and per-key scales 2^e, e in [-2, 0]: every
score is then a multiple of 2^-6 below 2^19 -- still exact in float32.

Random numbers come from torch.Generator objects seeded per tensor (seed, tensor
id), on the device the tensors are created on.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

import torch

# tensor ids used to derive independent streams from one workload seed
_T_QIDX, _T_W, _T_KIDX, _T_QMLA, _T_KV, _T_QSCALE, _T_KSCALE = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    n_seq: int                 # caches (sequences)
    L: int                     # rows per cache
    q_pos: tuple               # position of every query (len = n_q)
    q_seq: tuple               # sequence of every query
    idx_heads: int = 32
    idx_dim: int = 128
    topk: int = 2048
    mla_heads: int = 64
    d_lat: int = 512
    d_rope: int = 64
    scale: float = 1.0 / 16.0  # 1/sqrt(192 + 64)
    dtype: str = "bf16"        # storage dtype of q/k/cache ("bf16" or "f32")
    n_layers: int = 1          # IndexShare group size (layer 0 full)
    int_range: int = 4         # indexer ints in [-int_range, int_range]
    w_exp: tuple = (-3, 1)     # w = 2^e, e in [w_exp[0], w_exp[1]]
    seed: int = 0
    shared_cache: bool = False  # all sequences alias one cache (seq stride 0)
    note: str = ""

    @property
    def n_q(self) -> int:
        return len(self.q_pos)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def describe(self) -> dict:
        return {
            "workload": self.name, "n_seq": self.n_seq, "ctx": self.L, "n_q": self.n_q,
            "layers": self.n_layers, "topk": self.topk,
            "indexer": f"{self.idx_heads}x{self.idx_dim}",
            "mla": f"{self.mla_heads}x({self.d_lat}+{self.d_rope})", "dtype": self.dtype,
        }


def _decode(name, n_seq, L, seed, **kw):
    return Workload(name=name, n_seq=n_seq, L=L, q_pos=tuple([L - 1] * n_seq),
                    q_seq=tuple(range(n_seq)), seed=seed, **kw)


# The five named workloads, in their published order.
NAMED = {
    "tiny": Workload(
        name="tiny", n_seq=1, L=256, q_pos=tuple(range(240, 256)), q_seq=tuple([0] * 16),
        idx_heads=4, idx_dim=32, topk=64, mla_heads=4, d_lat=64, d_rope=16,
        scale=1.0 / math.sqrt(48.0), dtype="f32", int_range=3, w_exp=(-2, 1), seed=0,
        note="tiny single layer, fp32"),
    "decode_32k": _decode("decode_32k", 8, 32768, 1,
                          note="decode, one full layer: 8 queries each at context 32768"),
    "prefill_64k": Workload(
        name="prefill_64k", n_seq=1, L=65536, q_pos=tuple(range(61440, 65536)),
        q_seq=tuple([0] * 4096), seed=2,
        note="prefill chunk: 4096 queries at 61440..65535 over a 65536-row cache"),
    "indexshare_128k": _decode("indexshare_128k", 32, 131072, 3, n_layers=4,
                               note="IndexShare group decode: 1 full + 3 shared layers, "
                                    "32 queries at context 131072"),
    "decode_1m": _decode("decode_1m", 4, 1048576, 4,
                         note="long-context decode: 4 queries at context 1048576"),
}
NAMED_ORDER = ["tiny", "decode_32k", "prefill_64k", "indexshare_128k", "decode_1m"]


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tensor_id * 7_919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _ints(shape, a, gen, device, dtype):
    return torch.randint(-a, a + 1, shape, generator=gen, device=device, dtype=torch.int32).to(dtype)


def make_inputs(w: Workload, device="cpu", layers=None) -> dict:
    """Draw every input tensor of a workload.

    Returns a dict with
      q_seq, q_pos  int32 [n_q]
      q_idx  [n_q, idx_heads, idx_dim]  (bf16/fp32)
      w      [n_q, idx_heads]           fp32
      k_idx  [n_seq, L, idx_dim]        (only layer 0 has indexer keys)
      q_mla  list per layer of [n_q, mla_heads, d_lat + d_rope]
      kv     list per layer of [n_seq, L, d_lat + d_rope]  rows [c | r]
    With shared_cache the caches have one sequence ([1, L, ...]).
    `layers` limits which MLA layers are drawn (default: all).
    """
    device = torch.device(device)
    dt = w.torch_dtype
    n_cache = 1 if w.shared_cache else w.n_seq
    out = {
        "q_seq": torch.tensor(w.q_seq, dtype=torch.int32, device=device),
        "q_pos": torch.tensor(w.q_pos, dtype=torch.int32, device=device),
    }
    out["q_idx"] = _ints((w.n_q, w.idx_heads, w.idx_dim), w.int_range,
                         _gen(w.seed, _T_QIDX, device), device, dt)
    e = torch.randint(w.w_exp[0], w.w_exp[1] + 1, (w.n_q, w.idx_heads),
                      generator=_gen(w.seed, _T_W, device), device=device, dtype=torch.int32)
    out["w"] = torch.pow(2.0, e.to(torch.float32))
    # indexer keys: drawn one sequence at a time to bound temporary memory
    k = torch.empty((n_cache, w.L, w.idx_dim), dtype=dt, device=device)
    gk = _gen(w.seed, _T_KIDX, device)
    for b in range(n_cache):
        k[b] = _ints((w.L, w.idx_dim), w.int_range, gk, device, dt)
    out["k_idx"] = k
    dk = w.d_lat + w.d_rope
    layer_ids = range(w.n_layers) if layers is None else layers
    q_mla, kv = [], []
    for layer in layer_ids:
        gq = _gen(w.seed, _T_QMLA + 16 * layer, device)
        q_mla.append(torch.randn((w.n_q, w.mla_heads, dk), generator=gq, device=device,
                                 dtype=torch.float32).to(dt))
        gc = _gen(w.seed, _T_KV + 16 * layer, device)
        c = torch.empty((n_cache, w.L, dk), dtype=dt, device=device)
        for b in range(n_cache):
            c[b] = torch.randn((w.L, dk), generator=gc, device=device, dtype=torch.float32).to(dt)
        kv.append(c)
    out["q_mla"] = q_mla
    out["kv"] = kv
    return out


def random_scores(n_q, L, seed, device="cpu", mode="ties"):
    """Seeded float32 score matrices for testing top-k on its own.

    mode "ties": small integers (heavy ties); "normal": N(0,1) values with a few
    exact duplicates and signed zeros planted; "equal": every score the same.
    """
    g = _gen(seed, 99, device)
    if mode == "ties":
        return torch.randint(0, 7, (n_q, L), generator=g, device=device, dtype=torch.int32).float()
    if mode == "equal":
        return torch.full((n_q, L), 1.5, device=device)
    s = torch.randn((n_q, L), generator=g, device=device, dtype=torch.float32)
    if L >= 8:
        s[:, 1::7] = s[:, 0:1]          # duplicates of the first score
        s[:, 3::11] = 0.0
        s[:, 5::13] = -0.0
    return s


def fp8_indexer_inputs(w: Workload, x: dict, device="cpu") -> dict:
    """FP8 (E4M3) versions of a workload's indexer inputs: the same integer
    values as x["q_idx"] / x["k_idx"] stored as float8_e4m3fn, plus seeded
    power-of-two scales q_scale [n_q][heads] and k_scale [n_cache][L]."""
    n_cache = x["k_idx"].shape[0]
    gq = _gen(w.seed, _T_QSCALE, device)
    gk = _gen(w.seed, _T_KSCALE, device)
    eq = torch.randint(-1, 2, (w.n_q, w.idx_heads), generator=gq, device=device, dtype=torch.int32)
    ek = torch.randint(-2, 1, (n_cache, w.L), generator=gk, device=device, dtype=torch.int32)
    return {
        "q8": x["q_idx"].to(device).float().to(torch.float8_e4m3fn),
        "k8": x["k_idx"].to(device).float().to(torch.float8_e4m3fn),
        "q_scale": torch.pow(2.0, eq.to(torch.float32)),
        "k_scale": torch.pow(2.0, ek.to(torch.float32)),
    }


def fp8_row_bytes(d_lat: int, d_rope: int) -> int:
    """Bytes of one packed FP8 latent-cache row: d_lat E4M3 codes, d_rope bf16
    RoPE values, one float32 scale, padded to a multiple of 16 (656 for 512 + 64)."""
    return (d_lat + 2 * d_rope + 4 + 15) // 16 * 16


def fp8_latent_inputs(w: Workload, x: dict, device="cpu", layers=None) -> list:
    """Packed FP8 latent caches, one uint8 tensor [n_cache][L][row_bytes] per MLA
    layer of x (rows: codes | RoPE key | scale | zero padding), holding the
    layer's bf16 cache x["kv"][layer] in 8 bits: scale = amax(|c|) / 448 per row
    (448 is E4M3's largest finite value), codes = E4M3(c / scale) rounded by
    torch; the RoPE key is copied as bf16.  One sequence at a time."""
    device = torch.device(device)
    rb = fp8_row_bytes(w.d_lat, w.d_rope)
    layer_ids = range(len(x["kv"])) if layers is None else layers
    out = []
    for layer in layer_ids:
        kv = x["kv"][layer]
        n_cache = kv.shape[0]
        rows = torch.zeros((n_cache, w.L, rb), dtype=torch.uint8, device=device)
        for b in range(n_cache):
            c = kv[b, :, : w.d_lat].to(device=device, dtype=torch.float32)
            sigma = c.abs().amax(-1, keepdim=True).clamp_min(2.0 ** -60) / 448.0
            code = (c / sigma).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
            rope = kv[b, :, w.d_lat:].to(device=device, dtype=torch.bfloat16).contiguous()
            rows[b, :, : w.d_lat] = code.view(torch.uint8)
            rows[b, :, w.d_lat: w.d_lat + 2 * w.d_rope] = rope.view(torch.uint8)
            rows[b, :, w.d_lat + 2 * w.d_rope: w.d_lat + 2 * w.d_rope + 4] = sigma.view(torch.uint8)
        out.append(rows)
    return out
