"""The benchmark's algorithmic byte counts (the roofline numerators) against
closed forms for the named workloads: keys once per sequence, selected rows
once per query and layer, queries and outputs once."""
import bench
from dsa_indexer_top_b200 import workloads as wl


def test_decode_32k_bytes():
    w = wl.NAMED["decode_32k"]
    by = bench.path_bytes(w, 1)
    keys = 8 * 32768 * 128 * 2
    q_idx = 8 * 32 * (128 * 2 + 4)
    rows = 8 * 2048 * 576 * 2
    q_out = 8 * 64 * (576 * 2 + 512 * 2 + 4)
    assert by["indexer"] == keys + q_idx + 8 * 32768 * 4
    assert by["mla_per_layer"] == rows + q_out
    assert by["path"] == keys + rows + q_out + q_idx


def test_fp8_variants_bytes():
    w = wl.NAMED["indexshare_128k"]
    base = bench.path_bytes(w, 1)
    f8 = bench.path_bytes(w, 1, indexer_fp8=True, mla_fp8=True)
    n_sel = 32 * 2048
    # packed latent rows: 656 bytes instead of 1152 per selected row, on every layer
    assert base["mla_per_layer"] - f8["mla_per_layer"] == n_sel * (1152 - 656)
    # E4M3 keys with a float32 scale: 132 bytes instead of 256 per key row (layer 0 only)
    keys = 32 * 131072
    q_diff = 32 * 32 * ((128 * 2 + 4) - (128 + 8))
    assert base["path"] - f8["path"] == keys * (256 - 132) + 4 * n_sel * (1152 - 656) + q_diff
