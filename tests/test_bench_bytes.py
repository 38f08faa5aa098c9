"""The benchmark's algorithmic byte and FLOP counts (the roofline numerators)
against closed forms for the named workloads: keys once per sequence, selected
rows once per query and layer, queries and outputs once."""
import bench
from dsa_indexer_top_b200 import workloads as wl


def test_decode_32k_bytes():
    w = wl.NAMED["decode_32k"]
    by = bench.path_bytes(w)
    keys = 8 * 32768 * 128 * 2
    q_idx = 8 * 32 * (128 * 2 + 4)
    rows = 8 * 2048 * 576 * 2
    q_out = 8 * 64 * (576 * 2 + 512 * 2 + 4)
    assert by["indexer"] == keys + q_idx + 8 * 32768 * 4
    assert by["mla"] == rows + q_out
    assert by["path"] == keys + rows + q_out + q_idx


def test_indexshare_bytes_count_every_layer():
    w = wl.NAMED["indexshare_128k"]
    by = bench.path_bytes(w)
    rows = 32 * 2048 * 1152
    q_out = 32 * 64 * (1152 + 1024 + 4)
    assert by["mla"] == 4 * (rows + q_out)
    assert by["path"] == 32 * 131072 * 256 + 4 * (rows + q_out) + 32 * 32 * (256 + 4)


def test_fp8_variants_bytes():
    w = wl.NAMED["indexshare_128k"]
    base = bench.path_bytes(w)
    f8 = bench.path_bytes(w, indexer_fp8=True, mla_fp8=True)
    n_sel = 32 * 2048
    # packed latent rows: 656 bytes instead of 1152 per selected row, on every layer
    assert base["mla"] - f8["mla"] == 4 * n_sel * (1152 - 656)
    # E4M3 keys with a float32 scale: 132 bytes instead of 256 per key row (layer 0 only)
    keys = 32 * 131072
    q_diff = 32 * 32 * ((128 * 2 + 4) - (128 + 8))
    assert base["path"] - f8["path"] == keys * (256 - 132) + 4 * n_sel * (1152 - 656) + q_diff


def test_prefill_flops():
    w = wl.NAMED["prefill_64k"]
    fl = bench.path_flops(w)
    vis = sum(t + 1 for t in range(61440, 65536))
    assert fl["indexer"] == 2 * 32 * 128 * vis
    # every prefill query sees more than 2048 rows: 2048 selected rows, S over 576 dims, O over 512
    assert fl["mla"] == 2 * 64 * (576 + 512) * 2048 * 4096
