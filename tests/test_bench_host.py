"""Host-side arithmetic of bench.py (CPU only): the attention pair count that
the FLOP and roofline figures rest on, the per-token FLOPs of the headline
workload, the committed traffic line that feeds roofline.traffic, and the
profiling overrides of the workload's shape."""
import numpy as np
import pytest

import bench
import synth
from oracle import model as om


@pytest.mark.parametrize("T,window", [(1, -1), (7, -1), (64, 32), (200, 0), (333, 100), (130, 64), (50, 49), (50, 80)])
def test_attention_pairs_counts_the_oracle_mask(T, window):
    # the oracle's visibility mask is the definition; the closed form must count it
    assert bench.attention_pairs(T, window) == int(om.visible_mask(T, window).sum())


def test_attention_pairs_brute_force():
    for T in (1, 2, 5, 17):
        for W in (-1, 0, 1, 3, 16, 40):
            n = sum(1 for t in range(T) for s in range(T) if s <= t and (W < 0 or t - s <= W))
            assert bench.attention_pairs(T, W) == n


def test_flops_per_token_d24_by_hand():
    c = synth.config("d24")
    f = bench.flops_per_token(c)
    # per layer: qkv 1536x4608 + o 1536x1536 + fc/proj 2 x 1536x6144 = 28,311,552 weights;
    # x 24 layers + lm_head 1536 x 32768 = 729,808,896 matmul parameters
    assert f["matmul_params"] == 729_808_896
    # 6 per parameter + attention 12*hd*H per visible pair: 12*128*12 * (2048*2049/2) / 2048 * 24
    attn = 12 * 128 * 12 * (2048 * 2049 // 2) * 24 / 2048
    assert f["algorithmic"] == pytest.approx(6 * 729_808_896 + attn, rel=1e-12)
    assert f["algorithmic"] == pytest.approx(4.832059392e9, rel=1e-9)


def test_traffic_line_is_read_from_the_committed_summary():
    assert bench.profile_traffic("d24") == pytest.approx(5.065e8)
    assert bench.profile_traffic("no_such_workload") is None


def test_profiling_overrides_reshape_and_rename_the_workload():
    c = bench.workload_config("d24")
    assert (c["name"], c["B"], c["T"], c["n_layer"]) == ("d24", 16, 2048, 24)
    o = bench.workload_config("d24", batch=8, layers=2, seq_len=4096)
    assert (o["B"], o["T"], o["n_layer"]) == (8, 4096, 2)
    assert o["name"].startswith("d24_profiling_") and o["name"] != "d24"
    # the per-layer lists follow the layer count, the model width does not change
    assert len(o["window"]) == 2 and len(o["has_ve"]) == 2 and o["d"] == c["d"]
    # the FLOP count per token grows with T (attention) and shrinks with the layer count
    assert bench.flops_per_token(o)["algorithmic"] != bench.flops_per_token(c)["algorithmic"]
