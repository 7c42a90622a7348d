"""The workloads and the benchmark's accounting against the constants the
pages print for one K2 MoE layer (tests/golden/k2_moe_layer.txt, each line
cited).  A printed "~" value is compared within its rounding (1% for the
"~44M" / "~16.9B" counts, 0.1% for "~793M")."""
import os

import pytest

from moe_inputs import CONFIGS

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    vals = {}
    with open(os.path.join(HERE, "golden", "k2_moe_layer.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            key, val = line.split()[:2]
            vals[key] = (float(val.lstrip("~")), val.startswith("~"))
    return vals


G = _golden()


@pytest.mark.parametrize("name", ["k2_decode", "k2_prefill", "k2_skew"])
def test_k2_workloads_use_the_printed_shape(name):
    cfg = CONFIGS[name]
    assert (cfg.d, cfg.inter, cfg.E, cfg.k) == (G["d"][0], G["inter"][0], G["E"][0], G["k"][0])
    assert cfg.scale == G["scale"][0]


def test_expert_parameter_counts():
    cfg = CONFIGS["k2_decode"]
    per_expert = 3 * cfg.d * cfg.inter
    assert abs(per_expert - G["expert_params"][0]) <= 0.01 * G["expert_params"][0]
    assert abs(cfg.E * per_expert - G["layer_expert_params"][0]) <= \
        0.01 * G["layer_expert_params"][0]


def test_layer_flops_per_token_equal_the_printed_dense_ffn():
    """A token passes k routed experts and the shared one: (k + 1) x 2048 = 18432
    intermediate columns, the dense layer 0's width, so its FLOPs are the
    printed ~793M; the benchmark's accounting must give the same per token."""
    import bench
    cfg = CONFIGS["k2_prefill"]
    assert (cfg.k + int(G["shared"][0])) * cfg.inter == G["dense_ffn_inter"][0]
    acc = bench.layer_accounting(cfg, touched=cfg.E)
    per_token = (acc["gate_up_flops"] + acc["down_flops"]) / cfg.T
    assert per_token == 2 * 3 * cfg.d * G["dense_ffn_inter"][0]
    assert abs(per_token - G["dense_ffn_flops"][0]) <= 0.001 * G["dense_ffn_flops"][0]
    # weight bytes of one touched expert: 3 x d x inter bf16 values
    acc1 = bench.layer_accounting(cfg, touched=1)
    acc0 = bench.layer_accounting(cfg, touched=0)
    assert acc1["weight_bytes"] - acc0["weight_bytes"] == 3 * cfg.d * cfg.inter * 2
