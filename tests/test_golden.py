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


@pytest.mark.parametrize("weights,per_expert,shared", [
    # routed bytes per expert (gate|up + down) and the shared expert's, per format
    ("bf16", 3 * 7168 * 2048 * 2, 3 * 7168 * 2048 * 2),
    # E4M3 codes + one int8 exponent per 128 x 128 block; shared expert stays bf16
    ("fp8", 3 * 7168 * 2048 + (4096 // 128) * (7168 // 128) + (7168 // 128) * (2048 // 128),
     3 * 7168 * 2048 * 2),
    # INT4: half a byte per weight + one bf16 scale per 32 K elements; shared bf16
    ("w4a16", 3 * 7168 * 2048 // 2 + (4096 * (7168 // 32) + 7168 * (2048 // 32)) * 2,
     3 * 7168 * 2048 * 2),
    # FP8 compute: codes + one int8 exponent per row, shared expert included
    ("w8a8", 3 * 7168 * 2048 + 4096 + 7168, 3 * 7168 * 2048 + 4096 + 7168),
])
def test_weight_bytes_per_format(weights, per_expert, shared):
    import bench
    cfg = CONFIGS["k2_decode"]
    acc0 = bench.layer_accounting(cfg, touched=0, weights=weights)
    acc1 = bench.layer_accounting(cfg, touched=1, weights=weights)
    assert acc1["weight_bytes"] - acc0["weight_bytes"] == per_expert
    router = cfg.E * cfg.d * 2
    assert acc0["weight_bytes"] == shared + router
    # the FLOPs do not depend on the weight format
    assert acc1["flops"] == bench.layer_accounting(cfg, touched=1)["flops"]
