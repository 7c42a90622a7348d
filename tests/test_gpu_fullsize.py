"""Full-size layer shapes (K2 decode / prefill / skewed, DeepSeek-V3-shaped):
the CUDA path in the launch configuration the benchmark times, against the
oracle on every token's routing, on the full permutation, and on sampled
output rows (rows are independent, so a sample is exact)."""
import numpy as np
import pytest
import torch

import oracle
import parity as PR
from moe_inputs import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu

FULL = ["k2_decode", "k2_prefill", "k2_skew", "v3"]


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


@pytest.mark.parametrize("name", FULL)
def test_fullsize_layer(moe, name):
    cfg = CONFIGS[name]
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    g = make_inputs(cfg, seed=0, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(g["x"], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], k, cfg.scale, out)
    ws = torch.empty(moe.moe_workspace_size(T, d, E, k, I), dtype=torch.uint8, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(g["x"], g["w_router"], g["bias"], k, cfg.scale, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0

    # routing of every token
    x_h, wr_h, bias_h = g["x"].cpu(), g["w_router"].cpu(), g["bias"].cpu()
    ridx, rw, gap, scores = oracle.route(x_h, wr_h, bias_h, k, cfg.scale, want_scores=True)
    flagged = PR.check_routing(idx.cpu().numpy(), w.cpu().numpy(), ridx, scores, bias_h.numpy(),
                               cfg.scale)
    assert len(flagged) <= max(2, T // 1000), flagged

    # permutation of the oracle's routing, bit-exact
    counts, offsets, row_token, slot_row = oracle.permute(ridx, E)
    i32 = lambda n: torch.empty((n,), dtype=torch.int32, device="cuda")
    dc, do, dr, ds = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    moe.moe_permute(torch.from_numpy(ridx).cuda(), E, dc, do, dr, ds, ws)
    torch.cuda.synchronize()
    assert np.array_equal(dc.cpu().numpy(), counts)
    assert np.array_equal(do.cpu().numpy(), offsets)
    assert np.array_equal(dr.cpu().numpy(), row_token)
    assert np.array_equal(ds.cpu().numpy(), slot_row)

    # output rows at the tiles' edges: the busiest expert's last two token
    # tiles, the shared expert's last tile, a ragged multi-tile expert's last
    # tile, element by element against the oracle (one batch of experts on the
    # host at a time)
    sample, parts = PR.wide_sample(ridx, gap, E, T, k)
    print(f"{name}: {len(sample)} rows compared: {parts}")
    assert len(sample) >= min(T, 128) - 8, parts
    ref = PR.oracle_rows_by_expert(
        x_h, ridx, rw, sample,
        load_expert=lambda e: (PR.u16(g["w_gate_up"][e]), PR.u16(g["w_down"][e])),
        load_shared=lambda: (PR.u16(g["ws_gate_up"]), PR.u16(g["ws_down"])),
        row_fn=lambda xr, wts: oracle.swiglu_row(xr, *wts))
    got = PR.bf16_np(out[torch.tensor(sample, device="cuda")])
    PR.check_output(got, ref)
    del g, out, ws
    torch.cuda.empty_cache()
