"""The test-side helpers that pick full-size sample rows and assemble oracle
rows one expert at a time: the assembled rows equal the oracle's whole-layer
rows bit for bit, and the sample covers the tile edges it names."""
import numpy as np

import oracle
import parity as PR
from moe_inputs import CONFIGS, make_inputs, make_topk_idx


def test_rows_by_expert_equal_moe_rows():
    cfg = CONFIGS["tiny"]
    g = make_inputs(cfg, seed=3)
    ridx, rw, gap = oracle.route(g["x"], g["w_router"], g["bias"], cfg.k, cfg.scale)
    tokens = [0, 5, 17, 33, 63]
    want = oracle.moe_rows(g["x"], ridx, rw, list(g["w_gate_up"]), list(g["w_down"]),
                           g["ws_gate_up"], g["ws_down"], tokens=np.array(tokens, np.int32))
    got = PR.oracle_rows_by_expert(
        g["x"], ridx, rw, tokens,
        load_expert=lambda e: (PR.u16(g["w_gate_up"][e]), PR.u16(g["w_down"][e])),
        load_shared=lambda: (PR.u16(g["ws_gate_up"]), PR.u16(g["ws_down"])),
        row_fn=lambda xr, w: oracle.swiglu_row(xr, *w), batch=3)
    assert np.array_equal(got, want)


def test_wide_sample_covers_tile_edges():
    T, E, k = 4096, 64, 8
    ridx = make_topk_idx(T, E, k, seed=1, skew=3.0).numpy()
    gap = np.ones(T)
    tokens, parts = PR.wide_sample(ridx, gap, E, T, k, cap=10_000)
    counts, offsets, row_token, _ = oracle.permute(ridx, E)
    b = int(np.argmax(counts))
    # the busiest expert's last row and the batch's last token are compared
    assert int(row_token[offsets[b + 1] - 1]) in tokens
    assert T - 1 in tokens and 0 in tokens
    assert any(name.startswith("shared") for name in parts)
    gap[T - 1] = 0.0                       # a near tie is left out
    tokens2, _ = PR.wide_sample(ridx, gap, E, T, k, cap=10_000)
    assert T - 1 not in tokens2
    small, parts = PR.wide_sample(ridx[:64], np.ones(64), E, 64, k)
    assert small == list(range(64)) and parts == {"all": 64}
