"""CUDA path vs the fp64 oracle, stage by stage and end to end (B200 only).

Every call goes through the C ABI (the ctypes binding).  Inputs come from the
seeded generators in moe_inputs; expected values come only from the oracle.
Sizes span several tiles and ragged tails; the full-size layer shapes are
checked on sampled tokens (rows are independent) in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as PR
from moe_inputs import MoEConfig, make_combine_inputs, make_inputs, make_topk_idx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()          # start from a clean status word
    return m


def _ws(m, T, d, E, k, inter):
    return torch.empty(m.moe_workspace_size(T, d, E, k, inter), dtype=torch.uint8, device="cuda")


def _cuda(inp):
    return {k: v.cuda() for k, v in inp.items()}


def _status_ok(m):
    assert m.moe_device_status() == 0


# ------------------------------------------------------------------ routing

ROUTE_CASES = [
    MoEConfig("tiny", T=64, d=512, E=32, k=4, inter=128, scale=2.827),
    MoEConfig("ragged", T=37, d=256, E=48, k=6, inter=64, scale=2.827),
    MoEConfig("k1", T=50, d=192, E=7, k=1, inter=64, scale=2.5),
    MoEConfig("e_eq_k", T=20, d=64, E=5, k=5, inter=64, scale=2.827),
    MoEConfig("zipf", T=300, d=256, E=64, k=8, inter=64, scale=2.827, bias="zipf"),
    MoEConfig("max_e_k", T=70, d=128, E=1024, k=32, inter=64, scale=2.827),
    MoEConfig("many_tiles", T=700, d=640, E=200, k=8, inter=64, scale=2.827),
]


@pytest.mark.parametrize("cfg", ROUTE_CASES, ids=lambda c: c.name)
def test_route_parity(moe, cfg):
    inp = make_inputs(cfg, seed=1)
    g = _cuda(inp)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_route(g["x"], g["w_router"], g["bias"], cfg.k, cfg.scale, idx, w,
                  _ws(moe, cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter))
    torch.cuda.synchronize()
    _status_ok(moe)
    ridx, rw, gap, scores = oracle.route(inp["x"], inp["w_router"], inp["bias"], cfg.k, cfg.scale,
                                         want_scores=True)
    flagged = PR.check_routing(idx.cpu().numpy(), w.cpu().numpy(), ridx, scores,
                               inp["bias"].numpy(), cfg.scale)
    assert len(flagged) <= max(1, cfg.T // 100)


def test_bias_changes_selection_not_weights(moe):
    cfg = MoEConfig("bias", T=256, d=256, E=32, k=4, inter=64, scale=2.827)
    inp = make_inputs(cfg, seed=2)
    g = _cuda(inp)
    ws = _ws(moe, cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter)
    out = []
    for b in (torch.zeros_like(g["bias"]), g["bias"] * 5):
        idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
        w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
        moe.moe_route(g["x"], g["w_router"], b, cfg.k, cfg.scale, idx, w, ws)
        out.append((idx.cpu().numpy(), w.cpu().numpy()))
    _status_ok(moe)
    changed = 0
    for t in range(cfg.T):
        m0 = dict(zip(out[0][0][t].tolist(), out[0][1][t].tolist()))
        m1 = dict(zip(out[1][0][t].tolist(), out[1][1][t].tolist()))
        if set(m0) == set(m1):
            assert m0 == m1, f"token {t}: weights moved with the bias"
        else:
            changed += 1
    assert changed > 0


# -------------------------------------------------------------- permutation

PERMUTE_CASES = [(1, 8, 2, 0.0), (37, 32, 4, 0.0), (64, 384, 8, 0.0), (300, 384, 8, 3.0),
                 (1000, 16, 8, 0.0), (4096, 384, 8, 2.0), (8192, 384, 8, 0.0), (100, 1024, 32, 0.0),
                 (129, 5, 5, 0.0), (257, 1, 1, 0.0)]


@pytest.mark.parametrize("T,E,k,skew", PERMUTE_CASES)
def test_permute_bit_exact(moe, T, E, k, skew):
    idx = make_topk_idx(T, E, k, seed=T + E, skew=skew)
    counts, offsets, row_token, slot_row = oracle.permute(idx.numpy(), E)
    dev = dict(counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
               row_token=torch.full((T * k,), -7, dtype=torch.int32, device="cuda"),
               slot_row=torch.full((T * k,), -7, dtype=torch.int32, device="cuda"))
    moe.moe_permute(idx.cuda(), E, dev["counts"], dev["offsets"], dev["row_token"],
                    dev["slot_row"], _ws(moe, T, 64, E, k, 64))
    torch.cuda.synchronize()
    _status_ok(moe)
    assert np.array_equal(dev["counts"].cpu().numpy(), counts)
    assert np.array_equal(dev["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(dev["row_token"].cpu().numpy(), row_token)
    assert np.array_equal(dev["slot_row"].cpu().numpy(), slot_row)


def test_permute_flags_bad_index(moe):
    idx = make_topk_idx(40, 16, 4, seed=3)
    idx[5, 2] = 99
    z = lambda n: torch.zeros((n,), dtype=torch.int32, device="cuda")
    moe.moe_permute(idx.cuda(), 16, z(16), z(17), z(160), z(160), _ws(moe, 40, 64, 16, 4, 64))
    assert moe.moe_device_status() == -1
    _status_ok(moe)


# ------------------------------------------------------------------ combine

@pytest.mark.parametrize("T,d,k,shared", [(1, 64, 1, True), (37, 512, 4, True),
                                          (64, 7168, 8, True), (300, 1024, 8, False),
                                          (1000, 256, 32, True)])
def test_combine(moe, T, d, k, shared):
    c = make_combine_inputs(T, d, k, seed=T * k)
    ys = c["y_shared"] if shared else None
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(c["y"].cuda(), None if ys is None else ys.cuda(), c["topk_w"].cuda(),
                    c["slot_row"].cuda(), out)
    torch.cuda.synchronize()
    _status_ok(moe)
    y64 = oracle.bf16_to_f64(c["y"])
    ys64 = None if ys is None else oracle.bf16_to_f64(ys)
    w = c["topk_w"].numpy().astype(np.float64)
    sr = c["slot_row"].numpy()
    ref = oracle.combine(y64, ys64, w, sr.reshape(-1))
    got = PR.bf16_np(out)
    mag = np.abs(w)[:, :, None] * np.abs(y64[sr.reshape(T, k)])
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6 * (mag.sum(1) + (0 if ys64 is None else np.abs(ys64)))
    assert (np.abs(got - ref) <= bound + 1e-30).all()
    PR.check_output(got, ref)


# --------------------------------------------------------------- expert FFN

FFN_CASES = [
    MoEConfig("tiny", T=64, d=512, E=32, k=4, inter=128, scale=2.827),
    MoEConfig("ragged", T=37, d=320, E=7, k=3, inter=192, scale=2.827),
    MoEConfig("multi_token_tiles", T=600, d=256, E=1, k=1, inter=128, scale=1.0),
    MoEConfig("skewed", T=300, d=256, E=16, k=4, inter=256, scale=2.827),
    MoEConfig("k2_dims", T=16, d=7168, E=3, k=2, inter=2048, scale=2.827),
]


@pytest.mark.parametrize("cfg", FFN_CASES, ids=lambda c: c.name)
def test_expert_ffn_parity(moe, cfg):
    inp = make_inputs(cfg, seed=4)
    idx = make_topk_idx(cfg.T, cfg.E, cfg.k, seed=5, skew=3.0 if cfg.name == "skewed" else 0.0)
    counts, offsets, row_token, slot_row = oracle.permute(idx.numpy(), cfg.E)
    g = _cuda(inp)
    y = torch.empty((cfg.T * cfg.k, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(g["x"], torch.from_numpy(row_token).cuda(),
                       torch.from_numpy(offsets).cuda(), g["w_gate_up"], g["w_down"], cfg.k, y,
                       _ws(moe, cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter))
    torch.cuda.synchronize()
    _status_ok(moe)
    expert_of_row = np.repeat(np.arange(cfg.E), counts)
    ref = np.empty((cfg.T * cfg.k, cfg.d))
    for r in range(cfg.T * cfg.k):
        e = expert_of_row[r]
        ref[r] = oracle.swiglu_row(inp["x"][row_token[r]], inp["w_gate_up"][e], inp["w_down"][e])
    PR.check_output(PR.bf16_np(y), ref)


def test_expert_ffn_bad_row_token(moe):
    """Out-of-range token indices are reported and skipped; other rows are exact."""
    cfg = MoEConfig("bad_rows", T=40, d=256, E=4, k=2, inter=128, scale=1.0)
    inp = make_inputs(cfg, seed=21)
    idx = make_topk_idx(cfg.T, cfg.E, cfg.k, seed=22)
    counts, offsets, row_token, _ = oracle.permute(idx.numpy(), cfg.E)
    bad = row_token.copy()
    bad_rows = [3, 41, 70]
    bad[3], bad[41], bad[70] = cfg.T, -1, 1 << 30
    g = _cuda(inp)
    y = torch.empty((cfg.T * cfg.k, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(g["x"], torch.from_numpy(bad).cuda(), torch.from_numpy(offsets).cuda(),
                       g["w_gate_up"], g["w_down"], cfg.k, y,
                       _ws(moe, cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter))
    assert moe.moe_device_status() == -1          # MOE_ERR_INVALID_ARG
    expert_of_row = np.repeat(np.arange(cfg.E), counts)
    keep = [r for r in range(cfg.T * cfg.k) if r not in bad_rows]
    ref = np.stack([oracle.swiglu_row(inp["x"][row_token[r]], inp["w_gate_up"][expert_of_row[r]],
                                      inp["w_down"][expert_of_row[r]]) for r in keep])
    PR.check_output(PR.bf16_np(y)[keep], ref)


# -------------------------------------------------------------------- layer

LAYER_CASES = [
    MoEConfig("tiny", T=64, d=512, E=32, k=4, inter=128, scale=2.827),
    MoEConfig("one_token", T=1, d=512, E=32, k=4, inter=128, scale=2.827),
    MoEConfig("ragged", T=37, d=320, E=7, k=3, inter=192, scale=2.827),
    MoEConfig("e_eq_k", T=16, d=128, E=4, k=4, inter=64, scale=2.827),
    MoEConfig("k1", T=45, d=192, E=6, k=1, inter=128, scale=2.5),
    MoEConfig("zipf_multi_tile", T=600, d=256, E=16, k=4, inter=128, scale=2.827, bias="zipf"),
    MoEConfig("max_e_k", T=64, d=128, E=1024, k=32, inter=64, scale=2.827),
    # T >= 1024: the token rows are permuted token by token; rows of 16 and 48
    # 16-byte vectors leave part of the warp without a vector in the last round
    MoEConfig("token_major_d128", T=1100, d=128, E=64, k=8, inter=64, scale=2.827),
    MoEConfig("token_major_d384_k32", T=1030, d=384, E=48, k=32, inter=64, scale=2.827),
]


@pytest.mark.parametrize("cfg", LAYER_CASES, ids=lambda c: c.name)
def test_layer_parity(moe, cfg):
    inp = make_inputs(cfg, seed=6)
    g = _cuda(inp)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(g["x"], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)
    torch.cuda.synchronize()
    _status_ok(moe)
    ref, ridx, rw, gap = oracle.moe_forward(inp, cfg.k, cfg.scale)
    # near-tie tokens (oracle gap < TIE_EPS) may legitimately route differently
    skip = np.nonzero(gap < PR.TIE_EPS)[0]
    PR.check_output(PR.bf16_np(out), ref, skip_rows=skip)


def test_layer_deterministic_and_ws_variant(moe):
    cfg = MoEConfig("det", T=200, d=256, E=24, k=6, inter=128, scale=2.827)
    g = _cuda(make_inputs(cfg, seed=7))
    args = (g["x"], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"], g["ws_gate_up"],
            g["ws_down"], cfg.k, cfg.scale)
    o1 = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    o3 = torch.empty_like(o1)
    moe.moe_layer_forward(*args, o1)
    moe.moe_layer_forward(*args, o2)
    moe.moe_layer_forward_ws(*args, o3, _ws(moe, cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter))
    torch.cuda.synchronize()
    _status_ok(moe)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))
    kernels = [moe.moe_kernel_name(i) for i in range(32) if moe.moe_kernel_name(i)]
    # every slot but the activation quantizer of FP8 compute
    assert moe.moe_last_launch_count() == len([n for n in kernels if n != "quantize_h"])


def test_staged_calls_compose_to_layer(moe):
    """route -> permute -> expert_ffn (routed, then shared as E=1) -> combine."""
    cfg = MoEConfig("staged", T=96, d=256, E=16, k=4, inter=128, scale=2.827)
    g = _cuda(make_inputs(cfg, seed=8))
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    ws = _ws(moe, T, d, E, k, cfg.inter)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(g["x"], g["w_router"], g["bias"], k, cfg.scale, idx, w, ws)
    i32 = lambda n: torch.empty((n,), dtype=torch.int32, device="cuda")
    counts, offsets, row_token, slot_row = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    moe.moe_permute(idx, E, counts, offsets, row_token, slot_row, ws)
    y = torch.empty((T * k, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(g["x"], row_token, offsets, g["w_gate_up"], g["w_down"], k, y, ws)
    ysh = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    ident = torch.arange(T, dtype=torch.int32, device="cuda")
    off1 = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    moe.moe_expert_ffn(g["x"], ident, off1, g["ws_gate_up"][None], g["ws_down"][None], 1, ysh, ws)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(y, ysh, w, slot_row, out)
    fused = torch.empty_like(out)
    moe.moe_layer_forward(g["x"], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], k, cfg.scale, fused)
    torch.cuda.synchronize()
    _status_ok(moe)
    assert torch.equal(out.view(torch.int16), fused.view(torch.int16))


def test_zero_tokens_leaves_output_untouched(moe):
    cfg = MoEConfig("z", T=0, d=128, E=8, k=2, inter=64, scale=2.827)
    g = _cuda(make_inputs(MoEConfig("z1", T=1, d=128, E=8, k=2, inter=64, scale=2.827), seed=9))
    out = torch.full((1, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(g["x"][:0], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out[:0])
    torch.cuda.synchronize()
    assert (out == 3.0).all()
    _status_ok(moe)


def test_wait_timeout_is_reported_and_context_survives(moe):
    moe.moe_selftest_wait_timeout(2_000_000)           # 2 ms, nobody arrives
    assert moe.moe_device_status() == -4               # MOE_ERR_TIMEOUT
    _status_ok(moe)                                    # read clears it
    cfg = MoEConfig("after", T=32, d=128, E=8, k=2, inter=64, scale=2.827)
    inp = make_inputs(cfg, seed=10)
    g = _cuda(inp)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(g["x"], g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)
    torch.cuda.synchronize()
    _status_ok(moe)
    ref, _, _, gap = oracle.moe_forward(inp, cfg.k, cfg.scale)
    PR.check_output(PR.bf16_np(out), ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])
