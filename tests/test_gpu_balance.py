"""Load balancing on the GPU against the oracle ("Kimi K2.5 Q&A", Q7.2; "Kimi
K2.5 deep dive", CH10.2 step 2): the loss-free bias update (bit-exact: integer
load comparison, one fp32 add), the router scores it starts from, and the
sequence-level balance loss (fp32 against fp64)."""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import CONFIGS, MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


@pytest.mark.parametrize("T,E,k", [(64, 384, 8), (37, 7, 3), (1, 4, 4), (1000, 1024, 32),
                                   (7, 3, 1)])
def test_bias_update_bit_exact(moe, T, E, k):
    rng = np.random.default_rng(T + E + k)
    # loads of a real routing (every token picks k distinct experts), plus loads
    # equal to the mean where possible
    counts = np.zeros(E, np.int32)
    for _ in range(T):
        counts[rng.choice(E, k, replace=False)] += 1
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    gamma = np.float32(1e-3)
    ref = oracle.bias_update(counts, T, k, float(gamma), bias)
    dc, db = torch.from_numpy(counts).cuda(), torch.from_numpy(bias).cuda()
    moe.moe_bias_update(dc, T, k, float(gamma), db)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert np.array_equal(db.cpu().numpy(), ref)


def test_bias_update_from_the_layers_loads(moe):
    """route -> permute -> bias update, all on the GPU, against the oracle chain."""
    cfg = CONFIGS["k2_decode"].__class__(**{**CONFIGS["k2_decode"].as_dict(), "d": 512,
                                            "inter": 128})
    inp = make_inputs(cfg, seed=50)
    g = {k: v.cuda() for k, v in inp.items()}
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    ws = torch.empty(moe.moe_workspace_size(T, d, E, k, cfg.inter), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(g["x"], g["w_router"], g["bias"], k, cfg.scale, idx, w, ws)
    i32 = lambda n: torch.empty((n,), dtype=torch.int32, device="cuda")
    counts, offs, rt, sr = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    moe.moe_permute(idx, E, counts, offs, rt, sr, ws)
    bias = g["bias"].clone()
    moe.moe_bias_update(counts, T, k, 1e-3, bias)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    ridx, _, gap = oracle.route(inp["x"], inp["w_router"], inp["bias"], k, cfg.scale)
    assert (gap >= 1e-6).all()                      # no near-ties in this draw
    rcounts = np.bincount(ridx.reshape(-1), minlength=E).astype(np.int32)
    assert np.array_equal(counts.cpu().numpy(), rcounts)
    assert np.array_equal(bias.cpu().numpy(), oracle.bias_update(rcounts, T, k, 1e-3, inp["bias"]))


def test_router_scores(moe):
    cfg = MoEConfig("scores", T=70, d=512, E=48, k=6, inter=128, scale=2.827)
    inp = make_inputs(cfg, seed=51)
    g = {k: v.cuda() for k, v in inp.items()}
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    sc = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device="cuda")
    moe.moe_router_scores(g["x"], g["w_router"], sc, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    _, _, _, ref = oracle.route(inp["x"], inp["w_router"], inp["bias"], cfg.k, cfg.scale,
                                want_scores=True)
    # fp32 accumulation over d = 512 of bf16 products: |d logit| < 1e-5, sigmoid' <= 1/4
    assert np.abs(sc.cpu().numpy() - ref).max() < 5e-6


@pytest.mark.parametrize("B,S,E,k", [(4, 64, 384, 8), (3, 37, 7, 3), (1, 500, 1024, 32),
                                     (8, 1, 16, 4), (2, 4096, 384, 8)])
def test_seq_aux_loss(moe, B, S, E, k):
    rng = np.random.default_rng(B * S + E)
    T = B * S
    scores = (1.0 / (1.0 + np.exp(-rng.normal(0, 1, (T, E))))).astype(np.float32)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    loss = torch.empty(B, dtype=torch.float32, device="cuda")
    f = torch.empty((B, E), dtype=torch.float32, device="cuda")
    p = torch.empty((B, E), dtype=torch.float32, device="cuda")
    moe.moe_seq_aux_loss(torch.from_numpy(scores).cuda(), torch.from_numpy(idx).cuda(), S, 1e-3,
                         loss, f, p)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    rl, rf, rp = oracle.seq_aux_loss(scores.astype(np.float64), idx, S, 1e-3)
    # f is an integer count times E/(kS): exact up to one fp32 rounding
    assert np.allclose(f.cpu().numpy(), rf, rtol=2e-7, atol=0)
    # sums of S fp32 terms and of E products: a few hundred ulp at most
    assert np.allclose(p.cpu().numpy(), rp, rtol=1e-5, atol=1e-9)
    assert np.allclose(loss.cpu().numpy(), rl, rtol=1e-5, atol=0)
    # deterministic
    loss2 = torch.empty_like(loss)
    moe.moe_seq_aux_loss(torch.from_numpy(scores).cuda(), torch.from_numpy(idx).cuda(), S, 1e-3,
                         loss2)
    torch.cuda.synchronize()
    assert torch.equal(loss.view(torch.int32), loss2.view(torch.int32))
