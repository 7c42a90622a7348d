"""FP8 compute in every expert ("Kimi K2.5 Q&A", Q7.1 names V3's compute in
FP8; "Kimi K2 deep dive", 3.2), CUDA path against the fp64 oracle (B200 only).

- moe_quantize_fp8_rows: codes and per-row exponents bit-exact against the
  oracle's row quantizer (both sides decide from the exact value w * 2^-s).
- moe_layer_forward_w8a8: against the oracle's FP8-compute layer, which
  quantizes x and the bf16 activation per row exactly as the method states and
  evaluates everything else in fp64, with the weights the ORACLE's quantizer
  produces.  Tolerance: the bf16 output rule of the bf16 layer (relative L2
  5e-3, max 2% of max|ref|).  GPU and oracle form the same bf16 activation up to
  fp32 accumulation order; an activation element that lands next to an E4M3
  rounding boundary can take the neighbouring code (one step of 2^-3 of its own
  size), which moves the output far less than the bf16 rounding the rule allows.
No expected value comes from the CUDA path.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as PR
from moe_inputs import CONFIGS, MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _planted_rows(shape, seed):
    """bf16 rows of many magnitudes: an all-zero row, a row whose maximum is
    negative, a row at exactly 448 * 2^-3, a row below the clamp, ties."""
    rng = np.random.default_rng(seed)
    rows, cols = shape
    w = rng.normal(0, 1, shape) * 2.0 ** rng.integers(-40, 20, (rows, 1))
    w[0] = 0.0
    w[1, 3] = -100.0 * np.abs(w[1]).max()
    w[2] = rng.normal(0, 1e-3, cols)
    w[2, 5] = 56.0
    w[3] = rng.normal(0, 1e-39, cols)
    t = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)
    t[4, :4] = torch.tensor([448.0, 1.0625, -1.0625, 3.25 * 2 ** -9])   # ties after scaling
    return t


@pytest.mark.parametrize("shape", [(8, 128), (37, 208), (300, 7168), (2048 + 5, 48)])
def test_quantize_rows_bit_exact(moe, shape):
    w = _planted_rows(shape, seed=sum(shape))
    q, e = moe.moe_quantize_fp8_rows(w.cuda())
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    rq, re = oracle.quantize_fp8_rows(_u16(w))
    assert np.array_equal(e.cpu().numpy(), re)
    assert np.array_equal(q.cpu().numpy(), rq)


def _quantize_all(moe, g):
    qgu, egu = moe.moe_quantize_fp8_rows(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8_rows(g["w_down"])
    sqgu, segu = moe.moe_quantize_fp8_rows(g["ws_gate_up"])
    sqdn, sedn = moe.moe_quantize_fp8_rows(g["ws_down"])
    return (qgu, egu, qdn, edn, sqgu, segu, sqdn, sedn)


W8A8_CASES = [
    MoEConfig("w8a8_small", T=64, d=512, E=16, k=4, inter=256, scale=2.827),
    MoEConfig("w8a8_ragged", T=37, d=384, E=7, k=3, inter=128, scale=2.827),
    MoEConfig("w8a8_multi_tile", T=600, d=256, E=16, k=4, inter=128, scale=2.827, bias="zipf"),
    MoEConfig("w8a8_k2_dims", T=16, d=7168, E=4, k=2, inter=2048, scale=2.827),
    MoEConfig("w8a8_v3_scale", T=100, d=384, E=12, k=6, inter=256, scale=2.5),
    MoEConfig("w8a8_one_token_k_eq_E", T=2, d=128, E=8, k=8, inter=128, scale=2.827),
    # T >= 1024: token rows quantized token by token (rows of 16 and 48 vectors)
    MoEConfig("w8a8_token_major_d128", T=1100, d=128, E=32, k=8, inter=128, scale=2.827),
    MoEConfig("w8a8_token_major_d384", T=1030, d=384, E=16, k=4, inter=128, scale=2.827),
]


def _plant_token_rows(inp):
    """Token 0 all zero, token 1 one large element among tiny ones (its codes
    mostly subnormal or zero after the per-row scaling)."""
    x = inp["x"].float()
    x[0] = 0.0
    x[1] = x[1] * 1e-4
    x[1, 7] = 3.0
    inp["x"] = x.to(torch.bfloat16)
    return inp


@pytest.mark.parametrize("cfg", W8A8_CASES, ids=lambda c: c.name)
def test_w8a8_layer_parity(moe, cfg):
    inp = _plant_token_rows(make_inputs(cfg, seed=51))
    g = {k: v.cuda() for k, v in inp.items()}
    wq = _quantize_all(moe, g)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(g["x"], g["w_router"], g["bias"], *wq, cfg.k, cfg.scale, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    ref, ridx, rw, gap = oracle.moe_forward_fp8(inp, cfg.k, cfg.scale)
    o = PR.bf16_np(out)
    assert np.all(o[0] == 0.0)                         # a zero token row gives zero
    PR.check_output(o, ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])


def test_w8a8_layer_deterministic_and_ws(moe):
    cfg = W8A8_CASES[0]
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=52).items()}
    wq = _quantize_all(moe, g)
    args = (g["x"], g["w_router"], g["bias"], *wq, cfg.k, cfg.scale)
    o1 = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    o2, o3 = torch.empty_like(o1), torch.empty_like(o1)
    moe.moe_layer_forward_w8a8(*args, o1)
    moe.moe_layer_forward_w8a8(*args, o2)
    ws = torch.empty(moe.moe_workspace_size_w8a8(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_w8a8_ws(*args, o3, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))
    # every kernel slot runs in FP8 compute, the activation quantizer included
    names = [moe.moe_kernel_name(i) for i in range(32) if moe.moe_kernel_name(i)]
    assert "quantize_h" in names and moe.moe_last_launch_count() == len(names)


FULL = ["k2_decode", "k2_prefill", "k2_skew", "v3"]


def _sample_tokens(ridx, gap, E, T):
    """Token 0, T/2, T-1 and the first token of the busiest expert (near-ties out)."""
    counts, offsets, row_token, _ = oracle.permute(ridx, E)
    busiest = int(np.argmax(counts))
    first_of_busiest = int(row_token[offsets[busiest]])
    return sorted({0, T // 2, T - 1, first_of_busiest} - set(np.nonzero(gap < PR.TIE_EPS)[0]))


@pytest.mark.parametrize("name", FULL)
def test_w8a8_fullsize(moe, name):
    """Full K2 / DeepSeek-V3 shapes in the benchmark's launch configuration: the
    output rows at the GEMM tiles' ends (the last 64 rows of the busiest
    expert's segment, of the shared expert's last tile and of a ragged
    multi-tile expert's last tile) against the oracle with its own row
    quantizer; the GPU codes and exponents of every expert those rows select
    equal the oracle quantizer's."""
    cfg = CONFIGS[name]
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    g = make_inputs(cfg, seed=0, device="cuda")
    wq = _quantize_all(moe, g)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_w8a8(g["x"], g["w_router"], g["bias"], *wq, k, cfg.scale, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    x_h = g["x"].cpu()
    ridx, rw, gap = oracle.route(x_h, g["w_router"].cpu(), g["bias"].cpu(), k, cfg.scale)
    # each tile part's last 64 rows (the tiles' ends): the oracle's FP8 / INT4
    # rows cost more than bf16 ones
    sample, parts = PR.wide_sample(ridx, gap, E, T, k, tail=64)
    print(f"{name}: {len(sample)} rows compared: {parts}")
    assert len(sample) >= min(T, 64) - 4, parts

    def load_expert(e):
        q = oracle.quantize_fp8_rows(PR.u16(g["w_gate_up"][e])) + \
            oracle.quantize_fp8_rows(PR.u16(g["w_down"][e]))
        for got, want in zip((wq[0][e], wq[1][e], wq[2][e], wq[3][e]), q):
            assert np.array_equal(got.cpu().numpy(), want), f"expert {e} codes"
        return q

    ref = PR.oracle_rows_by_expert(
        x_h, ridx, rw, sample, load_expert=load_expert,
        load_shared=lambda: oracle.quantize_fp8_rows(PR.u16(g["ws_gate_up"])) +
        oracle.quantize_fp8_rows(PR.u16(g["ws_down"])),
        row_fn=lambda xr, q: oracle.swiglu_row_fp8(xr, *q))
    PR.check_output(PR.bf16_np(out[torch.tensor(sample, device="cuda")]), ref)
    del g, wq, out
    torch.cuda.empty_cache()
