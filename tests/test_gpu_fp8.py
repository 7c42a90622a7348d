"""FP8 storage of the routed experts' weights ("Kimi K2.5 Q&A", Q7.1: routed-
expert weight storage quantized, compute in BF16, shared experts exempt), CUDA
path against the fp64 oracle (B200 only).

- moe_quantize_fp8: codes and block exponents bit-exact against the oracle's
  quantizer (an integer result decided by floating point: both sides take the
  decision from the same exact value w * 2^-s).
- moe_layer_forward_fp8: against the oracle's layer evaluated with the weights
  the ORACLE's own quantizer produces, dequantized exactly; same tolerance as
  the bf16 layer, since the GPU computes with exactly those weights.
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


def _planted(shape, seed):
    """bf16 weights whose 128 x 128 blocks span many magnitudes, an all-zero
    block, a block of values in the E4M3 subnormal range, and exact ties."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, shape)
    rows, cols = shape[-2], shape[-1]
    w2 = w.reshape(-1, rows, cols)
    for m in range(w2.shape[0]):
        for i in range(rows // 128):
            for j in range(cols // 128):
                w2[m, i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] *= 2.0 ** ((i * 5 + j * 3 + m) % 23 - 11)
    w2[0, :128, :128] = 0.0
    if cols >= 256:
        w2[0, :128, 128:256] = rng.normal(0, 1e-6, (128, 128))
        w2[0, :128, 128] = 1.0                      # block max: s = -8, rest far below
    t = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)
    if rows >= 256 and cols >= 256:
        # ties between two E4M3 values after scaling: 1.0625 sits between 1.0 and 1.125
        t.view(-1, rows, cols)[0, 128, 256 % cols] = 448.0
        t.view(-1, rows, cols)[0, 129, 256 % cols] = 1.0625
    return t


@pytest.mark.parametrize("shape", [(128, 128), (256, 384), (3, 256, 512), (2, 384, 256)])
def test_quantize_bit_exact(moe, shape):
    w = _planted(shape, seed=sum(shape))
    q, e = moe.moe_quantize_fp8(w.cuda())
    torch.cuda.synchronize()
    rq, re = oracle.quantize_fp8(_u16(w))
    assert np.array_equal(e.cpu().numpy(), re)
    assert np.array_equal(q.cpu().numpy(), rq)


FP8_CASES = [
    MoEConfig("fp8_small", T=64, d=512, E=16, k=4, inter=256, scale=2.827),
    MoEConfig("fp8_ragged", T=37, d=384, E=7, k=3, inter=128, scale=2.827),
    MoEConfig("fp8_multi_tile", T=600, d=256, E=16, k=4, inter=128, scale=2.827, bias="zipf"),
    MoEConfig("fp8_k2_dims", T=16, d=7168, E=4, k=2, inter=2048, scale=2.827),
    # decode-sized batches (routed experts average <= 4 rows): the register-
    # dequantizing GEMMs with 16-row token tiles
    MoEConfig("fp8v_small", T=16, d=512, E=32, k=4, inter=128, scale=2.827),
    # experts 0 and 1 take all 32 tokens: two full token tiles each; d = 384
    # leaves the down tiles' second 128-row block half outside
    MoEConfig("fp8v_zipf_two_tiles", T=32, d=384, E=32, k=4, inter=256, scale=2.827,
              bias="zipf"),
    MoEConfig("fp8v_ragged", T=23, d=640, E=24, k=3, inter=384, scale=2.827),
    MoEConfig("fp8v_k2_dims", T=8, d=7168, E=16, k=8, inter=2048, scale=2.827),
]


def _oracle_fp8_inputs(inp):
    """The layer inputs with the routed experts' weights replaced by what the
    oracle's own quantizer stores, dequantized (shared expert unchanged)."""
    out = dict(inp)
    for key in ("w_gate_up", "w_down"):
        q, s = oracle.quantize_fp8(_u16(inp[key]))
        out[key] = oracle.dequantize_fp8(q, s)
    return out


@pytest.mark.parametrize("cfg", FP8_CASES, ids=lambda c: c.name)
def test_fp8_layer_parity(moe, cfg):
    inp = make_inputs(cfg, seed=31)
    g = {k: v.cuda() for k, v in inp.items()}
    qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8(g["w_down"])
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_fp8(g["x"], g["w_router"], g["bias"], qgu, egu, qdn, edn,
                              g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    ref, ridx, rw, gap = oracle.moe_forward(_oracle_fp8_inputs(inp), cfg.k, cfg.scale)
    PR.check_output(PR.bf16_np(out), ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])


def test_fp8_layer_deterministic_and_ws(moe):
    cfg = FP8_CASES[0]
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=32).items()}
    qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8(g["w_down"])
    args = (g["x"], g["w_router"], g["bias"], qgu, egu, qdn, edn, g["ws_gate_up"], g["ws_down"],
            cfg.k, cfg.scale)
    o1 = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    o2, o3 = torch.empty_like(o1), torch.empty_like(o1)
    moe.moe_layer_forward_fp8(*args, o1)
    moe.moe_layer_forward_fp8(*args, o2)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_fp8_ws(*args, o3, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_fp8_decode_path_deterministic_and_ws(moe):
    """The decode-sized path: identical bits on repeated calls and through the
    caller-workspace form."""
    cfg = next(c for c in FP8_CASES if c.name == "fp8v_zipf_two_tiles")
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=33).items()}
    qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8(g["w_down"])
    args = (g["x"], g["w_router"], g["bias"], qgu, egu, qdn, edn, g["ws_gate_up"], g["ws_down"],
            cfg.k, cfg.scale)
    o1 = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    o2, o3 = torch.empty_like(o1), torch.empty_like(o1)
    moe.moe_layer_forward_fp8(*args, o1)
    moe.moe_layer_forward_fp8(*args, o2)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_fp8_ws(*args, o3, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_fp8_fullsize_decode(moe):
    """K2 decode shape in the benchmark's launch configuration: every token's
    output row against the oracle evaluated with its own quantizer's weights
    (one batch of experts on the host at a time); the GPU's stored codes and
    exponents of every selected expert equal the oracle quantizer's."""
    cfg = CONFIGS["k2_decode"]
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    g = make_inputs(cfg, seed=0, device="cuda")
    qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8(g["w_down"])
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_fp8(g["x"], g["w_router"], g["bias"], qgu, egu, qdn, edn,
                              g["ws_gate_up"], g["ws_down"], k, cfg.scale, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    x_h = g["x"].cpu()
    ridx, rw, gap = oracle.route(x_h, g["w_router"].cpu(), g["bias"].cpu(), k, cfg.scale)
    sample, parts = PR.wide_sample(ridx, gap, E, T, k)

    def load_expert(e):
        wts = []
        for key, q_gpu, s_gpu in (("w_gate_up", qgu, egu), ("w_down", qdn, edn)):
            q, s = oracle.quantize_fp8(_u16(g[key][e]))
            assert np.array_equal(q_gpu[e].cpu().numpy(), q), f"expert {e} {key} codes"
            assert np.array_equal(s_gpu[e].cpu().numpy(), s), f"expert {e} {key} exponents"
            wts.append(oracle.dequantize_fp8(q, s))
        return tuple(wts)

    ref = PR.oracle_rows_by_expert(
        x_h, ridx, rw, sample, load_expert=load_expert,
        load_shared=lambda: (PR.u16(g["ws_gate_up"]), PR.u16(g["ws_down"])),
        row_fn=lambda xr, wts: oracle.swiglu_row(xr, *wts))
    PR.check_output(PR.bf16_np(out[torch.tensor(sample, device="cuda")]), ref)
    del g, qgu, qdn, out
    torch.cuda.empty_cache()


def test_fp8_layer_subnormal_codes(moe):
    """Routed gate|up weights whose codes are almost all E4M3 subnormals: each
    128 x 128 block holds one element of 1.0 (so s = -8) in K column 0 of the
    block, which x zeroes out, and values near 2e-5 elsewhere (codes 2^-9 .. 2^-7
    times 2^-8).  The shared expert is zero, so the output comes only through
    those subnormal codes; dequantizing them wrongly (flushed to zero, say)
    would change every row."""
    cfg = MoEConfig("fp8_subnormal", T=48, d=256, E=8, k=2, inter=128, scale=2.827)
    inp = make_inputs(cfg, seed=41)
    gu = inp["w_gate_up"].float() * 1e-3
    gu[:, :, ::128] = 0.0
    gu[:, ::128, ::128] = 1.0
    inp["w_gate_up"] = gu.to(torch.bfloat16)
    x = inp["x"].float()
    x[:, ::128] = 0.0
    inp["x"] = x.to(torch.bfloat16)
    inp["ws_gate_up"] = torch.zeros_like(inp["ws_gate_up"])
    q, s = oracle.quantize_fp8(_u16(inp["w_gate_up"]))
    sub = ((q & 0x78) == 0) & ((q & 0x07) != 0)
    assert sub.mean() > 0.5                      # most codes are subnormal
    assert np.all(s == -8)
    g = {k: v.cuda() for k, v in inp.items()}
    qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
    qdn, edn = moe.moe_quantize_fp8(g["w_down"])
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_fp8(g["x"], g["w_router"], g["bias"], qgu, egu, qdn, edn,
                              g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert np.array_equal(qgu.cpu().numpy(), q)
    ref, ridx, rw, gap = oracle.moe_forward(_oracle_fp8_inputs(inp), cfg.k, cfg.scale)
    assert np.abs(ref).max() > 0
    PR.check_output(PR.bf16_np(out), ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])
