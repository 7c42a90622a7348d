"""INT4 storage of the routed experts' weights ("Kimi K2.5 deep dive", CH7.2:
4-bit symmetric integers in groups of 32 along K; "Kimi K2.5 Q&A", Q7.1:
storage quantized, compute BF16), CUDA path against the fp64 oracle (B200 only).

- moe_quantize_int4: codes and group scales bit-exact against the oracle's
  quantizer (the test only re-packs the oracle's codes into the library's
  layout and transposes its scales: no arithmetic);
- moe_layer_forward_w4a16: against the oracle's bf16 layer evaluated with the
  weights the ORACLE's quantizer stands for, bf16(q * s); the bf16 layer's
  tolerance, since the GPU computes with exactly those weights.
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


def pack_codes(q):
    """The library's packing of int codes [.., rows, cols] (layout only): word j
    of a row holds elements 8j + 2i in bits 4i.. and 8j + 2i + 1 in bits 16 + 4i..,
    each as q + 8; returned as bytes [.., rows, cols / 2]."""
    n = (q.astype(np.int64) + 8).reshape(q.shape[:-1] + (q.shape[-1] // 8, 8))
    word = np.zeros(n.shape[:-1], dtype=np.uint64)
    for i in range(4):
        word |= (n[..., 2 * i].astype(np.uint64) << np.uint64(4 * i))
        word |= (n[..., 2 * i + 1].astype(np.uint64) << np.uint64(16 + 4 * i))
    return word.astype(np.uint32).view(np.uint8).reshape(q.shape[:-1] + (q.shape[-1] // 2,))


def _planted(shape, seed):
    """Groups of many magnitudes, an all-zero group, a negative group maximum,
    integer values (exact ties of w / s), bf16 subnormals."""
    rng = np.random.default_rng(seed)
    cols = shape[-1]
    w = rng.normal(0, 1, shape)
    w2 = w.reshape(-1, cols)
    w2 *= 2.0 ** rng.integers(-30, 12, (w2.shape[0], cols // 32)).repeat(32, 1)
    w2[0, :32] = 0.0
    w2[0, 32:64] = rng.normal(0, 1e-3, 32)
    w2[0, 40] = -3.0
    w2[1, :32] = np.arange(32) - 16.0
    w2[1, 32:64] = rng.normal(0, 1e-39, 32)
    return torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("shape", [(4, 64), (37, 192), (3, 256, 512), (2053, 128)])
def test_quantize_int4_bit_exact(moe, shape):
    w = _planted(shape, seed=sum(shape))
    codes, scales = moe.moe_quantize_int4(w.cuda())
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    q, sc = oracle.quantize_int4(_u16(w))
    assert np.array_equal(codes.cpu().numpy(), pack_codes(q))
    cols = shape[-1]
    want = sc.reshape(-1, cols // 32).T
    assert np.array_equal(scales.cpu().view(torch.int16).numpy().view(np.uint16), want)


W4_CASES = [
    MoEConfig("w4_small", T=64, d=512, E=16, k=4, inter=256, scale=2.827),
    MoEConfig("w4_ragged", T=37, d=384, E=7, k=3, inter=192, scale=2.827),
    MoEConfig("w4_multi_tile", T=600, d=256, E=16, k=4, inter=128, scale=2.827, bias="zipf"),
    MoEConfig("w4_k2_dims", T=16, d=7168, E=4, k=2, inter=2048, scale=2.827),
    MoEConfig("w4_one_token_k_eq_E", T=1, d=128, E=4, k=4, inter=64, scale=2.827),
    # decode-sized batches (routed experts average <= 4 rows, d and inter
    # multiples of 256): the register-dequantizing GEMMs with 16-row token tiles
    MoEConfig("w4v_small", T=16, d=512, E=32, k=4, inter=256, scale=2.827),
    # experts 0 and 1 take all 32 tokens: two full token tiles each (two MMA
    # n-tiles)
    MoEConfig("w4v_zipf_two_tiles", T=32, d=512, E=32, k=4, inter=256, scale=2.827,
              bias="zipf"),
    # the shared expert's 23 rows: a 16-row and a 7-row tile; inter = 512 (four
    # feature tiles), d = 768 (three down tiles)
    MoEConfig("w4v_ragged", T=23, d=768, E=24, k=3, inter=512, scale=2.827),
    MoEConfig("w4v_k2_dims", T=8, d=7168, E=16, k=8, inter=2048, scale=2.827),
    MoEConfig("w4v_one_token_k_eq_E", T=1, d=256, E=8, k=8, inter=256, scale=2.827),
]


def _oracle_w4_inputs(inp):
    """Layer inputs with the routed experts' weights replaced by what the
    oracle's own INT4 quantizer stands for (shared expert unchanged)."""
    out = dict(inp)
    for key in ("w_gate_up", "w_down"):
        out[key] = oracle.dequantize_int4(*oracle.quantize_int4(_u16(inp[key])))
    return out


def _run(moe, g, cfg, out=None, ws=None):
    qgu, sgu = moe.moe_quantize_int4(g["w_gate_up"])
    qdn, sdn = moe.moe_quantize_int4(g["w_down"])
    if out is None:
        out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    args = (g["x"], g["w_router"], g["bias"], qgu, sgu, qdn, sdn, g["ws_gate_up"], g["ws_down"],
            cfg.k, cfg.scale, out)
    if ws is None:
        moe.moe_layer_forward_w4a16(*args)
    else:
        moe.moe_layer_forward_w4a16_ws(*args, ws)
    return out, (qgu, sgu, qdn, sdn)


@pytest.mark.parametrize("cfg", W4_CASES, ids=lambda c: c.name)
def test_w4a16_layer_parity(moe, cfg):
    inp = make_inputs(cfg, seed=61)
    g = {k: v.cuda() for k, v in inp.items()}
    out, _ = _run(moe, g, cfg)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    ref, ridx, rw, gap = oracle.moe_forward(_oracle_w4_inputs(inp), cfg.k, cfg.scale)
    PR.check_output(PR.bf16_np(out), ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])


def test_w4a16_layer_deterministic_and_ws(moe):
    cfg = W4_CASES[0]
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=62).items()}
    o1, _ = _run(moe, g, cfg)
    o2, _ = _run(moe, g, cfg)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    o3, _ = _run(moe, g, cfg, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_w4a16_decode_path_deterministic_and_ws(moe):
    """The decode-sized path: identical bits on repeated calls and through the
    caller-workspace form."""
    cfg = next(c for c in W4_CASES if c.name == "w4v_zipf_two_tiles")
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=63).items()}
    o1, _ = _run(moe, g, cfg)
    o2, _ = _run(moe, g, cfg)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    o3, _ = _run(moe, g, cfg, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


FULL = ["k2_decode", "k2_prefill", "k2_skew", "v3"]


@pytest.mark.parametrize("name", FULL)
def test_w4a16_fullsize(moe, name):
    """Full K2 / DeepSeek-V3 shapes in the benchmark's launch configuration: the
    output rows at the GEMM tiles' ends (the last 64 rows of the busiest
    expert's segment, of the shared expert's last tile and of a ragged
    multi-tile expert's last tile) against the oracle with its own INT4
    quantizer; the GPU codes and scales of every expert those rows select equal
    the oracle quantizer's."""
    cfg = CONFIGS[name]
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    g = make_inputs(cfg, seed=0, device="cuda")
    out, (qgu, sgu, qdn, sdn) = _run(moe, g, cfg)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    x_h = g["x"].cpu()
    ridx, rw, gap = oracle.route(x_h, g["w_router"].cpu(), g["bias"].cpu(), k, cfg.scale)
    # each tile part's last 64 rows (the tiles' ends): the oracle's FP8 / INT4
    # rows cost more than bf16 ones
    sample, parts = PR.wide_sample(ridx, gap, E, T, k, tail=64)
    print(f"{name}: {len(sample)} rows compared: {parts}")
    assert len(sample) >= min(T, 64) - 4, parts
    sgu_h = PR.u16(sgu)
    sdn_h = PR.u16(sdn)

    def load_expert(e):
        q, sc = oracle.quantize_int4(_u16(g["w_gate_up"][e]))
        assert np.array_equal(qgu[e].cpu().numpy(), pack_codes(q)), f"expert {e} codes"
        assert np.array_equal(sgu_h[:, e * 2 * I:(e + 1) * 2 * I], sc.T), f"expert {e} scales"
        qd, scd = oracle.quantize_int4(_u16(g["w_down"][e]))
        assert np.array_equal(qdn[e].cpu().numpy(), pack_codes(qd)), f"expert {e} down codes"
        assert np.array_equal(sdn_h[:, e * d:(e + 1) * d], scd.T), f"expert {e} down scales"
        return oracle.dequantize_int4(q, sc), oracle.dequantize_int4(qd, scd)

    ref = PR.oracle_rows_by_expert(
        x_h, ridx, rw, sample, load_expert=load_expert,
        load_shared=lambda: (PR.u16(g["ws_gate_up"]), PR.u16(g["ws_down"])),
        row_fn=lambda xr, wts: oracle.swiglu_row(xr, *wts))
    PR.check_output(PR.bf16_np(out[torch.tensor(sample, device="cuda")]), ref)
    del g, qgu, qdn, out
    torch.cuda.empty_cache()
