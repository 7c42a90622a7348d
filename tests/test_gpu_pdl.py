"""Programmatic dependent launch (moe_set_pdl): with it on, each kernel of a
library call after the first may be scheduled while the call's previous kernel
still runs, and waits for it before reading its results.  The layer's output must be
bit-identical with it on and off, for the bf16, FP8-compute and INT4 decode
paths, eager and replayed from a CUDA graph captured with it on."""
import pytest
import torch

from moe_inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    yield m
    m.moe_set_pdl(False)


CASES = [
    MoEConfig("pdl_small", T=64, d=512, E=16, k=4, inter=256, scale=2.827),
    MoEConfig("pdl_decode_shape", T=16, d=512, E=32, k=4, inter=256, scale=2.827),
]


def _runners(moe, g, cfg):
    qgu, sgu = moe.moe_quantize_int4(g["w_gate_up"])
    qdn, sdn = moe.moe_quantize_int4(g["w_down"])
    wq = []
    for key in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        wq += list(moe.moe_quantize_fp8_rows(g[key]))
    torch.cuda.synchronize()

    def bf16(x, out):
        moe.moe_layer_forward(x, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                              g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)

    def w8a8(x, out):
        moe.moe_layer_forward_w8a8(x, g["w_router"], g["bias"], *wq, cfg.k, cfg.scale, out)

    def w4a16(x, out):
        moe.moe_layer_forward_w4a16(x, g["w_router"], g["bias"], qgu, sgu, qdn, sdn,
                                    g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)

    return {"bf16": bf16, "w8a8": w8a8, "w4a16": w4a16}


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_pdl_on_and_off_give_the_same_bits(moe, cfg):
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=81).items()}
    for name, run in _runners(moe, g, cfg).items():
        outs = []
        for pdl in (False, True, True):
            moe.moe_set_pdl(pdl)
            out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
            run(g["x"], out)
            torch.cuda.synchronize()
            assert moe.moe_device_status() == 0, name
            outs.append(out)
        for o in outs[1:]:
            assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16)), name


def test_pdl_layer_in_a_cuda_graph(moe):
    cfg = CASES[1]
    g = {k: v.cuda() for k, v in make_inputs(cfg, seed=82).items()}
    moe.moe_set_pdl(True)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    x_in = g["x"].clone()
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")

    def run(x, o):
        moe.moe_layer_forward_ws(x, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                                 g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, o, ws)

    run(x_in, out)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            run(x_in, out)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (3, 4):
        x_new = make_inputs(cfg, seed=seed)["x"].cuda()
        x_in.copy_(x_new)
        graph.replay()
        torch.cuda.synchronize()
        assert moe.moe_device_status() == 0
        moe.moe_set_pdl(False)
        ref = torch.empty_like(out)
        run(x_new, ref)
        torch.cuda.synchronize()
        moe.moe_set_pdl(True)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), seed
    del graph
    moe.moe_set_pdl(False)
