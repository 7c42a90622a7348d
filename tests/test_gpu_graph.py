"""The layer inside a CUDA graph: moe_layer_forward_ws / _w8a8_ws captured once
(caller-owned workspace, so the call allocates nothing), then replayed on new
token rows copied into the captured input.  Every replay must give the eager
call's bits (the path is deterministic)."""
import pytest
import torch

from moe_inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


CFG = MoEConfig("graph", T=64, d=512, E=16, k=4, inter=256, scale=2.827)


def _replay_matches_eager(moe, run, ws, g, cfg):
    x_in = g["x"].clone()
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    run(x_in, out, ws)                      # eager first: one-time host setup
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            run(x_in, out, ws)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (1, 2):
        x_new = make_inputs(cfg, seed=seed)["x"].cuda()
        x_in.copy_(x_new)
        graph.replay()
        torch.cuda.synchronize()
        assert moe.moe_device_status() == 0
        ref = torch.empty_like(out)
        run(x_new, ref, ws)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), seed
    del graph


def test_bf16_layer_in_a_cuda_graph(moe):
    g = {k: v.cuda() for k, v in make_inputs(CFG, seed=0).items()}
    ws = torch.empty(moe.moe_workspace_size(CFG.T, CFG.d, CFG.E, CFG.k, CFG.inter),
                     dtype=torch.uint8, device="cuda")

    def run(x, out, ws_):
        moe.moe_layer_forward_ws(x, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                                 g["ws_gate_up"], g["ws_down"], CFG.k, CFG.scale, out, ws_)

    _replay_matches_eager(moe, run, ws, g, CFG)


def test_w8a8_layer_in_a_cuda_graph(moe):
    g = {k: v.cuda() for k, v in make_inputs(CFG, seed=0).items()}
    wq = []
    for key in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        wq += list(moe.moe_quantize_fp8_rows(g[key]))
    ws = torch.empty(moe.moe_workspace_size_w8a8(CFG.T, CFG.d, CFG.E, CFG.k, CFG.inter),
                     dtype=torch.uint8, device="cuda")

    def run(x, out, ws_):
        moe.moe_layer_forward_w8a8_ws(x, g["w_router"], g["bias"], *wq, CFG.k, CFG.scale, out,
                                      ws_)

    _replay_matches_eager(moe, run, ws, g, CFG)
