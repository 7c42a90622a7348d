"""The expert-parallel layer's kernels on a B200: moe_ep_dispatch,
moe_ep_expert_ffn and moe_ep_combine with the exchange of sparse_moe_ffn_sigmoid_b200.ep.

- R = 2 and 4 ranks emulated as host threads of one process sharing one GPU:
  the all-to-all is a host-side exchange of device rows between the threads (no
  kernel waits on another rank; the threads meet on a host barrier).  Each
  rank's output must equal moe_layer_forward on that rank's tokens bit for bit,
  since every row meets the same kernels in the same K order.
- R = 1 over a real NCCL process group (one GPU): the same, through
  torch.distributed.all_to_all_single.
"""
import os
import socket
import threading

import pytest
import torch

from moe_inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


class ThreadComm:
    """All-to-all between R threads of one process on one device."""

    def __init__(self, shared, rank, world):
        self.shared, self.rank, self.world = shared, rank, world

    def all_to_all(self, out, inp, out_splits, in_splits):
        sh = self.shared
        sh["bufs"][self.rank] = (inp, list(in_splits))
        sh["barrier"].wait()
        off = 0
        for s in range(self.world):
            src, splits = sh["bufs"][s]
            start, n = sum(splits[:self.rank]), splits[self.rank]
            assert n == out_splits[s]
            if n:
                out[off:off + n].copy_(src[start:start + n])
            off += n
        torch.cuda.synchronize()
        sh["barrier"].wait()


def _ref(moe, g, x, cfg):
    out = torch.empty_like(x)
    if x.shape[0]:
        moe.moe_layer_forward(x, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                              g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, out)
    return out


CASES = [
    (MoEConfig("ep_small", T=96, d=512, E=32, k=4, inter=256, scale=2.827), 2, [48, 48]),
    (MoEConfig("ep_ragged", T=70, d=384, E=16, k=3, inter=128, scale=2.827), 4, [30, 0, 17, 23]),
    (MoEConfig("ep_zipf", T=600, d=256, E=16, k=4, inter=128, scale=2.827, bias="zipf"), 4,
     [150, 150, 150, 150]),
    (MoEConfig("ep_k2_dims", T=64, d=7168, E=32, k=8, inter=2048, scale=2.827), 4,
     [16, 16, 16, 16]),
]


@pytest.mark.parametrize("cfg,world,splits", CASES, ids=[c[0].name + f"_r{c[1]}" for c in CASES])
def test_ep_threads_equal_layer_forward(moe, cfg, world, splits):
    from sparse_moe_ffn_sigmoid_b200.ep import ExpertParallelMoE
    g = make_inputs(cfg, seed=71, device="cuda")
    El = cfg.E // world
    shared = {"bufs": [None] * world, "barrier": threading.Barrier(world)}
    outs, errors = [None] * world, []

    def rank_main(r):
        try:
            t0 = sum(splits[:r])
            x = g["x"][t0:t0 + splits[r]].contiguous()
            layer = ExpertParallelMoE(ThreadComm(shared, r, world), g["w_router"], g["bias"],
                                      g["w_gate_up"][r * El:(r + 1) * El], g["w_down"][r * El:(r + 1) * El],
                                      g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale)
            outs[r] = layer.forward(x, torch.empty_like(x))
        except BaseException as e:          # noqa: BLE001  (re-raised below)
            errors.append(e)
            shared["barrier"].abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    if errors:
        raise errors[0]
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    for r in range(world):
        t0 = sum(splits[:r])
        ref = _ref(moe, g, g["x"][t0:t0 + splits[r]].contiguous(), cfg)
        torch.cuda.synchronize()
        assert torch.equal(outs[r].view(torch.int16), ref.view(torch.int16)), f"rank {r}"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_nccl_one_rank(moe, monkeypatch):
    import datetime
    import torch.distributed as dist
    from sparse_moe_ffn_sigmoid_b200.ep import ExpertParallelMoE, TorchComm
    monkeypatch.setenv("MASTER_ADDR", "127.0.0.1")
    monkeypatch.setenv("MASTER_PORT", str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        cfg = CASES[0][0]
        g = make_inputs(cfg, seed=72, device="cuda")
        layer = ExpertParallelMoE(TorchComm(), g["w_router"], g["bias"], g["w_gate_up"],
                                  g["w_down"], g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale)
        out = layer.forward(g["x"], torch.empty_like(g["x"]))
        ref = _ref(moe, g, g["x"], cfg)
        torch.cuda.synchronize()
        assert moe.moe_device_status() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    finally:
        dist.destroy_process_group()


def test_ep_expert_ffn_rejects_count_mismatch(moe):
    """Counts that do not add up to the received rows: recorded in the device
    status, no expert computed, zero output rows."""
    cfg = CASES[0][0]
    g = make_inputs(cfg, seed=73, device="cuda")
    rows, R, El = 10, 2, cfg.E // 2
    recv = torch.randn((rows, cfg.d), device="cuda").to(torch.bfloat16)
    counts = torch.zeros((R, El), dtype=torch.int32, device="cuda")
    counts[0, 0] = 4
    counts[1, 3] = 5                        # 9 rows counted, 10 received
    y = torch.full_like(recv, float("nan"))
    ws = torch.empty(moe.moe_ep_expert_ffn_workspace_size(rows, cfg.d, R, El, cfg.inter),
                     dtype=torch.uint8, device="cuda")
    moe.moe_ep_expert_ffn(recv, counts, g["w_gate_up"][:El], g["w_down"][:El], y, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == -1    # MOE_ERR_INVALID_ARG
    assert torch.equal(y.float(), torch.zeros_like(y.float()))
