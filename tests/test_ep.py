"""The expert-parallel layer's exchange and bookkeeping as gloo ranks on CPU:
each rank owns E/R routed experts and routes its own tokens; the layer's kernel
calls are the oracle's (tests/ep_oracle_ops.py).  The ranks' outputs, put back
in token order, must equal the oracle's single-device layer on the whole batch
within the parity tolerance: rows cross the exchange twice (to their experts'
ranks and back) and every split, count and slot must land where it belongs."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import parity as PR
from moe_inputs import MoEConfig, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = [
    # (config, world, tokens per rank)
    (MoEConfig("ep_tiny", T=48, d=256, E=16, k=4, inter=128, scale=2.827), 2, [24, 24]),
    (MoEConfig("ep_tiny4", T=48, d=256, E=16, k=4, inter=128, scale=2.827), 4, [20, 0, 11, 17]),
    # Zipf-like loads: ranks owning the first experts receive most rows, the
    # last rank's experts almost none
    (MoEConfig("ep_zipf", T=40, d=128, E=8, k=2, inter=64, scale=2.5, bias="zipf"), 4,
     [10, 10, 10, 10]),
]


@pytest.mark.parametrize("cfg,world,splits", CASES, ids=[c[0].name + f"_r{c[1]}" for c in CASES])
def test_ep_layer_gloo_matches_oracle(cfg, world, splits, monkeypatch):
    import torch.multiprocessing as mp
    assert sum(splits) == cfg.T
    monkeypatch.setenv("PYTHONPATH", os.pathsep.join([ROOT, TESTS, os.environ.get("PYTHONPATH", "")]))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    import ep_worker
    procs = [ctx.Process(target=ep_worker.run, args=(r, world, port, cfg.as_dict(), splits, q))
             for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got = np.concatenate([results[r] for r in range(world)]).view(np.uint16)
    got = torch.from_numpy(got.view(np.int16)).view(torch.bfloat16)
    g = make_inputs(cfg, seed=5)
    ref, ridx, rw, gap = oracle.moe_forward(g, cfg.k, cfg.scale)
    PR.check_output(PR.bf16_np(got), ref, skip_rows=np.nonzero(gap < PR.TIE_EPS)[0])


class _OneRank:
    """A comm stand-in that only reports its size (no exchange is reached)."""

    def __init__(self, world):
        self.rank, self.world = 0, world

    def all_to_all(self, out, inp, out_splits, in_splits):
        raise AssertionError("the constructor checks run before any exchange")


def test_ep_layer_rejects_uneven_expert_split():
    from sparse_moe_ffn_sigmoid_b200 import ep
    cfg = MoEConfig("ep_check", T=4, d=64, E=6, k=2, inter=64, scale=2.827)
    g = make_inputs(cfg, seed=0)
    with pytest.raises(ValueError, match="do not split evenly"):
        ep.ExpertParallelMoE(_OneRank(4), g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                             g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, ops=object())


def test_ep_layer_rejects_wrong_local_expert_count():
    from sparse_moe_ffn_sigmoid_b200 import ep
    cfg = MoEConfig("ep_check", T=4, d=64, E=8, k=2, inter=64, scale=2.827)
    g = make_inputs(cfg, seed=0)
    # rank of 2 must hold E/R = 4 experts; give it all 8
    with pytest.raises(ValueError, match="expected E/R = 4"):
        ep.ExpertParallelMoE(_OneRank(2), g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                             g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, ops=object())
