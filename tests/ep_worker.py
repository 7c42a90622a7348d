"""Worker of tests/test_ep.py (a module of its own so spawned processes can
import it): one gloo rank of the expert-parallel layer on CPU tensors."""
import datetime
import os


def run(rank, world, port, cfg_dict, splits, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from ep_oracle_ops import OracleOps
        from moe_inputs import MoEConfig, make_inputs
        from sparse_moe_ffn_sigmoid_b200.ep import ExpertParallelMoE, TorchComm
        cfg = MoEConfig(**cfg_dict)
        g = make_inputs(cfg, seed=5)                     # every rank draws the same batch
        El = cfg.E // world
        t0 = sum(splits[:rank])
        x = g["x"][t0:t0 + splits[rank]].contiguous()
        layer = ExpertParallelMoE(TorchComm(), g["w_router"], g["bias"],
                                  g["w_gate_up"][rank * El:(rank + 1) * El].contiguous(),
                                  g["w_down"][rank * El:(rank + 1) * El].contiguous(),
                                  g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, ops=OracleOps())
        out = torch.empty_like(x)
        layer.forward(x, out)
        queue.put((rank, out.view(torch.int16).numpy().copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()
