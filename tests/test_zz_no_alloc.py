"""The allocation-free layer entry point, moe_layer_forward_noalloc.

Some callers of this library cannot allocate device memory.  A serving engine
may already have reserved the GPU's memory for weights and its KV cache and
give plugins no allocator.  A latency-critical loop cannot afford the
device-wide synchronisation that cudaMalloc may cause.  A deployment may run
on a fixed, audited memory plan.  Those callers use moe_layer_forward_noalloc,
which works in a scratch array compiled into the library and allocates
nothing.

These tests call it through the C ABI, twice in a row with different inputs,
and compare each result with moe_layer_forward (which manages its own
scratch), within the tolerance every parity test here uses.  They also check
the size limit.  This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import parity as PR
from moe_inputs import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_ok):
    import sparse_moe_ffn_sigmoid_b200 as m
    m.moe_device_status()
    return m


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_raw(moe, g, x, cfg, out):
    """The new entry point, called directly through the C ABI."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return moe.lib().moe_layer_forward_noalloc(
        _p(x), _p(g["w_router"]), _p(g["bias"]), _p(g["w_gate_up"]), _p(g["w_down"]),
        _p(g["ws_gate_up"]), _p(g["ws_down"]), x.shape[0], cfg.d, cfg.E, cfg.k, cfg.inter,
        ctypes.c_float(cfg.scale), _p(out), stream)


@pytest.mark.parametrize("name", ["tiny", "k2_decode"])
def test_noalloc_matches_layer_forward_on_two_calls(moe, name):
    cfg = CONFIGS[name]
    g = make_inputs(cfg, seed=11, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(12)
    xs = [g["x"], torch.randn(g["x"].shape, generator=gen, device="cuda").to(torch.bfloat16)]
    for call, x in enumerate(xs):
        ref = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_forward(x, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                              g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, ref)
        out = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = _noalloc_raw(moe, g, x, cfg, out)
        assert rc == 0, f"call {call}: {moe.moe_status_string(rc)}"
        torch.cuda.synchronize()
        assert moe.moe_device_status() == 0
        PR.check_output(PR.bf16_np(out), PR.bf16_np(ref))


def test_noalloc_size_limit(moe):
    cfg = CONFIGS["k2_decode"]
    limit = moe.NOALLOC_SCRATCH_BYTES
    fits = max(T for T in range(1, 200)
               if moe.moe_workspace_size(T, cfg.d, cfg.E, cfg.k, cfg.inter) <= limit)
    assert fits >= cfg.T            # the K2 decode batch fits
    # one weight set; only the token rows change with T
    g = make_inputs(cfg, seed=13, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(14)
    x_big = torch.randn((fits + 1, cfg.d), generator=gen, device="cuda").to(torch.bfloat16)
    out = torch.empty((fits + 1, cfg.d), dtype=torch.bfloat16, device="cuda")
    # one token more than the array holds: refused before any launch
    assert _noalloc_raw(moe, g, x_big, cfg, out) == -2      # MOE_ERR_UNSUPPORTED_SHAPE
    # the largest batch that fits runs, and its scratch reaches the array's
    # last bytes: compare it with the allocating entry point
    x_fit = x_big[:fits].contiguous()
    out2 = torch.full((fits, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _noalloc_raw(moe, g, x_fit, cfg, out2) == 0
    ref = torch.empty((fits, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(x_fit, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                          g["ws_gate_up"], g["ws_down"], cfg.k, cfg.scale, ref)
    torch.cuda.synchronize()
    assert moe.moe_device_status() == 0
    PR.check_output(PR.bf16_np(out2), PR.bf16_np(ref))


def _pool_bytes():
    """(used, reserved) bytes of the device's default CUDA memory pool, the pool
    cudaMallocAsync draws from, or None without the cuda-python bindings."""
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        return None
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess, err
    vals = []
    for attr in (rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemCurrent,
                 rt.cudaMemPoolAttr.cudaMemPoolAttrReservedMemCurrent):
        err, v = rt.cudaMemPoolGetAttribute(pool, attr)
        assert err == rt.cudaError_t.cudaSuccess, err
        vals.append(int(v))
    return tuple(vals)


def test_noalloc_allocates_nothing(moe):
    """The point of the entry point: two calls on a stream the library has never
    seen leave the device's free memory and the stream-ordered pool unchanged
    (the allocating entry point would take a new scratch buffer for a new
    stream)."""
    cfg = CONFIGS["tiny"]
    g = make_inputs(cfg, seed=15, device="cuda")
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    assert _noalloc_raw(moe, g, g["x"], cfg, out) == 0      # warm-up (symbol lookup)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    free0 = torch.cuda.mem_get_info()[0]
    pool0 = _pool_bytes()
    with torch.cuda.stream(side):
        for _ in range(2):
            assert _noalloc_raw(moe, g, g["x"], cfg, out) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert _pool_bytes() == pool0
    assert moe.moe_device_status() == 0
