"""Python binding of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: every function takes torch CUDA tensors (PyTorch
provides device memory and streams), checks dtype / device / contiguity,
passes raw pointers to the C entry point of the same name on the current
torch stream, and raises MoeError on a non-zero status.  All arithmetic runs
in the library's CUDA kernels; there is no CPU fallback, and importing this
package fails loudly if the library cannot be built or loaded.
"""
from __future__ import annotations

import ctypes

import torch

from . import build as _build

__all__ = [
    "MoeError", "lib", "moe_status_string", "moe_last_error_string", "moe_workspace_size", "moe_route", "moe_permute",
    "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_layer_forward_ws",
    "moe_device_status", "moe_set_wait_timeout_ns", "moe_set_pdl", "moe_selftest_wait_timeout",
    "moe_last_launch_count", "moe_profile_begin", "moe_profile_end", "moe_kernel_name",
    "moe_layer_forward_noalloc", "moe_quantize_fp8", "moe_layer_forward_fp8",
    "moe_layer_forward_fp8_ws", "moe_bias_update", "moe_router_scores", "moe_seq_aux_loss",
    "moe_quantize_fp8_rows", "moe_workspace_size_w8a8", "moe_layer_forward_w8a8",
    "moe_layer_forward_w8a8_ws", "moe_quantize_int4", "moe_layer_forward_w4a16",
    "moe_layer_forward_w4a16_ws", "moe_ep_dispatch", "moe_ep_expert_ffn", "moe_ep_combine",
    "moe_ep_dispatch_workspace_size", "moe_ep_expert_ffn_workspace_size",
    "moe_ep_combine_workspace_size", "NOALLOC_SCRATCH_BYTES", "EXPORTED_SYMBOLS",
]

# Every function declared in include/moe.h.
EXPORTED_SYMBOLS = [
    "moe_status_string", "moe_last_error_string", "moe_workspace_size", "moe_route",
    "moe_permute", "moe_expert_ffn",
    "moe_combine", "moe_layer_forward", "moe_layer_forward_ws", "moe_device_status",
    "moe_set_wait_timeout_ns", "moe_set_pdl", "moe_selftest_wait_timeout", "moe_last_launch_count",
    "moe_profile_begin", "moe_profile_end", "moe_kernel_name", "moe_layer_forward_noalloc",
    "moe_quantize_fp8", "moe_layer_forward_fp8", "moe_layer_forward_fp8_ws",
    "moe_bias_update", "moe_router_scores", "moe_seq_aux_loss", "moe_seq_aux_workspace_size",
    "moe_quantize_fp8_rows", "moe_workspace_size_w8a8", "moe_layer_forward_w8a8",
    "moe_layer_forward_w8a8_ws", "moe_quantize_int4", "moe_layer_forward_w4a16",
    "moe_layer_forward_w4a16_ws", "moe_ep_dispatch_workspace_size", "moe_ep_dispatch",
    "moe_ep_expert_ffn_workspace_size", "moe_ep_expert_ffn", "moe_ep_combine_workspace_size",
    "moe_ep_combine",
]

MOE_OK = 0
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024    # MOE_NOALLOC_SCRATCH_BYTES in include/moe.h


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        detail = f": {moe_last_error_string()}" if code == -3 else ""    # MOE_ERR_CUDA
        super().__init__(f"{fn} failed: {moe_status_string(code)} ({code}){detail}")


def _load():
    path = _build.build()
    L = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    SZ, U64, I64 = ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int64
    sig = {
        "moe_status_string": ([I], ctypes.c_char_p),
        "moe_last_error_string": ([], ctypes.c_char_p),
        "moe_workspace_size": ([I, I, I, I, I], SZ),
        "moe_route": ([P, P, P, I, I, I, I, F, P, P, P, SZ, P], I),
        "moe_permute": ([P, I, I, I, P, P, P, P, P, SZ, P], I),
        "moe_expert_ffn": ([P, P, P, P, P, I, I, I, I, I, P, P, SZ, P], I),
        "moe_combine": ([P, P, P, P, I, I, I, P, P], I),
        "moe_layer_forward": ([P, P, P, P, P, P, P, I, I, I, I, I, F, P, P], I),
        "moe_layer_forward_ws": ([P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, SZ, P], I),
        "moe_device_status": ([P, ctypes.POINTER(I)], I),
        "moe_set_wait_timeout_ns": ([U64], None),
        "moe_set_pdl": ([I], None),
        "moe_selftest_wait_timeout": ([U64, P], I),
        "moe_last_launch_count": ([], I),
        "moe_profile_begin": ([I], I),
        "moe_profile_end": ([ctypes.POINTER(F), I, ctypes.POINTER(I)], I),
        "moe_kernel_name": ([I], ctypes.c_char_p),
        "moe_layer_forward_noalloc": ([P, P, P, P, P, P, P, I, I, I, I, I, F, P, P], I),
        "moe_quantize_fp8": ([P, I64, I64, P, P, P], I),
        "moe_layer_forward_fp8": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P], I),
        "moe_layer_forward_fp8_ws": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, SZ, P],
                                     I),
        "moe_bias_update": ([P, I, I, I, F, P, P], I),
        "moe_router_scores": ([P, P, I, I, I, P, P, SZ, P], I),
        "moe_seq_aux_loss": ([P, P, I, I, I, I, F, P, P, P, P, SZ, P], I),
        "moe_seq_aux_workspace_size": ([I, I, I], SZ),
        "moe_quantize_fp8_rows": ([P, I64, I64, P, P, P], I),
        "moe_quantize_int4": ([P, I64, I64, P, P, P], I),
        "moe_layer_forward_w4a16": ([P] * 9 + [I, I, I, I, I, F, P, P], I),
        "moe_layer_forward_w4a16_ws": ([P] * 9 + [I, I, I, I, I, F, P, P, SZ, P], I),
        "moe_workspace_size_w8a8": ([I, I, I, I, I], SZ),
        "moe_layer_forward_w8a8": ([P] * 11 + [I, I, I, I, I, F, P, P], I),
        "moe_layer_forward_w8a8_ws": ([P] * 11 + [I, I, I, I, I, F, P, P, SZ, P], I),
        "moe_ep_dispatch_workspace_size": ([I, I, I, I], SZ),
        "moe_ep_dispatch": ([P, P, P, I, I, I, I, F, P, P, P, P, P, P, SZ, P], I),
        "moe_ep_expert_ffn_workspace_size": ([I, I, I, I, I], SZ),
        "moe_ep_expert_ffn": ([P, P, I, I, I, I, I, P, P, P, P, SZ, P], I),
        "moe_ep_combine_workspace_size": ([I, I, I], SZ),
        "moe_ep_combine": ([P] * 6 + [I, I, I, I, P, P, SZ, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


_LIB = _load()


def lib():
    return _LIB


# ------------------------------------------------------------- marshalling

def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, dtype, name, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check(fn, rc):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


# ------------------------------------------------------------------- calls

def moe_status_string(code: int) -> str:
    return _LIB.moe_status_string(int(code)).decode()


def moe_last_error_string() -> str:
    return _LIB.moe_last_error_string().decode()


def moe_workspace_size(T: int, d: int, E: int, k: int, inter: int) -> int:
    return int(_LIB.moe_workspace_size(T, d, E, k, inter))


def moe_route(x, w_router, bias, k: int, scale: float, topk_idx, topk_w, workspace, stream=None):
    T, d = x.shape
    E = w_router.shape[0]
    rc = _LIB.moe_route(_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"),
                        _ptr(bias, F32, "bias"), T, d, E, k, float(scale),
                        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"),
                        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                        _stream(stream))
    _check("moe_route", rc)


def moe_permute(topk_idx, E: int, counts, offsets, row_token, slot_row, workspace, stream=None):
    T, k = topk_idx.shape
    rc = _LIB.moe_permute(_ptr(topk_idx, I32, "topk_idx"), T, E, k, _ptr(counts, I32, "counts"),
                          _ptr(offsets, I32, "offsets"), _ptr(row_token, I32, "row_token"),
                          _ptr(slot_row, I32, "slot_row"),
                          _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                          _stream(stream))
    _check("moe_permute", rc)


def moe_expert_ffn(x, row_token, offsets, w_gate_up, w_down, k: int, y, workspace, stream=None):
    T, d = x.shape
    E, two_i, _ = w_gate_up.shape
    rc = _LIB.moe_expert_ffn(_ptr(x, BF16, "x"), _ptr(row_token, I32, "row_token"),
                             _ptr(offsets, I32, "offsets"), _ptr(w_gate_up, BF16, "w_gate_up"),
                             _ptr(w_down, BF16, "w_down"), T, d, E, k, two_i // 2,
                             _ptr(y, BF16, "y"), _ptr(workspace, torch.uint8, "workspace"),
                             workspace.numel(), _stream(stream))
    _check("moe_expert_ffn", rc)


def moe_combine(y, y_shared, topk_w, slot_row, out, stream=None):
    T, k = topk_w.shape
    d = y.shape[1]
    rc = _LIB.moe_combine(_ptr(y, BF16, "y"), _ptr(y_shared, BF16, "y_shared", optional=True),
                          _ptr(topk_w, F32, "topk_w"), _ptr(slot_row, I32, "slot_row"), T, d, k,
                          _ptr(out, BF16, "out"), _stream(stream))
    _check("moe_combine", rc)


def _layer_args(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down):
    T, d = x.shape
    E = w_router.shape[0]
    inter = w_gate_up.shape[1] // 2
    return ([_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"), _ptr(bias, F32, "bias"),
             _ptr(w_gate_up, BF16, "w_gate_up"), _ptr(w_down, BF16, "w_down"),
             _ptr(ws_gate_up, BF16, "ws_gate_up"), _ptr(ws_down, BF16, "ws_down")],
            T, d, E, inter)


def moe_layer_forward(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, k: int,
                      scale: float, out, stream=None):
    ptrs, T, d, E, inter = _layer_args(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward(*ptrs, T, d, E, k, inter, float(scale), _ptr(out, BF16, "out"),
                                _stream(stream))
    _check("moe_layer_forward", rc)


def moe_layer_forward_ws(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, k: int,
                         scale: float, out, workspace, stream=None):
    ptrs, T, d, E, inter = _layer_args(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_ws(*ptrs, T, d, E, k, inter, float(scale),
                                   _ptr(out, BF16, "out"),
                                   _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                   _stream(stream))
    _check("moe_layer_forward_ws", rc)


def moe_layer_forward_noalloc(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, k: int,
                              scale: float, out, stream=None):
    """moe_layer_forward without any device allocation: the scratch is a fixed
    array inside the library (see include/moe.h for the size limit and the
    rule that overlapping calls race on it)."""
    ptrs, T, d, E, inter = _layer_args(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_noalloc(*ptrs, T, d, E, k, inter, float(scale),
                                        _ptr(out, BF16, "out"), _stream(stream))
    _check("moe_layer_forward_noalloc", rc)


def moe_quantize_fp8(w, stream=None):
    """bf16 weights [..., rows, cols] (rows and cols multiples of 128) ->
    (E4M3 codes uint8 [..., rows, cols], int8 block exponents
    [..., rows/128, cols/128]), new tensors on w's device."""
    if w.dim() < 2:
        raise ValueError("w must have at least 2 dimensions")
    rows, cols = w.shape[-2], w.shape[-1]
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    exps = torch.empty(tuple(w.shape[:-2]) + (rows // 128, cols // 128), dtype=torch.int8,
                       device=w.device)
    rc = _LIB.moe_quantize_fp8(_ptr(w, BF16, "w"), w.numel() // cols, cols,
                               _ptr(q, torch.uint8, "q"), _ptr(exps, torch.int8, "exps"),
                               _stream(stream))
    _check("moe_quantize_fp8", rc)
    return q, exps


def _layer_fp8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                    ws_gate_up, ws_down):
    T, d = x.shape
    E = w_router.shape[0]
    inter = wq_gate_up.shape[1] // 2
    return ([_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"), _ptr(bias, F32, "bias"),
             _ptr(wq_gate_up, torch.uint8, "wq_gate_up"),
             _ptr(wq_gate_up_exp, torch.int8, "wq_gate_up_exp"),
             _ptr(wq_down, torch.uint8, "wq_down"), _ptr(wq_down_exp, torch.int8, "wq_down_exp"),
             _ptr(ws_gate_up, BF16, "ws_gate_up"), _ptr(ws_down, BF16, "ws_down")],
            T, d, E, inter)


def moe_layer_forward_fp8(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                          ws_gate_up, ws_down, k: int, scale: float, out, stream=None):
    """moe_layer_forward with the routed experts' weights as FP8 codes + block
    exponents (from moe_quantize_fp8); router and shared expert stay bf16."""
    ptrs, T, d, E, inter = _layer_fp8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp,
                                           wq_down, wq_down_exp, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_fp8(*ptrs, T, d, E, k, inter, float(scale),
                                    _ptr(out, BF16, "out"), _stream(stream))
    _check("moe_layer_forward_fp8", rc)


def moe_layer_forward_fp8_ws(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                             ws_gate_up, ws_down, k: int, scale: float, out, workspace,
                             stream=None):
    ptrs, T, d, E, inter = _layer_fp8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp,
                                           wq_down, wq_down_exp, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_fp8_ws(*ptrs, T, d, E, k, inter, float(scale),
                                       _ptr(out, BF16, "out"),
                                       _ptr(workspace, torch.uint8, "workspace"),
                                       workspace.numel(), _stream(stream))
    _check("moe_layer_forward_fp8_ws", rc)


def moe_quantize_int4(w, stream=None):
    """bf16 weights [..., rows, cols] (cols a multiple of 64) -> (packed INT4
    codes uint8 [..., rows, cols/2], group scales bf16 [cols/32, prod(...) *
    rows], group-major), new tensors on w's device."""
    if w.dim() < 2:
        raise ValueError("w must have at least 2 dimensions")
    cols = w.shape[-1]
    rows = w.numel() // cols
    codes = torch.empty(tuple(w.shape[:-1]) + (cols // 2,), dtype=torch.uint8, device=w.device)
    scales = torch.empty((cols // 32, rows), dtype=BF16, device=w.device)
    rc = _LIB.moe_quantize_int4(_ptr(w, BF16, "w"), rows, cols, _ptr(codes, torch.uint8, "codes"),
                                _ptr(scales, BF16, "scales"), _stream(stream))
    _check("moe_quantize_int4", rc)
    return codes, scales


def _layer_w4_args(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down, wq_down_scale,
                   ws_gate_up, ws_down):
    T, d = x.shape
    E = w_router.shape[0]
    inter = wq_gate_up.shape[1] // 2
    return ([_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"), _ptr(bias, F32, "bias"),
             _ptr(wq_gate_up, torch.uint8, "wq_gate_up"),
             _ptr(wq_gate_up_scale, BF16, "wq_gate_up_scale"),
             _ptr(wq_down, torch.uint8, "wq_down"), _ptr(wq_down_scale, BF16, "wq_down_scale"),
             _ptr(ws_gate_up, BF16, "ws_gate_up"), _ptr(ws_down, BF16, "ws_down")],
            T, d, E, inter)


def moe_layer_forward_w4a16(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down,
                            wq_down_scale, ws_gate_up, ws_down, k: int, scale: float, out,
                            stream=None):
    """moe_layer_forward with the routed experts' weights as INT4 codes + group
    scales (from moe_quantize_int4); router and shared expert stay bf16."""
    ptrs, T, d, E, inter = _layer_w4_args(x, w_router, bias, wq_gate_up, wq_gate_up_scale,
                                          wq_down, wq_down_scale, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_w4a16(*ptrs, T, d, E, k, inter, float(scale),
                                      _ptr(out, BF16, "out"), _stream(stream))
    _check("moe_layer_forward_w4a16", rc)


def moe_layer_forward_w4a16_ws(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down,
                               wq_down_scale, ws_gate_up, ws_down, k: int, scale: float, out,
                               workspace, stream=None):
    ptrs, T, d, E, inter = _layer_w4_args(x, w_router, bias, wq_gate_up, wq_gate_up_scale,
                                          wq_down, wq_down_scale, ws_gate_up, ws_down)
    rc = _LIB.moe_layer_forward_w4a16_ws(*ptrs, T, d, E, k, inter, float(scale),
                                         _ptr(out, BF16, "out"),
                                         _ptr(workspace, torch.uint8, "workspace"),
                                         workspace.numel(), _stream(stream))
    _check("moe_layer_forward_w4a16_ws", rc)


def moe_quantize_fp8_rows(w, stream=None):
    """bf16 weights [..., cols] (cols a multiple of 16) -> (E4M3 codes uint8
    [..., cols], one int8 exponent per row [...]), new tensors on w's device."""
    if w.dim() < 2:
        raise ValueError("w must have at least 2 dimensions")
    cols = w.shape[-1]
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    exps = torch.empty(tuple(w.shape[:-1]), dtype=torch.int8, device=w.device)
    rc = _LIB.moe_quantize_fp8_rows(_ptr(w, BF16, "w"), w.numel() // cols, cols,
                                    _ptr(q, torch.uint8, "q"), _ptr(exps, torch.int8, "exps"),
                                    _stream(stream))
    _check("moe_quantize_fp8_rows", rc)
    return q, exps


def moe_workspace_size_w8a8(T: int, d: int, E: int, k: int, inter: int) -> int:
    return int(_LIB.moe_workspace_size_w8a8(T, d, E, k, inter))


def _layer_w8a8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                     wsq_gate_up, wsq_gate_up_exp, wsq_down, wsq_down_exp):
    T, d = x.shape
    E = w_router.shape[0]
    inter = wq_gate_up.shape[1] // 2
    u8, i8 = torch.uint8, torch.int8
    return ([_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"), _ptr(bias, F32, "bias"),
             _ptr(wq_gate_up, u8, "wq_gate_up"), _ptr(wq_gate_up_exp, i8, "wq_gate_up_exp"),
             _ptr(wq_down, u8, "wq_down"), _ptr(wq_down_exp, i8, "wq_down_exp"),
             _ptr(wsq_gate_up, u8, "wsq_gate_up"), _ptr(wsq_gate_up_exp, i8, "wsq_gate_up_exp"),
             _ptr(wsq_down, u8, "wsq_down"), _ptr(wsq_down_exp, i8, "wsq_down_exp")],
            T, d, E, inter)


def moe_layer_forward_w8a8(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                           wsq_gate_up, wsq_gate_up_exp, wsq_down, wsq_down_exp, k: int,
                           scale: float, out, stream=None):
    """The layer with FP8 compute in every expert: codes + per-row exponents
    from moe_quantize_fp8_rows (routed [E, ...] and shared); router stays bf16."""
    ptrs, T, d, E, inter = _layer_w8a8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp,
                                            wq_down, wq_down_exp, wsq_gate_up, wsq_gate_up_exp,
                                            wsq_down, wsq_down_exp)
    rc = _LIB.moe_layer_forward_w8a8(*ptrs, T, d, E, k, inter, float(scale),
                                     _ptr(out, BF16, "out"), _stream(stream))
    _check("moe_layer_forward_w8a8", rc)


def moe_layer_forward_w8a8_ws(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down,
                              wq_down_exp, wsq_gate_up, wsq_gate_up_exp, wsq_down, wsq_down_exp,
                              k: int, scale: float, out, workspace, stream=None):
    ptrs, T, d, E, inter = _layer_w8a8_args(x, w_router, bias, wq_gate_up, wq_gate_up_exp,
                                            wq_down, wq_down_exp, wsq_gate_up, wsq_gate_up_exp,
                                            wsq_down, wsq_down_exp)
    rc = _LIB.moe_layer_forward_w8a8_ws(*ptrs, T, d, E, k, inter, float(scale),
                                        _ptr(out, BF16, "out"),
                                        _ptr(workspace, torch.uint8, "workspace"),
                                        workspace.numel(), _stream(stream))
    _check("moe_layer_forward_w8a8_ws", rc)


def moe_bias_update(counts, T: int, k: int, gamma: float, bias, stream=None):
    """One loss-free balancing step on `bias` (fp32 [E], in place) from the
    step's per-expert row counts (int32 [E])."""
    E = counts.numel()
    rc = _LIB.moe_bias_update(_ptr(counts, I32, "counts"), int(T), E, int(k), float(gamma),
                              _ptr(bias, F32, "bias"), _stream(stream))
    _check("moe_bias_update", rc)


def moe_router_scores(x, w_router, scores, workspace, stream=None):
    """Unbiased sigmoid router scores of every expert into scores [T, E] fp32."""
    T, d = x.shape
    E = w_router.shape[0]
    rc = _LIB.moe_router_scores(_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"), T, d, E,
                                _ptr(scores, F32, "scores"),
                                _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                _stream(stream))
    _check("moe_router_scores", rc)


def moe_seq_aux_workspace_size(B: int, S: int, E: int) -> int:
    return int(_LIB.moe_seq_aux_workspace_size(int(B), int(S), int(E)))


def moe_seq_aux_loss(scores, topk_idx, S: int, alpha: float, loss, f=None, p=None,
                     workspace=None, stream=None):
    """Sequence-level balance loss of the B = T / S sequences into loss [B]
    (and f, p [B, E] if given); workspace: moe_seq_aux_workspace_size bytes
    (allocated here if not given)."""
    T, E = scores.shape
    k = topk_idx.shape[1]
    B = T // S
    if workspace is None:
        workspace = torch.empty(max(moe_seq_aux_workspace_size(B, S, E), 16), dtype=torch.uint8,
                                device=scores.device)
    rc = _LIB.moe_seq_aux_loss(_ptr(scores, F32, "scores"), _ptr(topk_idx, I32, "topk_idx"),
                               B, int(S), E, k, float(alpha), _ptr(loss, F32, "loss"),
                               _ptr(f, F32, "f", optional=True), _ptr(p, F32, "p", optional=True),
                               _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                               _stream(stream))
    _check("moe_seq_aux_loss", rc)


def moe_device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    _check("moe_device_status", _LIB.moe_device_status(_stream(stream), ctypes.byref(v)))
    return v.value


def moe_set_wait_timeout_ns(ns: int) -> None:
    _LIB.moe_set_wait_timeout_ns(int(ns))


def moe_set_pdl(enable: bool) -> None:
    """Programmatic dependent launch of the library's kernels on / off (default off)."""
    _LIB.moe_set_pdl(1 if enable else 0)


def moe_selftest_wait_timeout(ns: int, stream=None) -> None:
    _check("moe_selftest_wait_timeout", _LIB.moe_selftest_wait_timeout(int(ns), _stream(stream)))


def moe_last_launch_count() -> int:
    return int(_LIB.moe_last_launch_count())


def moe_profile_begin(max_calls: int) -> None:
    _check("moe_profile_begin", _LIB.moe_profile_begin(int(max_calls)))


def moe_profile_end():
    """-> (n_calls, {kernel name: summed ms over the recorded calls})."""
    buf = (ctypes.c_float * 32)()
    n = ctypes.c_int(0)
    nk = _LIB.moe_profile_end(buf, 32, ctypes.byref(n))
    if nk < 0:
        raise MoeError("moe_profile_end", nk)
    return n.value, {moe_kernel_name(i): float(buf[i]) for i in range(nk)}


def moe_kernel_name(i: int) -> str:
    return _LIB.moe_kernel_name(int(i)).decode()


# ------------------------------------------------------ expert parallelism

def moe_ep_dispatch_workspace_size(T: int, d: int, E: int, k: int) -> int:
    return int(_LIB.moe_ep_dispatch_workspace_size(T, d, E, k))


def moe_ep_dispatch(x, w_router, bias, k: int, scale: float, topk_idx, topk_w, counts, slot_row,
                    send_rows, workspace, stream=None):
    T, d = x.shape
    E = w_router.shape[0]
    rc = _LIB.moe_ep_dispatch(_ptr(x, BF16, "x"), _ptr(w_router, BF16, "w_router"),
                              _ptr(bias, F32, "bias"), T, d, E, k, float(scale),
                              _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"),
                              _ptr(counts, I32, "counts"), _ptr(slot_row, I32, "slot_row"),
                              _ptr(send_rows, BF16, "send_rows"),
                              _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                              _stream(stream))
    _check("moe_ep_dispatch", rc)


def moe_ep_expert_ffn_workspace_size(rows: int, d: int, R: int, E_local: int, inter: int) -> int:
    return int(_LIB.moe_ep_expert_ffn_workspace_size(rows, d, R, E_local, inter))


def moe_ep_expert_ffn(recv_rows, recv_counts, w_gate_up, w_down, y, workspace, stream=None):
    rows, d = recv_rows.shape
    R, E_local = recv_counts.shape
    inter = w_gate_up.shape[1] // 2
    rc = _LIB.moe_ep_expert_ffn(_ptr(recv_rows, BF16, "recv_rows"),
                                _ptr(recv_counts, I32, "recv_counts"), rows, d, R, E_local, inter,
                                _ptr(w_gate_up, BF16, "w_gate_up"), _ptr(w_down, BF16, "w_down"),
                                _ptr(y, BF16, "y"), _ptr(workspace, torch.uint8, "workspace"),
                                workspace.numel(), _stream(stream))
    _check("moe_ep_expert_ffn", rc)


def moe_ep_combine_workspace_size(T: int, d: int, inter: int) -> int:
    return int(_LIB.moe_ep_combine_workspace_size(T, d, inter))


def moe_ep_combine(y_back, x, ws_gate_up, ws_down, topk_w, slot_row, out, workspace,
                   stream=None):
    T, d = x.shape
    k = topk_w.shape[1]
    inter = ws_gate_up.shape[0] // 2
    rc = _LIB.moe_ep_combine(_ptr(y_back, BF16, "y_back"), _ptr(x, BF16, "x"),
                             _ptr(ws_gate_up, BF16, "ws_gate_up"), _ptr(ws_down, BF16, "ws_down"),
                             _ptr(topk_w, F32, "topk_w"), _ptr(slot_row, I32, "slot_row"), T, d, k,
                             inter, _ptr(out, BF16, "out"),
                             _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                             _stream(stream))
    _check("moe_ep_combine", rc)
