"""Python wrapper of the fp64 CPU oracle (ctypes over liboracle.so).

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__.py
and bench.py's CPU-baseline / reference leg import this package; the product
(the CUDA library and its binding) never does, and this package never imports
the product.  Inputs come from numpy arrays: bf16 tensors as uint16 bit
patterns, everything else as int32 / float32 / float64.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None
_override = None


class use_library:
    """Context manager: route every call of this wrapper to another build of
    the oracle (the pin tests use it to run mutated copies)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _override
        self._saved = _override
        _override = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _override
        _override = self._saved
        return False


def lib():
    global _lib
    if _override is not None:
        return _override
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(L):
    P = ctypes.c_void_p
    i32, f64 = ctypes.c_int, ctypes.c_double
    L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_f64.restype = f64
    L.oracle_f64_to_bf16.argtypes = [f64]
    L.oracle_f64_to_bf16.restype = ctypes.c_uint16
    L.oracle_round_bf16.argtypes = [P, P, ctypes.c_size_t]
    L.oracle_round_bf16.restype = None
    L.oracle_sigmoid.argtypes = [f64]
    L.oracle_sigmoid.restype = f64
    L.oracle_silu.argtypes = [f64]
    L.oracle_silu.restype = f64
    L.oracle_route.argtypes = [P, P, P, i32, i32, i32, i32, f64, P, P, P, P, i32]
    L.oracle_route.restype = i32
    L.oracle_permute.argtypes = [P, i32, i32, i32, P, P, P, P]
    L.oracle_permute.restype = i32
    L.oracle_swiglu_row.argtypes = [P, P, P, i32, i32, P, P]
    L.oracle_swiglu_row.restype = None
    L.oracle_combine.argtypes = [P, P, P, P, i32, i32, i32, P]
    L.oracle_combine.restype = None
    L.oracle_moe_rows.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i32, P,
                                  i32]
    L.oracle_moe_rows.restype = i32
    i64 = ctypes.c_int64
    L.oracle_e4m3_encode.argtypes = [f64]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = f64
    L.oracle_fp8_block_exponent.argtypes = [f64]
    L.oracle_fp8_block_exponent.restype = i32
    L.oracle_quantize_fp8.argtypes = [P, i64, i64, P, P]
    L.oracle_quantize_fp8.restype = i32
    L.oracle_dequantize_fp8.argtypes = [P, P, i64, i64, P]
    L.oracle_dequantize_fp8.restype = i32
    L.oracle_quantize_int4.argtypes = [P, i64, i64, P, P]
    L.oracle_quantize_int4.restype = i32
    L.oracle_dequantize_int4.argtypes = [P, P, i64, i64, P]
    L.oracle_dequantize_int4.restype = i32
    L.oracle_quantize_fp8_rows.argtypes = [P, i64, i64, P, P]
    L.oracle_quantize_fp8_rows.restype = None
    L.oracle_swiglu_row_fp8.argtypes = [P, P, P, P, P, i32, i32, P]
    L.oracle_swiglu_row_fp8.restype = None
    L.oracle_moe_rows_fp8.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P,
                                      P, i32, P, i32]
    L.oracle_moe_rows_fp8.restype = i32
    L.oracle_bias_update.argtypes = [P, i32, i32, i32, ctypes.c_float, P]
    L.oracle_bias_update.restype = None
    L.oracle_seq_aux_loss.argtypes = [P, P, i32, i32, i32, i32, f64, P, P, P]
    L.oracle_seq_aux_loss.restype = None
    return L


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    """bf16 data as a C-contiguous uint16 numpy array (accepts torch or numpy)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy()
                                    .view(np.uint16))
    arr = np.ascontiguousarray(a)
    assert arr.dtype == np.uint16, arr.dtype
    return arr


def _np(a, dtype):
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def bf16_to_f64(a) -> np.ndarray:
    u = _u16(a)
    with np.errstate(invalid="ignore"):
        return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_ptr(a), _ptr(out), a.size)
    return out


def e4m3_encode(v: float) -> int:
    """E4M3 code of v (nearest, ties to even; saturating)."""
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code) & 0xFF)


def fp8_block_exponent(amax: float) -> int:
    return int(lib().oracle_fp8_block_exponent(float(amax)))


def quantize_fp8(w):
    """bf16 matrix [rows, cols] (rows, cols multiples of 128) -> (codes uint8
    [rows, cols], block exponents int8 [rows/128, cols/128])."""
    u = _u16(w)
    cols = u.shape[-1]
    rows = u.size // cols
    q = np.empty(u.shape, dtype=np.uint8)
    sexp = np.empty(u.shape[:-2] + (u.shape[-2] // 128, cols // 128), dtype=np.int8)
    rc = lib().oracle_quantize_fp8(_ptr(u), rows, cols, _ptr(q), _ptr(sexp))
    if rc != 0:
        raise ValueError("oracle_quantize_fp8: rows and cols must be multiples of 128")
    return q, sexp


def dequantize_fp8(q, sexp):
    """codes [.., rows, cols] + block exponents -> the exact bf16 weights (uint16)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sexp = np.ascontiguousarray(sexp, dtype=np.int8)
    cols = q.shape[-1]
    rows = q.size // cols
    out = np.empty(q.shape, dtype=np.uint16)
    rc = lib().oracle_dequantize_fp8(_ptr(q), _ptr(sexp), rows, cols, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequantize_fp8: rows and cols must be multiples of 128")
    return out


def quantize_int4(w):
    """bf16 matrix [.., rows, cols] (cols a multiple of 32) -> (codes int8 in
    [-8, 7], same shape; group scales as bf16 bits uint16 [.., rows, cols/32])."""
    u = _u16(w)
    cols = u.shape[-1]
    rows = u.size // cols
    q = np.empty(u.shape, dtype=np.int8)
    sc = np.empty(u.shape[:-1] + (cols // 32,), dtype=np.uint16)
    if lib().oracle_quantize_int4(_ptr(u), rows, cols, _ptr(q), _ptr(sc)) != 0:
        raise ValueError("oracle_quantize_int4: cols must be a multiple of 32")
    return q, sc


def dequantize_int4(q, scale):
    """codes + group scales -> the bf16 weights the model computes with (uint16)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    sc = np.ascontiguousarray(scale, dtype=np.uint16)
    cols = q.shape[-1]
    rows = q.size // cols
    out = np.empty(q.shape, dtype=np.uint16)
    if lib().oracle_dequantize_int4(_ptr(q), _ptr(sc), rows, cols, _ptr(out)) != 0:
        raise ValueError("oracle_dequantize_int4: cols must be a multiple of 32")
    return out


def quantize_fp8_rows(w):
    """bf16 matrix [.., rows, cols] -> (codes uint8 [.., rows, cols], one
    exponent per row int8 [.., rows]): the FP8-compute format."""
    u = _u16(w)
    cols = u.shape[-1]
    rows = u.size // cols
    q = np.empty(u.shape, dtype=np.uint8)
    sexp = np.empty(u.shape[:-1], dtype=np.int8)
    lib().oracle_quantize_fp8_rows(_ptr(u), rows, cols, _ptr(q), _ptr(sexp))
    return q, sexp


def swiglu_row_fp8(xrow, q_gate_up, s_gate_up, q_down, s_down):
    """One expert on one token in FP8 compute (see the C header) -> y f64 [d]."""
    xu = _u16(xrow)
    qg, sg = _np(q_gate_up, np.uint8), _np(s_gate_up, np.int8)
    qd, sd = _np(q_down, np.uint8), _np(s_down, np.int8)
    d = xu.shape[-1]
    inter = qg.shape[0] // 2
    y = np.empty((d,), np.float64)
    lib().oracle_swiglu_row_fp8(_ptr(xu), _ptr(qg), _ptr(sg), _ptr(qd), _ptr(sd), d, inter,
                                _ptr(y))
    return y


def moe_rows_fp8(x, topk_idx, topk_w, expert_q, shared_q, tokens=None,
                 nthreads: int | None = None):
    """Steps 5-7 in FP8 compute on the listed tokens.

    expert_q: sequence indexed by expert of (q_gate_up, s_gate_up, q_down,
    s_down) from quantize_fp8_rows, or None for experts no listed token
    selects; shared_q: the same tuple for the shared expert."""
    xu = _u16(x)
    T, d = xu.shape
    idx = _np(topk_idx, np.int32)
    w = _np(topk_w, np.float64)
    k = idx.shape[1]
    E = len(expert_q)
    keep = []
    ptrs = [(ctypes.c_void_p * E)() for _ in range(4)]
    for e in range(E):
        if expert_q[e] is None:
            continue
        arrs = [_np(expert_q[e][0], np.uint8), _np(expert_q[e][1], np.int8),
                _np(expert_q[e][2], np.uint8), _np(expert_q[e][3], np.int8)]
        keep += arrs
        for j in range(4):
            ptrs[j][e] = arrs[j].ctypes.data
    sq = [_np(shared_q[0], np.uint8), _np(shared_q[1], np.int8),
          _np(shared_q[2], np.uint8), _np(shared_q[3], np.int8)]
    inter = sq[0].shape[0] // 2
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok is None else tok.shape[0]
    out = np.empty((n, d), np.float64)
    rc = lib().oracle_moe_rows_fp8(_ptr(xu), T, d, E, k, inter, _ptr(idx), _ptr(w),
                                   *[ctypes.cast(p, ctypes.c_void_p) for p in ptrs],
                                   *[_ptr(a) for a in sq], _ptr(tok), n, _ptr(out),
                                   nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_moe_rows_fp8: a selected expert's weights are missing")
    del keep
    return out


def quantize_expert_rows(inputs: dict, experts):
    """The FP8-compute weights of the listed experts and of the shared expert,
    from the oracle's own row quantizer: ({e: (qgu, sgu, qdn, sdn)}, shared)."""
    from concurrent.futures import ThreadPoolExecutor

    def one(e):
        return quantize_fp8_rows(inputs["w_gate_up"][e]) + quantize_fp8_rows(inputs["w_down"][e])

    # the C quantizer runs outside the GIL: one expert per host thread
    with ThreadPoolExecutor(max_workers=max(1, min(default_threads(), len(experts)))) as ex:
        out = dict(zip(experts, ex.map(one, experts)))
    qg, sg = quantize_fp8_rows(inputs["ws_gate_up"])
    qd, sd = quantize_fp8_rows(inputs["ws_down"])
    return out, (qg, sg, qd, sd)


def moe_forward_fp8(inputs: dict, k: int, scale: float, tokens=None,
                    nthreads: int | None = None):
    """Whole layer with FP8 compute in every expert (routing stays bf16 /
    fp64): route all tokens, quantize the selected experts' weights per row
    with the oracle's quantizer, evaluate the listed rows.
    Returns (out f64 [n,d], topk_idx, topk_w, gap)."""
    idx, w, gap = route(inputs["x"], inputs["w_router"], inputs["bias"], k, scale, nthreads)
    E = inputs["w_router"].shape[0]
    need = sorted(set(np.unique(idx if tokens is None else idx[np.asarray(tokens)]).tolist()))
    qe, qs = quantize_expert_rows(inputs, need)
    expert_q = [qe.get(e) for e in range(E)]
    out = moe_rows_fp8(inputs["x"], idx, w, expert_q, qs, tokens=tokens, nthreads=nthreads)
    return out, idx, w, gap


def bias_update(counts, T: int, k: int, gamma: float, bias):
    """New fp32 bias after one loss-free balancing step (see the C header)."""
    c = _np(counts, np.int32)
    b = np.array(_np(bias, np.float32), copy=True)
    lib().oracle_bias_update(_ptr(c), int(T), c.size, int(k), float(gamma), _ptr(b))
    return b


def seq_aux_loss(scores, topk_idx, S: int, alpha: float):
    """Sequence-level balance loss per sequence of S tokens -> (loss [B], f [B,E], p [B,E])."""
    sc = _np(scores, np.float64)
    idx = _np(topk_idx, np.int32)
    T, E = sc.shape
    k = idx.shape[1]
    B = T // S
    loss = np.empty(B)
    f = np.empty((B, E))
    p = np.empty((B, E))
    lib().oracle_seq_aux_loss(_ptr(sc), _ptr(idx), B, int(S), E, k, float(alpha), _ptr(loss),
                              _ptr(f), _ptr(p))
    return loss, f, p


def sigmoid(z: float) -> float:
    return lib().oracle_sigmoid(float(z))


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def route(x, w_router, bias, k: int, scale: float, nthreads: int | None = None,
          want_scores: bool = False):
    """Steps 1-4: returns (topk_idx int32 [T,k], topk_w f64 [T,k], gap f64 [T][, scores])."""
    xu, wu = _u16(x), _u16(w_router)
    b = _np(bias, np.float32)
    T, d = xu.shape
    E = wu.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty((T,), np.float64)
    scores = np.empty((T, E), np.float64) if want_scores else None
    rc = lib().oracle_route(_ptr(xu), _ptr(wu), _ptr(b), T, d, E, k, float(scale),
                            _ptr(idx), _ptr(w), _ptr(scores), _ptr(gap),
                            nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_route: invalid arguments")
    return (idx, w, gap, scores) if want_scores else (idx, w, gap)


def permute(topk_idx, E: int):
    """Expert-contiguous permutation: (counts, offsets, row_token, slot_row)."""
    idx = _np(topk_idx, np.int32)
    T, k = idx.shape
    counts = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    row_token = np.empty((T * k,), np.int32)
    slot_row = np.empty((T * k,), np.int32)
    rc = lib().oracle_permute(_ptr(idx), T, E, k, _ptr(counts), _ptr(offsets),
                              _ptr(row_token), _ptr(slot_row))
    if rc != 0:
        raise ValueError("oracle_permute: invalid routing indices")
    return counts, offsets, row_token, slot_row


def swiglu_row(xrow, w_gate_up, w_down, want_act: bool = False):
    xu, gu, dn = _u16(xrow), _u16(w_gate_up), _u16(w_down)
    d = xu.shape[-1]
    inter = gu.shape[0] // 2
    y = np.empty((d,), np.float64)
    act = np.empty((inter,), np.float64)
    lib().oracle_swiglu_row(_ptr(xu), _ptr(gu), _ptr(dn), d, inter, _ptr(y), _ptr(act))
    return (y, act) if want_act else y


def combine(y, y_shared, topk_w, slot_row):
    y = _np(y, np.float64)
    ys = None if y_shared is None else _np(y_shared, np.float64)
    w = _np(topk_w, np.float64)
    sr = _np(slot_row, np.int32)
    T, k = w.shape
    d = y.shape[1]
    out = np.empty((T, d), np.float64)
    lib().oracle_combine(_ptr(y), _ptr(ys), _ptr(w), _ptr(sr), T, d, k, _ptr(out))
    return out


def moe_rows(x, topk_idx, topk_w, expert_gate_up, expert_down, shared_gate_up, shared_down,
             tokens=None, nthreads: int | None = None):
    """Steps 5-7 on the listed tokens (all tokens if None).

    expert_gate_up / expert_down: sequences indexed by expert (uint16 arrays or
    bf16 tensors, or None for experts no listed token selects)."""
    xu = _u16(x)
    T, d = xu.shape
    idx = _np(topk_idx, np.int32)
    w = _np(topk_w, np.float64)
    k = idx.shape[1]
    E = len(expert_gate_up)
    keep = []
    gu_ptrs = (ctypes.c_void_p * E)()
    dn_ptrs = (ctypes.c_void_p * E)()
    inter = None
    for e in range(E):
        if expert_gate_up[e] is None:
            continue
        g, dn = _u16(expert_gate_up[e]), _u16(expert_down[e])
        keep += [g, dn]
        inter = g.shape[0] // 2
        gu_ptrs[e] = g.ctypes.data
        dn_ptrs[e] = dn.ctypes.data
    sgu, sdn = _u16(shared_gate_up), _u16(shared_down)
    inter = sgu.shape[0] // 2
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok is None else tok.shape[0]
    out = np.empty((n, d), np.float64)
    rc = lib().oracle_moe_rows(_ptr(xu), T, d, E, k, inter, _ptr(idx), _ptr(w),
                               ctypes.cast(gu_ptrs, ctypes.c_void_p),
                               ctypes.cast(dn_ptrs, ctypes.c_void_p),
                               _ptr(sgu), _ptr(sdn), _ptr(tok), n, _ptr(out),
                               nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_moe_rows: a selected expert's weights are missing")
    del keep
    return out


def moe_forward(inputs: dict, k: int, scale: float, tokens=None, nthreads: int | None = None):
    """Whole layer: route all tokens, then evaluate the listed rows.

    inputs: dict from moe_inputs.make_inputs (CPU tensors).  Returns
    (out f64 [n,d], topk_idx, topk_w, gap)."""
    idx, w, gap = route(inputs["x"], inputs["w_router"], inputs["bias"], k, scale, nthreads)
    E = inputs["w_router"].shape[0]
    gu = inputs["w_gate_up"]
    dn = inputs["w_down"]
    need = set(np.unique(idx if tokens is None else idx[np.asarray(tokens)]).tolist())
    egu = [gu[e] if e in need else None for e in range(E)]
    edn = [dn[e] if e in need else None for e in range(E)]
    out = moe_rows(inputs["x"], idx, w, egu, edn, inputs["ws_gate_up"], inputs["ws_down"],
                   tokens=tokens, nthreads=nthreads)
    return out, idx, w, gap
