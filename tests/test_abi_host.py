"""C-ABI host logic without a GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import sparse_moe_ffn_sigmoid_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

OK, INVALID, SHAPE = 0, -1, -2
FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: checks fail first
NULL = None


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(moe.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    assert moe.moe_status_string(0) == "MOE_OK"
    assert moe.moe_status_string(-1) == "MOE_ERR_INVALID_ARG"
    assert moe.moe_status_string(-2) == "MOE_ERR_UNSUPPORTED_SHAPE"
    assert moe.moe_status_string(-4) == "MOE_ERR_TIMEOUT"
    assert moe.moe_status_string(-5) == "MOE_ERR_NO_MEMORY"


def _layer(T=64, d=7168, E=384, k=8, inter=2048, scale=2.827, ptrs=None, out=FAKE):
    p = ptrs if ptrs is not None else [FAKE] * 7
    return moe.lib().moe_layer_forward(*p, T, d, E, k, inter, ctypes.c_float(scale), out, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(d=7100), SHAPE), (dict(d=0), SHAPE), (dict(inter=2000), SHAPE), (dict(inter=32), SHAPE),
    (dict(E=0), SHAPE), (dict(E=1025), SHAPE), (dict(k=0), SHAPE), (dict(k=33, E=64), SHAPE),
    (dict(k=9, E=8), SHAPE), (dict(T=-1), INVALID), (dict(T=2**30, k=8), SHAPE),
    (dict(scale=float("nan")), INVALID),
])
def test_layer_rejects_bad_shapes(kw, code):
    assert _layer(**kw) == code


def test_layer_rejects_null_and_misaligned_pointers():
    for i in range(7):
        p = [FAKE] * 7
        p[i] = NULL
        assert _layer(ptrs=p) == INVALID
        p[i] = ctypes.c_void_p(0x10002)
        assert _layer(ptrs=p) == INVALID
    assert _layer(out=NULL) == INVALID


def test_zero_tokens_is_a_noop():
    # nothing is validated against memory and nothing launches for T == 0
    assert _layer(T=0) == OK
    L = moe.lib()
    assert L.moe_route(FAKE, FAKE, FAKE, 0, 512, 32, 4, ctypes.c_float(1.0), FAKE, FAKE, FAKE, 0,
                       NULL) == OK
    assert L.moe_permute(FAKE, 0, 32, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 0, NULL) == OK
    assert L.moe_combine(FAKE, NULL, FAKE, FAKE, 0, 512, 4, FAKE, NULL) == OK


def test_staged_calls_check_workspace_size():
    L = moe.lib()
    need = moe.moe_workspace_size(64, 512, 32, 4, 128)
    assert need > 0
    assert L.moe_route(FAKE, FAKE, FAKE, 64, 512, 32, 4, ctypes.c_float(1.0), FAKE, FAKE, FAKE, 16,
                       NULL) == INVALID
    assert L.moe_permute(FAKE, 64, 32, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 4, NULL) == INVALID
    assert L.moe_expert_ffn(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 512, 32, 4, 128, FAKE, FAKE, need - 1,
                            NULL) == INVALID
    assert L.moe_layer_forward_ws(*([FAKE] * 7), 64, 512, 32, 4, 128, ctypes.c_float(2.827), FAKE,
                                  FAKE, need - 1, NULL) == INVALID


def test_workspace_size_grows_with_the_layer():
    assert moe.moe_workspace_size(64, 512, 32, 4, 128) < moe.moe_workspace_size(128, 512, 32, 4, 128)
    assert moe.moe_workspace_size(64, 512, 0, 4, 128) == 0       # invalid shape -> 0
    dec = moe.moe_workspace_size(64, 7168, 384, 8, 2048)
    pre = moe.moe_workspace_size(8192, 7168, 384, 8, 2048)
    # prefill scratch: permuted x, h and y dominate (T*k*d + T*(k+1)*(inter+d) bf16)
    assert pre > 8192 * 8 * 7168 * 2 + 8192 * 9 * (2048 + 7168) * 2
    assert dec < 64 * 1024 * 1024


def test_combine_rejects_bad_shapes():
    L = moe.lib()
    assert L.moe_combine(FAKE, NULL, FAKE, FAKE, 4, 12, 4, FAKE, NULL) == SHAPE
    assert L.moe_combine(FAKE, NULL, FAKE, FAKE, 4, 512, 33, FAKE, NULL) == SHAPE
    assert L.moe_combine(NULL, NULL, FAKE, FAKE, 4, 512, 4, FAKE, NULL) == INVALID


# ------------------------------------------------------------ FP8 weights

def _layer_fp8(T=64, d=7168, E=384, k=8, inter=2048, scale=2.827, ptrs=None, out=FAKE, ws=None):
    p = ptrs if ptrs is not None else [FAKE] * 9
    L = moe.lib()
    if ws is None:
        return L.moe_layer_forward_fp8(*p, T, d, E, k, inter, ctypes.c_float(scale), out, NULL)
    return L.moe_layer_forward_fp8_ws(*p, T, d, E, k, inter, ctypes.c_float(scale), out, FAKE, ws,
                                      NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(d=7104), SHAPE), (dict(inter=2112), SHAPE), (dict(d=7100), SHAPE), (dict(E=0), SHAPE),
    (dict(k=9, E=8), SHAPE), (dict(T=-1), INVALID), (dict(scale=float("nan")), INVALID),
])
def test_fp8_layer_rejects_bad_shapes(kw, code):
    # FP8 blocks are 128 x 128: d and inter must be multiples of 128, not just 64
    assert _layer_fp8(**kw) == code


def test_fp8_layer_rejects_null_pointers_and_small_workspace():
    for i in range(9):
        p = [FAKE] * 9
        p[i] = NULL
        assert _layer_fp8(ptrs=p) == INVALID
    assert _layer_fp8(out=NULL) == INVALID
    need = moe.moe_workspace_size(64, 7168, 384, 8, 2048)
    assert _layer_fp8(ws=need - 1) == INVALID
    assert _layer_fp8(T=0) == OK


def test_quantize_fp8_rejects_bad_shapes():
    L = moe.lib()
    assert L.moe_quantize_fp8(FAKE, 100, 128, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_fp8(FAKE, 128, 100, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_fp8(FAKE, 128, 128 * 65536, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_fp8(FAKE, 0, 128, FAKE, FAKE, NULL) == OK
    assert L.moe_quantize_fp8(NULL, 128, 128, FAKE, FAKE, NULL) == INVALID
    assert L.moe_quantize_fp8(FAKE, 128, 128, FAKE, NULL, NULL) == INVALID


# ------------------------------------------------------------ INT4 weights

def _layer_w4(T=64, d=7168, E=384, k=8, inter=2048, scale=2.827, ptrs=None, out=FAKE, ws=None):
    p = ptrs if ptrs is not None else [FAKE] * 9
    L = moe.lib()
    if ws is None:
        return L.moe_layer_forward_w4a16(*p, T, d, E, k, inter, ctypes.c_float(scale), out, NULL)
    return L.moe_layer_forward_w4a16_ws(*p, T, d, E, k, inter, ctypes.c_float(scale), out, FAKE,
                                        ws, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(d=7100), SHAPE), (dict(inter=2000), SHAPE), (dict(E=0), SHAPE), (dict(k=9, E=8), SHAPE),
    (dict(T=-1), INVALID), (dict(scale=float("nan")), INVALID),
])
def test_w4a16_layer_rejects_bad_shapes(kw, code):
    assert _layer_w4(**kw) == code


def test_w4a16_layer_rejects_null_pointers_and_small_workspace():
    for i in range(9):
        p = [FAKE] * 9
        p[i] = NULL
        assert _layer_w4(ptrs=p) == INVALID
    assert _layer_w4(out=NULL) == INVALID
    need = moe.moe_workspace_size(64, 7168, 384, 8, 2048)
    assert _layer_w4(ws=need - 1) == INVALID
    assert _layer_w4(T=0) == OK


def test_quantize_int4_rejects_bad_shapes():
    L = moe.lib()
    assert L.moe_quantize_int4(FAKE, 8, 96, FAKE, FAKE, NULL) == SHAPE     # not a multiple of 64
    assert L.moe_quantize_int4(FAKE, -1, 128, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_int4(FAKE, 0, 128, FAKE, FAKE, NULL) == OK
    assert L.moe_quantize_int4(NULL, 8, 128, FAKE, FAKE, NULL) == INVALID
    assert L.moe_quantize_int4(FAKE, 8, 128, FAKE, NULL, NULL) == INVALID
    assert L.moe_quantize_int4(FAKE, 8, 128, ctypes.c_void_p(0x10004), FAKE, NULL) == INVALID


# ------------------------------------------------------------ FP8 compute

def _layer_w8a8(T=64, d=7168, E=384, k=8, inter=2048, scale=2.827, ptrs=None, out=FAKE,
                ws=None):
    p = ptrs if ptrs is not None else [FAKE] * 11
    L = moe.lib()
    if ws is None:
        return L.moe_layer_forward_w8a8(*p, T, d, E, k, inter, ctypes.c_float(scale), out, NULL)
    return L.moe_layer_forward_w8a8_ws(*p, T, d, E, k, inter, ctypes.c_float(scale), out, FAKE,
                                       ws, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(d=7104), SHAPE), (dict(inter=2112), SHAPE), (dict(d=7100), SHAPE), (dict(E=0), SHAPE),
    (dict(k=9, E=8), SHAPE), (dict(T=-1), INVALID), (dict(scale=float("nan")), INVALID),
])
def test_w8a8_layer_rejects_bad_shapes(kw, code):
    # K steps of 128 codes: d and inter must be multiples of 128
    assert _layer_w8a8(**kw) == code


def test_w8a8_layer_rejects_null_pointers_and_small_workspace():
    for i in range(11):
        p = [FAKE] * 11
        p[i] = NULL
        assert _layer_w8a8(ptrs=p) == INVALID
    assert _layer_w8a8(out=NULL) == INVALID
    need = moe.moe_workspace_size_w8a8(64, 7168, 384, 8, 2048)
    # the bf16 layer's workspace is too small: the codes' exponents and the
    # activation's codes need room of their own
    assert need > moe.moe_workspace_size(64, 7168, 384, 8, 2048)
    assert _layer_w8a8(ws=need - 1) == INVALID
    assert _layer_w8a8(T=0) == OK
    assert moe.moe_workspace_size_w8a8(64, 7100, 384, 8, 2048) == 0


def test_quantize_fp8_rows_rejects_bad_shapes():
    L = moe.lib()
    assert L.moe_quantize_fp8_rows(FAKE, 100, 120, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_fp8_rows(FAKE, -1, 128, FAKE, FAKE, NULL) == SHAPE
    assert L.moe_quantize_fp8_rows(FAKE, 0, 128, FAKE, FAKE, NULL) == OK
    assert L.moe_quantize_fp8_rows(FAKE, 5, 0, FAKE, FAKE, NULL) == OK
    assert L.moe_quantize_fp8_rows(NULL, 5, 128, FAKE, FAKE, NULL) == INVALID
    assert L.moe_quantize_fp8_rows(FAKE, 5, 128, ctypes.c_void_p(0x10008), FAKE, NULL) == INVALID
    assert L.moe_quantize_fp8_rows(FAKE, 5, 128, FAKE, NULL, NULL) == INVALID


# ------------------------------------------------------------ load balance

def test_balance_calls_reject_bad_arguments():
    L = moe.lib()
    f = ctypes.c_float
    assert L.moe_bias_update(FAKE, 64, 0, 8, f(1e-3), FAKE, NULL) == SHAPE
    assert L.moe_bias_update(FAKE, 64, 384, 33, f(1e-3), FAKE, NULL) == SHAPE
    assert L.moe_bias_update(FAKE, -1, 384, 8, f(1e-3), FAKE, NULL) == INVALID
    assert L.moe_bias_update(NULL, 64, 384, 8, f(1e-3), FAKE, NULL) == INVALID
    assert L.moe_bias_update(FAKE, 64, 384, 8, f(float("nan")), FAKE, NULL) == INVALID
    assert L.moe_bias_update(FAKE, 0, 384, 8, f(1e-3), FAKE, NULL) == OK
    assert L.moe_router_scores(FAKE, FAKE, 64, 7100, 384, FAKE, FAKE, 1 << 30, NULL) == SHAPE
    assert L.moe_router_scores(FAKE, FAKE, 64, 7168, 384, FAKE, FAKE, 16, NULL) == INVALID
    assert L.moe_router_scores(FAKE, FAKE, 0, 7168, 384, FAKE, FAKE, 0, NULL) == OK
    need = moe.moe_seq_aux_workspace_size(4, 64, 384)
    assert need >= 4 * 64 * 4
    aux = lambda *a, ws=need: L.moe_seq_aux_loss(*a, FAKE, NULL, NULL, FAKE, ws, NULL)
    assert aux(FAKE, FAKE, 4, 64, 2048, 8, f(1e-3)) == SHAPE
    assert aux(FAKE, FAKE, 4, 0, 384, 8, f(1e-3)) == INVALID
    assert aux(NULL, FAKE, 4, 64, 384, 8, f(1e-3)) == INVALID
    assert aux(FAKE, FAKE, 4, 64, 384, 8, f(1e-3), ws=need - 1) == INVALID
    assert aux(FAKE, FAKE, 0, 64, 384, 8, f(1e-3)) == OK
