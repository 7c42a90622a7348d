"""Checks that pin the fp64 oracle to something other than itself.

Each pin_* function raises AssertionError if the oracle (whichever build the
`oracle` wrapper currently points at) breaks a fact fixed by the pages or by
mathematics:
  - closed forms and identities (sigmoid(0) = 1/2, sigma(z) + sigma(-z) = 1,
    silu(z) - silu(-z) = z, weights summing to the scaling factor);
  - special cases that reduce to a library routine (numpy matmul + scipy expit
    for the router scores, torch's float->bf16 rounding);
  - brute force on tiny inputs (full sort for top-k, lexsort for the
    permutation, naive Python loops for a textbook SwiGLU MLP);
  - a dense all-experts-then-mask evaluation (the MoE definition) against the
    oracle's sparse path;
  - invariants (bias changes selection but never weights; rows independent).
tests/test_oracle_pins.py runs them on the oracle; tests/test_oracle_mutants.py
runs them on deliberately broken copies of the oracle and requires each copy
to fail at least one pin.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from scipy.special import expit

import oracle
from moe_inputs import MoEConfig, make_inputs, make_topk_idx

K2_SCALE = 2.827   # routed_scaling_factor of K2 (K2 team member's answer, "different")


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f64(t):
    return oracle.bf16_to_f64(t)


# ------------------------------------------------------------------ numbers

def pin_bf16_rounding():
    pats = np.arange(65536, dtype=np.uint16)
    vals = oracle.bf16_to_f64(pats)
    finite = np.isfinite(vals)
    back = oracle.f64_to_bf16(vals[finite])
    # every finite bf16 value is its own rounding (up to the sign of zero)
    same = (back == pats[finite]) | ((vals[finite] == 0) & ((back & 0x7FFF) == 0))
    assert same.all(), "bf16 values do not round-trip"
    # midpoints between neighbours round to the even significand
    rng = np.random.default_rng(1)
    a = rng.integers(0x0080, 0x7F00, size=2000).astype(np.uint16)
    lo, hi = oracle.bf16_to_f64(a), oracle.bf16_to_f64(a + 1)
    mid = (lo + hi) / 2.0
    got = oracle.f64_to_bf16(mid)
    want = np.where(a % 2 == 0, a, a + 1).astype(np.uint16)
    assert (got == want).all(), "ties do not go to even"
    # slightly off the midpoint goes to the nearer neighbour
    assert (oracle.f64_to_bf16(mid - (hi - lo) * 1e-3) == a).all()
    assert (oracle.f64_to_bf16(mid + (hi - lo) * 1e-3) == a + 1).all()
    # agrees with torch's fp32 -> bf16 rounding on values that are exact fp32
    f = rng.standard_normal(5000).astype(np.float32) * np.float32(37.0)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (oracle.f64_to_bf16(f.astype(np.float64)) == ref).all()


def pin_sigmoid_silu():
    assert oracle.sigmoid(0.0) == 0.5
    assert abs(oracle.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    for z in np.linspace(-30, 30, 61):
        s, sn = oracle.sigmoid(z), oracle.sigmoid(-z)
        assert abs(s + sn - 1.0) < 1e-15
        assert abs(s - expit(z)) < 1e-15
        assert abs(oracle.silu(z) - z * expit(z)) <= 1e-14 * max(1.0, abs(z))
        assert abs(oracle.silu(z) - oracle.silu(-z) - z) <= 1e-14 * max(1.0, abs(z))
    assert oracle.silu(0.0) == 0.0


# ------------------------------------------------------------------- router

def _rand_router(T, d, E, seed, bias_scale=0.01):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    w = (torch.randn((E, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    b = ((torch.rand((E,), generator=g) * 2 - 1) * bias_scale).to(torch.float32)
    return x, w, b


def pin_route_worked_example():
    """Hand-built: x = e_0, router column 0 carries the logits."""
    d, E, k = 8, 5, 2
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    L = np.array([0.0, 2.0, -2.0, 0.0, 1.0], np.float32)   # all exact in bf16
    w_r = np.zeros((E, d), np.float32)
    w_r[:, 0] = L
    # biased scores: [0.5, s(2), s(-2)+0.9, 0.5-0.1, s(1)-0.5] ->
    # order: e2 (1.019) > e1 (0.881) > e0 (0.5) > e3 (0.4) > e4 (0.231)
    bias = np.array([0.0, 0.0, 0.9, -0.1, -0.5], np.float32)
    idx, w, gap = oracle.route(_bf16(x), _bf16(w_r), bias, k, K2_SCALE)
    assert idx.tolist() == [[2, 1]], idx
    # unbiased: s(-2) + s(2) = 1 exactly in exact arithmetic
    s2 = 1.0 / (1.0 + math.exp(-2.0))
    assert abs(w[0, 0] - K2_SCALE * (1.0 - s2)) < 1e-14
    assert abs(w[0, 1] - K2_SCALE * s2) < 1e-14
    assert abs(gap[0] - (s2 - 0.5)) < 1e-7    # b_(2) - b_(3), bias is fp32 0.0
    # E = k: every expert, weights from all unbiased scores
    idx, w, gap = oracle.route(_bf16(x), _bf16(w_r), bias, E, K2_SCALE)
    assert idx.tolist() == [[2, 1, 0, 3, 4]]
    s = expit(L.astype(np.float64))
    assert np.allclose(w[0], K2_SCALE * s[[2, 1, 0, 3, 4]] / s.sum(), rtol=0, atol=1e-14)
    assert gap[0] == np.inf


def pin_router_scores_library():
    x, w, b = _rand_router(40, 64, 19, seed=3)
    idx, tw, gap, scores = oracle.route(x, w, b, 4, K2_SCALE, want_scores=True)
    ref = expit(_f64(x) @ _f64(w).T)
    assert np.abs(scores - ref).max() < 1e-13, "router scores differ from expit(x W^T)"


def pin_topk_brute_force():
    for (T, d, E, k, seed) in [(50, 32, 5, 1, 0), (50, 32, 9, 3, 1), (60, 64, 33, 8, 2),
                               (20, 16, 7, 7, 4), (30, 32, 40, 32, 5)]:
        x, w, b = _rand_router(T, d, E, seed, bias_scale=0.2)
        idx, tw, gap, scores = oracle.route(x, w, b, k, K2_SCALE, want_scores=True)
        bb = scores + b.numpy().astype(np.float64)[None, :]
        for t in range(T):
            order = sorted(range(E), key=lambda e: (-bb[t, e], e))
            assert idx[t].tolist() == order[:k], (t, idx[t], order[:k])
            want_gap = bb[t, order[k - 1]] - bb[t, order[k]] if k < E else np.inf
            assert gap[t] == want_gap
            assert len(set(idx[t].tolist())) == k


def pin_exact_ties():
    d, E, k = 16, 6, 3
    g = torch.Generator().manual_seed(7)
    row = torch.randn((1, d), generator=g)
    w = row.repeat(E, 1).to(torch.bfloat16)         # six identical router rows
    x = torch.randn((5, d), generator=g).to(torch.bfloat16)
    idx, tw, gap = oracle.route(x, w, np.zeros(E, np.float32), k, K2_SCALE)
    assert (idx == np.array([0, 1, 2])[None, :]).all(), idx   # ties -> lower index
    assert np.allclose(tw, K2_SCALE / k, rtol=0, atol=1e-15)
    assert (gap == 0).all()
    # a strictly larger bias on expert 4 lifts it to slot 0, the rest keep index order
    bias = np.zeros(E, np.float32)
    bias[4] = 1e-3
    idx, tw, gap = oracle.route(x, w, bias, k, K2_SCALE)
    assert (idx == np.array([4, 0, 1])[None, :]).all(), idx
    assert np.allclose(tw, K2_SCALE / k, rtol=0, atol=1e-15)


def pin_weights_closed_form():
    x, w, b = _rand_router(64, 64, 24, seed=9)
    k = 6
    idx, tw, gap = oracle.route(x, w, b, k, K2_SCALE)
    s = expit(_f64(x) @ _f64(w).T)
    sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    assert np.abs(tw.sum(1) - K2_SCALE).max() <= 1e-12 * K2_SCALE
    assert (tw > 0).all()
    assert np.abs(tw - K2_SCALE * sel / sel.sum(1, keepdims=True)).max() < 1e-12
    # the DeepSeek-V3 factor works the same way
    _, tw25, _ = oracle.route(x, w, b, k, 2.5)
    assert np.abs(tw25.sum(1) - 2.5).max() <= 1e-12 * 2.5


def pin_bias_selection_only():
    x, w, b = _rand_router(80, 64, 16, seed=11, bias_scale=0.05)
    k = 4
    idx0, tw0, _ = oracle.route(x, w, np.zeros(16, np.float32), k, K2_SCALE)
    idx1, tw1, _ = oracle.route(x, w, b, k, K2_SCALE)
    changed = 0
    for t in range(80):
        m0 = dict(zip(idx0[t].tolist(), tw0[t].tolist()))
        m1 = dict(zip(idx1[t].tolist(), tw1[t].tolist()))
        if set(m0) == set(m1):
            assert m0 == m1, "bias changed a weight of an unchanged selection"
        else:
            changed += 1
    assert changed > 0, "bias never changed a selection (test is too weak)"
    # a large bias forces expert 5 in; its weight still comes from unbiased scores
    big = np.zeros(16, np.float32)
    big[5] = 10.0
    idx2, tw2, _ = oracle.route(x, w, big, k, K2_SCALE)
    assert (idx2[:, 0] == 5).all()
    s = expit(_f64(x) @ _f64(w).T)
    sel = np.take_along_axis(s, idx2.astype(np.int64), axis=1)
    assert np.abs(tw2[:, 0] - K2_SCALE * s[:, 5] / sel.sum(1)).max() < 1e-12


# ------------------------------------------------------------- permutation

def pin_permute_brute_force():
    cases = [(37, 11, 3, 0, 0.0), (64, 32, 4, 1, 0.0), (200, 384, 8, 2, 0.0),
             (128, 16, 8, 3, 3.0), (1, 5, 5, 4, 0.0), (50, 9, 1, 5, 1.0)]
    for T, E, k, seed, skew in cases:
        idx = make_topk_idx(T, E, k, seed=seed, skew=skew).numpy()
        counts, offsets, row_token, slot_row = oracle.permute(idx, E)
        flat_e = idx.reshape(-1).astype(np.int64)
        flat_t = np.repeat(np.arange(T), k)
        order = np.lexsort((flat_t, flat_e))          # by expert, then token
        assert (counts == np.bincount(flat_e, minlength=E)).all()
        assert counts.sum() == T * k
        assert offsets[0] == 0 and (np.diff(offsets) == counts).all()
        assert (row_token == flat_t[order]).all()
        want_slot = np.empty(T * k, np.int64)
        want_slot[order] = np.arange(T * k)
        assert (slot_row == want_slot).all()
        assert sorted(slot_row.tolist()) == list(range(T * k))
        assert (row_token[slot_row] == flat_t).all()
        for e in range(E):
            seg = row_token[offsets[e]:offsets[e + 1]]
            assert (np.diff(seg) > 0).all()


# ------------------------------------------------------------------ experts

def pin_swiglu_textbook():
    """Naive loops: h_n = silu(sum_i G[n,i] x_i) * (sum_i U[n,i] x_i); y_o = sum_n D[o,n] h_n."""
    d, I = 12, 5
    g = torch.Generator().manual_seed(13)
    x = torch.randn((d,), generator=g).to(torch.bfloat16)
    gu = torch.randn((2 * I, d), generator=g).to(torch.bfloat16)
    dn = torch.randn((d, I), generator=g).to(torch.bfloat16)
    xf, guf, dnf = _f64(x), _f64(gu), _f64(dn)
    h = []
    for n in range(I):
        gate = sum(guf[n, i] * xf[i] for i in range(d))
        up = sum(guf[I + n, i] * xf[i] for i in range(d))
        h.append(gate * expit(gate) * up)
    y = [sum(dnf[o, n] * h[n] for n in range(I)) for o in range(d)]
    got, act = oracle.swiglu_row(x, gu, dn, want_act=True)
    assert np.abs(np.array(h) - act).max() < 1e-12
    assert np.abs(np.array(y) - got).max() < 1e-12


def _tiny_cfg():
    return MoEConfig("pin", T=24, d=64, E=10, k=3, inter=32, scale=K2_SCALE)


def pin_dense_vs_sparse():
    """MoE by definition: every expert on every token, masked by the routing weights."""
    cfg = _tiny_cfg()
    inp = make_inputs(cfg, seed=21)
    out, idx, tw, gap = oracle.moe_forward(inp, cfg.k, cfg.scale)
    xf = _f64(inp["x"])
    gu, dn = _f64(inp["w_gate_up"]), _f64(inp["w_down"])
    I = cfg.inter

    def ffn(gu_e, dn_e):
        G, U = xf @ gu_e[:I].T, xf @ gu_e[I:].T
        return (G * expit(G) * U) @ dn_e.T

    mask = np.zeros((cfg.T, cfg.E))
    np.put_along_axis(mask, idx.astype(np.int64), tw, axis=1)
    dense = ffn(_f64(inp["ws_gate_up"]), _f64(inp["ws_down"]))
    for e in range(cfg.E):
        dense += mask[:, e:e + 1] * ffn(gu[e], dn[e])
    assert np.abs(dense - out).max() <= 1e-12 * np.abs(dense).max()


def pin_special_cases():
    cfg = _tiny_cfg()
    inp = make_inputs(cfg, seed=22)
    I = cfg.inter
    xf = _f64(inp["x"])
    sg, sd = _f64(inp["ws_gate_up"]), _f64(inp["ws_down"])
    G = xf @ sg[:I].T
    shared_only = (G * expit(G) * (xf @ sg[I:].T)) @ sd.T
    # routed gate_proj = 0  =>  silu(0) = 0  =>  output is the shared expert alone
    z = dict(inp)
    z["w_gate_up"] = inp["w_gate_up"].clone()
    z["w_gate_up"][:, :I] = 0
    out, *_ = oracle.moe_forward(z, cfg.k, cfg.scale)
    assert np.abs(out - shared_only).max() <= 1e-12 * np.abs(shared_only).max()
    # the shared expert is always there: zeroing its down_proj leaves only routed rows
    z2 = dict(inp)
    z2["ws_down"] = torch.zeros_like(inp["ws_down"])
    out2, idx, tw, _ = oracle.moe_forward(z2, cfg.k, cfg.scale)
    full, *_ = oracle.moe_forward(inp, cfg.k, cfg.scale)
    assert np.abs((full - out2) - shared_only).max() <= 1e-11 * np.abs(shared_only).max()


def pin_row_independence():
    cfg = _tiny_cfg()
    inp = make_inputs(cfg, seed=23)
    full, idx, tw, _ = oracle.moe_forward(inp, cfg.k, cfg.scale)
    sub = np.array([5, 0, 23, 11, 11], np.int32)
    part, *_ = oracle.moe_forward(inp, cfg.k, cfg.scale, tokens=sub)
    assert np.array_equal(part, full[sub])


def pin_combine():
    T, d, k = 9, 16, 3
    rng = np.random.default_rng(5)
    y = rng.standard_normal((T * k, d))
    ys = rng.standard_normal((T, d))
    w = rng.random((T, k))
    slot_row = rng.permutation(T * k).astype(np.int32)
    out = oracle.combine(y, ys, w, slot_row)
    for t in range(T):
        want = ys[t] + sum(w[t, j] * y[slot_row[t * k + j]] for j in range(k))
        assert np.abs(out[t] - want).max() < 1e-13
    # one-hot weights pick the row the slot points at
    w1 = np.zeros((T, k))
    w1[:, 1] = 1.0
    out1 = oracle.combine(y, None, w1, slot_row)
    assert np.array_equal(out1, y[slot_row.reshape(T, k)[:, 1]])



# ------------------------------------------------------------ FP8 storage
# "Kimi K2.5 Q&A", Q7.1: routed-expert weights are stored quantized and
# computed in BF16; the element format is OCP FP8 E4M3 and the scale is one
# power of two per 128 x 128 block (the rule in the oracle header).

def _torch_e4m3(v):
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def pin_fp8_decode_library():
    """Every code decodes to torch's float8_e4m3fn value (NaN only at 0x7F/0xFF)."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_decode(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])


def pin_fp8_anchor_values():
    """Published values of the format: 448 max, 2^-6 smallest normal, 2^-9 smallest subnormal."""
    assert oracle.e4m3_encode(448.0) == 0x7E and oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_encode(2.0 ** -6) == 0x08
    assert oracle.e4m3_encode(2.0 ** -9) == 0x01
    assert oracle.e4m3_encode(1.0) == 0x38 and oracle.e4m3_encode(-2.0) == 0xC0
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(1000.0) == 0x7E and oracle.e4m3_encode(-1000.0) == 0xFE


def pin_fp8_encode_library():
    """Encoding matches torch's float -> float8_e4m3fn cast on random values and
    on every midpoint between adjacent codes (ties to the even code)."""
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 3000), rng.normal(0, 1, 3000),
                        rng.normal(0, 0.01, 3000), rng.uniform(-2.0 ** -6, 2.0 ** -6, 1000)])
    v = v.astype(np.float32).astype(np.float64)
    assert np.array_equal(np.array([oracle.e4m3_encode(x) for x in v], dtype=np.uint8),
                          _torch_e4m3(v))
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])     # 0 .. 448 ascending
    mids = (vals[:-1] + vals[1:]) / 2.0
    ours = np.array([oracle.e4m3_encode(m) for m in mids])
    assert np.all(ours % 2 == 0)
    assert np.array_equal(ours, _torch_e4m3(mids))
    assert np.array_equal(np.array([oracle.e4m3_encode(-m) for m in mids]), ours | 0x80)


def pin_fp8_block_exponent_brute_force():
    """s is the smallest integer with amax <= 448 * 2^s, clamped to [-124, 127]."""
    rng = np.random.default_rng(2)
    cases = [0.05, 1.0, 448.0, 449.0, 3.0e-3, 7.0, 224.0, 224.5, 1e-30, 3e38]
    cases += list(np.exp(rng.uniform(-20, 20, 40)))
    for amax in cases:
        brute = next(t for t in range(-300, 300) if amax <= 448.0 * 2.0 ** t)
        assert oracle.fp8_block_exponent(amax) == min(max(brute, -124), 127), amax
    assert oracle.fp8_block_exponent(0.0) == 0


def pin_fp8_quantize_bounds():
    """Per-element error within half a step of the format, each block's exponent
    from its own amax and on its own block, the block maximum in the top binade."""
    rng = np.random.default_rng(1)
    rows, cols = 256, 384
    w = rng.normal(0, 0.02, (rows, cols))
    for i in range(rows // 128):
        for j in range(cols // 128):
            w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] *= 2.0 ** (i + 3 * j)
    wb = _bf16(w).view(torch.int16).numpy().view(np.uint16)
    wf = oracle.bf16_to_f64(wb)
    q, sexp = oracle.quantize_fp8(wb)
    assert sexp.shape == (rows // 128, cols // 128)
    for i in range(rows // 128):
        for j in range(cols // 128):
            blk = wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            brute = next(t for t in range(-300, 300) if np.abs(blk).max() <= 448.0 * 2.0 ** t)
            assert sexp[i, j] == brute
    wq = oracle.bf16_to_f64(oracle.dequantize_fp8(q, sexp))
    scale = np.repeat(np.repeat(2.0 ** sexp.astype(float), 128, 0), 128, 1)
    y = np.abs(wf) / scale
    bound = np.where(y >= 2.0 ** -6, 2.0 ** -4 * np.abs(wf), 2.0 ** -10 * scale)
    assert np.all(np.abs(wq - wf) <= bound)
    assert np.all(np.sign(wq) * np.sign(wf) >= 0)
    for i in range(rows // 128):
        for j in range(cols // 128):
            top = np.abs(wq[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]).max()
            assert 224.0 <= top / 2.0 ** sexp[i, j] <= 448.0


# FP8 compute ("Kimi K2.5 Q&A", Q7.1 names V3's compute in FP8; "Kimi K2 deep
# dive", 3.2): E4M3 operands with one power-of-two exponent per row (weight
# output channel, token), which factors out of every K sum.

def _brute_exponent(amax):
    if amax == 0.0:
        return 0
    return min(max(next(t for t in range(-300, 300) if amax <= 448.0 * 2.0 ** t), -124), 127)


def _u16_of(w):
    return _bf16(w).view(torch.int16).numpy().view(np.uint16)


def _torch_e4m3_decode(q):
    return torch.from_numpy(np.ascontiguousarray(q, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def pin_fp8_rows_quantizer_library():
    """Each row's exponent by brute force from its own amax (negative maxima,
    an exact 448 * 2^s boundary, zero and clamped rows), its codes from torch's
    float8_e4m3fn cast of w * 2^-s."""
    rng = np.random.default_rng(5)
    rows, cols = 12, 200
    w = rng.normal(0, 1, (rows, cols)) * 2.0 ** rng.integers(-30, 30, (rows, 1))
    w[3] = 0.0
    w[4] = rng.normal(0, 1e-39, cols)              # amax below 448 * 2^-124: clamped
    w[5] = rng.normal(0, 1e-3, cols)
    w[5, 7] = 56.0                                 # = 448 * 2^-3 exactly: s = -3
    w[6, 9] = -50.0 * np.abs(w[6]).max()           # the row maximum is negative
    wb = _u16_of(w)
    wf = oracle.bf16_to_f64(wb)
    q, s = oracle.quantize_fp8_rows(wb)
    assert q.shape == (rows, cols) and s.shape == (rows,)
    for r in range(rows):
        se = _brute_exponent(np.abs(wf[r]).max())
        assert s[r] == se, (r, s[r], se)
        assert np.array_equal(q[r], _torch_e4m3(wf[r] * 2.0 ** -se)), r
    assert s[3] == 0 and s[4] == -124 and s[5] == -3


def _e4m3_exact(rng, shape, row_exp):
    """Values code * 2^e with E4M3 normal codes, random signs, each row's
    largest magnitude 448 * 2^e (so the row quantizer is exact on them)."""
    codes = rng.integers(0x08, 0x7F, shape)
    vals = _torch_e4m3_decode(codes.astype(np.uint8)) * rng.choice([-1.0, 1.0], shape)
    vals[:, 0] = 448.0
    return vals * 2.0 ** np.asarray(row_exp, dtype=float)[:, None]


def pin_fp8_compute_exact_inputs():
    """On inputs whose rows the quantizer represents exactly, FP8 compute is the
    bf16 oracle's SwiGLU activation rounded to bf16 and quantized per row (the
    exponent by brute force, the codes by torch's cast), then a matrix product."""
    rng = np.random.default_rng(6)
    d, inter = 96, 80
    x = _e4m3_exact(rng, (1, d), [-9])[0]
    wgu = _e4m3_exact(rng, (2 * inter, d), rng.integers(-16, -12, 2 * inter))
    wdn = _e4m3_exact(rng, (d, inter), rng.integers(-16, -12, d))
    xb, gub, dnb = _u16_of(x), _u16_of(wgu), _u16_of(wdn)
    assert np.array_equal(oracle.bf16_to_f64(gub), wgu)     # exact in bf16
    qg, sg = oracle.quantize_fp8_rows(gub)
    qd, sd = oracle.quantize_fp8_rows(dnb)
    y = oracle.swiglu_row_fp8(xb, qg, sg, qd, sd)
    _, act = oracle.swiglu_row(xb, gub, dnb, want_act=True)
    h = oracle.bf16_to_f64(oracle.f64_to_bf16(act))
    sh = _brute_exponent(np.abs(h).max())
    hq = _torch_e4m3_decode(_torch_e4m3(h * 2.0 ** -sh)) * 2.0 ** sh
    ref = wdn @ hq
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def pin_fp8_compute_exponent_bookkeeping():
    """Power-of-two rescalings that leave every code unchanged move the result
    exactly: x * 2^3 with the gate|up rows * 2^-3 gives the same y; the up rows
    * 2^5 give y * 2^5 (through the activation's exponent); one down row * 2^-4
    scales that output alone."""
    rng = np.random.default_rng(7)
    d, inter = 128, 64
    x = rng.normal(0, 1, d)
    wgu = rng.normal(0, 0.05, (2 * inter, d))
    wdn = rng.normal(0, 0.05, (d, inter))

    def run(x_, gu_, dn_):
        qg, sg = oracle.quantize_fp8_rows(_u16_of(gu_))
        qd, sd = oracle.quantize_fp8_rows(_u16_of(dn_))
        return oracle.swiglu_row_fp8(_u16_of(x_), qg, sg, qd, sd)

    y = run(x, wgu, wdn)
    assert np.abs(y).max() > 0
    assert np.array_equal(run(x * 8.0, wgu / 8.0, wdn), y)
    up = wgu.copy()
    up[inter:] *= 32.0
    assert np.array_equal(run(x, up, wdn), y * 32.0)
    dn = wdn.copy()
    dn[5] /= 16.0
    want = y.copy()
    want[5] /= 16.0
    assert np.array_equal(run(x, wgu, dn), want)


def pin_fp8_compute_layer_identities():
    """Whole layer in FP8 compute with expert e = the base expert with its up
    rows * 2^e, shared expert = base: row t is exactly
    y_base(x_t) (1 + sum_j w_tj 2^(e_tj)); a token subset gives the same rows."""
    rng = np.random.default_rng(8)
    T, d, inter, E, k = 5, 64, 32, 4, 2
    x = rng.normal(0, 1, (T, d))
    gu = rng.normal(0, 0.05, (2 * inter, d))
    dn = rng.normal(0, 0.05, (d, inter))
    base = oracle.quantize_fp8_rows(_u16_of(gu)) + oracle.quantize_fp8_rows(_u16_of(dn))
    experts = []
    for e in range(E):
        g = gu.copy()
        g[inter:] *= 2.0 ** e
        experts.append(oracle.quantize_fp8_rows(_u16_of(g)) + base[2:])
    idx = np.array([[0, 3], [2, 1], [3, 0], [1, 2], [2, 3]], np.int32)
    w = rng.uniform(0.1, 1.5, (T, k))
    xb = _u16_of(x)
    out = oracle.moe_rows_fp8(xb, idx, w, experts, base)
    for t in range(T):
        yb = oracle.swiglu_row_fp8(xb[t], *base)
        want = yb * (1.0 + sum(w[t, j] * 2.0 ** idx[t, j] for j in range(k)))
        assert np.allclose(out[t], want, rtol=1e-13, atol=1e-13 * np.abs(want).max()), t
    sub = oracle.moe_rows_fp8(xb, idx, w, experts, base, tokens=np.array([4, 1]))
    assert np.array_equal(sub, out[[4, 1]])


# INT4 storage ("Kimi K2.5 deep dive", CH7.2: 4-bit integer weights, group of
# 32, symmetric; "Kimi K2.5 Q&A", Q7.1: storage quantized, compute BF16).

def _int4_weights(seed):
    rng = np.random.default_rng(seed)
    rows, cols = 6, 256
    w = rng.normal(0, 1, (rows, cols)) * 2.0 ** rng.integers(-20, 10, (rows, cols // 32)).repeat(32, 1)
    w[0, :32] = 0.0                                   # all-zero group
    w[1, 32:64] = rng.normal(0, 1e-3, 32)
    w[1, 40] = -5.0                                   # the group's maximum is negative
    w[2, 64:96] = np.arange(32) - 16.0                # integers: exact ties of w / s
    w[3, 96:128] = rng.normal(0, 1e-39, 32)           # bf16 subnormals: amax / 7 may round to 0
    return _u16_of(w)


def pin_int4_scale_library():
    """Each group's scale is torch's bf16 rounding of (its amax / 7) in fp32."""
    wb = _int4_weights(11)
    wf = oracle.bf16_to_f64(wb)
    q, sc = oracle.quantize_int4(wb)
    assert q.shape == wb.shape and sc.shape == (wb.shape[0], wb.shape[1] // 32)
    amax = np.abs(wf.reshape(wf.shape[0], -1, 32)).max(axis=2)
    ref = (torch.from_numpy(amax.astype(np.float32)) / 7.0).to(torch.bfloat16)
    assert np.array_equal(sc, ref.view(torch.int16).numpy().view(np.uint16))
    assert sc[0, 0] == 0 and np.all(q[0, :32] == 0)


def pin_int4_codes_brute_force():
    """q minimises |w - q s| over the 16 codes, ties to the even code; zero
    scale gives zero codes."""
    wb = _int4_weights(12)
    wf = oracle.bf16_to_f64(wb)
    q, sc = oracle.quantize_int4(wb)
    s = oracle.bf16_to_f64(sc)
    cand = np.arange(-8, 8, dtype=np.float64)
    for r in range(wf.shape[0]):
        for c in range(wf.shape[1]):
            sv = s[r, c // 32]
            if sv == 0.0:
                assert q[r, c] == 0
                continue
            err = np.abs(wf[r, c] - cand * sv)
            best = cand[err == err.min()]
            want = best[0] if len(best) == 1 else best[(best % 2) == 0][0]
            assert q[r, c] == want, (r, c, wf[r, c], sv, q[r, c], want)


def pin_int4_dequantize_library():
    """Dequantized weights are torch's bf16 rounding of q * s (exact in fp32),
    within half a step of w, and every nonzero group reaches |q| = 7."""
    wb = _int4_weights(13)
    wf = oracle.bf16_to_f64(wb)
    q, sc = oracle.quantize_int4(wb)
    deq = oracle.dequantize_int4(q, sc)
    s = torch.from_numpy(sc.view(np.int16)).view(torch.bfloat16).float()
    ref = (torch.from_numpy(q.astype(np.float32)) * s.repeat_interleave(32, 1)).to(torch.bfloat16)
    assert np.array_equal(deq, ref.view(torch.int16).numpy().view(np.uint16))
    sv = oracle.bf16_to_f64(sc).repeat(32, 1)
    d = oracle.bf16_to_f64(deq)
    assert np.all(np.abs(wf - d) <= sv / 2 + np.abs(d) * 2.0 ** -8 + 1e-300)
    g = np.abs(q.reshape(q.shape[0], -1, 32)).max(axis=2)
    assert np.all((g == 7) | (oracle.bf16_to_f64(sc) == 0))


# ---------------------------------------------------------- load balancing
# "Kimi K2.5 Q&A", Q7.2 and "Kimi K2.5 deep dive", CH10.2 step 2: the selection
# bias is a non-learned buffer lowered for over-loaded and raised for
# under-loaded experts; a weak sequence-level balance loss (alpha = 0.001).

def pin_bias_update_worked_example():
    """Hand-computed steps: loads against the exact mean T*k/E, fp32 buffer."""
    b = oracle.bias_update(np.array([3, 1, 2, 2]), T=4, k=2, gamma=0.125,
                           bias=np.array([0.0, 0.0, 0.5, -0.25], np.float32))
    assert np.array_equal(b, np.array([-0.125, 0.125, 0.5, -0.25], np.float32))
    # mean 7/3 is not an integer: 2 < 7/3 < 3, none sits at the mean
    b = oracle.bias_update(np.array([3, 2, 2]), T=7, k=1, gamma=0.5,
                           bias=np.zeros(3, np.float32))
    assert np.array_equal(b, np.array([-0.5, 0.5, 0.5], np.float32))
    # the update is made in fp32: 1 + 2^-25 rounds back to 1
    b = oracle.bias_update(np.array([0, 2]), T=2, k=1, gamma=2.0 ** -25,
                           bias=np.array([1.0, 1.0], np.float32))
    assert b[0] == np.float32(1.0) and b[1] == np.float32(1.0)


def pin_bias_update_invariants():
    rng = np.random.default_rng(5)
    for _ in range(20):
        E = int(rng.integers(2, 64))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(1, 200))
        counts = np.bincount(rng.integers(0, E, T * k), minlength=E)
        bias = (rng.integers(-64, 64, E) * 2.0 ** -10).astype(np.float32)
        gamma = 2.0 ** -7
        nb = oracle.bias_update(counts, T, k, gamma, bias)
        d = nb.astype(np.float64) - bias
        over = counts * E > T * k
        under = counts * E < T * k
        assert np.all(d[over] == -gamma) and np.all(d[under] == gamma)
        assert np.all(d[~over & ~under] == 0.0)


def pin_bias_update_moves_load():
    """Lowering an over-loaded expert's bias (and raising the others' by at most
    gamma) cannot give it more tokens, and the least-loaded expert cannot lose
    any: checked with the oracle's own router."""
    x, wr, bias = _rand_router(96, 64, 16, seed=77)
    k = 4
    idx, _, _ = oracle.route(x, wr, bias, k, K2_SCALE)
    counts = np.bincount(idx.reshape(-1), minlength=16)
    nb = oracle.bias_update(counts, 96, k, 0.05, bias.numpy() if hasattr(bias, "numpy") else bias)
    idx2, _, _ = oracle.route(x, wr, torch.as_tensor(nb), k, K2_SCALE)
    c2 = np.bincount(idx2.reshape(-1), minlength=16)
    hi, lo = int(np.argmax(counts)), int(np.argmin(counts))
    assert c2[hi] <= counts[hi] and c2[lo] >= counts[lo]
    assert c2[hi] < counts[hi] or c2[lo] > counts[lo]      # and the step does move load


def pin_seq_aux_loss_closed_forms():
    alpha = 0.001
    # uniform affinities and a perfectly even selection: f_i = 1, P_i = 1/E, L = alpha
    E, k, S = 8, 2, 4
    scores = np.full((S, E), 0.3)
    idx = np.array([[0, 1], [2, 3], [4, 5], [6, 7]], np.int32)
    loss, f, p = oracle.seq_aux_loss(scores, idx, S, alpha)
    assert abs(loss[0] - alpha) < 1e-15 and np.allclose(f, 1.0) and np.allclose(p, 1.0 / E)
    # hand example: E=4, k=1, S=2, both tokens pick expert 0
    sc = np.array([[0.5, 0.5, 0.5, 0.5], [0.6, 0.2, 0.1, 0.1]])
    loss, f, p = oracle.seq_aux_loss(sc, np.array([[0], [0]], np.int32), 2, alpha)
    assert np.allclose(f[0], [4.0, 0.0, 0.0, 0.0]) and np.allclose(p[0], [0.425, 0.225, 0.175, 0.175])
    assert abs(loss[0] - 1.7 * alpha) < 1e-15
    # each sequence on its own; a token's affinities matter only up to a factor
    sc2 = np.concatenate([sc, sc * np.array([[3.0], [0.5]])])
    loss2, _, _ = oracle.seq_aux_loss(sc2, np.array([[0], [0], [0], [0]], np.int32), 2, alpha)
    assert np.allclose(loss2, [1.7 * alpha, 1.7 * alpha], rtol=0, atol=1e-15)

ALL_PINS = [pin_bf16_rounding, pin_sigmoid_silu, pin_route_worked_example,
            pin_router_scores_library, pin_topk_brute_force, pin_exact_ties,
            pin_weights_closed_form, pin_bias_selection_only, pin_permute_brute_force,
            pin_swiglu_textbook, pin_dense_vs_sparse, pin_special_cases,
            pin_row_independence, pin_combine, pin_fp8_decode_library, pin_fp8_anchor_values,
            pin_fp8_encode_library, pin_fp8_block_exponent_brute_force, pin_fp8_quantize_bounds,
            pin_bias_update_worked_example, pin_bias_update_invariants, pin_bias_update_moves_load,
            pin_seq_aux_loss_closed_forms, pin_fp8_rows_quantizer_library,
            pin_fp8_compute_exact_inputs, pin_fp8_compute_exponent_bookkeeping,
            pin_fp8_compute_layer_identities, pin_int4_scale_library,
            pin_int4_codes_brute_force, pin_int4_dequantize_library]


def failing_pins():
    """Names of the pins the current oracle build fails (exceptions count as failures)."""
    bad = []
    for p in ALL_PINS:
        try:
            p()
        except Exception:  # noqa: BLE001 - any error is a caught mistake
            bad.append(p.__name__)
    return bad
