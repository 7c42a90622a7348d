"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (stated once, used by every GPU parity test):
  - routing: the selected expert lists are bit-exact, except for tokens whose
    biased scores near the cut are within TIE_EPS of each other (the 8th/9th
    gap, or two slots' order): those are FLAGGED, not failed, and must still
    be a valid choice under the oracle's own fp64 scores;
  - routing weights (fp32 on the GPU): |w_gpu - w_ref| <= W_ATOL;
  - permutation: bit-exact;
  - bf16 outputs: relative L2 error <= REL_L2 and max abs error
    <= MAX_ABS_FRAC * max|ref|, rows of flagged tokens left out.
"""
from __future__ import annotations

import numpy as np

TIE_EPS = 1e-6
W_ATOL = 2e-5
REL_L2 = 5e-3
MAX_ABS_FRAC = 2e-2


def bf16_np(t):
    """bf16 torch tensor (any device) -> float64 numpy."""
    import torch
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


def check_routing(gpu_idx, gpu_w, ref_idx, ref_scores, bias, scale, eps=TIE_EPS):
    """Returns the list of flagged (near-tie) tokens; raises on any real mismatch."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_w = np.asarray(gpu_w, dtype=np.float64)
    T, k = ref_idx.shape
    b = ref_scores + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    flagged = []
    for t in range(T):
        g = gpu_idx[t]
        assert len(set(g.tolist())) == k, f"token {t}: repeated expert {g}"
        assert (g >= 0).all() and (g < b.shape[1]).all(), f"token {t}: index out of range {g}"
        if not np.array_equal(g, ref_idx[t]):
            bg = b[t, g]
            cut = np.sort(b[t])[::-1][k - 1]
            valid = (bg >= cut - eps).all() and (np.diff(bg) <= eps).all()
            assert valid, (f"token {t}: gpu {g.tolist()} vs oracle {ref_idx[t].tolist()}, "
                           f"gpu scores {bg}, k-th {cut}")
            flagged.append(t)
        # weights: scale * s / sum(s) over the GPU's own selection, oracle scores
        s = ref_scores[t, g]
        want = scale * s / s.sum()
        err = np.abs(gpu_w[t] - want).max()
        assert err <= W_ATOL, f"token {t}: weight error {err}"
    return flagged


def check_output(gpu, ref, skip_rows=()):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if len(skip_rows):
        keep = np.ones(ref.shape[0], bool)
        keep[list(skip_rows)] = False
        gpu, ref = gpu[keep], ref[keep]
    assert np.isfinite(gpu).all(), "non-finite output"
    denom = np.linalg.norm(ref)
    rel = np.linalg.norm(gpu - ref) / max(denom, 1e-300)
    mx = np.abs(gpu - ref).max() if ref.size else 0.0
    lim = MAX_ABS_FRAC * np.abs(ref).max() if ref.size else 0.0
    assert rel <= REL_L2, f"relative L2 error {rel:.3e} > {REL_L2}"
    assert mx <= lim, f"max abs error {mx:.3e} > {lim:.3e}"
    return rel, mx
