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


def u16(t):
    """bf16 tensor (any device) or uint16 array -> C-contiguous uint16 numpy (the
    bit patterns the oracle reads)."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16, t.dtype
        return np.ascontiguousarray(t)
    import torch
    return np.ascontiguousarray(t.detach().to("cpu").contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


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


# ------------------------------------------------------ wide full-size samples

def plan_tile_rows(T: int, E: int, k: int) -> int:
    """Largest token tile of the layer's expert GEMMs for a batch shape (the
    launch configuration the library picks: 192 rows when T > 256 and the routed
    experts average at most 64 rows, else 256)."""
    return 192 if (T > 256 and T * k <= 64 * E) else 256


def _tiles(c: int, tn: int):
    """(number of token tiles, rows per tile) of an expert with c rows."""
    nt = -(-c // tn)
    chunk = ((-(-c // nt)) + 15) // 16 * 16
    return nt, chunk


def wide_sample(ridx, gap, E: int, T: int, k: int, cap: int = 640, tail: int | None = None):
    """Tokens whose output rows a full-size parity test compares, chosen from the
    oracle's own routing to cover the GEMM tiles' edges:
      - every token when T <= 64;
      - the busiest expert's last two token tiles (its whole segment when it
        fits one or two tiles), tail rows included;
      - the shared expert's last token tile (T rows cut like any expert's);
      - the last tile of the most loaded expert whose last tile is ragged;
      - tokens 0, T/2 and T-1.
    With `tail`, each tile part keeps only its last `tail` rows (the tile's end).
    Near-tie tokens (gap < TIE_EPS) are left out.  Returns (sorted tokens,
    {part: token count}) with at most `cap` tokens."""
    import oracle
    counts, offsets, row_token, _ = oracle.permute(ridx, E)
    tn = plan_tile_rows(T, E, k)
    parts = {}
    def rows(r0, r1):        # rows [r0, r1) of a part, the last `tail` of them with tail
        return (max(r0, r1 - tail) if tail else r0), r1

    if T <= 64:
        parts["all"] = set(range(T))
    else:
        b = int(np.argmax(counts))
        nt, chunk = _tiles(int(counts[b]), tn)
        r0, r1 = rows(max(0, (nt - 2) * chunk), int(counts[b]))
        parts[f"expert {b} rows {r0}..{r1 - 1}"] = set(
            row_token[offsets[b] + r0:offsets[b] + r1].tolist())
        nt_s, chunk_s = _tiles(T, tn)
        r0, r1 = rows((nt_s - 1) * chunk_s, T)
        parts[f"shared rows {r0}..{r1 - 1}"] = set(range(r0, r1))
        ragged = [e for e in range(E) if counts[e] > tn and counts[e] % _tiles(int(counts[e]), tn)[1]]
        if ragged:
            e = max(ragged, key=lambda i: (counts[i], -i))
            nt_e, chunk_e = _tiles(int(counts[e]), tn)
            r0, r1 = rows((nt_e - 1) * chunk_e, int(counts[e]))
            parts[f"expert {e} rows {r0}..{r1 - 1}"] = set(
                row_token[offsets[e] + r0:offsets[e] + r1].tolist())
        parts["0, T/2, T-1"] = {0, T // 2, T - 1}
    ties = set(np.nonzero(np.asarray(gap) < TIE_EPS)[0].tolist())
    tokens = sorted(set().union(*parts.values()) - ties)
    if len(tokens) > cap:
        keep = np.linspace(0, len(tokens) - 1, cap).round().astype(int)
        tokens = [tokens[i] for i in sorted(set(keep.tolist()))]
    return tokens, {name: len(v) for name, v in parts.items()}


def oracle_rows_by_expert(x_host, ridx, rw, tokens, load_expert, load_shared, row_fn,
                          nthreads=None, batch=16):
    """The oracle's output rows (fp64) of `tokens`, with one batch of experts'
    weights on the host at a time: each (token, slot) row is the oracle's
    single-expert row function on that token, the shared expert's row too, and
    the rows are summed by the oracle's combine in slot order.

    load_expert(e) / load_shared() -> the host weights row_fn takes;
    row_fn(x_row, weights) -> y f64 [d]."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    tokens = np.asarray(tokens, dtype=np.int64)
    n, k = len(tokens), ridx.shape[1]
    xu = u16(x_host)
    d = xu.shape[1]
    y = np.zeros((n * k, d), np.float64)
    ysh = np.zeros((n, d), np.float64)
    slots = {}
    for i, t in enumerate(tokens):
        for j in range(k):
            slots.setdefault(int(ridx[t, j]), []).append((i, j))
    threads = nthreads or len(os.sched_getaffinity(0))
    experts = sorted(slots)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        sh = load_shared()
        futs = [ex.submit(row_fn, xu[tokens[i]], sh) for i in range(n)]
        for i, f in enumerate(futs):
            ysh[i] = f.result()
        del sh
        for b0 in range(0, len(experts), batch):
            group = experts[b0:b0 + batch]
            weights = dict(zip(group, ex.map(load_expert, group)))
            work = [(e, i, j) for e in group for (i, j) in slots[e]]
            futs = [ex.submit(row_fn, xu[tokens[i]], weights[e]) for (e, i, j) in work]
            for (e, i, j), f in zip(work, futs):
                y[i * k + j] = f.result()
            del weights
    w = np.asarray(rw, dtype=np.float64)[tokens]
    return oracle.combine(y, ysh, w, np.arange(n * k, dtype=np.int32))
