"""Comparison of the CUDA library against the CPU oracle (shared by the GPU tests and the
smoke check).

Bars (the parity contract of the block):
  - routing: selected experts equal the oracle's exactly, ties to the lower index; the only
    exempt tokens are those whose K-th and (K+1)-th oracle logits are within 1e-4 relative
    (for them the GPU's set must be one of the admissible sets); slot order is checked where
    neighbouring logits differ by more than the same band;
  - gates: within 1e-5 absolute of the oracle's softmax for the GPU's expert set;
  - bf16 outputs: max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the oracle's
    output rounded once to bf16; fp32 outputs: relative L2 error <= 1e-5 (and max-abs
    <= 1e-5 * max|y|);
  - permutation (counts, offsets, rows): exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_REL = 1e-4
BF16_MAX_ABS, BF16_REL_L2 = 2e-2, 5e-3
F32_REL = 1e-5
GATE_ABS = 1e-5


def check_routing(logits: np.ndarray, idx_gpu: np.ndarray, gate_gpu: np.ndarray, K: int):
    """Returns (exempt token list, errors list).  logits: oracle logits [T, n] (f64)."""
    T, n = logits.shape
    exempt, errors = [], []
    for t in range(T):
        l = logits[t]
        g_idx = [int(v) for v in idx_gpu[t]]
        if len(set(g_idx)) != K or min(g_idx) < 0 or max(g_idx) >= n:
            errors.append((t, "invalid expert set", g_idx))
            continue
        is_ex, sets = oracle.tie_band(l, K, TIE_REL)
        if is_ex:
            exempt.append(t)
            if tuple(sorted(g_idx)) not in sets:
                errors.append((t, "not an admissible set", g_idx, sets))
                continue
        else:
            order = sorted(range(n), key=lambda i: (-l[i], i))[:K]
            if sorted(g_idx) != sorted(order):
                errors.append((t, "expert set", g_idx, order))
                continue
        # slot order: descending logits; neighbours within the tie band may come either way
        bad_order = False
        for k in range(K - 1):
            a, b = l[g_idx[k]], l[g_idx[k + 1]]
            if abs(a - b) > TIE_REL * max(abs(a), abs(b)) and a < b:
                bad_order = True
        if bad_order:
            errors.append((t, "slot order", g_idx))
            continue
        # gates: softmax of the oracle's logits over the GPU's selection, in its slot order
        kept = np.array([l[i] for i in g_idx])
        ref = np.exp(kept - kept.max()) / np.exp(kept - kept.max()).sum()
        if np.max(np.abs(gate_gpu[t] - ref)) > GATE_ABS:
            errors.append((t, "gate", gate_gpu[t].tolist(), ref.tolist()))
    return exempt, errors


def check_permutation(idx_gpu, counts, offsets, rows, n, K, row_align=None):
    """Exact checks of the grouping: counts are the histogram of the selections, groups are
    contiguous and ordered by expert, every (token, slot) has a distinct row inside its
    expert's group, and rows of an expert are ordered by (token, slot)."""
    idx = np.asarray(idx_gpu).reshape(-1, K)
    counts = np.asarray(counts)
    offsets = np.asarray(offsets)
    rows = np.asarray(rows).reshape(-1, K)
    hist = np.bincount(idx.reshape(-1), minlength=n)
    assert np.array_equal(hist, counts), (hist, counts)
    assert offsets[0] == 0 and np.all(np.diff(offsets) >= counts)
    if row_align:
        assert np.all(offsets % row_align == 0)
    flat_rows = rows.reshape(-1)
    assert len(np.unique(flat_rows)) == flat_rows.size, "rows not distinct"
    e = idx.reshape(-1)
    assert np.all(flat_rows >= offsets[e]) and np.all(flat_rows < offsets[e] + counts[e])
    for ex in range(n):  # stable: rows follow (token, slot) order inside each group
        r = flat_rows[e == ex]
        assert np.all(np.diff(r) == 1) if r.size else True


def oracle_outputs(x, Wg, W1, W3, W2, n, K, tokens, idx_gpu, exempt):
    """Oracle block outputs (float64, rounded once to the output dtype) for `tokens`; exempt
    tokens are evaluated with the admissible expert set the GPU chose."""
    dt = oracle.BF16 if x.dtype == torch.bfloat16 else oracle.F32
    y, _, _ = oracle.moe_forward(x, Wg, W1, W3, W2, n, K, tokens=tokens)
    ex = set(exempt)
    for r, t in enumerate(tokens):
        if int(t) in ex:
            y[r] = oracle.moe_token_with_experts(x, Wg, W1, W3, W2, n, int(t), idx_gpu[int(t)])
    return oracle.round_array(y, dt)


def compare_outputs(out_gpu: np.ndarray, ref: np.ndarray, dtype, stacked: bool = False) -> dict:
    """stacked=True: the residual stream of stacked blocks grows past the magnitudes the
    absolute bar was set for, so each element may also differ by 2^-7 |ref| (two bf16 ulps)
    on top of 2e-2; the relative L2 bar is unchanged."""
    err = out_gpu.astype(np.float64) - ref
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)) if err.size else 0.0
    if dtype == torch.bfloat16 and stacked:
        ok = bool(np.all(np.abs(err) <= BF16_MAX_ABS + 2.0 ** -7 * np.abs(ref))) and \
            rel_l2 <= BF16_REL_L2
    elif dtype == torch.bfloat16:
        ok = max_abs <= BF16_MAX_ABS and rel_l2 <= BF16_REL_L2
    else:
        ok = rel_l2 <= F32_REL and max_abs <= F32_REL * max(float(np.max(np.abs(ref))), 1e-30)
    return {"max_abs": max_abs, "rel_l2": rel_l2, "ok": ok}


def sample_tokens(T: int, idx: np.ndarray, exempt, n: int, budget: int, seed: int = 0,
                  rows=None, offsets=None, counts=None, tile: int = 128):
    """All tokens if T <= budget; else a seeded sample covering the first and last token,
    every exempt token, every expert pair present (first token of each pair), and -- when the
    grouping (token_rows, offsets, counts) is given -- one token in every `tile`-row tile of
    every expert's group plus the token of each group's last row (the tail tile), so that
    every GEMM tile of the permuted layout has a checked output row.  Topped up with random
    tokens to `budget`."""
    if T <= budget:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    chosen = {0, T - 1, *[int(t) for t in exempt]}
    if rows is not None:
        rows = np.asarray(rows).reshape(T, -1)
        offsets = np.asarray(offsets)
        counts = np.asarray(counts)
        row_tok = np.full(int(offsets[-1]) + 1, -1, np.int64)
        flat = rows.reshape(-1)
        row_tok[flat] = np.repeat(np.arange(T), rows.shape[1])
        for e in range(len(counts)):
            c = int(counts[e])
            if c == 0:
                continue
            first = int(offsets[e])
            for r in list(range(first, first + c, tile)) + [first + c - 1]:
                chosen.add(int(row_tok[r]))
    seen = {}
    for t in range(T):
        key = tuple(sorted(idx[t].tolist()))
        if key not in seen:
            seen[key] = t
    for t in seen.values():
        chosen.add(int(t))
    while len(chosen) < budget:
        chosen.add(int(rng.integers(0, T)))
    return np.array(sorted(chosen))


# Parity results of the GPU tests, printed in pytest's terminal summary (tests/conftest.py)
# so that exempt-token counts and errors appear in every run's log, pass or fail.
REPORTS: list[tuple[str, dict]] = []


def record(name: str, rep: dict):
    REPORTS.append((name, {k: rep[k] for k in ("tokens", "exempt", "max_abs", "rel_l2", "ok")
                           if k in rep}))


def plain_scales(sf_tile, rows, cols):
    """MXFP8 block scales from the library's tile order (include/moe.h: the code of row r,
    elements [32c, 32c + 32) at byte ((r / 128) (cols / 128) + c / 4) 512 + 16 (r % 32)
    + 4 ((r % 128) / 32) + c % 4) to the oracle's plain [rows][cols / 32]."""
    r = np.arange(rows)[:, None]
    c = np.arange(cols // 32)[None, :]
    at = ((r // 128) * (cols // 128) + c // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + c % 4
    return np.asarray(sf_tile).reshape(-1)[at]
