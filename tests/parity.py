"""Comparison rules shared by the GPU parity tests.

Outputs: fp32 workloads within 1e-4 max-abs; bf16 workloads within 2e-2
max-abs and 5e-3 relative L2.  Top-k sets: identical wherever the oracle's
k-th and (k+1)-th scores differ by more than 1e-3 relative, IoU >= 0.999
overall, and every selected entry consistent with the oracle's fp64 scores up
to the fp32 accumulation error bound of the GPU's dot products.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

FP32_MAX_ABS = 1e-4
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
GAP_REL = 1e-3
IOU_MIN = 0.999


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else \
        t.detach().cpu().double().numpy()


def check_close(got, want, dtype: str, what: str):
    got, want = np.asarray(got, dtype=np.float64), np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    if dtype == "f32":
        assert max_abs <= FP32_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {FP32_MAX_ABS}"
        return {"max_abs": max_abs}
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert max_abs <= BF16_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
    assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return {"max_abs": max_abs, "rel_l2": rel, "max_abs_over_max": max_abs / max(float(np.abs(want).max()), 1e-30)}


def acc_bound(q: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Bound on |fp32 dot - exact dot| for bf16/fp32 operands: 2 n u sum|q_e k_e|."""
    n = q.shape[-1]
    return 2.0 * n * 2.0 ** -24 * (np.abs(keys) @ np.abs(q))


def topk_row_check(got: np.ndarray, scores: np.ndarray, ids: np.ndarray, k: int, eps: np.ndarray,
                   what: str):
    """Checks one GPU idx row against oracle scores of the candidate ids.

    Returns (iou, exact_required)."""
    n = len(ids)
    valid = got[got >= 0]
    assert np.all(got[len(valid):] == -1), f"{what}: -1 padding not at the end"
    assert len(valid) == min(k, n), f"{what}: {len(valid)} selected, want {min(k, n)}"
    assert np.all(np.diff(valid) > 0), f"{what}: selection not strictly ascending"
    want = O.select_topk(scores, ids, k)
    want_set = set(int(v) for v in want if v >= 0)
    got_set = set(int(v) for v in valid)
    assert got_set <= set(int(v) for v in ids), f"{what}: selected a non-candidate"
    if n <= k:
        assert got_set == want_set, f"{what}: all candidates must be selected"
        return 1.0, True
    order = np.lexsort((ids, -scores))
    s_k, s_k1 = scores[order[k - 1]], scores[order[k]]
    exact = (s_k - s_k1) > GAP_REL * max(abs(s_k), abs(s_k1))
    if exact:
        assert got_set == want_set, f"{what}: set differs although the k-th gap is {s_k - s_k1:.3e}"
    pos = {int(j): i for i, j in enumerate(ids)}
    for j in got_set - want_set:      # a swapped-in entry must be tied with the k-th within the bound
        i = pos[j]
        assert scores[i] >= s_k - eps[i] - eps[order[k - 1]], f"{what}: entry {j} is not a near-tie"
    for j in want_set - got_set:
        i = pos[j]
        assert scores[i] <= s_k + eps[i] + eps[order[k - 1]], f"{what}: dropped entry {j} is not a near-tie"
    inter = len(got_set & want_set)
    return inter / len(got_set | want_set), exact


def sample_rows(T: int, n: int, seed: int, extra=()) -> np.ndarray:
    """First/last rows, a seeded spread of the rest, plus the given rows."""
    rs = np.random.default_rng(seed)
    base = set(range(min(16, T))) | set(range(max(0, T - 16), T)) | set(int(x) for x in extra if 0 <= x < T)
    if T > len(base):
        base |= set(rs.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(base))
