"""Host checks of the figures bench.py derives from kernel outputs: the selection
IoU and planted-key recall it reports for the indexers, and the attention flop
count its roofline divides by.  Each is compared with a direct restatement of
its definition (sets for the IoU, the oracle's key-set sizes for the flops)."""
import types

import numpy as np
import pytest
import torch

import bench
import oracle as O


def _rows_with_padding(rng, R, k, n):
    out = np.full((R, k), -1, dtype=np.int32)
    for i in range(R):
        m = int(rng.integers(0, k + 1))
        out[i, :m] = np.sort(rng.choice(n, size=m, replace=False))
    return out


def test_selection_iou_matches_set_definition():
    rng = np.random.default_rng(3)
    R, k, n = 200, 16, 40
    a, b = _rows_with_padding(rng, R, k, n), _rows_with_padding(rng, R, k, n)
    b[:5] = a[:5]                      # identical rows
    b[5] = -1                          # one side empty
    a[6] = -1
    b[6] = -1                          # both empty: counted as 0 overlap
    want = []
    for i in range(R):
        sa, sb = set(a[i][a[i] >= 0].tolist()), set(b[i][b[i] >= 0].tolist())
        u = len(sa | sb)
        want.append(len(sa & sb) / u if u else 0.0)
    got = bench.selection_iou(torch.from_numpy(a), torch.from_numpy(b))
    assert got == pytest.approx(float(np.mean(want)), abs=1e-6)
    full = a[(a >= 0).any(1)]           # a row compared with itself: 1 unless the row is empty
    assert bench.selection_iou(torch.from_numpy(full), torch.from_numpy(full)) == pytest.approx(1.0)


def test_planted_recall_counts_selected_planted_pairs():
    # four entries; entries 1 and 3 are planted.  Query 0 points at entry 1 (cosine 1),
    # query 1 at entry 3 (cosine 1), query 2 at neither (cosine 0 with both).
    ic = torch.tensor([[1.0, 0, 0], [0, 1.0, 0], [1.0, 1.0, 0], [0, 0, 1.0]])
    qi = torch.tensor([[0, 2.0, 0], [0, 0, 3.0], [1.0, 0, 0]])
    planted = [1, 3]
    # query 0 selected entry 1; query 1 did not select entry 3
    idx = torch.tensor([[1, 2], [0, 2], [0, -1]], dtype=torch.int32)
    assert bench.planted_recall(idx, qi, ic, planted) == pytest.approx(0.5)
    idx[1, 1] = 3
    assert bench.planted_recall(idx, qi, ic, planted) == pytest.approx(1.0)
    assert np.isnan(bench.planted_recall(idx, qi, ic, []))


@pytest.mark.parametrize("kind,r,k,W,n_c", [("csa", 4, 8, 5, 30), ("hca", 16, 0, 7, 9), ("csa", 1, 3, 0, 100)])
def test_attention_flops_equal_the_oracle_key_sets(kind, r, k, W, n_c):
    H, D = 3, 5
    w = types.SimpleNamespace(H=H, D=D, W=W)
    ly = types.SimpleNamespace(kind=kind, r=r, k=k)
    q_pos = np.array([0, 1, 3, 17, 40, 63, 64, 200])
    keys = 0
    for t in q_pos.tolist():
        vis = O.visible_entries(t, r, n_c)
        comp = min(k, vis) if kind == "csa" else vis
        keys += comp + len(O.window_positions(t, W)) if W > 0 else comp
    assert bench.attention_flops(w, ly, q_pos, n_c) == 4.0 * H * D * keys
