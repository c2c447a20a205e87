"""Pins of the fp64 oracle against facts fixed outside the oracle itself:
hand-worked examples, closed forms, brute force on tiny inputs, special cases
that reduce to plain causal attention, and algebraic identities.  CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rs(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- rounding


def test_round_bf16_matches_torch_on_fp32_values():
    x = _rs(0).standard_normal(200000) * np.exp(_rs(1).uniform(-30, 30, 200000))
    x = x.astype(np.float32).astype(np.float64)            # exactly representable in fp32
    want = torch.from_numpy(x).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_bf16(x), want)


def test_round_bf16_ties_and_single_rounding():
    one = 1.0
    assert O.round_bf16(one + 2 ** -8) == 1.0                    # tie -> even
    assert O.round_bf16(one + 3 * 2 ** -8) == one + 2 ** -6      # tie -> even (up)
    assert O.round_bf16(one + 2 ** -8 + 2 ** -30) == one + 2 ** -7   # no double rounding via fp32
    assert O.round_bf16(-(one + 2 ** -8 + 2 ** -30)) == -(one + 2 ** -7)
    assert O.round_bf16(2.0 ** -133 * 0.75) == 2.0 ** -133       # subnormal spacing
    assert np.isinf(O.round_bf16(3.4e38))
    assert O.round_store(1 + 2 ** -30, "f32") == 1.0


# --------------------------------------------------------------------------- S1 compression


def test_compress_worked_examples():
    g = json.load(open(os.path.join(GOLDEN, "worked_compress.json")))
    x = np.array(g["x"], dtype=np.float64)
    for case in g["cases"]:
        z = np.log(np.array(case["a"], dtype=np.float64))
        b = np.log(np.array(case["c"], dtype=np.float64))
        n = x.shape[0] // case["r"]
        (got,) = O.compress([x], z, b, case["r"], case["overlap"], 0, n, "f32")
        want = np.array([[float(Fraction(v)) for v in row] for row in case["expected"]])
        np.testing.assert_allclose(got, want, rtol=1e-6, err_msg=case["name"])


@pytest.mark.parametrize("r,overlap", [(4, True), (128, False), (3, True), (5, False)])
def test_compress_equal_logits_zero_bias_is_window_mean(r, overlap):
    L, C = 40 * r, 6
    x = _rs(2).standard_normal((L, C))
    z = np.full(L, 0.37)
    span = 2 * r if overlap else r
    (got,) = O.compress([x], z, np.zeros(span), r, overlap, 0, L // r, "f32")
    for j in range(L // r):
        lo = max(0, (j - 1) * r) if overlap else j * r
        np.testing.assert_allclose(got[j], x[lo:(j + 1) * r].mean(axis=0), rtol=1e-6, atol=1e-7)


def test_compress_ratio_one_without_overlap_is_identity():
    x = _rs(3).standard_normal((64, 8)).astype(np.float32).astype(np.float64)
    (got,) = O.compress([x], _rs(4).standard_normal(64), _rs(5).standard_normal(1), 1, False, 0, 64, "f32")
    np.testing.assert_array_equal(got, x)


def test_compress_identical_rows_pool_to_that_row():
    r, L = 4, 64
    row = _rs(6).standard_normal(16).astype(np.float32).astype(np.float64)
    x = np.tile(row, (L, 1))
    (got,) = O.compress([x], _rs(7).standard_normal(L) * 5, _rs(8).standard_normal(2 * r), r, True, 0, L // r, "f32")
    np.testing.assert_allclose(got, np.tile(row, (L // r, 1)), rtol=1e-6)


def test_compress_bias_is_indexed_by_position_in_unclipped_window():
    r, L = 4, 32
    x = np.arange(L, dtype=np.float64)[:, None] * np.ones((1, 3))
    bias = np.zeros(2 * r)
    bias[r + 1] = 60.0                                   # one dominant window position
    (got,) = O.compress([x], np.zeros(L), bias, r, True, 0, L // r, "f32")
    # window of entry j starts at (j-1)r, so position r+1 is token j*r+1 (entry 0 included)
    np.testing.assert_allclose(got[:, 0], np.arange(L // r) * r + 1, rtol=0, atol=1e-12 * L)
    bias_h = np.zeros(r)
    bias_h[2] = 60.0
    (got_h,) = O.compress([x], np.zeros(L), bias_h, r, False, 0, L // r, "f32")
    np.testing.assert_allclose(got_h[:, 0], np.arange(L // r) * r + 2, atol=1e-12 * L)


def test_compress_weights_normalised_and_shift_invariant():
    r, L = 4, 48
    z = _rs(9).standard_normal(L) * 3
    b = _rs(10).standard_normal(2 * r)
    for j in range(L // r):
        _, w = O.pooling_weights(z, b, j, r, True)
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(w > 0)
    x = _rs(11).standard_normal((L, 5))
    (a,) = O.compress([x], z, b, r, True, 0, L // r, "f32")
    (c,) = O.compress([x], z + 123.0, b - 7.0, r, True, 0, L // r, "f32")
    np.testing.assert_allclose(a, c, rtol=1e-6, atol=1e-7)
    (h,) = O.compress([x], z * 0 + 1000.0 * (np.arange(L) % r == 3), np.zeros(r), r, False, 0, L // r, "f32")
    np.testing.assert_allclose(h, x[3::r].astype(np.float32), rtol=1e-6)   # huge logit: no overflow


def test_compress_same_weights_for_all_tensors_and_chunking():
    r, L = 4, 4 * 50
    xs = [_rs(12 + i).standard_normal((L, 4)) for i in range(3)]
    z, b = _rs(20).standard_normal(L), _rs(21).standard_normal(2 * r)
    full = O.compress(xs, z, b, r, True, 0, L // r, "f32", chunk=7)
    for j in (0, 1, 17, 49):
        s, w = O.pooling_weights(z, b, j, r, True)
        for x, out in zip(xs, full):
            np.testing.assert_allclose(out[j], (w[:, None] * x[s]).sum(0), rtol=1e-6, atol=1e-7)
    part = O.compress(xs, z, b, r, True, 10, 20, "f32")
    for a, c in zip(full, part):
        np.testing.assert_array_equal(a[10:20], c)


# --------------------------------------------------------------------------- S2a flat indexer


def _brute_topk(scores, k):
    n = len(scores)
    keep = []
    for j in range(n):
        rank = sum(1 for i in range(n) if scores[i] > scores[j] or (scores[i] == scores[j] and i < j))
        if rank < k:
            keep.append(j)
    return sorted(keep)


@pytest.mark.parametrize("seed", range(6))
def test_flat_topk_matches_rank_definition_with_ties(seed):
    rs = _rs(100 + seed)
    n, d, k = 60, 4, 9
    ic = rs.integers(-2, 3, (n, d)).astype(np.float64)   # small integers: many exact ties
    q = rs.integers(-2, 3, d).astype(np.float64)
    for n_vis in (0, 5, 9, 10, 37, 60):
        got = O.flat_topk(q, ic, n_vis, k)
        valid = sorted(int(v) for v in got if v >= 0)
        assert valid == _brute_topk(ic[:n_vis] @ q, k)
        assert list(got[len(valid):]) == [-1] * (k - len(valid))
        assert len(valid) == min(k, n_vis)


def test_visibility_boundaries():
    for j in range(0, 50):
        assert O.visible_entries(4 * j + 3, 4, 10 ** 9) == j + 1      # entry j complete at its last token
        assert O.visible_entries(4 * j + 2, 4, 10 ** 9) == j
    assert O.visible_entries(126, 128, 10 ** 9) == 0
    assert O.visible_entries(127, 128, 10 ** 9) == 1
    assert O.visible_entries(10 ** 6, 4, 77) == 77


def test_page_settings_and_scale_of_hca_cache():
    g = json.load(open(os.path.join(GOLDEN, "page_settings.json")))
    cfg = W.configs
    assert cfg.HCA128.r == g["hca_ratio"]["value"] and not cfg.HCA128.overlap
    for w in cfg.ALL[1:]:
        assert w.W == g["window"]["value"]
        assert w.layer("csa").r == g["csa_ratio"]["value"]
    h = cfg.PREFILL_128K.layer("csa")
    assert (h.block, h.top_m, h.k, h.q_chunk) == tuple(g["hisa"][k] for k in ("block", "top_m", "top_k", "q_chunk"))
    n_1m = O.visible_entries((1 << 20) - 1, 128, 10 ** 9)
    assert n_1m == 8192 and abs(n_1m - g["hca_entries_at_1m"]["approx"]) / 8000 < 0.05


# --------------------------------------------------------------------------- S2b HISA


@pytest.mark.parametrize("seed", range(4))
def test_hisa_with_all_blocks_equals_flat(seed):
    rs = _rs(200 + seed)
    n_c, d, B, k = 300, 8, 16, 25
    ic = rs.standard_normal((n_c, d))
    reps = O.block_reps(ic, B, "f32")
    for _ in range(20):
        q = rs.standard_normal(d)
        n_vis = int(rs.integers(0, n_c + 1))
        m = n_vis // B + 1
        np.testing.assert_array_equal(O.hisa_topk(q, ic, reps, n_vis, B, m, k), O.flat_topk(q, ic, n_vis, k))


def test_hisa_block_size_one_equals_flat():
    rs = _rs(210)
    ic = rs.standard_normal((120, 6))
    reps = O.block_reps(ic, 1, "f32")
    np.testing.assert_array_equal(reps, ic.astype(np.float32))
    ic32 = ic.astype(np.float32).astype(np.float64)
    for _ in range(20):
        q = rs.standard_normal(6)
        n_vis = int(rs.integers(0, 121))
        for m in (10, 17):
            np.testing.assert_array_equal(O.hisa_topk(q, ic32, reps, n_vis, 1, m, 10), O.flat_topk(q, ic32, n_vis, 10))


def test_hisa_worked_example_differs_from_flat():
    # 3 full blocks of B=2 (1-d keys).  Block means: 5, 0, -1.  The best single
    # entry (score 9) sits in block 2 whose mean is the lowest.
    ic = np.array([[5.0], [5.0], [1.0], [-1.0], [9.0], [-11.0]])
    reps = O.block_reps(ic, 2, "f32")
    np.testing.assert_array_equal(reps[:, 0], [5.0, 0.0, -1.0])
    q = np.array([1.0])
    assert list(O.hisa_blocks(q, reps, 6, 2, 1)) == [0]
    assert sorted(O.hisa_topk(q, ic, reps, 6, 2, 1, 2)) == [0, 1]
    assert sorted(O.flat_topk(q, ic, 6, 2)) == [1, 4] or sorted(O.flat_topk(q, ic, 6, 2)) == [0, 4]
    assert sorted(O.flat_topk(q, ic, 6, 2)) == [0, 4]                # tie 5 = 5 -> lower index
    # 5 visible entries: blocks 0,1 full, block 2 partial (entry 4 only) and always kept
    assert list(O.hisa_blocks(q, reps, 5, 2, 2)) == [0, 2]
    assert sorted(O.hisa_topk(q, ic, reps, 5, 2, 2, 2)) == [0, 4]
    assert list(O.hisa_blocks(-q, reps, 5, 2, 1)) == [2]            # m=1: only the partial block
    assert list(O.hisa_blocks(-q, reps, 5, 2, 2)) == [1, 2]


def test_block_reps_of_constant_blocks():
    B, nb = 8, 5
    vals = np.arange(nb, dtype=np.float64) * 1.5 - 2
    ic = np.repeat(vals, B)[:, None] * np.ones((1, 3))
    ic = np.vstack([ic, np.full((3, 3), 99.0)])          # a trailing partial block has no representative
    reps = O.block_reps(ic, B, "bf16")
    assert reps.shape == (nb, 3)
    np.testing.assert_array_equal(reps[:, 0], O.round_bf16(vals))


# --------------------------------------------------------------------------- S3 attention


def _causal_mqa(q, k, v, scale):
    """Plain causal MQA in matrix form: q [T,H,D], k/v [T,D]."""
    T = q.shape[0]
    s = np.einsum("thd,jd->thj", q, k) * scale
    mask = np.arange(T)[None, :] > np.arange(T)[:, None]
    s = np.where(mask[:, None, :], -np.inf, s)
    p = np.exp(s - s.max(axis=2, keepdims=True))
    p /= p.sum(axis=2, keepdims=True)
    lse = np.log(np.exp(s - s.max(axis=2, keepdims=True)).sum(axis=2)) + s.max(axis=2)
    return np.einsum("thj,jd->thd", p, v), lse


def _rows(p, q, qi, kc, vc, ic, reps, kw, vw, ring, pos):
    res = [O.layer_row(p, q[i], None if qi is None else qi[i], int(pos[i]), kc, vc, ic, reps, kw, vw, ring) for i in range(len(pos))]
    return np.stack([r[1] for r in res]), np.stack([r[2] for r in res])


def _f32(a):
    return a.astype(np.float32).astype(np.float64)


def test_ratio_one_full_topk_no_window_is_dense_causal_mqa():
    rs = _rs(300)
    T, H, D = 40, 4, 16
    xk, xv, q = _f32(rs.standard_normal((T, D))), _f32(rs.standard_normal((T, D))), rs.standard_normal((T, H, D))
    xi, qi = rs.standard_normal((T, 8)), rs.standard_normal((T, 8))
    z = rs.standard_normal(T)
    scale = 1 / math.sqrt(D)
    want_o, want_l = _causal_mqa(q, xk, xv, scale)
    p = O.LayerParams("csa", r=1, overlap=False, W=0, scale=scale, dtype="f32", k=T)
    kc, vc, ic = O.build_caches(p, xk, xv, xi, z, np.zeros(1))
    o, l = _rows(p, q, qi, kc, vc, ic, None, xk, xv, T, np.arange(T))
    np.testing.assert_allclose(o, want_o, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(l, want_l, rtol=1e-6, atol=1e-6)
    ph = O.LayerParams("hca", r=1, overlap=False, W=0, scale=scale, dtype="f32")
    kc, vc, _ = O.build_caches(ph, xk, xv, None, z, np.zeros(1))
    o, l = _rows(ph, q, qi, kc, vc, None, None, xk, xv, T, np.arange(T))
    np.testing.assert_allclose(o, want_o, rtol=1e-5, atol=1e-6)


def test_no_selection_full_window_is_causal_attention_and_union_counts_twice():
    rs = _rs(301)
    T, H, D = 33, 3, 8
    xk, xv, q = _f32(rs.standard_normal((T, D))), _f32(rs.standard_normal((T, D))), rs.standard_normal((T, H, D))
    scale = 0.3
    want_o, want_l = _causal_mqa(q, xk, xv, scale)
    p = O.LayerParams("csa", r=4, overlap=True, W=T, scale=scale, dtype="f32", k=0)
    kc, vc, ic = O.build_caches(p, xk, xv, xk, rs.standard_normal(T), rs.standard_normal(8))
    o, l = _rows(p, q, q[:, 0], kc, vc, ic, None, xk, xv, T, np.arange(T))
    np.testing.assert_allclose(o, want_o, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(l, want_l, rtol=1e-6, atol=1e-6)
    # HCA with r=1: every raw token is both a compressed entry and a window key.
    ph = O.LayerParams("hca", r=1, overlap=False, W=T, scale=scale, dtype="f32")
    kc, vc, _ = O.build_caches(ph, xk, xv, None, np.zeros(T), np.zeros(1))
    o, l = _rows(ph, q, None, kc, vc, None, None, xk, xv, T, np.arange(T))
    np.testing.assert_allclose(o, want_o, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(l, want_l + math.log(2), rtol=1e-6, atol=1e-6)


def test_attend_split_merge_identity_and_closed_forms():
    rs = _rs(302)
    H, D, n = 5, 12, 30
    q, k, v = rs.standard_normal((H, D)), rs.standard_normal((n, D)), rs.standard_normal((n, D))
    o, l = O.attend(q, k, v, 0.7)
    o1, l1 = O.attend(q, k[:11], v[:11], 0.7)
    o2, l2 = O.attend(q, k[11:], v[11:], 0.7)
    lm = np.logaddexp(l1, l2)
    om = (o1 * np.exp(l1 - lm)[:, None] + o2 * np.exp(l2 - lm)[:, None])
    np.testing.assert_allclose(o, om, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l, lm, rtol=1e-12)
    o0, l0 = O.attend(np.zeros((H, D)), k, v, 0.7)
    np.testing.assert_allclose(o0, np.tile(v.mean(0), (H, 1)), rtol=1e-12)
    np.testing.assert_allclose(l0, np.full(H, math.log(n)), rtol=1e-12)
    o1k, l1k = O.attend(q, k[:1], v[:1], 0.7)
    np.testing.assert_allclose(o1k, np.tile(v[0], (H, 1)), rtol=1e-12)
    np.testing.assert_allclose(l1k, 0.7 * q @ k[0], rtol=1e-12)


def test_decode_ring_row_equals_prefill_row():
    rs = _rs(303)
    L, H, D, dI, Wn = 300, 4, 16, 8, 24
    xk, xv, xi = (_f32(rs.standard_normal((L, c))) for c in (D, D, dI))
    z, q, qi = rs.standard_normal(L), rs.standard_normal((L, H, D)), rs.standard_normal((L, dI))
    for p in (O.LayerParams("csa", 4, True, Wn, 0.25, "f32", k=7),
              O.LayerParams("csa", 4, True, Wn, 0.25, "f32", k=7, index_mode="hisa", block=8, top_m=3),
              O.LayerParams("hca", 16, False, Wn, 0.25, "f32")):
        bias = rs.standard_normal(2 * p.r if p.overlap else p.r)
        kc, vc, ic = O.build_caches(p, xk, xv, xi, z, bias)
        reps = O.block_reps(ic, p.block, "f32") if p.kind == "csa" else None
        for t in (0, 5, 23, 24, 150, 299):
            a = O.layer_row(p, q[t], qi[t], t, kc, vc, ic, reps, xk, xv, L)
            # decode: ring of Wn slots holding positions t-Wn+1..t at slot s mod Wn
            ring_k, ring_v = np.zeros((Wn, D)), np.zeros((Wn, D))
            for s in range(max(0, t - Wn + 1), t + 1):
                ring_k[s % Wn], ring_v[s % Wn] = xk[s], xv[s]
            n_c = (t + 1) // p.r
            ic_t = ic[:n_c] if ic is not None else None
            reps_t = O.block_reps(ic_t, p.block, "f32") if p.kind == "csa" else None
            b = O.layer_row(p, q[t], qi[t], t, kc[:n_c], vc[:n_c], ic_t, reps_t, ring_k, ring_v, Wn)
            if a[0] is not None:
                np.testing.assert_array_equal(a[0], b[0])
            np.testing.assert_allclose(a[1], b[1], rtol=1e-12)
            np.testing.assert_allclose(a[2], b[2], rtol=1e-12)


# --------------------------------------------------------------------------- workloads


def test_planted_keys_are_selected_by_the_oracle():
    w = W.configs.scaled(W.configs.PREFILL_32K, L=2048, T=2048, plant_frac=0.02)
    ly = w.layer("csa")
    raw, qs = W.make.make_raw(w), W.make.make_queries(w)
    js = W.make.plant_prefill(w, ly, raw, qs)
    bias = W.make.make_bias(w, ly)
    np64 = lambda t: t[0].double().numpy()
    p = O.LayerParams("csa", ly.r, ly.overlap, w.W, w.D ** -0.5, w.dtype, k=ly.k)
    kc, vc, ic = O.build_caches(p, np64(raw["xk"]), np64(raw["xv"]), np64(raw["xi"]), np64(raw["z"]), bias.double().numpy())
    qi = np64(qs["qi"])
    u = ic[js]
    assert np.allclose(np.linalg.norm(u, axis=1), 1.0, atol=2e-2)      # pooled planted key = u_j
    hits = 0
    for j in js.tolist():
        cos = (qi @ ic[j]) / np.linalg.norm(qi, axis=1) / np.linalg.norm(ic[j])
        rows = np.nonzero(np.abs(cos - 0.5) < 0.02)[0]
        for t in rows[:8]:
            t = int(t)
            if O.visible_entries(t, 4, ic.shape[0]) > j:
                idx = O.flat_topk(qi[t], ic, O.visible_entries(t, 4, ic.shape[0]), ly.k)
                assert j in idx
                hits += 1
    assert hits > 20


# --------------------------------------------------------------------------- decode-step state update


def test_decode_append_token_by_token_equals_full_sequence_build():
    """Appending a sequence one token at a time (rings of 128, a CSA entry every 4
    tokens, an HCA entry every 128, a representative every 4 CSA entries) leaves the
    same caches and representatives as S1 over the whole sequence, and the rings hold
    the last 128 raw rows at slot s mod 128."""
    rs = _rs(11)
    L, D, dI, ring, B = 600, 16, 8, 128, 4
    xk, xv, xi = rs.normal(size=(L, D)), rs.normal(size=(L, D)), rs.normal(size=(L, dI))
    z = rs.normal(size=L)
    csa = O.LayerParams("csa", 4, True, ring, 0.25, "f32")
    hca = O.LayerParams("hca", 128, False, ring, 0.25, "f32")
    biases = {"csa": 0.1 * rs.normal(size=8), "hca": 0.1 * rs.normal(size=128)}
    st = O.DecodeState(ring, D, dI, (csa, hca), B, "f32")
    for t in range(L):
        O.decode_append(st, xk[t], xv[t], xi[t], z[t], biases)
    kc, vc, ic = O.build_caches(csa, xk, xv, xi, z, biases["csa"])
    kh, vh, _ = O.build_caches(hca, xk, xv, None, z, biases["hca"])
    assert len(st.kc["csa"]) == L // 4 and len(st.kc["hca"]) == L // 128 and len(st.reps) == (L // 4) // B
    for got, want in ((st.kc["csa"], kc), (st.vc["csa"], vc), (st.ic, ic), (st.kc["hca"], kh), (st.vc["hca"], vh),
                      (st.reps, O.block_reps(ic, B, "f32"))):
        got = np.array(got)
        assert got.shape == want.shape and np.all(np.isfinite(got))
        np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-7)
    pos = np.arange(L - ring, L)
    np.testing.assert_array_equal(st.kw[pos % ring], xk[pos])
    np.testing.assert_array_equal(st.zw[pos % ring], z[pos])


# --------------------------------------------------------------------------- per-channel compression weights


@pytest.mark.parametrize("r,overlap", [(4, True), (128, False), (3, True)])
def test_compress_per_channel_with_equal_channels_is_scalar_compress(r, overlap):
    """Every channel given the same logit and bias reduces to the scalar-weight S1."""
    rs = _rs(21)
    L, C = 7 * r + 5, 12
    x = rs.normal(size=(L, C))
    z1 = rs.normal(size=L)
    b1 = 0.3 * rs.normal(size=2 * r if overlap else r)
    zc, bc = np.repeat(z1[:, None], C, axis=1), np.repeat(b1[:, None], C, axis=1)
    got = O.compress_per_channel(x, zc, bc, r, overlap, 0, L // r, "f32")
    want = O.compress([x], z1, b1, r, overlap, 0, L // r, "f32")[0]
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-7)


def test_compress_per_channel_channels_are_independent():
    """Channel c depends only on column c of x, z and bias: each channel equals the
    scalar S1 run on that channel alone."""
    rs = _rs(22)
    r, L, C = 4, 41, 5
    x, z, b = rs.normal(size=(L, C)), rs.normal(size=(L, C)), 0.5 * rs.normal(size=(8, C))
    got = O.compress_per_channel(x, z, b, r, True, 0, L // r, "f32")
    for c in range(C):
        want = O.compress([x[:, c:c + 1]], z[:, c], b[:, c], r, True, 0, L // r, "f32")[0][:, 0]
        np.testing.assert_allclose(got[:, c], want, rtol=1e-6, atol=1e-7)


# --------------------------------------------------------------------------- real K/V reading of CSA attention


def _dense_causal(q_t, xk, xv, t, scale):
    """Plain causal attention of query t over raw positions 0..t, one head at a time."""
    H = q_t.shape[0]
    o, lse = np.empty((H, xk.shape[1])), np.empty(H)
    for h in range(H):
        s = [float(q_t[h] @ xk[j]) * scale for j in range(t + 1)]
        m = max(s)
        e = [math.exp(v - m) for v in s]
        den = sum(e)
        o[h] = sum(e[j] * xv[j] for j in range(t + 1)) / den
        lse[h] = m + math.log(den)
    return o, lse


@pytest.mark.parametrize("r,W", [(4, 8), (4, 0), (1, 3), (3, 64)])
def test_real_kv_with_every_entry_selected_is_dense_causal_attention(r, W):
    """Selecting every visible entry covers raw tokens 0 .. r*V-1, the window covers
    the rest up to t: the real-K/V key set is exactly positions 0..t once each."""
    rs = _rs(31)
    L, H, D = 50, 3, 8
    xk, xv, q = rs.normal(size=(L, D)), rs.normal(size=(L, D)), rs.normal(size=(L, H, D))
    for t in (0, 3, 17, 49):
        n_vis = (t + 1) // r
        pos = O.real_kv_positions(t, np.arange(n_vis), r, W)
        if r * n_vis + W >= t + 1:
            np.testing.assert_array_equal(pos, np.arange(t + 1))
            keys, vals = O.key_set_real_kv(t, np.arange(n_vis), r, xk, xv, L, W)
            o, lse = O.attend(q[t], keys, vals, 0.5)
            o2, lse2 = _dense_causal(q[t], xk, xv, t, 0.5)
            np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse, lse2, rtol=1e-12, atol=1e-12)


def test_real_kv_positions_by_brute_force():
    """Tokens of the selected entries, minus nothing, plus the window, as a set."""
    rs = _rs(32)
    for _ in range(50):
        r, W = int(rs.integers(1, 6)), int(rs.integers(0, 20))
        t = int(rs.integers(0, 200))
        n_vis = (t + 1) // r
        sel = rs.choice(max(n_vis, 1), size=min(n_vis, int(rs.integers(0, 8))), replace=False) if n_vis else []
        sel = np.concatenate([np.asarray(sel, dtype=np.int64), [-1, -1]])
        want = set()
        for j in sel:
            if j >= 0:
                want |= set(range(j * r, j * r + r))
        want |= set(range(max(0, t - W + 1), t + 1))
        assert O.real_kv_positions(t, sel, r, W).tolist() == sorted(want)
        assert all(p <= t for p in want)
