"""GPU parity of each libhyb stage against the fp64 oracle on identical seeded
inputs: several tiles plus ragged tails, both storage types, edge cases
(nothing visible, fewer candidates than k, partial HISA blocks, split-KV)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import make, rng

from parity import (acc_bound, check_close, to64, topk_row_check)

pytestmark = pytest.mark.gpu

dev = "cuda"


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_hyb_b200 as S
    S.abi.lib()
    return S


@pytest.fixture(autouse=True)
def _status_clean(S):
    S.abi.hyb_get_device_status()
    yield
    assert S.abi.hyb_get_device_status() == 0


def _normal(name, shape, std, dtype, seed=1):
    return make.normal_tensor(seed, name, shape, std, dtype)


def _ulp_bf16(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


# --------------------------------------------------------------------------- S1


@pytest.mark.parametrize("dtype,B,L,D,dI,r,overlap,j0,j1", [
    ("f32", 1, 512, 64, 32, 4, True, 0, 128),
    ("f32", 1, 512, 64, 32, 128, False, 0, 4),
    ("bf16", 2, 1003, 128, 128, 4, True, 0, 250),
    ("bf16", 2, 1003, 128, 64, 4, True, 37, 201),
    ("bf16", 3, 1000, 128, 128, 128, False, 0, 7),
    ("bf16", 1, 777, 96, 32, 3, True, 0, 259),
])
def test_compress(S, dtype, B, L, D, dI, r, overlap, j0, j1):
    sc = 1.0 if dtype == "f32" else 128 ** -0.5
    xk, xv = _normal("k", (B, L, D), sc, dtype), _normal("v", (B, L, D), sc, dtype)
    xi = _normal("i", (B, L, dI), sc, dtype) if overlap else None
    z = _normal("z", (B, L), 1.0, "f32")
    bias = _normal("b", (2 * r if overlap else r,), 0.1, "f32")
    nc = L // r
    kc = torch.zeros(B, nc, D, dtype=xk.dtype, device=dev)
    vc, ic = torch.zeros_like(kc), (torch.zeros(B, nc, dI, dtype=xk.dtype, device=dev) if overlap else None)
    g = lambda t: None if t is None else t.to(dev)
    S.abi.hyb_compress(g(xk), g(xv), g(xi), g(z), g(bias), r, overlap, j0, j1, kc, vc, ic)
    torch.cuda.synchronize()
    for b in range(B):
        xs = [to64(xk[b]), to64(xv[b])] + ([to64(xi[b])] if overlap else [])
        want = O.compress(xs, to64(z[b]), to64(bias), r, overlap, j0, j1, dtype)
        got = [kc[b, j0:j1], vc[b, j0:j1]] + ([ic[b, j0:j1]] if overlap else [])
        for gt, wt, nm in zip(got, want, "kvi"):
            g64 = to64(gt)
            check_close(g64, wt, dtype, f"compress {nm} b={b}")
            if dtype == "bf16":   # one bf16 ulp from the fp64 result, plus the fp32 accumulation error
                slack = 2.0 ** -20 * max(1.0, float(np.abs(wt).max()))
                assert np.all(np.abs(g64 - wt) <= _ulp_bf16(wt) * 1.0001 + slack), f"{nm}: more than one ulp"
        assert torch.all(kc[b, :j0] == 0) and torch.all(kc[b, j1:] == 0)   # nothing outside the range


@pytest.mark.parametrize("dtype,B,L,D,dI,r,overlap,j0,j1", [
    ("f32", 1, 130, 64, 32, 4, True, 0, 32),
    ("bf16", 2, 3001, 128, 128, 4, True, 0, 750),
    ("bf16", 2, 3001, 128, 128, 4, True, 7, 301),     # ragged range
    ("bf16", 1, 1000, 128, 0, 128, False, 0, 7),      # HCA geometry, no indexer keys
])
def test_compress_per_channel(S, dtype, B, L, D, dI, r, overlap, j0, j1):
    sc = 1.0 if dtype == "f32" else 128 ** -0.5
    span = 2 * r if overlap else r
    xk, xv = _normal("pk", (B, L, D), sc, dtype), _normal("pv", (B, L, D), sc, dtype)
    xi = _normal("pi", (B, L, dI), sc, dtype) if dI else None
    zkv, bkv = _normal("pzkv", (B, L, D), 1.0, "f32"), _normal("pbkv", (span, D), 0.3, "f32")
    zi = _normal("pzi", (B, L, dI), 1.0, "f32") if dI else None
    bi = _normal("pbi", (span, dI), 0.3, "f32") if dI else None
    nc = L // r
    kc = torch.zeros(B, nc, D, dtype=xk.dtype, device=dev)
    vc = torch.zeros_like(kc)
    ic = torch.zeros(B, nc, dI, dtype=xk.dtype, device=dev) if dI else None
    g = lambda t: None if t is None else t.to(dev)
    S.abi.hyb_compress_pc(g(xk), g(xv), g(xi), g(zkv), g(bkv), g(zi), g(bi), r, overlap, j0, j1, kc, vc, ic)
    torch.cuda.synchronize()
    for b in range(B):
        wants = [O.compress_per_channel(to64(xk[b]), to64(zkv[b]), to64(bkv), r, overlap, j0, j1, dtype),
                 O.compress_per_channel(to64(xv[b]), to64(zkv[b]), to64(bkv), r, overlap, j0, j1, dtype)]
        gots = [kc[b, j0:j1], vc[b, j0:j1]]
        if dI:
            wants.append(O.compress_per_channel(to64(xi[b]), to64(zi[b]), to64(bi), r, overlap, j0, j1, dtype))
            gots.append(ic[b, j0:j1])
        for gt, wt, nm in zip(gots, wants, "kvi"):
            g64 = to64(gt)
            check_close(g64, wt, dtype, f"compress_pc {nm} b={b}")
            if dtype == "bf16":   # one bf16 ulp from the fp64 result, plus the fp32 accumulation error
                slack = 2.0 ** -20 * max(1.0, float(np.abs(wt).max()))
                assert np.all(np.abs(g64 - wt) <= _ulp_bf16(wt) * 1.0001 + slack), f"{nm}: more than one ulp"
        assert torch.all(kc[b, :j0] == 0) and torch.all(kc[b, j1:] == 0)   # nothing outside the range


def test_block_reps(S):
    B, nc, dI, blk = 2, 1000, 128, 128
    ic = _normal("ic", (B, nc, dI), 0.1, "bf16")
    reps = torch.zeros(B, 8, dI, dtype=torch.bfloat16, device=dev)
    S.abi.hyb_block_reps(ic.to(dev), blk, 0, nc // blk, reps)
    torch.cuda.synchronize()
    for b in range(B):
        want = O.block_reps(to64(ic[b]), blk, "bf16")
        got = to64(reps[b, :nc // blk])
        assert np.all(np.abs(got - want) <= _ulp_bf16(want) * 1.0001 + 2.0 ** -20)
    assert torch.all(reps[:, nc // blk:] == 0)


# --------------------------------------------------------------------------- S2


def _positions(B, T, hi, seed):
    p = rng.randint_below(seed, "pos", 0, B * T, hi).view(B, T).to(torch.int32)
    if T >= 8:
        p[:, :4] = torch.tensor([0, 2, 3, 7], dtype=torch.int32)  # nothing / one entry visible
        p[:, 4] = hi - 1
    return p


@pytest.mark.parametrize("dtype,B,T,nc,dI,r,k,chunk", [
    ("f32", 1, 300, 128, 32, 4, 16, 0),
    ("bf16", 2, 700, 3000, 128, 4, 64, 0),
    ("bf16", 2, 700, 3000, 128, 4, 64, 128),
    ("bf16", 64, 1, 8192, 128, 4, 512, 0),
    ("bf16", 1, 200, 33000, 128, 4, 2048, 0),
    ("bf16", 2, 300, 2000, 64, 4, 64, 0),      # tensor-core scorer, one 64-wide K block
    ("bf16", 2, 300, 1000, 96, 4, 32, 0),      # CUDA-core scorer (width not built for tensor cores)
    ("bf16", 1, 48, 131072, 128, 1, 2048, 0),  # token level (r = 1): 128K raw tokens, k = 2048
    # decode scorer (one or two query rows per pass): both key widths, both row counts,
    # passes of 2, 2 and 1 rows, and the fp32 variant
    ("bf16", 2, 1, 3000, 64, 4, 128, 0),
    ("bf16", 3, 2, 5000, 64, 4, 256, 0),
    ("bf16", 4, 2, 6000, 128, 4, 512, 0),
    ("bf16", 2, 5, 4000, 128, 4, 256, 2),
    ("f32", 2, 2, 1000, 64, 4, 32, 0),
])
def test_index_flat(S, dtype, B, T, nc, dI, r, k, chunk):
    sc = 1.0 if dtype == "f32" else dI ** -0.5
    ic = _normal("ic", (B, nc, dI), sc, dtype)
    qi = _normal("qi", (B, T, dI), sc, dtype)
    q_pos = _positions(B, T, r * nc + 40, 5)
    idx = S.layer.index_topk(qi.to(dev), q_pos.to(dev), ic.to(dev), nc, r, k, q_chunk=chunk)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    ious = []
    for b in range(B):
        ic64, qi64 = to64(ic[b]), to64(qi[b])
        for i in range(T):
            t = int(q_pos[b, i])
            n = O.visible_entries(t, r, nc)
            ids = np.arange(n)
            s = O.index_scores(qi64[i], ic64, ids)
            iou, _ = topk_row_check(idx[b, i], s, ids, k, acc_bound(qi64[i], ic64[:n]), f"b{b} t{t}")
            ious.append(iou)
    assert np.mean(ious) >= 0.999


@pytest.mark.parametrize("T,nc,dI,k,lo,hi", [
    (40, 6000, 32, 512, -3, 4),     # scores: small integers, hundreds of keys per value
    (40, 9000, 8, 2048, -1, 2),     # a few dozen distinct values, thousands of keys each
    (24, 20000, 16, 1024, -2, 3),   # rows of up to 20000 keys (the 1024-thread select)
])
def test_index_flat_exact_ties(S, T, nc, dI, k, lo, hi):
    """Integer-valued fp32 keys and queries make every score exact (sums of small
    integer products) and put whole groups of keys at the k-th score: the selection
    must equal the oracle's rule exactly, ties going to the lower entry.  Query row 4
    (which sees every entry) is all zeros, so all of its scores tie."""
    B = 2
    ic = (rng.randint_below(11, "tie_ic", 0, B * nc * dI, hi - lo) + lo).view(B, nc, dI).to(torch.float32)
    qi = (rng.randint_below(11, "tie_qi", 0, B * T * dI, hi - lo) + lo).view(B, T, dI).to(torch.float32)
    qi[:, 4] = 0.0
    q_pos = _positions(B, T, 4 * nc + 40, 6)
    idx = S.layer.index_topk(qi.to(dev), q_pos.to(dev), ic.to(dev), nc, 4, k)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    for b in range(B):
        ic64, qi64 = to64(ic[b]), to64(qi[b])
        for i in range(T):
            n = O.visible_entries(int(q_pos[b, i]), 4, nc)
            ids = np.arange(n)
            want = O.select_topk(O.index_scores(qi64[i], ic64, ids), ids, k)
            want = np.concatenate([np.sort(want[want >= 0]), want[want < 0]])   # ascending, then -1
            assert np.array_equal(idx[b, i], want), f"b{b} row {i} (n = {n})"


@pytest.mark.parametrize("dtype,B,T,nc,dI,blk,m,k,r", [
    ("f32", 1, 200, 300, 32, 16, 4, 20, 4),
    ("bf16", 2, 400, 5000, 128, 128, 8, 256, 4),
    ("bf16", 1, 64, 32768, 128, 128, 64, 2048, 4),
    ("bf16", 1, 48, 131072, 128, 128, 64, 2048, 1),   # token level (r = 1): 1024 blocks of 128 raw tokens
    ("bf16", 2, 2, 20000, 128, 128, 16, 512, 4),      # decode: stage 1 on the decode scorer
    ("f32", 2, 3, 3000, 32, 16, 6, 40, 4),            # a few queries: stage 2 by kept-block slot, B = 16
])
def test_index_hisa(S, dtype, B, T, nc, dI, blk, m, k, r):
    sc = 1.0 if dtype == "f32" else dI ** -0.5
    ic = _normal("ic", (B, nc, dI), sc, dtype)
    qi = _normal("qi", (B, T, dI), sc, dtype)
    q_pos = _positions(B, T, r * nc + 40, 6)
    icd, qid, qpd = ic.to(dev), qi.to(dev), q_pos.to(dev)
    reps = S.layer.block_reps(icd, nc, blk)
    idx = S.layer.index_topk(qid, qpd, icd, nc, r, k, S.HYB_INDEX_HISA, reps, blk, m, 128)
    # with every block kept, HISA must reproduce the flat indexer exactly (where that many
    # candidates per row are supported: at most 51200)
    if (nc // blk + 1) * blk <= 51200:
        idx_all = S.layer.index_topk(qid, qpd, icd, nc, r, k, S.HYB_INDEX_HISA, reps, blk, nc // blk + 1, 0)
        idx_flat = S.layer.index_topk(qid, qpd, icd, nc, r, k)
        torch.cuda.synchronize()
        assert torch.equal(idx_all, idx_flat)
    idx = idx.cpu().numpy()
    exact_rows = 0
    for b in range(B):
        ic64, qi64 = to64(ic[b]), to64(qi[b])
        reps64 = O.block_reps(ic64, blk, dtype)
        for i in range(T):
            t = int(q_pos[b, i])
            n = O.visible_entries(t, r, nc)
            full = n // blk
            m_full = m - (1 if n % blk else 0)
            # stage-1 near ties (blocks) may legitimately pick other blocks: skip those rows
            if 0 < m_full < full:
                bs = reps64[:full] @ qi64[i]
                srt = np.sort(bs)[::-1]
                if srt[m_full - 1] - srt[m_full] <= 1e-3 * max(abs(srt[m_full - 1]), abs(srt[m_full])):
                    continue
            blocks = O.hisa_blocks(qi64[i], reps64, n, blk, m)
            ids = np.concatenate([np.arange(g * blk, min((g + 1) * blk, n)) for g in blocks]) \
                if len(blocks) else np.empty(0, dtype=np.int64)
            s = O.index_scores(qi64[i], ic64, ids)
            topk_row_check(idx[b, i], s, ids, k, acc_bound(qi64[i], ic64[ids]), f"hisa b{b} t{t}")
            exact_rows += 1
    assert exact_rows >= 0.9 * B * T


# --------------------------------------------------------------------------- S3


def _random_sel(B, T, k, q_pos, r, nc, seed):
    """Random distinct visible entries per query (ascending), -1 padded: an input
    for testing attention on its own."""
    out = np.full((B, T, k), -1, dtype=np.int32)
    for b in range(B):
        for i in range(T):
            n = O.visible_entries(int(q_pos[b, i]), r, nc)
            if n == 0:
                continue
            keys = rng.raw_u64(seed, f"sel_{b}_{i}", 0, n)
            pick = np.sort(torch.argsort(keys)[:min(k, n)].numpy())
            cut = min(len(pick), k - (i % 3))           # some rows shorter than k
            out[b, i, :cut] = pick[:cut]
    return torch.from_numpy(out)


@pytest.mark.parametrize("dtype,B,T,H,D,nc,r,k,W,L,mode", [
    ("f32", 1, 120, 8, 64, 128, 4, 16, 32, 512, "prefill"),
    ("f32", 1, 120, 8, 64, 4, 128, 0, 32, 512, "prefill"),
    ("bf16", 2, 150, 64, 128, 2000, 4, 96, 128, 8000, "prefill"),
    ("bf16", 2, 150, 64, 128, 60, 128, 0, 128, 7680, "prefill"),
    ("bf16", 2, 150, 64, 128, 2000, 4, 96, 128, 8000, "decode"),   # 300 queries: keys not split
    ("bf16", 3, 2, 64, 128, 60, 128, 0, 128, 7680, "decode"),      # split-KV: 2 slices
    ("bf16", 1, 8, 64, 128, 60, 128, 0, 128, 7680, "decode"),      # split-KV: 2 slices; rows at t < 127 see
                                                                   # no entry: their second slice is empty
    ("bf16", 2, 4, 64, 128, 2000, 4, 96, 128, 8000, "decode"),     # split-KV: 2 slices
    ("bf16", 1, 8, 64, 128, 2000, 4, 512, 128, 8000, "decode"),    # split-KV: 5 slices; rows at t = 0..7 see
                                                                   # at most two entries: slices of masked keys
])
def test_attention(S, dtype, B, T, H, D, nc, r, k, W, L, mode):
    sc = 1.0 if dtype == "f32" else D ** -0.5
    q = _normal("q", (B, T, H, D), sc, dtype)
    kc, vc = _normal("kc", (B, nc, D), sc, dtype), _normal("vc", (B, nc, D), sc, dtype)
    kw, vw = _normal("kw", (B, L, D), sc, dtype), _normal("vw", (B, L, D), sc, dtype)
    q_pos = _positions(B, T, L, 7)
    idx = _random_sel(B, T, k, q_pos, r, nc, 8) if k > 0 else None
    md = S.HYB_ATTN_PREFILL if mode == "prefill" else S.HYB_ATTN_DECODE
    scale = 1.0 / math.sqrt(D)
    g = lambda t: None if t is None else t.to(dev)
    o, lse = S.layer.attention(g(q), g(q_pos), g(kc), g(vc), nc, r, g(idx), g(kw), g(vw), W, scale, md)
    torch.cuda.synchronize()
    kind = "csa" if k > 0 else "hca"
    p = O.LayerParams(kind, r, kind == "csa", W, scale, dtype, k=k)
    want_o, want_l = [], []
    for b in range(B):
        kc64, vc64, kw64, vw64 = to64(kc[b]), to64(vc[b]), to64(kw[b]), to64(vw[b])
        for i in range(T):
            t = int(q_pos[b, i])
            n = O.visible_entries(t, r, nc)
            sel = idx[b, i].numpy() if k > 0 else np.arange(n)
            keys, vals = O.key_set(t, sel[sel >= 0], kc64, vc64, kw64, vw64, L, W)
            oo, ll = O.attend(to64(q[b, i]), keys, vals, scale)
            want_o.append(O.round_store(oo, dtype))
            want_l.append(ll)
    check_close(to64(o).reshape(B * T, H, D), np.stack(want_o), dtype, f"attention {mode}")
    np.testing.assert_allclose(to64(lse).reshape(B * T, H), np.stack(want_l), rtol=0,
                               atol=1e-4 if dtype == "f32" else 1e-3)


@pytest.mark.parametrize("B,T,nc,r,k,W,L,mode", [
    (2, 150, 2000, 4, 96, 128, 8000, "prefill"),
    (2, 150, 2000, 4, 96, 0, 8000, "prefill"),       # no window: the selected tokens alone
    (1, 100, 700, 4, 512, 128, 2800, "prefill"),     # k > visible entries for many rows
    (2, 150, 2000, 4, 96, 128, 8000, "decode"),      # 300 queries: keys not split
    (2, 4, 2000, 4, 96, 128, 8000, "decode"),        # split-KV: 4 slices
])
def test_attention_real_kv(S, B, T, nc, r, k, W, L, mode):
    """The real-K/V reading: selected entries attend their raw tokens (from the ring,
    here the raw sequence), together with the window as one set of positions."""
    H, D, dtype = 64, 128, "bf16"
    sc = D ** -0.5
    q = _normal("q", (B, T, H, D), sc, dtype)
    kw, vw = _normal("kw", (B, L, D), sc, dtype), _normal("vw", (B, L, D), sc, dtype)
    q_pos = _positions(B, T, L, 9)
    idx = _random_sel(B, T, k, q_pos, r, nc, 10)
    md = (S.HYB_ATTN_PREFILL if mode == "prefill" else S.HYB_ATTN_DECODE) | S.HYB_ATTN_REAL_KV
    scale = 1.0 / math.sqrt(D)
    o, lse = S.layer.attention(q.to(dev), q_pos.to(dev), None, None, nc, r, idx.to(dev), kw.to(dev), vw.to(dev), W,
                               scale, md)
    torch.cuda.synchronize()
    want_o, want_l = [], []
    for b in range(B):
        kw64, vw64 = to64(kw[b]), to64(vw[b])
        for i in range(T):
            t = int(q_pos[b, i])
            keys, vals = O.key_set_real_kv(t, idx[b, i].numpy(), r, kw64, vw64, L, W)
            if len(keys) == 0:   # no key at all (no window, nothing selected yet): o = 0, lse = -inf
                want_o.append(np.zeros((H, D)))
                want_l.append(np.full(H, -np.inf))
                continue
            oo, ll = O.attend(to64(q[b, i]), keys, vals, scale)
            want_o.append(O.round_store(oo, dtype))
            want_l.append(ll)
    check_close(to64(o).reshape(B * T, H, D), np.stack(want_o), dtype, f"real-K/V attention {mode}")
    np.testing.assert_allclose(to64(lse).reshape(B * T, H), np.stack(want_l), rtol=0, atol=1e-3)


def test_attention_real_kv_reports_tokens_outside_the_ring(S):
    B, T, H, D, nc, k, W, ring = 1, 4, 64, 128, 250, 8, 128, 256
    q = _normal("q", (B, T, H, D), 0.1, "bf16").to(dev)
    kw = _normal("kw", (B, ring, D), 0.1, "bf16").to(dev)
    q_pos = torch.full((B, T), 999, dtype=torch.int32, device=dev)
    idx = torch.arange(k, dtype=torch.int32, device=dev).repeat(B, T, 1).contiguous()   # tokens 0..31: gone
    S.layer.attention(q, q_pos, None, None, nc, 4, idx, kw, kw, W, 0.1, S.HYB_ATTN_PREFILL | S.HYB_ATTN_REAL_KV)
    assert S.abi.hyb_get_device_status() == S.abi.HYB_ERR_DEVICE_CHECK


def test_attention_reports_bad_index(S):
    B, T, H, D, nc, k, W, L = 1, 4, 64, 128, 100, 8, 128, 600
    q = _normal("q", (B, T, H, D), 0.1, "bf16").to(dev)
    kc = _normal("kc", (B, nc, D), 0.1, "bf16").to(dev)
    kw = _normal("kw", (B, L, D), 0.1, "bf16").to(dev)
    q_pos = torch.full((B, T), 500, dtype=torch.int32, device=dev)
    idx = torch.arange(k, dtype=torch.int32, device=dev).repeat(B, T, 1).contiguous()
    idx[0, 2, 3] = 10 ** 6                                   # out of range: skipped and reported
    S.layer.attention(q, q_pos, kc, kc, nc, 4, idx, kw, kw, W, 0.1)
    assert S.abi.hyb_get_device_status() == S.abi.HYB_ERR_DEVICE_CHECK
