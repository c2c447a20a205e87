"""fp64 CPU oracle of the forward pass of one hybrid compressed attention layer.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
CPU-baseline / reference arm may import or run this module.  The CUDA library
shares no code with it, and it never reads anything the CUDA path produced.

What it computes, and where the pages state it:
  * Hybrid attention = CSA (compress the KV cache along the sequence, then
    DeepSeek sparse attention) + HCA (heavier compression, dense attention):
    "Hybrid Attention" explainer (process-cxr.github.io), section
    "DeepSeek V4 中的定义" (Definition in DeepSeek V4).
  * S1 compression: raw KV and per-token compression weights are computed first;
    every r entries are combined with "softmax weights plus a learnable
    positional bias"; HCA uses r = 128 and adjacent blocks do not overlap, so CSA
    blocks do; CSA uses r = 4: HCA article (daiw.net, "前代 · HCA：128 倍压缩后
    再做稠密注意力"), section "怎么压" (How it is compressed) and the CSA/HCA
    comparison table; trdm.cn news 749237, section 2.1.
  * S2a flat indexer: score every prefix entry per query, keep the top-k:
    HISA write-up (my.qihongyi.cn "DeepSeek速度狂飙4倍还不丢精度"), section 01.
  * S2b HISA: blocks of B entries, one pooled representative per block, the
    query scores representatives and keeps the top-m blocks (stage 1), then
    the original indexer runs on the tokens of those blocks and keeps the
    top-k (stage 2); output format identical to the flat indexer: same
    write-up, section 02 (stage 1 / stage 2), section 05 step 3, Fig. 2.
  * S3 attention: all query heads share one K/V (MQA); CSA attends the selected
    entries, HCA attends every compressed entry; both add a branch over the
    most recent 128 raw tokens: HCA article, section "怎么压"; trdm.cn 2.1.

Readings where the pages are silent (each one is listed in the design notes):
  * one scalar compression logit per token and one scalar bias per window
    position; the same weights pool K, V and the indexer keys;
  * CSA entry j pools tokens [(j-1)r, (j+1)r) clipped at 0, the bias indexed by
    the position in the unclipped window; HCA entry j pools [jr, (j+1)r);
  * an entry is visible to the query at position t once complete:
    j < floor((t+1)/r);
  * indexer score = q_I . I_c (single head, no scale or activation);
  * ties go to the lower index (entries and blocks); fewer than k candidates:
    keep all, pad with -1;
  * HISA representative = mean of the B indexer keys of a full block; a query's
    partial last block is always kept and takes one of the m slots;
  * the window covers positions max(0, t-W+1) .. t; compressed and window keys
    are one set under one joint softmax; scores are q.k / sqrt(D) (the scale
    is an argument); lse is the natural log of the softmax denominator.

Rounding model: arithmetic in fp64; every value the CUDA path stores (K_c,
V_c, I_c, block representatives, o, lse) is rounded to its storage type here
too, with round-to-nearest-even.

Parity status: every function below is pinned by the CPU tests against
closed forms, brute force and special cases; none is "parity unpinned".
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

# --------------------------------------------------------------------------- rounding


def round_bf16(x) -> np.ndarray:
    """fp64 -> nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits and the fp32 exponent range.  Normal values
    drop the low 45 of fp64's 52 fraction bits with round-half-even on the bit
    pattern; values below 2^-126 are rounded to a multiple of 2^-133 (the bf16
    subnormal spacing); magnitudes past the largest bf16 become infinities.
    """
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64).copy()
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    bits = (bits + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    y = bits.view(np.float64)
    tiny = np.abs(x) < 2.0 ** -126
    if np.any(tiny):
        y = np.where(tiny, np.round(x / 2.0 ** -133) * 2.0 ** -133, y)
    big = np.abs(x) >= (2.0 - 2.0 ** -8) * 2.0 ** 127   # half an ulp above the largest bf16
    if np.any(big):
        y = np.where(big & np.isfinite(x), np.copysign(np.inf, x), y)
    return y


def round_store(x, dtype: str) -> np.ndarray:
    """Round fp64 values to a storage type ('f32' or 'bf16'); result in fp64."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


# --------------------------------------------------------------------------- S1 compression


def window_start(j: int, r: int, overlap: bool) -> int:
    """First token of entry j's (unclipped) pooling window: (j-1)r with overlap, else jr."""
    return (j - 1) * r if overlap else j * r


def pooling_weights(z: np.ndarray, bias: np.ndarray, j: int, r: int, overlap: bool):
    """Tokens of entry j and their weights softmax_i(z_i + b_p), p = position in the window."""
    start = window_start(j, r, overlap)
    end = (j + 1) * r
    s = np.arange(max(start, 0), end)
    a = z[s].astype(np.float64) + bias[s - start].astype(np.float64)
    e = np.exp(a - a.max())
    return s, e / e.sum()


def compress(xs, z, bias, r: int, overlap: bool, j_begin: int, j_end: int, dtype: str,
             chunk: int = 4096):
    """Entries j_begin..j_end-1 of every raw tensor in ``xs`` ([L, C] each), pooled
    with the same weights.  Returns a list of [j_end-j_begin, C] arrays, rounded."""
    span = 2 * r if overlap else r
    z = np.asarray(z, dtype=np.float64)
    bias = np.asarray(bias, dtype=np.float64)
    outs = [np.empty((j_end - j_begin, np.asarray(x).shape[1])) for x in xs]
    for c0 in range(j_begin, j_end, chunk):
        js = np.arange(c0, min(c0 + chunk, j_end))
        start = np.array([window_start(int(j), r, overlap) for j in js])
        tok = start[:, None] + np.arange(span)[None, :]          # [n, span]
        valid = tok >= 0
        a = np.where(valid, z[np.maximum(tok, 0)] + bias[None, :], -np.inf)
        e = np.exp(a - a.max(axis=1, keepdims=True))
        w = e / e.sum(axis=1, keepdims=True)                      # zero weight outside [0, L)
        for x, out in zip(xs, outs):
            xv = np.asarray(x, dtype=np.float64)[np.maximum(tok, 0)]  # [n, span, C]
            out[js - j_begin] = np.einsum("ns,nsc->nc", w, xv)
    return [round_store(o, dtype) for o in outs]


def compress_per_channel(x, z, bias, r: int, overlap: bool, j_begin: int, j_end: int, dtype: str):
    """S1 with per-channel compression weights (the other reading of "compression
    weights" in the HCA article, section "怎么压"): channel c of entry j is
    sum_i w[i, c] x[i, c] with w[., c] = softmax over the window's in-range tokens
    of (z[i, c] + bias[p, c]), p the position in the unclipped window.
    x, z: [L, C]; bias: [span, C].  Returns [j_end - j_begin, C], rounded."""
    span = 2 * r if overlap else r
    x = np.asarray(x, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    bias = np.asarray(bias, dtype=np.float64)
    out = np.empty((j_end - j_begin, x.shape[1]))
    for j in range(j_begin, j_end):
        start = window_start(j, r, overlap)
        s = np.arange(max(start, 0), (j + 1) * r)
        a = z[s] + bias[s - start]                       # [n, C]
        e = np.exp(a - a.max(axis=0, keepdims=True))
        w = e / e.sum(axis=0, keepdims=True)
        out[j - j_begin] = (w * x[s]).sum(axis=0)
    return round_store(out, dtype)


# --------------------------------------------------------------------------- S2 indexer


def visible_entries(t: int, r: int, n_c: int) -> int:
    """Number of entries whose window has ended by position t: min(floor((t+1)/r), n_c)."""
    return min((t + 1) // r, n_c)


def select_topk(scores: np.ndarray, ids: np.ndarray, k: int) -> np.ndarray:
    """The k best ids by (score descending, id ascending), padded with -1 to length k."""
    order = np.lexsort((ids, -scores))
    chosen = ids[order[:k]]
    out = np.full(k, -1, dtype=np.int64)
    out[:len(chosen)] = chosen
    return out


def index_scores(qi_t: np.ndarray, ic: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Indexer scores q_I . I_c[j] for the given entries."""
    return np.asarray(ic, dtype=np.float64)[ids] @ np.asarray(qi_t, dtype=np.float64)


def flat_topk(qi_t, ic, n_vis: int, k: int) -> np.ndarray:
    """Flat indexer: score all visible entries, keep the top-k."""
    ids = np.arange(n_vis)
    return select_topk(index_scores(qi_t, ic, ids), ids, k)


def block_reps(ic, B: int, dtype: str) -> np.ndarray:
    """HISA block representatives: mean of the indexer keys of each full block of B entries."""
    ic = np.asarray(ic, dtype=np.float64)
    nb = ic.shape[0] // B
    return round_store(ic[:nb * B].reshape(nb, B, ic.shape[1]).mean(axis=1), dtype)


def hisa_blocks(qi_t, reps, n_vis: int, B: int, m: int) -> np.ndarray:
    """Stage 1: blocks kept for a query (ascending).  The partial block, if any,
    always; the best of the full visible blocks fill the other slots."""
    full = n_vis // B
    partial = n_vis % B != 0
    m_full = m - 1 if partial else m
    ids = np.arange(full)
    bsc = np.asarray(reps, dtype=np.float64)[:full] @ np.asarray(qi_t, dtype=np.float64)
    kept = select_topk(bsc, ids, m_full) if m_full > 0 else np.empty(0, dtype=np.int64)
    kept = kept[kept >= 0]
    if partial:
        kept = np.append(kept, full)
    return np.sort(kept)


def hisa_topk(qi_t, ic, reps, n_vis: int, B: int, m: int, k: int) -> np.ndarray:
    """Stage 2: the flat rule on the visible entries of the stage-1 blocks."""
    blocks = hisa_blocks(qi_t, reps, n_vis, B, m)
    ids = np.concatenate([np.arange(b * B, min((b + 1) * B, n_vis)) for b in blocks]) \
        if len(blocks) else np.empty(0, dtype=np.int64)
    return select_topk(index_scores(qi_t, ic, ids), ids, k)


# --------------------------------------------------------------------------- S3 attention


def window_positions(t: int, W: int) -> np.ndarray:
    """Raw positions in query t's sliding window: max(0, t-W+1) .. t."""
    return np.arange(max(0, t - W + 1), t + 1)


def attend(q_t, keys, vals, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """One query, all heads: o[h] = sum_j softmax_j(scale * q[h].k_j) v_j, and the
    natural-log softmax denominator lse[h] (of the scaled scores)."""
    q_t = np.asarray(q_t, dtype=np.float64)
    s = (q_t @ np.asarray(keys, dtype=np.float64).T) * scale      # [H, n]
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    den = e.sum(axis=1, keepdims=True)
    o = (e @ np.asarray(vals, dtype=np.float64)) / den
    return o, (mx + np.log(den))[:, 0]


def key_set(t: int, sel: np.ndarray, kc, vc, kw, vw, ring: int, W: int):
    """Keys and values of query t: compressed entries ``sel`` then its window (ring slot s mod ring)."""
    pos = window_positions(t, W)
    sel = np.asarray(sel, dtype=np.int64)
    keys = np.concatenate([np.asarray(kc)[sel], np.asarray(kw)[pos % ring]])
    vals = np.concatenate([np.asarray(vc)[sel], np.asarray(vw)[pos % ring]])
    return keys, vals


def real_kv_positions(t: int, sel: np.ndarray, r: int, W: int) -> np.ndarray:
    """The "real K/V" reading of CSA attention (the block-sparse methods the
    pages compare against attend the real keys and values behind a selection):
    each selected entry j stands for its r raw tokens jr .. jr+r-1, and the key
    set is those tokens together with the window as a set of raw positions (a
    token the window already holds is not repeated), ascending."""
    sel = np.asarray(sel, dtype=np.int64)
    sel = sel[sel >= 0]
    toks = (sel[:, None] * r + np.arange(r)[None, :]).reshape(-1)
    win = window_positions(t, W)
    return np.union1d(toks, win)


def key_set_real_kv(t: int, sel: np.ndarray, r: int, raw_k, raw_v, ring: int, W: int):
    """Keys and values of query t under the real-K/V reading, read from a raw ring
    holding at least positions 0 .. t (slot s mod ring)."""
    pos = real_kv_positions(t, sel, r, W)
    return np.asarray(raw_k)[pos % ring], np.asarray(raw_v)[pos % ring]


# --------------------------------------------------------------------------- whole layer


@dataclass(frozen=True)
class LayerParams:
    kind: str            # "csa" or "hca"
    r: int
    overlap: bool
    W: int
    scale: float
    dtype: str           # storage type: "f32" or "bf16"
    k: int = 0
    index_mode: str = "flat"
    block: int = 128
    top_m: int = 64


def build_caches(p: LayerParams, xk, xv, xi, z, bias, n_entries: Optional[int] = None):
    """S1 over a raw sequence: K_c, V_c (and I_c for CSA) for entries 0..n_entries-1."""
    n = np.asarray(xk).shape[0] // p.r if n_entries is None else n_entries
    xs = [xk, xv] + ([xi] if p.kind == "csa" else [])
    out = compress(xs, z, bias, p.r, p.overlap, 0, n, p.dtype)
    return out[0], out[1], (out[2] if p.kind == "csa" else None)


def layer_row(p: LayerParams, q_t, qi_t, t: int, kc, vc, ic, reps, kw, vw, ring: int):
    """S2 + S3 + S4 for one query at position t given the caches.

    Returns (idx or None, o [H, D] rounded to storage, lse [H] rounded to fp32)."""
    n_c = np.asarray(kc).shape[0]
    n_vis = visible_entries(t, p.r, n_c)
    idx = None
    if p.kind == "csa":
        if p.index_mode == "flat":
            idx = flat_topk(qi_t, ic, n_vis, p.k)
        else:
            idx = hisa_topk(qi_t, ic, reps, n_vis, p.block, p.top_m, p.k)
        sel = idx[idx >= 0]
    else:
        sel = np.arange(n_vis)
    keys, vals = key_set(t, sel, kc, vc, kw, vw, ring, p.W)
    o, lse = attend(q_t, keys, vals, p.scale)
    return idx, round_store(o, p.dtype), round_store(lse, "f32")


# --------------------------------------------------------------------------- decode-step state update


class DecodeState:
    """What one sequence keeps between decode steps: the window rings (raw K, V,
    indexer key and compression logit of the last `ring` tokens, token s at slot
    s mod ring) and, per layer, the compressed entries emitted so far and the
    HISA block representatives of the full blocks."""

    def __init__(self, ring: int, D: int, dI: int, layers, block: int, dtype: str):
        self.ring, self.block, self.dtype = ring, block, dtype
        self.length = 0
        self.kw = np.zeros((ring, D))
        self.vw = np.zeros((ring, D))
        self.iw = np.zeros((ring, dI))
        self.zw = np.zeros(ring)
        self.layers = {p.kind: p for p in layers}
        self.kc = {p.kind: [] for p in layers}
        self.vc = {p.kind: [] for p in layers}
        self.ic = []      # CSA indexer keys
        self.reps = []    # CSA block representatives


def _ring_view(st: DecodeState, rows: np.ndarray) -> np.ndarray:
    """The ring's rows placed at their absolute positions 0..length-1; positions
    that have left the ring are NaN, so a read of one would poison the result."""
    n = st.length
    out = np.full((n,) + rows.shape[1:], np.nan)
    lo = max(0, n - st.ring)
    pos = np.arange(lo, n)
    out[pos] = rows[pos % st.ring]
    return out


def decode_append(st: DecodeState, k_t, v_t, i_t, z_t: float, biases) -> None:
    """One decode step's state update for the token at position t = st.length:
    append it to the rings; when t closes a window of a layer ((t+1) a multiple
    of r), emit that layer's next entry with the pooling of S1 (`compress`, so
    the same definition as over the full sequence); when a CSA entry completes a
    block of `block` entries, add that block's representative (`block_reps`).
    HCA article, section "怎么压" (one entry per r tokens, softmax weights plus
    position bias); HISA write-up, section 02, stage 1 (block representatives)."""
    t = st.length
    slot = t % st.ring
    st.kw[slot], st.vw[slot] = np.asarray(k_t, np.float64), np.asarray(v_t, np.float64)
    if i_t is not None:
        st.iw[slot] = np.asarray(i_t, np.float64)
    st.zw[slot] = float(z_t)
    st.length = t + 1
    for kind, p in st.layers.items():
        if (t + 1) % p.r:
            continue
        j = (t + 1) // p.r - 1
        xs = [_ring_view(st, st.kw), _ring_view(st, st.vw)] + ([_ring_view(st, st.iw)] if kind == "csa" else [])
        out = compress(xs, _ring_view(st, st.zw), biases[kind], p.r, p.overlap, j, j + 1, st.dtype)
        st.kc[kind].append(out[0][0])
        st.vc[kind].append(out[1][0])
        if kind == "csa":
            st.ic.append(out[2][0])
            if st.block > 0 and (j + 1) % st.block == 0:
                st.reps.append(block_reps(np.array(st.ic[-st.block:]), st.block, st.dtype)[0])
