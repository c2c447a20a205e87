"""Seeded synthetic inputs for the workloads in ``configs``.

Everything here is input construction: random tensors of the stated shapes and
distributions, rounded to the workload's storage type, plus the planted
indexer keys.  No step of the attention method is computed here.

Tensor layouts (row-major, batch outermost):
  raw K / raw V   [B, L_raw, D]     raw indexer keys [B, L_raw, dI]
  logits          [B, L_raw] fp32   bias (per layer)  [span] fp32
  q               [B, T, H, D]      q_I               [B, T, dI]
  q_pos           [B, T] int32 (absolute positions)
  decode caches   K_c / V_c [B, N_c, D], I_c [B, N_c, dI], ring [B, W, D]
"""
from __future__ import annotations

import math
from typing import Dict

import torch

from . import rng
from .configs import LayerSpec, Workload

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_storage(x64: torch.Tensor, dtype: str) -> torch.Tensor:
    """fp64 values -> storage type: round to fp32 (nearest-even), then to bf16 if asked."""
    x = x64.to(torch.float32)
    return x if dtype == "f32" else x.to(torch.bfloat16)


def normal_tensor(seed: int, name: str, shape, std: float, dtype: str, device="cpu") -> torch.Tensor:
    n = math.prod(shape)
    x = rng.normal(seed, name, 0, n, device).view(*shape) * std
    return to_storage(x, dtype)


def raw_length(w: Workload) -> int:
    """Raw tokens to generate: the prefix, plus the new tokens of a decode step."""
    return w.L + (w.T if w.mode == "decode" else 0)


def query_positions(w: Workload, device="cpu") -> torch.Tensor:
    p = torch.arange(w.q_pos0, w.q_pos0 + w.T, dtype=torch.int32, device=device)
    return p.unsqueeze(0).expand(w.batch, w.T).contiguous()


def make_queries(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    return {
        "q": normal_tensor(w.seed, "q", (w.batch, w.T, w.H, w.D), w.x_scale, w.dtype, device),
        "qi": normal_tensor(w.seed, "q_index", (w.batch, w.T, w.dI), w.i_scale, w.dtype, device),
        "q_pos": query_positions(w, device),
    }


def make_bias(w: Workload, ly: LayerSpec, device="cpu") -> torch.Tensor:
    return normal_tensor(w.seed, f"bias_{ly.kind}", (ly.span,), w.bias_std, "f32", device)


def make_raw(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    L = raw_length(w)
    out = {
        "xk": normal_tensor(w.seed, "raw_k", (w.batch, L, w.D), w.x_scale, w.dtype, device),
        "xv": normal_tensor(w.seed, "raw_v", (w.batch, L, w.D), w.x_scale, w.dtype, device),
        "z": normal_tensor(w.seed, "logits", (w.batch, L), 1.0, "f32", device),
    }
    if any(ly.kind == "csa" for ly in w.layers):
        out["xi"] = normal_tensor(w.seed, "raw_i", (w.batch, L, w.dI), w.i_scale, w.dtype, device)
    return out


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def _plant_vectors(w: Workload, name: str, n: int, device) -> torch.Tensor:
    """n planted key directions, unit in fp64 then rounded to storage (returned as fp64)."""
    u = _unit_rows(rng.normal(w.seed, name, 0, n * w.dI, device).view(n, w.dI))
    return to_storage(u, w.dtype).to(torch.float64)


def _correlated_query(w: Workload, qi_rows64: torch.Tensor, u64: torch.Tensor, tag: int, device):
    """Rows rescaled to their own norm along 0.5*u_hat + sqrt(0.75)*w_hat (w_hat orthogonal to u)."""
    n = qi_rows64.shape[0]
    g = rng.normal(w.seed, "plant_w", tag * 4096 * w.dI, n * w.dI, device).view(n, w.dI)
    uh = u64 / u64.norm()
    g = g - (g @ uh).unsqueeze(1) * uh.unsqueeze(0)
    wh = _unit_rows(g)
    return qi_rows64.norm(dim=1, keepdim=True) * (0.5 * uh.unsqueeze(0) + math.sqrt(0.75) * wh)


def plant_prefill(w: Workload, ly: LayerSpec, raw: Dict[str, torch.Tensor],
                  qs: Dict[str, torch.Tensor], device="cpu") -> torch.Tensor:
    """Plant keys in the raw indexer keys of a sequence; returns planted entry indices.

    Planted entries sit at j = 3s+1, so no two pooling windows of 2r overlap.
    Every raw indexer key in entry j's window is set to u_j, so its pooled key
    is u_j.  ``plant_queries`` queries that can see j get cos 0.5 with u_j.
    """
    if w.plant_frac <= 0 or ly.kind != "csa":
        return torch.empty(0, dtype=torch.int64)
    L = raw.get("xi").shape[1]
    r = ly.r
    n_c = L // r
    slots = (n_c - 2) // 3
    n = max(1, round(w.plant_frac * n_c))
    order = torch.argsort(rng.raw_u64(w.seed, "plant_pos", 0, slots, device))
    js = torch.sort(order[:n] * 3 + 1).values
    u = _plant_vectors(w, "plant_u", n, device)
    xi, qi = raw["xi"], qs["qi"]
    last_q = w.q_pos0 + w.T - 1
    picks = rng.uniform(w.seed, "plant_q", 0, n * w.plant_queries, device).view(n, w.plant_queries)
    for p in range(n):
        j = int(js[p])
        lo = max(0, (j - 1) * r) if ly.overlap else j * r
        xi[:, lo:(j + 1) * r, :] = to_storage(u[p], w.dtype).to(xi.device)
        first_t = (j + 1) * r - 1
        if first_t > last_q:
            continue
        i_min = max(0, first_t - w.q_pos0)
        rows = (i_min + (picks[p] * (w.T - i_min)).to(torch.int64)).clamp(max=w.T - 1)
        # each picked row once: a row picked twice would get two different correlated
        # values, and which write of a repeated index lands is unspecified on a GPU
        rows = torch.unique(rows)
        for b in range(w.batch):
            q64 = qi[b, rows].to(torch.float64)
            qi[b, rows] = to_storage(_correlated_query(w, q64, u[p], p, device), w.dtype)
    return js


def make_decode_cache(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Compressed caches and the window ring generated directly (no raw sequence).

    Ring slot s mod W holds the raw key/value of position s, for the W
    positions q_pos0-W+1 .. q_pos0 (the new token included).
    """
    out = {}
    for ly in w.layers:
        n_c = w.L // ly.r
        out[f"kc_{ly.kind}"] = normal_tensor(w.seed, f"cache_k_{ly.kind}", (w.batch, n_c, w.D), w.x_scale, w.dtype, device)
        out[f"vc_{ly.kind}"] = normal_tensor(w.seed, f"cache_v_{ly.kind}", (w.batch, n_c, w.D), w.x_scale, w.dtype, device)
        if ly.kind == "csa":
            out["ic"] = normal_tensor(w.seed, "cache_i", (w.batch, n_c, w.dI), w.i_scale, w.dtype, device)
    out["kw"] = normal_tensor(w.seed, "ring_k", (w.batch, w.W, w.D), w.x_scale, w.dtype, device)
    out["vw"] = normal_tensor(w.seed, "ring_v", (w.batch, w.W, w.D), w.x_scale, w.dtype, device)
    return out


def plant_decode(w: Workload, ly: LayerSpec, cache: Dict[str, torch.Tensor],
                 qs: Dict[str, torch.Tensor], device="cpu") -> torch.Tensor:
    """Plant keys directly in I_c: per sequence, plant_frac of the entries get u_j,
    and the sequence's query gets cos 0.5 with one of them.  Returns [B, n] indices."""
    if w.plant_frac <= 0 or ly.kind != "csa":
        return torch.empty(0, dtype=torch.int64)
    ic, qi = cache["ic"], qs["qi"]
    n_c = ic.shape[1]
    n = max(1, round(w.plant_frac * n_c))
    all_js = []
    for b in range(w.batch):
        order = torch.argsort(rng.raw_u64(w.seed, f"plant_pos_{b}", 0, n_c, device))
        js = torch.sort(order[:n]).values
        u = _plant_vectors(w, f"plant_u_{b}", n, device)
        ic[b, js] = to_storage(u, w.dtype).to(ic.device)
        pick = int(rng.randint_below(w.seed, "plant_pick", b, 1, n, device)[0])
        q64 = qi[b, :].to(torch.float64)
        qi[b, :] = to_storage(_correlated_query(w, q64, u[pick], b, device), w.dtype)
        all_js.append(js)
    return torch.stack(all_js)


def ring_from_raw(w: Workload, raw: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Window ring [B, W, D] of a decode step, taken from a raw sequence.

    For new tokens at positions q_pos0..q_pos0+T-1 the ring holds positions
    q_pos0+T-W .. q_pos0+T-1, position s at slot s mod W.
    """
    last = w.q_pos0 + w.T - 1
    pos = torch.arange(last - w.W + 1, last + 1)
    pos = pos[pos >= 0]
    kw = torch.zeros(w.batch, w.W, w.D, dtype=raw["xk"].dtype, device=raw["xk"].device)
    vw = torch.zeros_like(kw)
    kw[:, pos % w.W] = raw["xk"][:, pos]
    vw[:, pos % w.W] = raw["xv"][:, pos]
    return {"kw": kw, "vw": vw}
