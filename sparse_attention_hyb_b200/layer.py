"""One hybrid compressed attention layer composed from the libhyb entry points.

Output tensors and workspaces are allocated with torch (device memory only);
every computation is a libhyb kernel.  Shapes as in include/hyb.h.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import abi


@dataclass
class LayerOut:
    o: torch.Tensor
    lse: torch.Tensor
    idx: Optional[torch.Tensor] = None


def _ws(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def compress(xk, xv, xi, z, bias, r: int, overlap: bool, n_entries: Optional[int] = None,
             out=None, j_begin: int = 0, stream=None):
    """S1: entries [j_begin, n_entries) of K_c, V_c (and I_c when xi is given)."""
    B, L, D = xk.shape
    n = L // r if n_entries is None else n_entries
    if out is None:
        kc = torch.empty(B, n, D, dtype=xk.dtype, device=xk.device)
        vc = torch.empty_like(kc)
        ic = torch.empty(B, n, xi.shape[2], dtype=xi.dtype, device=xi.device) if xi is not None else None
    else:
        kc, vc, ic = out
    abi.hyb_compress(xk, xv, xi, z, bias, r, overlap, j_begin, n, kc, vc, ic, stream)
    return kc, vc, ic


def block_reps(ic, nc: int, block: int, stream=None):
    B, _, dI = ic.shape
    nb = nc // block
    reps = torch.empty(B, max(nb, 1), dI, dtype=ic.dtype, device=ic.device)
    abi.hyb_block_reps(ic, block, 0, nb, reps, stream)
    return reps


def index_topk(qi, q_pos, ic, nc: int, r: int, k: int, mode: int = abi.HYB_INDEX_FLAT, reps=None,
               block: int = 0, top_m: int = 0, q_chunk: int = 0, stream=None):
    B, T, dI = qi.shape
    dt = abi._dtype_code(qi)
    ws = _ws(abi.hyb_index_topk_workspace_size(dt, B, T, nc, dI, k, mode, block, top_m, q_chunk), qi.device)
    idx = torch.empty(B, T, k, dtype=torch.int32, device=qi.device)
    abi.hyb_index_topk(qi, q_pos, ic, nc, r, k, mode, reps, block, top_m, q_chunk, idx, ws, stream)
    return idx


def attention(q, q_pos, kc, vc, nc: int, r: int, idx, kw, vw, W: int, scale: float,
              mode: int = abi.HYB_ATTN_PREFILL, stream=None):
    B, T, H, D = q.shape
    k = idx.shape[2] if idx is not None else 0
    dt = abi._dtype_code(q)
    ws = _ws(abi.hyb_attn_fwd_workspace_size(dt, B, T, H, D, k, nc, W, mode), q.device)
    o = torch.empty_like(q)
    lse = torch.empty(B, T, H, dtype=torch.float32, device=q.device)
    abi.hyb_attn_fwd(q, q_pos, kc, vc, nc, r, idx, k, kw, vw, W, scale, o, lse, mode, ws, stream)
    return o, lse
