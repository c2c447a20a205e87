"""The five workloads of the hybrid compressed attention layer, as data.

Shapes and settings follow the HCA article (section "How it is compressed":
ratio 128 without overlap, shared-KV MQA, 128-token sliding window) and the
HISA write-up (section 02 and the Fig. 2 caption: block size 128, top-m 64
blocks, top-k 2048, query chunk 1024).  CSA uses ratio 4 with windows of 2r
at stride r.

Value distributions (the pages fix only the shapes):
  * tiny: every tensor ~ N(0, 1); positional bias ~ N(0, 0.1^2).
  * others: q, raw K, raw V ~ N(0,1)/sqrt(D); indexer q_I and raw indexer
    keys ~ N(0,1)/sqrt(d_I); compression logits ~ N(0,1); bias ~ N(0, 0.1^2);
    1% of compressed positions carry a planted indexer key with cos 0.5 to a
    random subset of queries that can see it.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class LayerSpec:
    kind: str                 # "csa" (compressed + top-k) or "hca" (compressed, dense)
    r: int                    # compression ratio
    overlap: bool             # CSA windows of 2r at stride r; HCA windows of r
    k: int = 0                # top-k entries per query (CSA)
    index_mode: str = "flat"  # "flat" or "hisa" (CSA)
    block: int = 128          # HISA block size B (entries)
    top_m: int = 64           # HISA blocks kept per query
    q_chunk: int = 1024       # HISA query chunk (scheduling unit only)

    @property
    def span(self) -> int:
        """Tokens in one pooling window (= length of the positional bias)."""
        return 2 * self.r if self.overlap else self.r


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                # "f32" or "bf16"
    mode: str                 # "prefill" (queries are rows of the raw sequence) or "decode"
    batch: int
    L: int                    # raw tokens present (prefill: raw sequence length; decode: cached tokens)
    T: int                    # queries per sequence
    q_pos0: int               # position of the first query
    H: int
    D: int
    dI: int
    W: int                    # sliding window (tokens)
    layers: Tuple[LayerSpec, ...]
    seed: int = 0
    x_scale: float = 1.0      # std of q / raw K / raw V
    i_scale: float = 1.0      # std of q_I / raw indexer keys
    bias_std: float = 0.1
    plant_frac: float = 0.0   # fraction of compressed CSA positions with a planted key
    plant_queries: int = 64   # queries correlated with each planted key
    cache_from_raw: bool = True  # decode: compressed cache made by S1 from a raw sequence

    def layer(self, kind: str) -> LayerSpec:
        for ly in self.layers:
            if ly.kind == kind:
                return ly
        raise KeyError(kind)


CSA4_FLAT_16 = LayerSpec("csa", 4, True, k=16)
HCA128 = LayerSpec("hca", 128, False)

TINY = Workload(
    name="tiny_f32_prefill_L512", dtype="f32", mode="prefill", batch=1, L=512, T=512, q_pos0=0,
    H=8, D=64, dI=32, W=32, layers=(CSA4_FLAT_16, HCA128), x_scale=1.0, i_scale=1.0)

_S = 128 ** -0.5

PREFILL_32K = Workload(
    name="csa_prefill_32k_bf16", dtype="bf16", mode="prefill", batch=1, L=32768, T=32768, q_pos0=0,
    H=64, D=128, dI=128, W=128, layers=(LayerSpec("csa", 4, True, k=512),),
    x_scale=_S, i_scale=_S, plant_frac=0.01)

PREFILL_128K = Workload(
    name="csa_prefill_128k_bf16_hisa_vs_flat", dtype="bf16", mode="prefill", batch=1, L=131072,
    T=131072, q_pos0=0, H=64, D=128, dI=128, W=128,
    layers=(LayerSpec("csa", 4, True, k=2048, index_mode="hisa", block=128, top_m=64, q_chunk=1024),),
    x_scale=_S, i_scale=_S, plant_frac=0.01)

DECODE_BS64_128K = Workload(
    name="decode_bs64_ctx128k_bf16", dtype="bf16", mode="decode", batch=64, L=131072, T=1,
    q_pos0=131072, H=64, D=128, dI=128, W=128,
    layers=(LayerSpec("csa", 4, True, k=512), HCA128),
    x_scale=_S, i_scale=_S, plant_frac=0.01, cache_from_raw=False)

_M = 1 << 20
CTX_1M_DECODE = Workload(
    name="decode_bs1_ctx1m_bf16", dtype="bf16", mode="decode", batch=1, L=_M, T=1, q_pos0=_M,
    H=64, D=128, dI=128, W=128,
    layers=(LayerSpec("csa", 4, True, k=2048, index_mode="hisa", block=128, top_m=64), HCA128),
    x_scale=_S, i_scale=_S, plant_frac=0.01, cache_from_raw=True)

CTX_1M_CHUNK = Workload(
    name="chunk_prefill_8k_at_1m_bf16", dtype="bf16", mode="prefill", batch=1, L=_M, T=8192,
    q_pos0=_M - 8192, H=64, D=128, dI=128, W=128,
    layers=(LayerSpec("csa", 4, True, k=2048, index_mode="hisa", block=128, top_m=64), HCA128),
    x_scale=_S, i_scale=_S, plant_frac=0.01)

ALL = (TINY, PREFILL_32K, PREFILL_128K, DECODE_BS64_128K, CTX_1M_DECODE, CTX_1M_CHUNK)


def by_name(name: str) -> Workload:
    for w in ALL:
        if w.name == name:
            return w
    raise KeyError(name)


def scaled(w: Workload, **kw) -> Workload:
    """A copy with some fields replaced (used for small parity cases)."""
    return replace(w, **kw)
