#!/usr/bin/env python
"""Benchmark of one hybrid compressed attention layer on B200.

Headline: CSA prefill of a 32K-token sequence (bf16, 64 query heads sharing one
128-d K/V, r = 4 with windows of 8 at stride 4, indexer dim 128, flat top-512,
128-token window).  One step = S1 compression of the whole sequence + S2 flat
indexer and top-k for every query + S3/S4 attention for every query.
value = tokens/s over all ranks (replicas: each rank runs the whole layer).
Also reported: the decode step of 64 sequences x 128K context (CSA flat top-512
+ HCA dense), per-stage times, the roofline of the dominant kernel, an
end-to-end figure through host buffers, SM clocks during the timed region, and
the fp64 CPU oracle timed on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import configs as C  # noqa: E402
from workloads import make, rng  # noqa: E402

METRIC = "prefill tok/s & decode tok/s per hybrid layer at 1 B200; % of HBM/TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU oracle sample")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the HCA prefill, 128K indexer and 1M-context measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-only", action="store_true", help="time only the prefill step (profiling runs)")
    ap.add_argument("--L", type=int, default=None, help="override the prefill length (profiling runs)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: d[k] for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- distributed plumbing


def dist_setup(n_gpus, timeout_s: float = 300.0):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the launcher):
    NCCL between GPUs; without a GPU (host-side tests of the replica plumbing) gloo."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        timeout = datetime.timedelta(seconds=timeout_s)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (step times are taken as the max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, world: int, max_step_ms: float) -> float:
    """Whole-job rate of `world` independent replicas: every rank's units over the
    slowest rank's step time."""
    return world * units_per_rank / (max_step_ms / 1e3)


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- workload


def prefill_inputs(w, device):
    ly = w.layer("csa")
    raw, qs = make.make_raw(w, device), make.make_queries(w, device)
    make.plant_prefill(w, ly, raw, qs, device)
    bias = make.make_bias(w, ly, device)
    return raw, qs, bias


def attention_flops(w, ly, q_pos: np.ndarray, n_c: int) -> float:
    """4*H*D per (query, key): keys = min(k, visible entries) + window length (CSA),
    or all visible entries + window length (HCA)."""
    t = q_pos.astype(np.int64)
    vis = np.minimum((t + 1) // ly.r, n_c)
    comp = np.minimum(vis, ly.k) if ly.kind == "csa" else vis
    win = np.minimum(w.W, t + 1)
    return 4.0 * w.H * w.D * float((comp + win).sum())


# Sources that define each profiled kernel (its code, helpers and launch).
KERNEL_SOURCES = {"attention": ["attn_hm.cuh", "attn_tc.cuh", "attn.cuh", "sm100.cuh", "common.cuh"]}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "sparse_attention_hyb_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was
    taken on the current sources of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("source_hash") != source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch")


class PrefillStep:
    """All buffers of one CSA prefill layer, preallocated; run() enqueues the three calls."""

    def __init__(self, S, w, raw, qs, bias):
        self.S, self.w, self.ly = S, w, w.layer("csa")
        self.raw, self.qs, self.bias = raw, qs, bias
        ly, dev = self.ly, raw["xk"].device
        L = raw["xk"].shape[1]
        self.n_c = L // ly.r
        self.kc = torch.empty(1, self.n_c, w.D, dtype=raw["xk"].dtype, device=dev)
        self.vc = torch.empty_like(self.kc)
        self.ic = torch.empty(1, self.n_c, w.dI, dtype=raw["xk"].dtype, device=dev)
        self.idx = torch.empty(1, w.T, ly.k, dtype=torch.int32, device=dev)
        self.o = torch.empty_like(qs["q"])
        self.lse = torch.empty(1, w.T, w.H, dtype=torch.float32, device=dev)
        A = S.abi
        nb = A.hyb_index_topk_workspace_size(A.HYB_DTYPE_BF16, 1, w.T, self.n_c, w.dI, ly.k, A.HYB_INDEX_FLAT)
        self.ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
        self.scale = 1.0 / math.sqrt(w.D)

    def run(self, ev=None):
        A, ly, raw, qs = self.S.abi, self.ly, self.raw, self.qs
        if ev:
            ev[0].record()
        A.hyb_compress(raw["xk"], raw["xv"], raw["xi"], raw["z"], self.bias, ly.r, ly.overlap, 0, self.n_c,
                       self.kc, self.vc, self.ic)
        if ev:
            ev[1].record()
        A.hyb_index_topk(qs["qi"], qs["q_pos"], self.ic, self.n_c, ly.r, ly.k, A.HYB_INDEX_FLAT, None, 0, 0, 0,
                         self.idx, self.ws)
        if ev:
            ev[2].record()
        A.hyb_attn_fwd(qs["q"], qs["q_pos"], self.kc, self.vc, self.n_c, ly.r, self.idx, ly.k, raw["xk"],
                       raw["xv"], self.w.W, self.scale, self.o, self.lse, A.HYB_ATTN_PREFILL, None)
        if ev:
            ev[3].record()


def capture(fn, n_events):
    """Captures fn(events) into a CUDA graph (after one eager run on the capture
    stream); returns (graph, events).  Replaying re-records the same events."""
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_events)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(None)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(ev)
    return g, ev


def bench_prefill(S, w, steps, warmup, world, flush):
    raw, qs, bias = prefill_inputs(w, "cuda")
    st = PrefillStep(S, w, raw, qs, bias)
    for _ in range(warmup):
        st.run()
    torch.cuda.synchronize()
    if S.abi.hyb_get_device_status() != 0:
        raise RuntimeError("device status error during warm-up")
    n0 = S.abi.hyb_kernel_launches()
    graph, ev = capture(st.run, 4)
    per_step = (S.abi.hyb_kernel_launches() - n0) // 2     # one eager run + one captured run
    barrier(world)
    torch.cuda.synchronize()
    stage = []
    for i in range(steps):
        flush.zero_()                      # evict L2 between timed steps (outside the events)
        graph.replay()
        torch.cuda.synchronize()
        stage.append([ev[j].elapsed_time(ev[j + 1]) for j in range(3)])
    torch.cuda.synchronize()
    barrier(world)
    launches = per_step * steps
    stage = np.array(stage)
    step_ms = float(stage.sum(axis=1).mean())
    median_ms = float(np.median(stage.sum(axis=1)))
    flops = attention_flops(w, st.ly, qs["q_pos"][0].cpu().numpy(), st.n_c)
    return st, {"step_ms": step_ms, "median_ms": median_ms, "stage_ms": stage.mean(axis=0).tolist(), "launches": launches,
                "attn_flops": flops}


def bench_e2e(S, st, steps):
    """The same step through host buffers: every step's inputs are copied from
    pinned host memory and its outputs (o, lse) back, inside the timed region.
    The copies overlap the compute: two device buffer sets, step i+1's inputs go
    up on one stream and step i-1's outputs come down on another while step i
    computes.  Returns (ms per step, H2D bytes per step, D2H bytes per step)."""
    names = ["xk", "xv", "xi", "z"]
    host_raw = {k: st.raw[k].cpu().pin_memory() for k in names}
    host_q = {k: st.qs[k].cpu().pin_memory() for k in ("q", "qi", "q_pos")}
    host_b = st.bias.cpu().pin_memory()
    out_o = [torch.empty(st.o.shape, dtype=st.o.dtype, pin_memory=True) for _ in range(2)]
    out_l = [torch.empty(st.lse.shape, dtype=st.lse.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in list(host_raw.values()) + list(host_q.values())) \
        + host_b.numel() * 4
    d2h = out_o[0].numel() * out_o[0].element_size() + out_l[0].numel() * 4
    # a second buffer set: inputs, caches, outputs and workspace of its own
    raw2 = {k: torch.empty_like(v) for k, v in st.raw.items()}
    qs2 = {k: torch.empty_like(v) for k, v in st.qs.items()}
    sets = [st, PrefillStep(S, st.w, raw2, qs2, torch.empty_like(st.bias))]
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i % 2
        x = sets[b]
        with torch.cuda.stream(up):
            up.wait_event(done[b])          # step i-2 no longer reads this set's inputs
            for k in names:
                x.raw[k].copy_(host_raw[k], non_blocking=True)
            for k in host_q:
                x.qs[k].copy_(host_q[k], non_blocking=True)
            x.bias.copy_(host_b, non_blocking=True)
            in_ready[b].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(in_ready[b])
            comp.wait_event(out_read[b])    # step i-2's outputs have left this set
            x.run()
            done[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(done[b])
            out_o[b].copy_(x.o, non_blocking=True)
            out_l[b].copy_(x.lse, non_blocking=True)
            out_read[b].record(down)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(steps):
        step(i)
    e1.record(down)                          # after the last D2H, which follows every copy and call
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def bench_decode(S, steps, warmup, flush):
    w = C.DECODE_BS64_128K
    qs = make.make_queries(w, "cuda")
    cache = make.make_decode_cache(w, "cuda")
    make.plant_decode(w, w.layer("csa"), cache, qs, "cuda")
    A = S.abi
    csa, hca = w.layer("csa"), w.layer("hca")
    nc_c, nc_h = w.L // csa.r, w.L // hca.r
    idx = torch.empty(w.batch, 1, csa.k, dtype=torch.int32, device="cuda")
    o = torch.empty_like(qs["q"])
    o2 = torch.empty_like(qs["q"])
    lse = torch.empty(w.batch, 1, w.H, dtype=torch.float32, device="cuda")
    lse2 = torch.empty_like(lse)
    wsi = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, w.batch, 1, nc_c, w.dI, csa.k, 0)),
                      dtype=torch.uint8, device="cuda")
    wsa = torch.empty(max(256, A.hyb_attn_fwd_workspace_size(1, w.batch, 1, w.H, w.D, csa.k, nc_c, w.W, 1)),
                      dtype=torch.uint8, device="cuda")
    wsh = torch.empty(max(256, A.hyb_attn_fwd_workspace_size(1, w.batch, 1, w.H, w.D, 0, nc_h, w.W, 1)),
                      dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(w.D)

    def step(ev=None):
        if ev:
            ev[0].record()
        A.hyb_index_topk(qs["qi"], qs["q_pos"], cache["ic"], nc_c, csa.r, csa.k, A.HYB_INDEX_FLAT, None, 0, 0, 0,
                         idx, wsi)
        A.hyb_attn_fwd(qs["q"], qs["q_pos"], cache["kc_csa"], cache["vc_csa"], nc_c, csa.r, idx, csa.k,
                       cache["kw"], cache["vw"], w.W, scale, o, lse, A.HYB_ATTN_DECODE, wsa)
        if ev:
            ev[1].record()
        A.hyb_attn_fwd(qs["q"], qs["q_pos"], cache["kc_hca"], cache["vc_hca"], nc_h, hca.r, None, 0,
                       cache["kw"], cache["vw"], w.W, scale, o2, lse2, A.HYB_ATTN_DECODE, wsh)
        if ev:
            ev[2].record()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph, ev = capture(step, 3)
    times = []
    for i in range(steps):
        flush.zero_()
        graph.replay()
        torch.cuda.synchronize()
        times.append((ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])))
    csa_ms = float(np.mean([t[0] for t in times]))
    hca_ms = float(np.mean([t[1] for t in times]))
    bytes_csa = w.batch * (nc_c * w.dI * 2 + (csa.k + w.W) * 2 * w.D * 2 + 2 * w.H * w.D * 2)
    bytes_hca = w.batch * ((nc_h + w.W) * 2 * w.D * 2 + 2 * w.H * w.D * 2)
    return {"workload": w.name, "tokens_per_s_csa_plus_hca": w.batch / ((csa_ms + hca_ms) / 1e3),
            "tokens_per_s_csa": w.batch / (csa_ms / 1e3), "tokens_per_s_hca": w.batch / (hca_ms / 1e3),
            "ms_csa": csa_ms, "ms_hca": hca_ms,
            "hbm_gbs_csa": bytes_csa / (csa_ms / 1e3) / 1e9, "hbm_gbs_hca": bytes_hca / (hca_ms / 1e3) / 1e9,
            "algorithmic_bytes_csa": bytes_csa, "algorithmic_bytes_hca": bytes_hca}


def decode_batch(decode) -> int:
    return C.by_name(decode["workload"]).batch


def bench_decode_append(S, warmup, flush, n_steps=512):
    """The fused decode-step state update for batch 64 at 128K: n_steps
    consecutive tokens (a CSA entry every 4, an HCA entry every 128, a HISA
    representative every 512), replayed as one CUDA graph; amortized time per step."""
    w = C.DECODE_BS64_128K
    A = S.abi
    csa, hca, blk = w.layer("csa"), w.layer("hca"), 128
    B, D, dI, ring, t0 = w.batch, w.D, w.dI, w.W, w.L
    dt = torch.bfloat16
    ncap, nhcap = (t0 + n_steps) // csa.r, (t0 + n_steps) // hca.r
    kc = torch.zeros(B, ncap, D, dtype=dt, device="cuda")
    vc, ic = torch.zeros_like(kc), torch.zeros(B, ncap, dI, dtype=dt, device="cuda")
    kh = torch.zeros(B, nhcap, D, dtype=dt, device="cuda")
    vh = torch.zeros_like(kh)
    reps = torch.zeros(B, ncap // blk, dI, dtype=dt, device="cuda")
    kw = torch.zeros(B, ring, D, dtype=dt, device="cuda")
    vw, iw = torch.zeros_like(kw), torch.zeros(B, ring, dI, dtype=dt, device="cuda")
    zw = torch.zeros(B, ring, dtype=torch.float32, device="cuda")
    xk = make.normal_tensor(7, "ak", (B, D), 0.1, "bf16", "cuda")
    xv = make.normal_tensor(7, "av", (B, D), 0.1, "bf16", "cuda")
    xi = make.normal_tensor(7, "ai", (B, dI), 0.1, "bf16", "cuda")
    z = make.normal_tensor(7, "az", (B,), 1.0, "f32", "cuda")
    bc, bh = make.make_bias(w, csa, "cuda"), make.make_bias(w, hca, "cuda")
    pos = (t0 + torch.arange(n_steps, dtype=torch.int32, device="cuda"))[:, None].repeat(1, B).contiguous()

    def step(ev):
        _rec(ev, 0)
        for i in range(n_steps):
            A.hyb_decode_append(xk, xv, xi, z, pos[i], kw, vw, iw, zw, bias_csa=bc, r_csa=csa.r, overlap=csa.overlap,
                                kc=kc, vc=vc, ic=ic, bias_hca=bh, r_hca=hca.r, kc_hca=kh, vc_hca=vh, block=blk,
                                reps=reps)
        _rec(ev, 1)

    (ms,) = graph_times(step, 1, 3, warmup, flush)
    if A.hyb_get_device_status() != 0:
        raise RuntimeError("device status error in the decode state update")
    return {"batch": B, "steps_timed_together": n_steps, "us_per_step": ms * 1e3 / n_steps,
            "what": "ring append of K, V, indexer key and logit; CSA entry every 4 tokens, HCA entry every 128, "
                    "HISA representative every 512 (one fused launch per step)"}


# --------------------------------------------------------------------------- the other configs


def _rec(ev, i):
    if ev:
        ev[i].record()


def graph_times(step, n_seg, steps, warmup, flush):
    """Median time (ms) of each of the n_seg segments of step(ev), replayed as one
    CUDA graph per step with L2 flushed between replays (outside the events)."""
    for _ in range(warmup):
        step(None)
    torch.cuda.synchronize()
    graph, ev = capture(step, n_seg + 1)
    seg = []
    for _ in range(steps):
        flush.zero_()
        graph.replay()
        torch.cuda.synchronize()
        seg.append([ev[j].elapsed_time(ev[j + 1]) for j in range(n_seg)])
    del graph
    return [float(x) for x in np.median(np.array(seg), axis=0)]


def selection_iou(a, b) -> float:
    """Mean over rows of |A & B| / |A | B| for two index sets per row ([R, k] int32,
    valid entries ascending then -1 padding, as the indexer writes them)."""
    a, b = a.reshape(-1, a.shape[-1]).long(), b.reshape(-1, b.shape[-1]).long()
    s, _ = torch.sort(torch.cat([a, b], 1), dim=1)
    inter = ((s[:, 1:] == s[:, :-1]) & (s[:, 1:] >= 0)).sum(1).float()
    union = ((a >= 0).sum(1) + (b >= 0).sum(1)).float() - inter
    return float((inter / union.clamp(min=1)).mean())


def planted_recall(idx, qi, ic, planted) -> float:
    """Fraction of (query, planted entry) pairs with cosine above 0.4 -- the planted
    construction gives 0.5 -- whose entry the query selected."""
    if len(planted) == 0:
        return float("nan")
    js = torch.as_tensor(planted, device=ic.device).long()
    q = qi.reshape(-1, qi.shape[-1]).float()
    kp = ic.reshape(-1, ic.shape[-1])[js].float()
    cos = (q @ kp.T) / (q.norm(dim=1, keepdim=True) * kp.norm(dim=1)[None, :]).clamp(min=1e-30)
    r, c = torch.nonzero(cos > 0.4, as_tuple=True)
    if r.numel() == 0:
        return float("nan")
    sel = idx.reshape(-1, idx.shape[-1]).long()
    return float((sel[r] == js[c][:, None]).any(1).float().mean())


def _dense_flops(w, r, n_c, q_pos):
    t = q_pos.astype(np.int64)
    return 4.0 * w.H * w.D * float((np.minimum((t + 1) // r, n_c) + np.minimum(w.W, t + 1)).sum())


def bench_hca_prefill(S, st, csa_step_ms, steps, warmup, flush, pk):
    """HCA layer (r=128, dense over all visible entries + window) on the 32K prefill
    inputs, and the CSA+HCA pair."""
    w, raw, qs, A = st.w, st.raw, st.qs, S.abi
    ly = C.HCA128
    n_c = w.L // ly.r
    bias = make.make_bias(w, ly, "cuda")
    kc = torch.empty(1, n_c, w.D, dtype=raw["xk"].dtype, device="cuda")
    vc = torch.empty_like(kc)
    o = torch.empty_like(qs["q"])
    lse = torch.empty(1, w.T, w.H, dtype=torch.float32, device="cuda")

    def step(ev):
        _rec(ev, 0)
        A.hyb_compress(raw["xk"], raw["xv"], None, raw["z"], bias, ly.r, ly.overlap, 0, n_c, kc, vc, None)
        _rec(ev, 1)
        A.hyb_attn_fwd(qs["q"], qs["q_pos"], kc, vc, n_c, ly.r, None, 0, raw["xk"], raw["xv"], w.W, st.scale,
                       o, lse, A.HYB_ATTN_PREFILL, None)
        _rec(ev, 2)

    comp_ms, attn_ms = graph_times(step, 2, steps, warmup, flush)
    fl = _dense_flops(w, ly.r, n_c, qs["q_pos"][0].cpu().numpy())
    ms = comp_ms + attn_ms
    return {"workload": "hca_prefill_32k_bf16", "tokens_per_s": w.T / (ms / 1e3), "ms": ms,
            "stages_ms": {"compress": comp_ms, "attention": attn_ms},
            "attention_tflops": fl / (attn_ms / 1e3) / 1e12,
            "attention_frac_of_bf16_peak": fl / (attn_ms / 1e3) / 1e12 / pk["bf16_tflops"],
            "csa_plus_hca_tokens_per_s": w.T / ((csa_step_ms + ms) / 1e3)}


def bench_compress_pc(S, st, steps, warmup, flush, pk):
    """S1 of the 32K CSA layer with per-channel compression weights (logits [L, D]
    for K and V, [L, dI] for the indexer keys): HBM-bound streaming pass."""
    w, raw, A = st.w, st.raw, S.abi
    ly = st.ly
    span = 2 * ly.r if ly.overlap else ly.r
    L = raw["xk"].shape[1]
    zkv = make.normal_tensor(w.seed, "z_kv", (1, L, w.D), 1.0, "f32", "cuda")
    zi = make.normal_tensor(w.seed, "z_i", (1, L, w.dI), 1.0, "f32", "cuda")
    bkv = make.normal_tensor(w.seed, "b_kv", (span, w.D), w.bias_std, "f32", "cuda")
    bi = make.normal_tensor(w.seed, "b_i", (span, w.dI), w.bias_std, "f32", "cuda")

    def step(ev):
        _rec(ev, 0)
        A.hyb_compress_pc(raw["xk"], raw["xv"], raw["xi"], zkv, bkv, zi, bi, ly.r, ly.overlap, 0, st.n_c, st.kc, st.vc,
                          st.ic)
        _rec(ev, 1)

    (ms,) = graph_times(step, 1, steps, warmup, flush)
    byts = L * (2 * w.D + w.dI) * 2 + L * (w.D + w.dI) * 4 + st.n_c * (2 * w.D + w.dI) * 2
    return {"workload": "csa_compress_per_channel_32k_bf16", "ms": ms, "algorithmic_bytes": byts,
            "hbm_gbs": byts / (ms / 1e3) / 1e9, "frac_of_hbm": byts / (ms / 1e3) / 1e9 / pk["hbm_gbs"]}


def bench_real_kv(S, st, steps, warmup, flush):
    """CSA attention at 32K under the real-K/V reading: the 512 selected entries of
    each query stand for their 4 raw tokens each (up to 2048 raw keys + the window)."""
    w, raw, qs, A = st.w, st.raw, st.qs, S.abi
    ly = st.ly
    o = torch.empty_like(qs["q"])
    lse = torch.empty(1, w.T, w.H, dtype=torch.float32, device="cuda")

    def step(ev):
        _rec(ev, 0)
        A.hyb_attn_fwd(qs["q"], qs["q_pos"], None, None, st.n_c, ly.r, st.idx, ly.k, raw["xk"], raw["xv"], w.W,
                       st.scale, o, lse, A.HYB_ATTN_PREFILL | A.HYB_ATTN_REAL_KV, None)
        _rec(ev, 1)

    (ms,) = graph_times(step, 1, steps, warmup, flush)
    t = qs["q_pos"][0].cpu().numpy().astype(np.int64)
    keys = np.minimum(np.minimum((t + 1) // ly.r, st.n_c), ly.k) * ly.r + np.minimum(w.W, t + 1)
    fl = 4.0 * w.H * w.D * float(keys.sum())
    return {"workload": "csa_real_kv_attention_32k_bf16", "ms": ms, "tokens_per_s": w.T / (ms / 1e3),
            "tflops_upper": fl / (ms / 1e3) / 1e12,
            "note": "flops counted with every selected token (a token inside the window is attended once)"}


def bench_index_128k(S, steps, warmup, flush):
    """Indexer latency of the last query chunk of a 128K prefill (queries
    130048..131071, chunk 1024): flat top-2048 over all visible entries vs HISA
    (128-entry blocks, top-64 blocks, then top-2048 of their entries)."""
    w = C.PREFILL_128K
    ly = w.layer("csa")
    wq = C.scaled(w, T=ly.q_chunk, q_pos0=w.L - ly.q_chunk)
    A = S.abi
    n_c = w.L // ly.r
    raw = make.make_raw(w, "cuda")
    qs = make.make_queries(wq, "cuda")
    planted = make.plant_prefill(wq, ly, raw, qs, "cuda").tolist()
    bias = make.make_bias(w, ly, "cuda")
    kc, vc, ic = S.layer.compress(raw["xk"], raw["xv"], raw["xi"], raw["z"], bias, ly.r, ly.overlap, n_c)
    del raw, kc, vc
    reps = S.layer.block_reps(ic, n_c, ly.block)
    idx = torch.empty(1, wq.T, ly.k, dtype=torch.int32, device="cuda")
    idx2 = torch.empty_like(idx)
    wsf = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, wq.T, n_c, w.dI, ly.k, A.HYB_INDEX_FLAT, 0, 0,
                                                               0)), dtype=torch.uint8, device="cuda")
    wsh = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, wq.T, n_c, w.dI, ly.k, A.HYB_INDEX_HISA,
                                                               ly.block, ly.top_m, ly.q_chunk)),
                      dtype=torch.uint8, device="cuda")

    def step(ev):
        _rec(ev, 0)
        A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, ly.r, ly.k, A.HYB_INDEX_FLAT, None, 0, 0, 0, idx, wsf)
        _rec(ev, 1)
        A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, ly.r, ly.k, A.HYB_INDEX_HISA, reps, ly.block, ly.top_m,
                         ly.q_chunk, idx2, wsh)
        _rec(ev, 2)

    flat_ms, hisa_ms = graph_times(step, 2, steps, warmup, flush)
    step(None)
    torch.cuda.synchronize()
    return {"workload": "csa_index_128k_last_chunk_bf16", "queries": wq.T, "k": ly.k,
            "flat_ms": flat_ms, "hisa_ms": hisa_ms, "hisa_speedup": flat_ms / hisa_ms,
            "hisa_vs_flat_iou": selection_iou(idx2, idx),
            "planted_recall_flat": planted_recall(idx, qs["qi"], ic, planted),
            "planted_recall_hisa": planted_recall(idx2, qs["qi"], ic, planted),
            "planted_entries": len(planted)}


def bench_prefill_128k(S, steps, warmup, flush, pk):
    """The whole CSA layer over a 128K-token prefill (all 131072 queries): S1, the
    flat or the HISA indexer (128-entry blocks, top-64 blocks, query chunk 1024),
    then attention over the selected top-2048 entries and the window."""
    w = C.PREFILL_128K
    ly = w.layer("csa")
    A = S.abi
    raw, qs, bias = prefill_inputs(w, "cuda")
    n_c = w.L // ly.r
    nb = n_c // ly.block
    dt = raw["xk"].dtype
    kc = torch.empty(1, n_c, w.D, dtype=dt, device="cuda")
    vc, ic = torch.empty_like(kc), torch.empty(1, n_c, w.dI, dtype=dt, device="cuda")
    reps = torch.empty(1, nb, w.dI, dtype=dt, device="cuda")
    idx = torch.empty(1, w.T, ly.k, dtype=torch.int32, device="cuda")
    o, lse = torch.empty_like(qs["q"]), torch.empty(1, w.T, w.H, dtype=torch.float32, device="cuda")
    wsf = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, w.T, n_c, w.dI, ly.k, A.HYB_INDEX_FLAT, 0, 0, 0)),
                      dtype=torch.uint8, device="cuda")
    wsh = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, w.T, n_c, w.dI, ly.k, A.HYB_INDEX_HISA,
                                                               ly.block, ly.top_m, ly.q_chunk)),
                      dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(w.D)

    def layer(hisa):
        def step(ev):
            _rec(ev, 0)
            A.hyb_compress(raw["xk"], raw["xv"], raw["xi"], raw["z"], bias, ly.r, ly.overlap, 0, n_c, kc, vc, ic)
            if hisa:
                A.hyb_block_reps(ic, ly.block, 0, nb, reps)
            _rec(ev, 1)
            if hisa:
                A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, ly.r, ly.k, A.HYB_INDEX_HISA, reps, ly.block,
                                 ly.top_m, ly.q_chunk, idx, wsh)
            else:
                A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, ly.r, ly.k, A.HYB_INDEX_FLAT, None, 0, 0, 0, idx,
                                 wsf)
            _rec(ev, 2)
            A.hyb_attn_fwd(qs["q"], qs["q_pos"], kc, vc, n_c, ly.r, idx, ly.k, raw["xk"], raw["xv"], w.W, scale, o,
                           lse, A.HYB_ATTN_PREFILL, None)
            _rec(ev, 3)
        return step

    out = {"workload": "csa_prefill_128k_bf16", "queries": w.T, "k": ly.k}
    flops = attention_flops(w, ly, qs["q_pos"][0].cpu().numpy(), n_c)
    for name, hisa in (("flat", False), ("hisa", True)):
        c_ms, i_ms, a_ms = graph_times(layer(hisa), 3, max(3, steps // 4), warmup, flush)
        tot = c_ms + i_ms + a_ms
        out[f"tokens_per_s_{name}"] = w.T / (tot / 1e3)
        out[f"stages_ms_{name}"] = {"compress": c_ms, "index_topk": i_ms, "attention": a_ms}
        out[f"attention_frac_of_bf16_peak_{name}"] = flops / (a_ms / 1e3) / 1e12 / pk["bf16_tflops"]
    return out


def bench_index_128k_tokens(S, steps, warmup, flush):
    """Token-level indexer (r = 1, no compression: the raw indexer keys are the
    keys, as in DSA) for the last 1024 queries of a 128K sequence: flat top-2048
    over all previous tokens vs HISA (128-token blocks, top-64 blocks, top-2048 of
    their tokens) -- the setting of the pages' flat-vs-HISA comparison."""
    w = C.PREFILL_128K
    ly = w.layer("csa")
    wq = C.scaled(w, T=ly.q_chunk, q_pos0=w.L - ly.q_chunk)
    A = S.abi
    n_c = w.L
    ic = make.normal_tensor(w.seed, "raw_index", (1, w.L, w.dI), w.i_scale, w.dtype, "cuda")
    reps = S.layer.block_reps(ic, n_c, ly.block)
    qs = make.make_queries(wq, "cuda")
    idx = torch.empty(1, wq.T, ly.k, dtype=torch.int32, device="cuda")
    idx2 = torch.empty_like(idx)
    wsf = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, wq.T, n_c, w.dI, ly.k, A.HYB_INDEX_FLAT, 0, 0,
                                                               0)), dtype=torch.uint8, device="cuda")
    wsh = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, wq.T, n_c, w.dI, ly.k, A.HYB_INDEX_HISA,
                                                               ly.block, ly.top_m, ly.q_chunk)),
                      dtype=torch.uint8, device="cuda")

    def step(ev):
        _rec(ev, 0)
        A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, 1, ly.k, A.HYB_INDEX_FLAT, None, 0, 0, 0, idx, wsf)
        _rec(ev, 1)
        A.hyb_index_topk(qs["qi"], qs["q_pos"], ic, n_c, 1, ly.k, A.HYB_INDEX_HISA, reps, ly.block, ly.top_m,
                         ly.q_chunk, idx2, wsh)
        _rec(ev, 2)

    flat_ms, hisa_ms = graph_times(step, 2, steps, warmup, flush)
    step(None)
    torch.cuda.synchronize()
    return {"workload": "token_index_128k_last_chunk_bf16", "queries": wq.T, "k": ly.k, "r": 1,
            "flat_ms": flat_ms, "hisa_ms": hisa_ms, "hisa_speedup": flat_ms / hisa_ms,
            "hisa_vs_flat_iou": selection_iou(idx2, idx)}


def bench_1m(S, steps, warmup, flush, pk):
    """1M-token context: S1 over the whole prefix (CSA with indexer keys, HCA, HISA
    block representatives), a batch-1 decode step (CSA with the HISA indexer, HCA)
    and an 8K-query chunked prefill at the end of the context."""
    wd, wc = C.CTX_1M_DECODE, C.CTX_1M_CHUNK
    csa, hca = wd.layer("csa"), wd.layer("hca")
    A = S.abi
    L, dt = wd.L, torch.bfloat16
    raw = make.make_raw(wd, "cuda")                       # L + 1 tokens (the decode token last)
    ring = make.ring_from_raw(wd, raw)
    xk, xv, xi, z = (raw[n][:, :L] for n in ("xk", "xv", "xi", "z"))
    ncc, nch = L // csa.r, L // hca.r
    bias_c, bias_h = make.make_bias(wd, csa, "cuda"), make.make_bias(wd, hca, "cuda")
    kc_c = torch.empty(1, ncc, wd.D, dtype=dt, device="cuda")
    vc_c, ic_c = torch.empty_like(kc_c), torch.empty(1, ncc, wd.dI, dtype=dt, device="cuda")
    kc_h = torch.empty(1, nch, wd.D, dtype=dt, device="cuda")
    vc_h = torch.empty_like(kc_h)
    nb = ncc // csa.block
    reps = torch.empty(1, nb, wd.dI, dtype=dt, device="cuda")

    def s1(ev):
        _rec(ev, 0)
        A.hyb_compress(xk, xv, xi, z, bias_c, csa.r, csa.overlap, 0, ncc, kc_c, vc_c, ic_c)
        A.hyb_block_reps(ic_c, csa.block, 0, nb, reps)
        _rec(ev, 1)
        A.hyb_compress(xk, xv, None, z, bias_h, hca.r, hca.overlap, 0, nch, kc_h, vc_h, None)
        _rec(ev, 2)

    s1_csa_ms, s1_hca_ms = graph_times(s1, 2, steps, warmup, flush)
    s1_bytes_csa = L * (2 * wd.D + wd.dI) * 2 + L * 4 + ncc * (2 * wd.D + wd.dI) * 2 + nb * wd.dI * 2
    s1_bytes_hca = L * 2 * wd.D * 2 + L * 4 + nch * 2 * wd.D * 2
    scale = 1.0 / math.sqrt(wd.D)
    # ---- decode step, batch 1
    qd = make.make_queries(wd, "cuda")
    idx_d = torch.empty(1, 1, csa.k, dtype=torch.int32, device="cuda")
    od, od2 = torch.empty_like(qd["q"]), torch.empty_like(qd["q"])
    lsed = torch.empty(1, 1, wd.H, dtype=torch.float32, device="cuda")
    lsed2 = torch.empty_like(lsed)
    wsi = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, 1, ncc, wd.dI, csa.k, A.HYB_INDEX_HISA,
                                                               csa.block, csa.top_m, 0)), dtype=torch.uint8,
                      device="cuda")
    wsa = torch.empty(max(256, A.hyb_attn_fwd_workspace_size(1, 1, 1, wd.H, wd.D, csa.k, ncc, wd.W, 1)),
                      dtype=torch.uint8, device="cuda")
    wsh = torch.empty(max(256, A.hyb_attn_fwd_workspace_size(1, 1, 1, wd.H, wd.D, 0, nch, wd.W, 1)),
                      dtype=torch.uint8, device="cuda")

    def dec(ev):
        _rec(ev, 0)
        A.hyb_index_topk(qd["qi"], qd["q_pos"], ic_c, ncc, csa.r, csa.k, A.HYB_INDEX_HISA, reps, csa.block,
                         csa.top_m, 0, idx_d, wsi)
        A.hyb_attn_fwd(qd["q"], qd["q_pos"], kc_c, vc_c, ncc, csa.r, idx_d, csa.k, ring["kw"], ring["vw"], wd.W,
                       scale, od, lsed, A.HYB_ATTN_DECODE, wsa)
        _rec(ev, 1)
        A.hyb_attn_fwd(qd["q"], qd["q_pos"], kc_h, vc_h, nch, hca.r, None, 0, ring["kw"], ring["vw"], wd.W, scale,
                       od2, lsed2, A.HYB_ATTN_DECODE, wsh)
        _rec(ev, 2)

    dec_csa_ms, dec_hca_ms = graph_times(dec, 2, steps, warmup, flush)
    cand = csa.top_m * csa.block
    dec_bytes_csa = nb * wd.dI * 2 + cand * wd.dI * 2 + (csa.k + wd.W) * 2 * wd.D * 2 + 2 * wd.H * wd.D * 2
    dec_bytes_hca = (nch + wd.W) * 2 * wd.D * 2 + 2 * wd.H * wd.D * 2
    # ---- 8K-query chunked prefill at the end of the context
    qc = make.make_queries(wc, "cuda")
    idx_c = torch.empty(1, wc.T, csa.k, dtype=torch.int32, device="cuda")
    oc, oc2 = torch.empty_like(qc["q"]), torch.empty_like(qc["q"])
    lsec = torch.empty(1, wc.T, wd.H, dtype=torch.float32, device="cuda")
    lsec2 = torch.empty_like(lsec)
    wsc = torch.empty(max(256, A.hyb_index_topk_workspace_size(1, 1, wc.T, ncc, wd.dI, csa.k, A.HYB_INDEX_HISA,
                                                               csa.block, csa.top_m, 1024)), dtype=torch.uint8,
                      device="cuda")

    def chunk(ev):
        _rec(ev, 0)
        A.hyb_index_topk(qc["qi"], qc["q_pos"], ic_c, ncc, csa.r, csa.k, A.HYB_INDEX_HISA, reps, csa.block,
                         csa.top_m, 1024, idx_c, wsc)
        _rec(ev, 1)
        A.hyb_attn_fwd(qc["q"], qc["q_pos"], kc_c, vc_c, ncc, csa.r, idx_c, csa.k, xk, xv, wd.W, scale, oc, lsec,
                       A.HYB_ATTN_PREFILL, None)
        _rec(ev, 2)
        A.hyb_attn_fwd(qc["q"], qc["q_pos"], kc_h, vc_h, nch, hca.r, None, 0, xk, xv, wd.W, scale, oc2, lsec2,
                       A.HYB_ATTN_PREFILL, None)
        _rec(ev, 3)

    idx_ms, attn_c_ms, attn_h_ms = graph_times(chunk, 3, steps, warmup, flush)
    # HISA-vs-flat selection IoU (not timed): the decode row, and the chunk's last 1024 queries
    torch.cuda.synchronize()
    iou_dec = selection_iou(idx_d, S.layer.index_topk(qd["qi"], qd["q_pos"], ic_c, ncc, csa.r, csa.k))
    tail = slice(wc.T - 1024, wc.T)
    flat_tail = S.layer.index_topk(qc["qi"][:, tail].contiguous(), qc["q_pos"][:, tail].contiguous(), ic_c, ncc, csa.r,
                                   csa.k)
    iou_chunk = selection_iou(idx_c[:, tail], flat_tail)
    del flat_tail
    qp = qc["q_pos"][0].cpu().numpy().astype(np.int64)
    fl_c = 4.0 * wd.H * wd.D * float((np.minimum(np.minimum((qp + 1) // csa.r, ncc), csa.k)
                                       + np.minimum(wd.W, qp + 1)).sum())
    fl_h = _dense_flops(wc, hca.r, nch, qp)
    hbm = pk["hbm_gbs"]
    return {
        "s1_1m": {"csa_ms": s1_csa_ms, "hca_ms": s1_hca_ms,
                  "csa_hbm_gbs": s1_bytes_csa / (s1_csa_ms / 1e3) / 1e9,
                  "hca_hbm_gbs": s1_bytes_hca / (s1_hca_ms / 1e3) / 1e9,
                  "csa_frac_of_hbm": s1_bytes_csa / (s1_csa_ms / 1e3) / 1e9 / hbm,
                  "hca_frac_of_hbm": s1_bytes_hca / (s1_hca_ms / 1e3) / 1e9 / hbm},
        "decode_bs1_ctx1m": {"csa_hisa_ms": dec_csa_ms, "hca_ms": dec_hca_ms,
                             "tokens_per_s_csa_plus_hca": 1.0 / ((dec_csa_ms + dec_hca_ms) / 1e3),
                             "csa_hbm_gbs": dec_bytes_csa / (dec_csa_ms / 1e3) / 1e9,
                             "hca_hbm_gbs": dec_bytes_hca / (dec_hca_ms / 1e3) / 1e9,
                             "hisa_vs_flat_iou": iou_dec},
        "chunk_prefill_8k_at_1m": {"csa_index_hisa_ms": idx_ms, "csa_attention_ms": attn_c_ms,
                                   "hca_attention_ms": attn_h_ms,
                                   "tokens_per_s_csa": wc.T / ((idx_ms + attn_c_ms) / 1e3),
                                   "tokens_per_s_hca": wc.T / (attn_h_ms / 1e3),
                                   "csa_attention_tflops": fl_c / (attn_c_ms / 1e3) / 1e12,
                                   "hca_attention_tflops": fl_h / (attn_h_ms / 1e3) / 1e12,
                                   "hisa_vs_flat_iou_last_1024": iou_chunk},
    }


# --------------------------------------------------------------------------- CPU oracle


def _oracle_rows_worker(args):
    """One host core of the CPU baseline: runs the oracle's S2+S3 on its rows (the
    caches come from the parent through memory-mapped files) until its time budget
    is spent.  Returns (rows done, seconds spent on them)."""
    cache_dir, rows, budget, wname = args
    os.environ["OMP_NUM_THREADS"] = "1"
    torch.set_num_threads(1)
    import oracle as O
    w = {c.name: c for c in (C.PREFILL_32K, C.PREFILL_128K)}[wname]
    ly = w.layer("csa")
    ld = lambda n: np.load(os.path.join(cache_dir, n + ".npy"), mmap_mode="r")
    kc, vc, ic, xk, xv, qi64 = (ld(n) for n in ("kc", "vc", "ic", "xk", "xv", "qi"))
    p = O.LayerParams("csa", ly.r, ly.overlap, w.W, 1.0 / math.sqrt(w.D), w.dtype, k=ly.k)
    hd = w.H * w.D
    done, t_rows = 0, 0.0
    for i in rows:
        if t_rows >= budget:
            break
        q_row = make.to_storage(rng.normal(w.seed, "q", int(i) * hd, hd) * w.x_scale, w.dtype).float().double()
        t1 = time.perf_counter()
        O.layer_row(p, q_row.view(w.H, w.D).numpy(), qi64[i], w.q_pos0 + int(i), kc, vc, ic, None, xk, xv,
                    xk.shape[0])
        t_rows += time.perf_counter() - t1
        done += 1
    return done, t_rows


def oracle_sample(w, seconds: float):
    """Times the fp64 oracle on the host's cores: S1 over the whole sequence in
    this process, then S2+S3 row by row on every core of the process's affinity
    mask (one single-threaded worker per core, started with `spawn`) until each
    worker's budget is spent.  Returns (tokens/s, rows, seconds, cores)."""
    import multiprocessing as mp
    import oracle as O
    ly = w.layer("csa")
    raw = make.make_raw(w)
    qi = make.normal_tensor(w.seed, "q_index", (w.batch, w.T, w.dI), w.i_scale, w.dtype)
    qs = {"qi": qi, "q_pos": make.query_positions(w)}
    make.plant_prefill(w, ly, raw, qs)
    bias = make.make_bias(w, ly)
    f64 = lambda t: t.float().double().numpy()
    p = O.LayerParams("csa", ly.r, ly.overlap, w.W, 1.0 / math.sqrt(w.D), w.dtype, k=ly.k)
    t0 = time.perf_counter()
    kc, vc, ic = O.build_caches(p, f64(raw["xk"][0]), f64(raw["xv"][0]), f64(raw["xi"][0]), f64(raw["z"][0]),
                                f64(bias))
    t_s1 = time.perf_counter() - t0
    order = torch.argsort(rng.raw_u64(w.seed, "cpu_rows", 0, w.T)).numpy()
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    cores = max(1, min(cores, 64))
    with tempfile.TemporaryDirectory() as d:
        for n, a in (("kc", kc), ("vc", vc), ("ic", ic), ("xk", f64(raw["xk"][0])), ("xv", f64(raw["xv"][0])),
                     ("qi", f64(qs["qi"][0]))):
            np.save(os.path.join(d, n + ".npy"), a)
        jobs = [(d, order[c::cores], seconds, w.name) for c in range(cores)]
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        os.environ.update({k: "1" for k in saved})   # one BLAS thread per worker (read at the workers' start)
        try:
            with mp.get_context("spawn").Pool(cores) as pool:
                res = pool.map(_oracle_rows_worker, jobs)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
    done = sum(r[0] for r in res)
    wall = max(r[1] for r in res)        # the workers run side by side
    per_row = wall / done + t_s1 / w.T
    return 1.0 / per_row, done, wall + t_s1, cores


# --------------------------------------------------------------------------- arms


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = C.PREFILL_32K
    tok_s, rows, secs, cores = oracle_sample(w, max(2.0, args.cpu_seconds / max(1, args.steps)))
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.T / tok_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "T": w.T, "H": w.H, "D": w.D, "dI": w.dI, "r": 4, "k": 512,
                   "W": w.W},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"S1 over all {w.L} tokens (1 core) + S2/S3 for {rows} seeded rows on {cores} "
                                   f"single-threaded workers ({secs:.1f} s)"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import sparse_attention_hyb_b200 as S
    S.abi.lib()
    w = C.PREFILL_32K if args.L is None else C.scaled(C.PREFILL_32K, L=args.L, T=args.L)
    pk, pk_src = peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    clock = ClockSampler(local)
    clock.start()
    st, res = bench_prefill(S, w, args.steps, args.warmup, world, flush)
    clocks = clock.stop()
    step_ms = max_over_ranks(res["step_ms"], world)
    value = replica_throughput(w.T, world, step_ms)
    attn_ms = res["stage_ms"][2]
    achieved = res["attn_flops"] / (attn_ms / 1e3) / 1e12
    peak = pk["bf16_tflops"]
    traffic = measured_traffic("attention")
    if args.prefill_only:
        args.no_decode = args.no_cpu_baseline = args.no_extras = True
        e2e_ms, h2d, d2h = float("nan"), 0, 0
    else:
        e2e_ms, h2d, d2h = bench_e2e(S, st, max(3, args.steps // 2))
        e2e_ms = max_over_ranks(e2e_ms, world)
    decode = None if args.no_decode else bench_decode(S, args.steps, args.warmup, flush)
    if decode is not None:
        upd = bench_decode_append(S, args.warmup, flush)
        decode["state_update"] = upd
        dstep_ms = decode["ms_csa"] + decode["ms_hca"] + upd["us_per_step"] / 1e3
        decode["tokens_per_s_csa_plus_hca_with_update"] = decode_batch(decode) / (dstep_ms / 1e3)
    extras = None
    if not args.no_extras:
        extras = {"hca_prefill_32k": bench_hca_prefill(S, st, step_ms, args.steps, args.warmup, flush, pk),
                  "compress_per_channel_32k": bench_compress_pc(S, st, args.steps, args.warmup, flush, pk),
                  "real_kv_attention_32k": bench_real_kv(S, st, args.steps, args.warmup, flush)}
        del st
        torch.cuda.empty_cache()
        extras["index_128k_last_chunk"] = bench_index_128k(S, args.steps, args.warmup, flush)
        torch.cuda.empty_cache()
        extras["prefill_128k"] = bench_prefill_128k(S, args.steps, args.warmup, flush, pk)
        torch.cuda.empty_cache()
        extras["token_index_128k_last_chunk"] = bench_index_128k_tokens(S, args.steps, args.warmup, flush)
        torch.cuda.empty_cache()
        extras.update(bench_1m(S, args.steps, args.warmup, flush, pk))
        extras["timing"] = "median of the timed steps, CUDA-graph replay, L2 flushed between steps"
    if S.abi.hyb_get_device_status() != 0:
        raise RuntimeError("device status error after the benchmark")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, rows, secs, cores = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"S1 over all {w.L} tokens (1 core) + S2/S3 for {rows} seeded query rows on {cores} "
                         f"single-threaded workers ({secs:.1f} s)"}
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "median_ms_per_step": res["median_ms"],
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "T": w.T, "H": w.H, "D": w.D, "dI": w.dI, "r": 4,
                   "window_span": 8, "k": 512, "W": w.W, "parallelism": f"replicas{world}",
                   "l2": "flushed (256 MiB write) between timed steps, outside the timed events",
                   "launch": "each step is one CUDA-graph replay of the three libhyb calls"},
        "stages_ms": {"compress": res["stage_ms"][0], "index_topk": res["stage_ms"][1],
                      "attention": res["stage_ms"][2]},
        "roofline": {"kernel": "attention (hyb_attn_fwd, prefill)", "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{pk_src} bf16 burst", "flops_per_launch": res["attn_flops"]},
        "gpu_launches": res["launches"],
        "e2e": {"value": None if math.isnan(e2e_ms) else replica_throughput(w.T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clocks,
        "decode": decode,
        "extras": extras,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
