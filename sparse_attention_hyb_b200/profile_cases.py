"""Small cases of the kernels whose counters the profiles summarise (for ncu captures).

    python sparse_attention_hyb_b200/profile_cases.py {prefill8k|s1_1m|hisa128k|decode} [reps]

prefill8k: S1 + flat indexer + attention of an 8K-token CSA prefill; s1_1m: CSA and HCA
compression of a 1M-token sequence; hisa128k: the HISA indexer on the last 1024 queries of a
128K prefill; decode: one decode step of 64 sequences x 128K (CSA index + attention, HCA
attention).  Each case runs `reps` times and checks the device status word.  The inputs are the
seeded synthetic workloads; a capture of a few launches holds at most a few GB on the device.
"""
import sys, os, math, torch
sys.path.insert(0, os.environ.get("GRAFT_REPO_ROOT", "/root/repo"))
import sparse_attention_hyb_b200 as S
from workloads import configs as C, make
A = S.abi
which = sys.argv[1]
reps = int(sys.argv[2]) if len(sys.argv) > 2 else 2
if which == "prefill8k":      # compress, indexer scores + select, attention of a CSA prefill of 8K tokens
    w = C.scaled(C.PREFILL_32K, L=8192, T=8192)
    raw, qs = make.make_raw(w, "cuda"), make.make_queries(w, "cuda")
    make.plant_prefill(w, w.layer("csa"), raw, qs, "cuda")
    bias = make.make_bias(w, w.layer("csa"), "cuda")
    for _ in range(reps):
        kc, vc, ic = S.layer.compress(raw["xk"], raw["xv"], raw["xi"], raw["z"], bias, 4, True, 2048)
        idx = S.layer.index_topk(qs["qi"], qs["q_pos"], ic, 2048, 4, 512)
        S.layer.attention(qs["q"], qs["q_pos"], kc, vc, 2048, 4, idx, raw["xk"], raw["xv"], 128, 1 / math.sqrt(128))
elif which == "s1_1m":        # compression of a 1M-token sequence, CSA and HCA
    w = C.CTX_1M_DECODE
    raw = make.make_raw(w, "cuda")
    L = w.L
    for _ in range(reps):
        for ly in w.layers:
            bias = make.make_bias(w, ly, "cuda")
            xi = raw["xi"][:, :L] if ly.kind == "csa" else None
            S.layer.compress(raw["xk"][:, :L], raw["xv"][:, :L], xi, raw["z"][:, :L].contiguous(), bias, ly.r, ly.overlap, L // ly.r)
elif which == "hisa128k":     # HISA indexer of the last 1024 queries of a 128K prefill
    w = C.PREFILL_128K
    ly = w.layer("csa")
    wq = C.scaled(w, T=1024, q_pos0=w.L - 1024)
    raw = make.make_raw(w, "cuda")
    qs = make.make_queries(wq, "cuda")
    bias = make.make_bias(w, ly, "cuda")
    n_c = w.L // 4
    kc, vc, ic = S.layer.compress(raw["xk"], raw["xv"], raw["xi"], raw["z"], bias, 4, True, n_c)
    reps_ = S.layer.block_reps(ic, n_c, 128)
    for _ in range(reps):
        S.layer.index_topk(qs["qi"], qs["q_pos"], ic, n_c, 4, 2048, S.HYB_INDEX_HISA, reps_, 128, 64, 1024)
elif which == "decode":       # decode step, batch 64 x 128K: CSA flat index + attention, HCA attention
    w = C.DECODE_BS64_128K
    qs = make.make_queries(w, "cuda")
    cache = make.make_decode_cache(w, "cuda")
    for _ in range(reps):
        idx = S.layer.index_topk(qs["qi"], qs["q_pos"], cache["ic"], 32768, 4, 512)
        S.layer.attention(qs["q"], qs["q_pos"], cache["kc_csa"], cache["vc_csa"], 32768, 4, idx, cache["kw"], cache["vw"], 128,
                          1 / math.sqrt(128), S.HYB_ATTN_DECODE)
        S.layer.attention(qs["q"], qs["q_pos"], cache["kc_hca"], cache["vc_hca"], 1024, 128, None, cache["kw"], cache["vw"], 128,
                          1 / math.sqrt(128), S.HYB_ATTN_DECODE)
torch.cuda.synchronize()
assert A.hyb_get_device_status() == 0
print("ok", which)
