"""The C ABI without a GPU: libhyb.so loads, exports every entry point that
include/hyb.h declares, and rejects bad arguments on the host before any
launch (these paths touch no CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def A():
    from sparse_attention_hyb_b200 import abi, build
    build.build()
    abi.lib()
    return abi


def _declared():
    src = open(os.path.join(ROOT, "include", "hyb.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hyb_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(A):
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(A.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
        assert n in A.SIGNATURES, f"binding lacks {n}"


def test_status_strings_and_version(A):
    assert A.hyb_abi_version() == 100
    for code in range(7):
        assert A.status_string(code).startswith("HYB_")
    assert A.status_string(99) == "HYB_ERR_UNKNOWN"


def test_host_argument_checks(A):
    L = A.lib()
    # unsupported dtype, null pointers, inconsistent ranges: rejected before any launch
    assert L.hyb_compress(7, 1, 8, 4, 4, 1, 1, None, 1, 1, 4, 1, 0, 1, 1, 1, None, 2, None) == A.HYB_ERR_UNSUPPORTED
    assert L.hyb_compress(1, 1, 8, 4, 4, None, 1, None, 1, 1, 4, 1, 0, 1, 1, 1, None, 2, None) == A.HYB_ERR_INVALID_ARG
    assert L.hyb_compress(1, 1, 8, 4, 4, 1, 1, None, 1, 1, 4, 1, 0, 3, 1, 1, None, 3, None) == A.HYB_ERR_INVALID_ARG
    assert L.hyb_compress(1, 1, 1024, 4, 4, 1, 1, None, 1, 1, 200, 1, 0, 1, 1, 1, None, 1, None) == A.HYB_ERR_UNSUPPORTED
    assert L.hyb_compress(1, 1, 8, 6, 4, 1, 1, None, 1, 1, 4, 1, 0, 1, 1, 1, None, 2, None) == A.HYB_ERR_UNSUPPORTED
    assert L.hyb_block_reps(1, 1, 128, 1, 100, 128, 0, 1, 1, 1, None) == A.HYB_ERR_INVALID_ARG
    # decode append: (dtype, batch, D, dI, xk, xv, xi, z, pos, kw, vw, iw, zw, ring, bias_c, r_c, overlap,
    # kc, vc, ic, nc_cap, bias_h, r_h, kc_h, vc_h, nch_cap, block, reps, nb_cap, stream)
    ok = [1, 2, 128, 128, 1, 1, 1, 1, 1, 1, 1, 1, 1, 128, 1, 4, 1, 1, 1, 1, 64, 1, 128, 1, 1, 4, 16, 1, 4, None]
    bad = list(ok); bad[0] = 9
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_UNSUPPORTED          # dtype
    bad = list(ok); bad[8] = None
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_INVALID_ARG          # no positions
    bad = list(ok); bad[11] = None
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_INVALID_ARG          # indexer key without its ring
    bad = list(ok); bad[13] = 6
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_UNSUPPORTED          # ring shorter than the 2r window
    bad = list(ok); bad[22] = 256
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_UNSUPPORTED          # HCA window longer than the ring
    bad = list(ok); bad[2] = 126
    assert L.hyb_decode_append(*bad) == A.HYB_ERR_UNSUPPORTED          # D not a multiple of 4
    bad = list(ok); bad[1] = 0
    assert L.hyb_decode_append(*bad) == A.HYB_OK                       # empty batch: nothing to do
    # index: bad mode, missing workspace, HISA without representatives
    args = [1, 1, 16, 128, 1, 1, 1, 64, 64, 4, 8]
    assert L.hyb_index_topk(*args, 5, None, 0, 0, 0, 0, 1, None, 0, None) == A.HYB_ERR_INVALID_ARG
    assert L.hyb_index_topk(*args, 0, None, 0, 0, 0, 0, 1, None, 0, None) == A.HYB_ERR_WORKSPACE
    assert L.hyb_index_topk(*args, 1, None, 0, 16, 4, 0, 1, 256, 1 << 20, None) == A.HYB_ERR_INVALID_ARG
    assert L.hyb_index_topk(*args, 0, None, 0, 0, 0, 0, 1, 256 + 8, 1 << 30, None) == A.HYB_ERR_WORKSPACE
    # attention: ring smaller than the window, unsupported head geometry, missing workspace
    a = [1, 1, 4, 64, 128, 1, 1, 1, 1, 10, 10, 4, None, 0, 1, 1]
    assert L.hyb_attn_fwd(*a, 64, 128, ctypes.c_float(0.1), 1, None, 0, None, 0, None) == A.HYB_ERR_INVALID_ARG
    b = [1, 1, 4, 48, 128, 1, 1, 1, 1, 10, 10, 4, None, 0, 1, 1]
    assert L.hyb_attn_fwd(*b, 128, 128, ctypes.c_float(0.1), 1, None, 0, None, 0, None) == A.HYB_ERR_UNSUPPORTED
    assert L.hyb_attn_fwd(*a, 128, 128, ctypes.c_float(0.1), 1, None, 1, None, 0, None) == A.HYB_ERR_WORKSPACE
    # empty problems are fine and launch nothing
    assert L.hyb_attn_fwd(1, 0, 4, 64, 128, None, None, None, None, 0, 0, 4, None, 0, None, None, 128, 128,
                          ctypes.c_float(0.1), None, None, 0, None, 0, None) == A.HYB_OK


def test_workspace_sizes(A):
    f = A.hyb_index_topk_workspace_size
    flat = f(1, 1, 32768, 8192, 128, 512, A.HYB_INDEX_FLAT)
    assert flat >= 64 * 8192 * 4 and flat % 256 == 0
    hisa = f(1, 1, 131072, 32768, 128, 2048, A.HYB_INDEX_HISA, 128, 64, 1024)
    assert hisa >= 1024 * 64 * 128 * 4
    assert A.hyb_attn_fwd_workspace_size(1, 1, 32768, 64, 128, 512, 8192, 128, A.HYB_ATTN_PREFILL) == 0
    # decode splits a query's keys (partials in the workspace) only while fewer than half
    # of the 148 SMs would hold a query: one sequence splits, 64 do not
    assert A.hyb_attn_fwd_workspace_size(1, 1, 1, 64, 128, 512, 32768, 128, A.HYB_ATTN_DECODE) > 0
    assert A.hyb_attn_fwd_workspace_size(1, 64, 1, 64, 128, 512, 32768, 128, A.HYB_ATTN_DECODE) == 0


def test_flat_workspace_budget(A):
    f = A.hyb_index_topk_workspace_size
    # the default pass keeps about 512 MiB of fp32 scores, however long the prefill
    assert f(1, 1, 32768, 8192, 128, 512, A.HYB_INDEX_FLAT) >= 16384 * 8192 * 4
    assert f(1, 1, 131072, 32768, 128, 2048, A.HYB_INDEX_FLAT) <= (512 << 20) + (1 << 20)
    # a smaller q_chunk shrinks it (2048 queries x 8192 entries x 4 B = 64 MiB)
    assert f(1, 1, 32768, 8192, 128, 512, A.HYB_INDEX_FLAT, 0, 0, 2048) <= (64 << 20) + (1 << 20)


def test_decode_split_rule(A):
    # split a query's keys into slices only while fewer than half of the 148 SMs would hold
    # a query: 148 // (2 * queries) slices, at most one per 64 keys; the workspace holds the
    # fp32 partial outputs and lse of every slice (256-byte aligned)
    def ws(batch, ns, H=64, D=128):
        rows = batch * ns * H
        al = lambda x: (x + 255) // 256 * 256
        return al(rows * D * 4) + al(rows * 4)
    f = lambda batch, k, nc: A.hyb_attn_fwd_workspace_size(1, batch, 1, 64, 128, k, nc, 128, A.HYB_ATTN_DECODE)
    assert f(1, 512, 32768) == ws(1, 10)      # 640 keys: capped at one slice per 64 keys
    assert f(1, 0, 8192) == ws(1, 64)         # HCA at 1M (8192 entries + 128): 74 capped at 64
    assert f(37, 512, 32768) == ws(37, 2)     # 148 // 74
    assert f(38, 512, 32768) == 0             # 148 // 76 = 1: no split


def test_binding_checks_shapes_and_types_before_the_call(A):
    """The Python binding refuses output and position tensors whose shape or type
    differs from what the other arguments imply (the kernels would write past them);
    the checks run before the library is called, so host tensors suffice here."""
    import torch
    B, T, dI, nc, k, H, D = 2, 3, 16, 40, 8, 64, 128
    qi, ic = torch.zeros(B, T, dI), torch.zeros(B, nc, dI)
    q_pos = torch.zeros(B, T, dtype=torch.int32)
    idx = torch.zeros(B, T, k, dtype=torch.int32)
    bad_idx = [torch.zeros(B, T, k - 1, dtype=torch.int32), torch.zeros(B, T, k, dtype=torch.int64), None]
    for bi in bad_idx:
        with pytest.raises(ValueError, match="idx"):
            A.hyb_index_topk(qi, q_pos, ic, nc, 4, k, 0, None, 0, 0, 0, bi, None)
        with pytest.raises(ValueError, match="idx"):
            A.hyb_index_topk_noalloc(qi, q_pos, ic, nc, 4, k, bi)
    with pytest.raises(ValueError, match="q_pos"):
        A.hyb_index_topk(qi, q_pos.long(), ic, nc, 4, k, 0, None, 0, 0, 0, idx, None)
    q = torch.zeros(B, T, H, D, dtype=torch.bfloat16)
    kw = torch.zeros(B, 128, D, dtype=torch.bfloat16)
    o, lse = torch.zeros_like(q), torch.zeros(B, T, H)
    args = (q, q_pos, None, None, 0, 4, idx, k, kw, kw, 128, 0.1)
    with pytest.raises(ValueError, match="o:"):
        A.hyb_attn_fwd(*args, o.float(), lse, 0, None)
    with pytest.raises(ValueError, match="lse"):
        A.hyb_attn_fwd(*args, o, lse[:, :, :-1], 0, None)
    with pytest.raises(ValueError, match="idx"):
        A.hyb_attn_fwd(q, q_pos, None, None, 0, 4, bad_idx[0], k, kw, kw, 128, 0.1, o, lse, 0, None)
