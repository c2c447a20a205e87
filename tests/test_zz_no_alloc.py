"""hyb_index_topk_noalloc: the flat indexer for callers that cannot give the
library device memory (an engine whose pool allocator owns all of HBM, a plugin
whose host framework makes every device allocation).  Its scratch is a fixed
array inside libhyb, so it must agree with hyb_index_topk exactly, including
when the array still holds the previous call's scores.

The file name sorts last on purpose: the array persists for the whole
process, so a run that stops at the first failure has already run every other
test before this one touches it.  The tests pass alone in a fresh process as
well as after the rest of the suite (the array then holds earlier scores)."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import make, rng

from parity import acc_bound, to64, topk_row_check

pytestmark = pytest.mark.gpu
dev = "cuda"


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_hyb_b200 as S
    S.abi.lib()
    return S


def _case(B, T, nc, dI, r, seed, dtype="bf16"):
    sc = dI ** -0.5
    ic = make.normal_tensor(seed, "na_ic", (B, nc, dI), sc, dtype, device=dev)
    qi = make.normal_tensor(seed, "na_qi", (B, T, dI), sc, dtype, device=dev)
    pos = rng.randint_below(seed, "na_pos", 0, B * T, r * nc + 40, device=dev).view(B, T).to(torch.int32)
    return qi, pos, ic


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_two_calls(S, dtype):
    A = S.abi
    cases = [(2, 700, 3000, 128, 4, 64, 11), (1, 2000, 8192, 128, 4, 512, 12)]
    if dtype == "f32":
        cases = [(1, 300, 128, 32, 4, 16, 13), (2, 200, 500, 32, 4, 40, 14)]
    for (B, T, nc, dI, r, k, seed) in cases:      # two calls in a row, different shapes and data
        qi, pos, ic = _case(B, T, nc, dI, r, seed, dtype)
        got = torch.full((B, T, k), -7, dtype=torch.int32, device=dev)
        A.hyb_index_topk_noalloc(qi, pos, ic, nc, r, k, got)
        want = S.layer.index_topk(qi, pos, ic, nc, r, k)
        torch.cuda.synchronize()
        assert A.hyb_get_device_status() == 0
        assert torch.equal(got, want), f"case {(B, T, nc)}: {(got != want).sum().item()} differing indices"


def test_noalloc_decode_rows_that_fill_the_array_exactly(S):
    """Decode shape at the limit: 128 sequences x 32768 entries of fp32 scores is
    exactly the 16 MiB array, so each pass scores one query row per sequence (the
    streaming decode scorer).  Two calls in a row; sampled rows against the oracle."""
    A = S.abi
    B, T, nc, dI, r, k = 128, 2, 32768, 64, 4, 512
    assert B * nc * 4 == 16 << 20
    for seed in (21, 22):
        ic = make.normal_tensor(seed, "na_ic", (B, nc, dI), dI ** -0.5, "bf16", device=dev)
        qi = make.normal_tensor(seed, "na_qi", (B, T, dI), dI ** -0.5, "bf16", device=dev)
        pos = torch.tensor([[r * nc - 1, r * nc - 9]], dtype=torch.int32, device=dev).repeat(B, 1)
        got = torch.full((B, T, k), -7, dtype=torch.int32, device=dev)
        A.hyb_index_topk_noalloc(qi, pos, ic, nc, r, k, got)
        want = S.layer.index_topk(qi, pos, ic, nc, r, k)
        torch.cuda.synchronize()
        assert A.hyb_get_device_status() == 0
        assert torch.equal(got, want), f"seed {seed}: {(got != want).sum().item()} differing indices"
        g = got.cpu().numpy()
        for b in (0, 77, B - 1):
            ic64, qi64 = to64(ic[b]), to64(qi[b])
            for i in range(T):
                n = O.visible_entries(int(pos[b, i]), r, nc)
                ids = np.arange(n)
                s = O.index_scores(qi64[i], ic64, ids)
                iou, _ = topk_row_check(g[b, i], s, ids, k, acc_bound(qi64[i], ic64[:n]), f"b{b} i{i}")
                assert iou >= 0.99


def test_noalloc_rejects_rows_beyond_its_array(S):
    qi, pos, ic = _case(1, 4, 40000, 128, 4, 15)
    idx = torch.empty(1, 4, 16, dtype=torch.int32, device=dev)
    with pytest.raises(S.abi.HybError) as e:
        S.abi.hyb_index_topk_noalloc(qi, pos, ic, 40000, 4, 16, idx)
    assert e.value.status == S.abi.HYB_ERR_UNSUPPORTED
    # one more sequence than the boundary case above: 129 x 32768 x 4 B > 16 MiB
    qi, pos, ic = _case(129, 1, 32768, 64, 4, 16)
    idx = torch.empty(129, 1, 16, dtype=torch.int32, device=dev)
    with pytest.raises(S.abi.HybError) as e:
        S.abi.hyb_index_topk_noalloc(qi, pos, ic, 32768, 4, 16, idx)
    assert e.value.status == S.abi.HYB_ERR_UNSUPPORTED
