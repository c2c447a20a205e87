"""hyb_index_topk_noalloc: the flat indexer for callers that cannot give the
library device memory (an engine whose pool allocator owns all of HBM, a plugin
whose host framework makes every device allocation).  Its scratch is a fixed
array inside libhyb, so it must agree with hyb_index_topk exactly, including
when the array still holds the previous call's scores.

Kept in a file of its own that pytest collects last."""
import pytest
import torch

from workloads import make, rng

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
    ic = make.normal_tensor(seed, "na_ic", (B, nc, dI), sc, dtype).to(dev)
    qi = make.normal_tensor(seed, "na_qi", (B, T, dI), sc, dtype).to(dev)
    pos = rng.randint_below(seed, "na_pos", 0, B * T, r * nc + 40).view(B, T).to(torch.int32).to(dev)
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


def test_noalloc_rejects_rows_beyond_its_array(S):
    qi, pos, ic = _case(1, 4, 40000, 128, 4, 15)
    idx = torch.empty(1, 4, 16, dtype=torch.int32, device=dev)
    with pytest.raises(S.abi.HybError) as e:
        S.abi.hyb_index_topk_noalloc(qi, pos, ic, 40000, 4, 16, idx)
    assert e.value.status == S.abi.HYB_ERR_UNSUPPORTED
