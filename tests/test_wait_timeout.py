"""The failure path of the bounded device waits, made to run on purpose.

hyb_attn_fwd_wait_test runs the tensor-core attention with a short wait limit
and one K-tile arrival withheld in the first CTA: that CTA's waits expire, it
stops without trapping (its issued MMAs finish, its tensor memory is freed)
and the status word reports HYB_ERR_TIMEOUT.  Nothing faults: the same stream
then runs normal calls whose results equal those from before the failure."""
import math

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


def _inputs(B, T, nc, k, L, r=4):
    D, H = 128, 64
    sc = D ** -0.5
    q = make.normal_tensor(41, "wt_q", (B, T, H, D), sc, "bf16", device=dev)
    kc = make.normal_tensor(41, "wt_kc", (B, nc, D), sc, "bf16", device=dev)
    vc = make.normal_tensor(41, "wt_vc", (B, nc, D), sc, "bf16", device=dev)
    kw = make.normal_tensor(41, "wt_kw", (B, L, D), sc, "bf16", device=dev)
    vw = make.normal_tensor(41, "wt_vw", (B, L, D), sc, "bf16", device=dev)
    pos = (rng.randint_below(41, "wt_pos", 0, B * T, L - r * 8, device=dev) + r * 8).view(B, T).to(torch.int32)
    vis = (pos + 1) // r
    u = rng.uniform(41, "wt_idx", 0, B * T * k, device=dev).view(B, T, k)
    idx = torch.sort((u * vis[..., None]).floor().to(torch.int32), dim=-1).values.contiguous()
    return q, pos, kc, vc, kw, vw, idx


@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_expired_wait_reports_timeout_and_the_stream_stays_usable(S, mode):
    A = S.abi
    B, T, nc, k, W, L = (1, 600, 2000, 256, 128, 8000) if mode == "prefill" else (2, 2, 2000, 512, 128, 8000)
    q, pos, kc, vc, kw, vw, idx = _inputs(B, T, nc, k, L)
    md = A.HYB_ATTN_PREFILL if mode == "prefill" else A.HYB_ATTN_DECODE
    scale = 1.0 / math.sqrt(128)
    A.hyb_get_device_status()
    o1, l1 = S.layer.attention(q, pos, kc, vc, nc, 4, idx, kw, vw, W, scale, md)
    torch.cuda.synchronize()
    assert A.hyb_get_device_status() == A.HYB_OK

    ws_n = A.hyb_attn_fwd_workspace_size(A.HYB_DTYPE_BF16, B, T, 64, 128, k, nc, W, md)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev) if ws_n else None
    # the hook with nothing withheld and a 1 s limit is an ordinary call
    o0, l0 = torch.empty_like(o1), torch.empty_like(l1)
    A.hyb_attn_fwd_wait_test(q, pos, kc, vc, nc, 4, idx, k, kw, vw, W, scale, o0, l0, md, ws, 10 ** 9, False)
    torch.cuda.synchronize()
    assert A.hyb_get_device_status() == A.HYB_OK
    assert torch.equal(o0, o1) and torch.equal(l0, l1)

    # one arrival withheld, 2 ms limit: the first CTA gives up and reports it
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    A.hyb_attn_fwd_wait_test(q, pos, kc, vc, nc, 4, idx, k, kw, vw, W, scale, o2, l2, md, ws, 2 * 10 ** 6, True)
    torch.cuda.synchronize()
    assert A.hyb_get_device_status() == A.HYB_ERR_TIMEOUT
    assert A.hyb_get_device_status() == A.HYB_OK          # reading clears the word

    # the same stream runs normal calls afterwards, with the same results
    o3, l3 = S.layer.attention(q, pos, kc, vc, nc, 4, idx, kw, vw, W, scale, md)
    torch.cuda.synchronize()
    assert A.hyb_get_device_status() == A.HYB_OK
    assert torch.equal(o3, o1) and torch.equal(l3, l1)


def test_hook_rejects_what_it_does_not_cover(S):
    A = S.abi
    q, pos, kc, vc, kw, vw, idx = _inputs(1, 4, 100, 16, 600)
    o, l = torch.empty_like(q), torch.empty(1, 4, 64, dtype=torch.float32, device=dev)
    for wait_ns in (0, 2 * 10 ** 9):
        with pytest.raises(A.HybError) as e:
            A.hyb_attn_fwd_wait_test(q, pos, kc, vc, 100, 4, idx, 16, kw, vw, 128, 0.1, o, l, 0, None, wait_ns, True)
        assert e.value.status == A.HYB_ERR_INVALID_ARG
    with pytest.raises(A.HybError) as e:
        A.hyb_attn_fwd_wait_test(q, pos, None, None, 100, 4, idx, 16, kw, vw, 128, 0.1, o, l,
                                 A.HYB_ATTN_PREFILL | A.HYB_ATTN_REAL_KV, None, 10 ** 6, True)
    assert e.value.status == A.HYB_ERR_UNSUPPORTED
