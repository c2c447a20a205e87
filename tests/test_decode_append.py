"""GPU parity of the fused decode-step state update (hyb_decode_append): appending
tokens one step at a time from a prefix state must give exactly the caches,
representatives and rings that S1 over the whole sequence gives on the GPU
(same arithmetic), and match the fp64 oracle like S1 does."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import make

from parity import check_close, to64

pytestmark = pytest.mark.gpu

dev = "cuda"


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_hyb_b200 as S
    S.abi.lib()
    return S


def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_append_matches_full_compress(S, dtype):
    A = S.abi
    B, D, dI, ring, blk = 2, 128, 128, 128, 128
    r_c, r_h = 4, 128
    P0 = [1000, 1271]            # prefix lengths (different per sequence)
    n = 520                      # appended tokens: 130 CSA entries, 4 HCA entries, one more block
    L = max(P0) + n
    sc = 128 ** -0.5
    xk = make.normal_tensor(5, "dk", (B, L, D), sc, dtype)
    xv = make.normal_tensor(5, "dv", (B, L, D), sc, dtype)
    xi = make.normal_tensor(5, "di", (B, L, dI), sc, dtype)
    z = make.normal_tensor(5, "dz", (B, L), 1.0, "f32")
    bias_c = make.normal_tensor(5, "dbc", (2 * r_c,), 0.1, "f32").to(dev)
    bias_h = make.normal_tensor(5, "dbh", (r_h,), 0.1, "f32").to(dev)
    xk_d, xv_d, xi_d, z_d = xk.to(dev), xv.to(dev), xi.to(dev), z.to(dev)
    ncap, nhcap, nbcap = L // r_c, L // r_h, (L // r_c) // blk
    tdt = xk.dtype
    kc = torch.zeros(B, ncap, D, dtype=tdt, device=dev)
    vc, ic = torch.zeros_like(kc), torch.zeros(B, ncap, dI, dtype=tdt, device=dev)
    kh = torch.zeros(B, nhcap, D, dtype=tdt, device=dev)
    vh = torch.zeros_like(kh)
    reps = torch.zeros(B, nbcap, dI, dtype=tdt, device=dev)
    kw = torch.zeros(B, ring, D, dtype=tdt, device=dev)
    vw, iw = torch.zeros_like(kw), torch.zeros(B, ring, dI, dtype=tdt, device=dev)
    zw = torch.zeros(B, ring, dtype=torch.float32, device=dev)
    # prefix state of each sequence: S1 over its prefix, representatives, rings
    for b in range(B):
        p = P0[b]
        sl = slice(b, b + 1)
        A.hyb_compress(xk_d[sl, :p], xv_d[sl, :p], xi_d[sl, :p], z_d[sl, :p], bias_c, r_c, True, 0, p // r_c,
                       kc[sl], vc[sl], ic[sl])
        A.hyb_compress(xk_d[sl, :p], xv_d[sl, :p], None, z_d[sl, :p], bias_h, r_h, False, 0, p // r_h,
                       kh[sl], vh[sl], None)
        A.hyb_block_reps(ic[sl], blk, 0, (p // r_c) // blk, reps[sl])
        pos = torch.arange(p - ring, p, device=dev)
        kw[b, pos % ring], vw[b, pos % ring] = xk_d[b, pos], xv_d[b, pos]
        iw[b, pos % ring], zw[b, pos % ring] = xi_d[b, pos], z_d[b, pos]
    # n decode steps
    p0 = torch.tensor(P0, dtype=torch.int32, device=dev)
    bidx = torch.arange(B, device=dev)
    for i in range(n):
        t = p0 + i
        tl = t.long()
        A.hyb_decode_append(xk_d[bidx, tl].contiguous(), xv_d[bidx, tl].contiguous(), xi_d[bidx, tl].contiguous(),
                            z_d[bidx, tl].contiguous(), t.contiguous(), kw, vw, iw, zw,
                            bias_csa=bias_c, r_csa=r_c, overlap=True, kc=kc, vc=vc, ic=ic,
                            bias_hca=bias_h, r_hca=r_h, kc_hca=kh, vc_hca=vh, block=blk, reps=reps)
    torch.cuda.synchronize()
    assert A.hyb_get_device_status() == 0
    for b in range(B):
        p = P0[b] + n
        sl = slice(b, b + 1)
        nc_b, nh_b, nb_b = p // r_c, p // r_h, (p // r_c) // blk
        # the same S1 over the whole sequence on the GPU: bit-identical
        fk, fv, fi = torch.zeros_like(kc[sl]), torch.zeros_like(vc[sl]), torch.zeros_like(ic[sl])
        fkh, fvh = torch.zeros_like(kh[sl]), torch.zeros_like(vh[sl])
        fr = torch.zeros_like(reps[sl])
        A.hyb_compress(xk_d[sl, :p], xv_d[sl, :p], xi_d[sl, :p], z_d[sl, :p], bias_c, r_c, True, 0, nc_b, fk, fv, fi)
        A.hyb_compress(xk_d[sl, :p], xv_d[sl, :p], None, z_d[sl, :p], bias_h, r_h, False, 0, nh_b, fkh, fvh, None)
        A.hyb_block_reps(fi, blk, 0, nb_b, fr)
        torch.cuda.synchronize()
        for got, want, n_ok, nm in ((kc, fk, nc_b, "kc"), (vc, fv, nc_b, "vc"), (ic, fi, nc_b, "ic"),
                                    (kh, fkh, nh_b, "kc_hca"), (vh, fvh, nh_b, "vc_hca"), (reps, fr, nb_b, "reps")):
            assert torch.equal(got[b, :n_ok], want[0, :n_ok]), f"{nm} b={b}: differs from S1 over the sequence"
        pos = torch.arange(p - ring, p, device=dev)
        assert torch.equal(kw[b, pos % ring], xk_d[b, pos]) and torch.equal(zw[b, pos % ring], z_d[b, pos])
        # and the fp64 oracle, as for S1
        want_c = O.compress([to64(xk[b, :p]), to64(xv[b, :p]), to64(xi[b, :p])], to64(z[b, :p]),
                            to64(bias_c.cpu()), r_c, True, 0, nc_b, dtype)
        want_h = O.compress([to64(xk[b, :p]), to64(xv[b, :p])], to64(z[b, :p]), to64(bias_h.cpu()), r_h, False, 0,
                            nh_b, dtype)
        want_r = O.block_reps(want_c[2], blk, dtype)
        for got, wt, nm in ((kc[b, :nc_b], want_c[0], "kc"), (ic[b, :nc_b], want_c[2], "ic"),
                            (kh[b, :nh_b], want_h[0], "kc_hca"), (vh[b, :nh_b], want_h[1], "vc_hca")):
            g64 = to64(got)
            check_close(g64, wt, dtype, f"decode append {nm} b={b}")
            if dtype == "bf16":   # one bf16 ulp from the fp64 result, plus the fp32 accumulation error
                slack = 2.0 ** -20 * max(1.0, float(np.abs(wt).max()))
                assert np.all(np.abs(g64 - wt) <= _ulp_bf16(wt) * 1.0001 + slack), f"{nm}: more than one ulp"
        check_close(to64(reps[b, :nb_b]), want_r, dtype, f"decode append reps b={b}")
