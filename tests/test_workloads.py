"""The seeded generator: SplitMix64 on int64 lanes equals the published
definition on Python integers, values are a pure function of the counter, the
synthetic distributions have the stated moments (all on the CPU), and the
planted prefill inputs are reproducible on the GPU."""
import numpy as np
import pytest
import torch

import workloads as W
from workloads import rng


def test_splitmix64_matches_integer_definition():
    key = rng.stream_key(0, "x")
    got = rng.raw_u64(0, "x", 5, 40)
    for i in range(40):
        want = rng.mix64_int(key + (5 + i) * rng.GAMMA)
        assert int(got[i]) & rng.MASK64 == want


def test_splitmix64_reference_vector():
    # SplitMix64 seeded with 0: first outputs of the reference C implementation
    # (state += gamma; mix) are 0xE220A8397B1DCDAF and 0x6E789E6AA1B965F4.
    assert rng.mix64_int(1 * rng.GAMMA) == 0xE220A8397B1DCDAF
    assert rng.mix64_int(2 * rng.GAMMA) == 0x6E789E6AA1B965F4


def test_counter_based_slices_and_moments():
    a = rng.normal(3, "s", 0, 100000)
    b = rng.normal(3, "s", 777, 1000)
    torch.testing.assert_close(a[777:1777], b, rtol=0, atol=0)
    assert abs(a.mean().item()) < 0.01 and abs(a.std().item() - 1) < 0.01
    u = rng.uniform(1, "u", 0, 100000)
    assert 0 < u.min().item() and u.max().item() < 1


def test_workload_shapes_and_planting():
    w = W.configs.scaled(W.configs.PREFILL_32K, L=1024, T=1024)
    raw, qs = W.make.make_raw(w), W.make.make_queries(w)
    assert raw["xk"].shape == (1, 1024, 128) and raw["xk"].dtype == torch.bfloat16
    assert qs["q"].shape == (1, 1024, 64, 128)
    assert abs(raw["xk"].float().std().item() - 128 ** -0.5) < 2e-3
    js = W.make.plant_prefill(w, w.layer("csa"), raw, qs)
    assert len(js) == round(0.01 * 256) and bool(torch.all(js[1:] - js[:-1] >= 3))
    c = W.make.make_decode_cache(W.configs.scaled(W.configs.DECODE_BS64_128K, batch=2, L=4096))
    assert c["ic"].shape == (2, 1024, 128) and c["kc_hca"].shape == (2, 32, 128) and c["kw"].shape == (2, 128, 128)


@pytest.mark.gpu
def test_prefill_inputs_are_reproducible_on_the_gpu():
    # the planted queries are written by indexed assignment; a repeated row index would
    # make the result depend on which GPU write lands
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    w = W.configs.PREFILL_32K
    out = []
    for _ in range(2):
        raw, qs = W.make.make_raw(w, "cuda"), W.make.make_queries(w, "cuda")
        W.make.plant_prefill(w, w.layer("csa"), raw, qs, "cuda")
        out.append((raw["xi"].cpu(), qs["qi"].cpu()))
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
