"""Host-side arithmetic of bench.py: step sizing, algorithmic work of the layer, peaks."""
import math
import sys

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_rounds_per_step_reaches_the_target():
    assert bench.rounds_per_step(0.001, 0.06) == 60
    assert bench.rounds_per_step(0.0007, 0.06) == 86         # ceil(85.7)
    assert bench.rounds_per_step(1.0, 0.06) == 1
    assert bench.rounds_per_step(0.0, 0.06) == 1
    assert bench.rounds_per_step(float("nan"), 0.06) == 1


def test_sweeps_separate_each_tensors_transforms_by_more_than_twice_l2():
    # a tensor of view p is touched by fwd p and inv p; between them lie the rest of
    # its own pool and the whole other view's pool
    pool_bytes = bench.POOL * bench.ELEMS * 2
    assert pool_bytes >= 2 * 126 * 1000 * 1000
    kinds = [d for d, _ in bench.SWEEPS]
    assert kinds == ["fwd", "fwd", "inv", "inv"]
    assert {p for _, p in bench.SWEEPS} == set(bench.PS)
    for p in bench.PS:
        i_f = bench.SWEEPS.index(("fwd", p))
        i_i = bench.SWEEPS.index(("inv", p))
        assert i_i - i_f == len(bench.PS)                     # every other sweep lies between


def test_layer_work_counts_the_method():
    B, D, p = 256, 4096, 128
    q = D // p
    w = bench.layer_work(B, D, p, 2)
    fft = 2.5 * p * math.log2(p)
    contr = q * q * (8 * (p // 2 - 1) + 4)
    assert w["fwd"]["flops"] == B * (2 * q * fft + contr)
    assert w["fwd"]["bytes"] == 2 * B * D * 2 + 4 * q * q * p
    assert w["grad_x"] == w["fwd"]
    assert w["bwd"]["bytes"] == 3 * B * D * 2 + 8 * q * q * p
    assert w["bwd"]["flops"] == B * (3 * q * fft + 2 * contr) + q * q * fft
    # contraction per token at this shape: q^2 (4p - 4) = 520,192 flops (78% of the forward)
    assert contr == 520192
    assert abs(contr / (w["fwd"]["flops"] / B) - 0.78) < 0.01


def test_fp32_peak_from_lanes_and_clock():
    assert abs(bench.fp32_peak_tflops(1965.0, 148) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
    assert bench.fp32_peak_tflops(None, 148) == bench.fp32_peak_tflops(bench.NOMINAL_SM_MHZ, 148)


def test_clock_summary_reads_reasons():
    s = bench.ClockSampler(None)
    s.lines = [(10.0, "0, 1965, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active"),
               (10.1, "0, 1950, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"),
               (20.0, "0, 300, 1965, 90.0, 0x1, Not Active, Not Active, Not Active, Not Active")]
    d = s.summary(9.9, 10.2)
    assert d["samples"] == 2 and d["sm_max_mhz"] == 1965.0 and d["reasons"] == ["sw_power_cap"]
    assert d["sm_mhz"] == statistics_median([1965.0, 1950.0])


def statistics_median(v):
    import statistics
    return statistics.median(v)


def test_torch_fft_reference_matches_the_oracle():
    """The torch.fft circulant the bench measures for context computes the same layer as
    the oracle's dense circulant (paper-notes page, "Circulant matrix training
    adaptation"), so its memory and time figures describe the same work."""
    import numpy as np
    import torch

    import oracle

    gen = torch.Generator().manual_seed(11)
    for q, p in ((1, 16), (4, 16), (3, 8)):
        x = torch.randn(5, q * p, generator=gen)
        c = torch.randn(q, q, p, generator=gen)
        y = bench.torch_fft_circulant(torch, x, c).double().numpy()
        ref = oracle.circ_forward(x.double().numpy(), c.double().numpy())
        assert np.abs(y - ref).max() <= 1e-5 * np.abs(ref).max()
