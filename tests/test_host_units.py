"""Host-side units on CPU: the algorithmic FLOPs and bytes behind every
roofline fraction, and the seeded input generators (their determinism and
the distributions the workloads state)."""
import math
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gemm_epilogues_tcgen05_b200 import synth  # noqa: E402

W = synth.WORKLOADS


# ------------------------------------------------ algorithmic FLOPs and bytes
def test_ffn_units_match_the_worked_table():
    # FFN (bf16, T=K=4096, N=11008, D2=4096): 369.4 GFLOP per call; forward
    # X 33.6 + W 90.2 + Y 90.2 + mask 5.6 MB, backward dY2 + W2 + mask + dZ + dbias
    a = bench.algorithmic(W["ffn"], "RELU_AUX_BIAS", True)
    assert a["fwd"]["flops"] == pytest.approx(369.4e9, rel=1e-3)
    assert a["bwd"]["flops"] == a["fwd"]["flops"]
    assert a["fwd"]["bytes"] / 1e6 == pytest.approx(219.6, rel=2e-3)
    assert a["bwd"]["bytes"] / 1e6 == pytest.approx(219.6, rel=2e-3)


def test_skinny_and_large_units():
    a = bench.algorithmic(W["skinny-1"], "RELU_BIAS", True)
    assert a["fwd"]["bytes"] / 1e6 == pytest.approx(90.2, rel=2e-3)  # the weight dominates
    assert a["fwd"]["flops"] == pytest.approx(2 * 4096 * 11008)
    big = bench.algorithmic(W["large"], "RELU_AUX_BIAS", False)
    assert set(big) == {"fwd"}
    assert big["fwd"]["bytes"] / 1e6 == pytest.approx(3556, rel=2e-3)  # X 2147 + W 268 + Y 1074 + mask 67


def test_mode_units():
    w = W["ffn"]
    g = 2.0 * w.T * w.K * w.N
    wg = bench.algorithmic(w, "WGRAD", False)["fwd"]
    assert wg["flops"] == g and wg["bytes"] == 2 * (w.T * w.K + w.T * w.N + w.K * w.N)
    st = bench.algorithmic(w, "FFN_STEP", True)
    assert st["fwd"]["flops"] == 2 * g and st["bwd"]["flops"] == 4 * g
    assert bench.algorithmic(w, "RELU_BIAS", False)["fwd"]["bytes"] < bench.algorithmic(w, "RELU_AUX_BIAS", False)["fwd"]["bytes"]


def test_step_spec_modes():
    class A:  # an argparse namespace stand-in
        ffn_step = False
        wgrad = False
        fwd_epilog = None
    assert bench.step_spec(W["ffn"], A()) == ("RELU_AUX_BIAS", True)
    assert bench.step_spec(W["square"], A()) == ("RELU_BIAS", False)
    a = A(); a.fwd_epilog = "GELU_BIAS"
    assert bench.step_spec(W["ffn"], a) == ("GELU_BIAS", False)
    a = A(); a.wgrad = True
    assert bench.step_spec(W["ffn"], a) == ("WGRAD", False)
    a = A(); a.ffn_step = True
    assert bench.step_spec(W["ffn"], a) == ("FFN_STEP", True)


# ------------------------------------------------------------ input generators
def test_generators_are_seeded():
    a = synth.make_shape_inputs(33, 40, 24, "bf16", seed=9, D2=16)
    b = synth.make_shape_inputs(33, 40, 24, "bf16", seed=9, D2=16)
    c = synth.make_shape_inputs(33, 40, 24, "bf16", seed=10, D2=16)
    for k in a:
        assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16))
    assert not torch.equal(a["X"].view(torch.int16), c["X"].view(torch.int16))
    assert {k: tuple(v.shape) for k, v in a.items()} == {"X": (33, 24), "W": (24, 40), "bias": (40,),
                                                        "dY2": (33, 16), "W2": (16, 40)}


def test_stated_distributions():
    K, N = 1024, 2048
    inp = synth.make_shape_inputs(512, N, K, "fp16", seed=4, D2=256)
    std = {k: float(v.float().std()) for k, v in inp.items()}
    assert std["X"] == pytest.approx(1.0, rel=0.02)
    assert std["W"] == pytest.approx(K ** -0.5, rel=0.02)
    assert std["bias"] == pytest.approx(math.sqrt(0.1), rel=0.1)  # N(0, 0.1) read as a variance
    assert std["dY2"] == pytest.approx(1.0, rel=0.02)
    assert std["W2"] == pytest.approx(N ** -0.5, rel=0.02)


def test_masked_grad_stand_in():
    T, N, D2 = 256, 1024, 4096
    g = synth.masked_grad(T, N, D2, torch.bfloat16, seed=3).float()
    zero = float((g == 0).float().mean())
    assert zero == pytest.approx(0.5, abs=0.02)  # the inactive half of a ReLU layer
    assert float(g[g != 0].std()) == pytest.approx(math.sqrt(D2 / N), rel=0.03)


def test_ffn_step_inputs():
    n = synth.ffn_step_inputs(16, 64, 96, "bf16", seed=1)
    assert {k: tuple(v.shape) for k, v in n.items()} == {"X": (16, 64), "W1": (96, 64), "b1": (96,),
                                                        "W2": (64, 96), "b2": (64,), "dY": (16, 64)}
    i = synth.ffn_step_inputs(16, 64, 96, "fp16", seed=1, kind="int")
    for k, v in i.items():
        vals = v.float()
        assert torch.equal(vals, vals.round())
        assert float(vals.abs().max()) <= (2 if k in ("b1", "b2") else 1)


def test_sample_indices_distinct_and_seeded():
    a = synth.sample_indices(4096, 256, seed=7)
    assert len(set(a)) == 256 and all(0 <= x < 4096 for x in a)
    assert a == synth.sample_indices(4096, 256, seed=7)


# ------------------------------------------------------------ roofline object
PEAKS = {"hbm_gbs": 6542.1, "bf16_tflops": 1671.6, "bf16_tflops_sustained": 1407.4}


def _res(w, fwd_epi, fwd_ms, bwd_ms, reasons=(), kernel=2):
    alg = bench.algorithmic(w, fwd_epi, bwd_ms > 0)
    return {"alg": alg, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "step_ms": fwd_ms + bwd_ms, "kernel": kernel,
            "clocks": {"reasons": list(reasons)}}


def test_roofline_takes_the_slower_call_and_the_burst_peak():
    w = W["ffn"]
    r = bench.roofline(w, "RELU_AUX_BIAS", _res(w, "RELU_AUX_BIAS", 0.270, 0.280), PEAKS, "measured")
    assert r["bound"] == "tensor" and r["kernel"].startswith("bwd: tile2_kernel")
    assert r["achieved"] == pytest.approx(369.4e9 / 0.280e-3 / 1e12, rel=1e-3)
    assert r["peak"] == 1671.6 and r["peak_kind"].startswith("burst")
    assert r["frac"] == pytest.approx(r["achieved"] / 1671.6)
    # the whole step against its roofline time (FLOPs at the tensor peak for both calls)
    assert r["step_roofline_frac"] == pytest.approx(2 * 369.4e9 / 1671.6e12 / 0.550e-3, rel=2e-3)


def test_roofline_uses_the_sustained_peak_under_the_power_cap_or_for_long_launches():
    w = W["ffn"]
    capped = bench.roofline(w, "RELU_AUX_BIAS", _res(w, "RELU_AUX_BIAS", 0.27, 0.28, ["sw_power_cap"]), PEAKS, "measured")
    assert capped["peak"] == 1407.4 and "power cap" in capped["peak_kind"]
    assert capped["frac_of_burst"] == pytest.approx(capped["achieved"] / 1671.6)
    big = W["large"]
    long_ = bench.roofline(big, "RELU_AUX_BIAS", _res(big, "RELU_AUX_BIAS", 15.0, 0.0, kernel=0), PEAKS, "measured")
    assert long_["peak"] == 1407.4 and "1 ms" in long_["peak_kind"] and long_["kernel"].startswith("fwd: tile_kernel")


def test_roofline_is_hbm_bound_for_the_few_row_workloads():
    w = W["skinny-1"]
    r = bench.roofline(w, "RELU_BIAS", _res(w, "RELU_BIAS", 0.0246, 0.0227, kernel=1), PEAKS, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6542.1
    assert r["achieved"] == pytest.approx(bench.algorithmic(w, "RELU_BIAS", True)["fwd"]["bytes"] / 0.0246e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6542.1)
