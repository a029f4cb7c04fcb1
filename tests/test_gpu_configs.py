"""Parity at the benchmark workloads' full sizes, in the launch configuration
bench.py times (the plans' default tile choice).

pr1 and the skinny sweep are checked on every output. square, ffn and large
are checked on a seeded sample of 256 full rows and 256 full columns (every
output of those rows and columns), and dbias on the sampled columns (a full
column gives the exact bias gradient of that feature).
"""
import numpy as np
import pytest
import torch

import oracle
from gemm_epilogues_tcgen05_b200 import Plan, synth

from _parity import (Y_REL, assert_dbias, assert_dbias_is_column_sum, assert_within, check_forward, check_wgrad, odt,
                     run_forward, run_wgrad, unit_roundoff)

pytestmark = pytest.mark.gpu

SAMPLE = 256


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _fwd_epilog(w):
    return "RELU_BIAS" if w.name == "square" or w.name.startswith("skinny") else "RELU_AUX_BIAS"


def _check_y(w, inp, Y_rows, Y_cols, aux_rows, aux_cols, rows, cols, epilog):
    bits = synth.bits_u16
    dt = w.torch_dtype
    u = unit_roundoff(dt)
    X, W, b = bits(inp["X"]), bits(inp["W"]), bits(inp["bias"])
    for sel, Yg, auxg, kw in ((rows, Y_rows, aux_rows, {"rows": rows}), (cols, Y_cols, aux_cols, {"cols": cols})):
        ref = oracle.linear_fwd(X, W, b, odt(dt), epilog, **kw)
        assert_within(Yg, ref["Y"], ref["S"], Y_REL, f"{w.name} Y ({list(kw)[0]} sample)", u)
        if epilog == "RELU_AUX_BIAS":
            sure = np.abs(ref["Z"]) > Y_REL * ref["S"]
            assert not ((auxg != ref["bits"]) & sure).any(), f"{w.name} relu_aux mismatch"
            assert sure.mean() > 0.5  # the bit-exact check covers most elements


def _run(w, full: bool):
    dev = "cuda"
    dt = w.torch_dtype
    inp = synth.make_inputs(w, device="cpu")
    g = {k: v.to(dev) for k, v in inp.items()}
    epilog = _fwd_epilog(w)
    aux_words = (w.N + 31) // 32
    if full:
        rows, cols = None, None
    else:
        rows = synth.sample_indices(w.T, SAMPLE, seed=w.seed + 11)
        cols = synth.sample_indices(w.N, SAMPLE, seed=w.seed + 12)
    with Plan(w.T, w.N, w.K, dt, epilog) as fp:
        Y = torch.empty((w.T, w.N), dtype=dt, device=dev)
        aux = torch.empty((w.T, aux_words), dtype=torch.int32, device=dev)
        fp.gemm_epi_execute(g["X"], g["W"], g["bias"], Y, aux if epilog == "RELU_AUX_BIAS" else None)
        torch.cuda.synchronize()
        assert fp.status() == 0
    if w.has_backward and epilog != "RELU_AUX_BIAS":
        with Plan(w.T, w.N, w.K, dt, "RELU_AUX_BIAS") as mp:  # the backward's mask
            Ym = torch.empty_like(Y)
            mp.gemm_epi_execute(g["X"], g["W"], g["bias"], Ym, aux)
            torch.cuda.synchronize()
            del Ym
    aux_np = aux.cpu().numpy().view(np.uint32)
    all_bits = oracle.relu_aux_bits(aux_np, w.N)

    def take(t, r, c):
        if r is None and c is None:
            return t
        if r is not None:
            return t[torch.tensor(r, device=t.device)]
        return t[:, torch.tensor(c, device=t.device)]

    if full:
        ref = oracle.linear_fwd(*(synth.bits_u16(inp[k]) for k in ("X", "W", "bias")), odt(dt), epilog)
        assert_within(Y.double().cpu().numpy(), ref["Y"], ref["S"], Y_REL, f"{w.name} Y", unit_roundoff(dt))
        if epilog == "RELU_AUX_BIAS":
            sure = np.abs(ref["Z"]) > Y_REL * ref["S"]
            assert not ((all_bits != ref["bits"]) & sure).any()
    else:
        _check_y(w, inp, take(Y, rows, None).double().cpu().numpy(), take(Y, None, cols).double().cpu().numpy(),
                 all_bits[rows], all_bits[:, cols], rows, cols, epilog)
    del Y
    if not w.has_backward:
        return
    with Plan(w.T, w.N, w.D2, dt, "DRELU_BGRAD") as bp:
        dZ = torch.empty((w.T, w.N), dtype=dt, device=dev)
        dbias = torch.empty((w.N,), dtype=torch.float32, device=dev)
        bp.drelu_bgrad_execute(g["dY2"], g["W2"], aux, dZ, dbias)
        torch.cuda.synchronize()
        assert bp.status() == 0
    bits = synth.bits_u16
    u = unit_roundoff(dt)
    if full:
        rb = oracle.drelu_bgrad(bits(inp["dY2"]), bits(inp["W2"]), aux_np, odt(dt), w.N)
        assert_within(dZ.double().cpu().numpy(), rb["dZ"], rb["S"], Y_REL, f"{w.name} dZ", u)
        assert_dbias(dbias.double().cpu().numpy(), rb, w.D2, f"{w.name} (full size, every column)")
        assert_dbias_is_column_sum(dbias.cpu(), dZ.cpu(), dt)
    else:
        rr = oracle.drelu_bgrad(bits(inp["dY2"]), bits(inp["W2"]), aux_np, odt(dt), w.N, rows=rows)
        assert_within(take(dZ, rows, None).double().cpu().numpy(), rr["dZ"], rr["S"], Y_REL, f"{w.name} dZ rows", u)
        rc = oracle.drelu_bgrad(bits(inp["dY2"]), bits(inp["W2"]), aux_np, odt(dt), w.N, cols=cols)
        assert_within(take(dZ, None, cols).double().cpu().numpy(), rc["dZ"], rc["S"], Y_REL, f"{w.name} dZ cols", u)
        ci = torch.tensor(cols, device=dev)
        assert_dbias(dbias[ci].double().cpu().numpy(), rc, w.D2, f"{w.name} (full size, {len(cols)} sampled columns)")
        assert_dbias_is_column_sum(dbias[ci].cpu(), dZ[:, ci].cpu(), dt)


def test_pr1_full():
    _run(synth.WORKLOADS["pr1"], full=True)


@pytest.mark.parametrize("t", [1, 8, 64, 256])
def test_skinny_full(t):
    _run(synth.WORKLOADS[f"skinny-{t}"], full=True)


def test_square_sampled():
    _run(synth.WORKLOADS["square"], full=False)


def test_ffn_sampled():
    _run(synth.WORKLOADS["ffn"], full=False)


def test_ffn_wgrad_sampled():
    """Weight gradient on the FFN shape: dW (4096 x 11008) = X^T dZ over T = 4096,
    checked on 256 sampled rows and 256 sampled columns."""
    w = synth.WORKLOADS["ffn"]
    inp = {"X": synth.make_inputs(w, parts=("fwd",))["X"],
           "dZ": synth.masked_grad(w.T, w.N, w.D2, w.torch_dtype, seed=w.seed + 21)}
    gpu = run_wgrad(inp, w.torch_dtype, dz_key="dZ")
    assert gpu["info"]["kernel"] == 2
    rows = synth.sample_indices(w.K, SAMPLE, seed=w.seed + 13)
    cols = synth.sample_indices(w.N, SAMPLE, seed=w.seed + 14)
    check_wgrad(inp, w.torch_dtype, gpu, rows=rows, dz_key="dZ")
    check_wgrad(inp, w.torch_dtype, gpu, cols=cols, dz_key="dZ")


@pytest.mark.parametrize("epilog", ["GELU_BIAS", "GELU_AUX_BIAS"])
def test_ffn_gelu_sampled(epilog):
    """The GELU epilogs on the FFN shape, in the launch configuration the bench
    times (CTA pairs with eight epilogue warps), checked on 256 sampled rows
    and 256 sampled columns of Y (and of Z for GELU_AUX_BIAS)."""
    w = synth.WORKLOADS["ffn"]
    inp = synth.make_inputs(w, parts=("fwd",))
    gpu = run_forward(inp, epilog, w.torch_dtype)
    assert gpu["info"]["kernel"] == 2
    rows = synth.sample_indices(w.T, SAMPLE, seed=w.seed + 15)
    cols = synth.sample_indices(w.N, SAMPLE, seed=w.seed + 16)
    check_forward(inp, epilog, w.torch_dtype, gpu, rows=rows)
    check_forward(inp, epilog, w.torch_dtype, gpu, cols=cols)


@pytest.mark.slow
def test_large_sampled():
    _run(synth.WORKLOADS["large"], full=False)
