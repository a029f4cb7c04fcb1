"""The allocation-free DRELU_BGRAD entry point against the plan-based one.

drelu_bgrad_execute_noalloc serves callers that may not allocate device
memory: code running under a host framework that owns all of the device's
memory (a caching allocator, a fixed memory budget), and enqueue callbacks
that must not call cudaMalloc because it can synchronise the device. It keeps
its column partials in a fixed static scratch array instead of a plan's
workspace. This file is collected last on purpose, so that a run stopping at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gemm_epilogues_tcgen05_b200 import binding, synth

from _parity import DBIAS_REL, Y_REL, check_backward, run_forward, unit_roundoff

pytestmark = pytest.mark.gpu


def _noalloc(inp, aux_words, dtype):
    dev = "cuda"
    dY2, W2 = inp["dY2"].to(dev), inp["W2"].to(dev)
    T, N = dY2.shape[0], W2.shape[1]
    aux = torch.from_numpy(np.ascontiguousarray(aux_words).view(np.int32)).to(dev)
    dZ = torch.empty((T, N), dtype=dtype, device=dev)
    dbias = torch.empty((N,), dtype=torch.float32, device=dev)
    binding.drelu_bgrad_execute_noalloc(dY2, W2, aux, dZ, dbias)
    return dZ, dbias


def _plan(inp, aux_words, dtype):
    dev = "cuda"
    dY2, W2 = inp["dY2"].to(dev), inp["W2"].to(dev)
    T, D2 = dY2.shape
    N = W2.shape[1]
    aux = torch.from_numpy(np.ascontiguousarray(aux_words).view(np.int32)).to(dev)
    with binding.Plan(T, N, D2, dtype, "DRELU_BGRAD") as plan:
        dZ, dbias = plan.backward(dY2, W2, aux)
        torch.cuda.synchronize()
        assert plan.status() == 0
    return dZ, dbias


def test_noalloc_matches_plan_entry_point_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dtype = torch.bfloat16
    cases = [(1000, 520, 264, 11), (300, 1032, 136, 12)]  # different shapes, so stale scratch would show
    results = []
    for T, N, D2, seed in cases:
        inp = synth.make_shape_inputs(T, N, 64, "bf16", seed=seed, D2=D2)
        aux = run_forward(inp, "RELU_AUX_BIAS", dtype)["aux"]
        results.append((inp, aux, _noalloc(inp, aux, dtype)))  # two no-alloc calls back to back
    torch.cuda.synchronize()
    u = unit_roundoff(dtype)
    for inp, aux, (dZ_n, db_n) in results:
        dZ_p, db_p = _plan(inp, aux, dtype)
        S = (inp["dY2"].double().abs() @ inp["W2"].double().abs()).numpy()
        dzp = dZ_p.double().cpu().numpy()
        dzn = dZ_n.double().cpu().numpy()
        assert np.all(np.abs(dzn - dzp) <= Y_REL * S + u * np.abs(dzp)), "dZ differs from the plan entry point"
        Sb = np.abs(dzp).sum(axis=0)
        dbp, dbn = db_p.double().cpu().numpy(), db_n.double().cpu().numpy()
        assert np.all(np.isfinite(dbn)), "watchdog fired (dbias is NaN)"
        assert np.all(np.abs(dbn - dbp) <= DBIAS_REL * Sb), "dbias differs from the plan entry point"
        # and both agree with the oracle
        check_backward(inp, aux, dtype, {"dZ": dZ_n.cpu(), "dbias": db_n.cpu()})


def test_noalloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = binding.lib()
    T, N, K = 128 * 64, 16400, 64  # 64 row tiles x 16400 floats x 4 B > 4 MiB
    rc = L.drelu_bgrad_execute_noalloc(T, N, K, binding.BF16, 16, 16, 16, 16, 16, None)
    assert rc == binding.ERR_INVALID_ARG
    assert "scratch" in binding.gemm_epi_last_error()
