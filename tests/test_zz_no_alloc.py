"""The allocation-free DRELU_BGRAD entry point against the plan-based one.

drelu_bgrad_execute_noalloc serves callers that may not allocate device
memory: code running under a host framework that owns all of the device's
memory (a caching allocator, a fixed memory budget), and enqueue callbacks
that must not call cudaMalloc because it can synchronise the device. It keeps
its column partials in a fixed static scratch array instead of a plan's
workspace. This file is collected last on purpose, so that a run stopping at
the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from gemm_epilogues_tcgen05_b200 import binding, synth

from _parity import Y_REL, check_backward, dbias_scale, run_forward, unit_roundoff

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


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


def _same_as_plan(inp, aux, dZ_n, db_n, dtype):
    """Both entry points agree with the oracle, and with each other within the
    sum of their two parity bounds (they may accumulate in different orders:
    different kernels)."""
    dZ_p, db_p = _plan(inp, aux, dtype)
    db_n_cpu = db_n.cpu()
    assert torch.all(torch.isfinite(db_n_cpu)), "watchdog fired (dbias is NaN)"
    ref = check_backward(inp, aux, dtype, {"dZ": dZ_n.cpu(), "dbias": db_n_cpu}, record="allocation-free entry point")
    check_backward(inp, aux, dtype, {"dZ": dZ_p.cpu(), "dbias": db_p.cpu()})
    dzp, dzn = dZ_p.double().cpu().numpy(), dZ_n.double().cpu().numpy()
    bound = 2 * (Y_REL * ref["S"] + unit_roundoff(dtype) * np.abs(ref["dZ"]))
    assert np.all(np.abs(dzn - dzp) <= bound), "dZ differs from the plan entry point"
    D2 = inp["dY2"].shape[1]
    dbp, dbn = db_p.double().cpu().numpy(), db_n_cpu.double().numpy()
    assert np.all(np.abs(dbn - dbp) <= 2 * dbias_scale(ref, D2)), "dbias differs from the plan entry point"


def test_noalloc_matches_plan_entry_point_on_two_calls_in_a_row():
    dtype = torch.bfloat16
    cases = [(1000, 520, 264, 11), (300, 1032, 136, 12)]  # different shapes, so stale scratch would show
    results = []
    for T, N, D2, seed in cases:
        inp = synth.make_shape_inputs(T, N, 64, "bf16", seed=seed, D2=D2)
        aux = run_forward(inp, "RELU_AUX_BIAS", dtype)["aux"]
        results.append((inp, aux, _noalloc(inp, aux, dtype)))  # two no-alloc calls back to back
    torch.cuda.synchronize()
    for inp, aux, (dZ_n, db_n) in results:
        _same_as_plan(inp, aux, dZ_n, db_n, dtype)


@pytest.mark.parametrize("T", [1, 64])
def test_noalloc_few_rows(T):
    """Few-row shapes (N = 11008, D2 = 4096, one row tile, rows past T): a plan
    runs them on the few-row kernel, this entry point on the tile kernel."""
    dtype = torch.bfloat16
    inp = synth.make_shape_inputs(T, 11008, 64, "bf16", seed=40 + T, D2=4096)
    aux = run_forward(inp, "RELU_AUX_BIAS", dtype)["aux"]
    dZ_n, db_n = _noalloc(inp, aux, dtype)
    torch.cuda.synchronize()
    _same_as_plan(inp, aux, dZ_n, db_n, dtype)


def test_noalloc_allocates_no_device_memory():
    """After a first call (the per-device set-up, and the first load of its
    kernels), a call of another shape changes neither the device's free memory
    nor torch's allocated bytes."""
    dtype = torch.bfloat16
    first = synth.make_shape_inputs(1000, 520, 64, "bf16", seed=21, D2=264)  # both shapes get 64-column tiles
    second = synth.make_shape_inputs(300, 1032, 64, "bf16", seed=22, D2=136)
    bufs = []
    for inp in (first, second):
        aux = run_forward(inp, "RELU_AUX_BIAS", dtype)["aux"]
        T, N = inp["dY2"].shape[0], inp["W2"].shape[1]
        bufs.append((inp["dY2"].cuda(), inp["W2"].cuda(),
                     torch.from_numpy(np.ascontiguousarray(aux).view(np.int32)).cuda(),
                     torch.empty((T, N), dtype=dtype, device="cuda"),
                     torch.empty((N,), dtype=torch.float32, device="cuda")))
    binding.drelu_bgrad_execute_noalloc(*bufs[0])
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    binding.drelu_bgrad_execute_noalloc(*bufs[1])
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    assert torch.all(torch.isfinite(bufs[1][4]))


def test_noalloc_watchdog_reports_nan_and_next_call_is_correct(monkeypatch):
    """The bounded waits of this entry point follow GEMM_EPI_WAIT_TIMEOUT_MS
    like a plan's; with the stall hook the epilogue's wait runs out, every
    dbias entry comes back NaN, and the next call (hook off) matches the plan
    entry point (its status block starts from zero again)."""
    dtype = torch.bfloat16
    inp = synth.make_shape_inputs(512, 512, 64, "bf16", seed=31, D2=256)
    aux = run_forward(inp, "RELU_AUX_BIAS", dtype)["aux"]
    monkeypatch.setenv("GEMM_EPI_FORCE_KERNEL", "tile")
    monkeypatch.setenv("GEMM_EPI_FORCE_BN", "64")
    monkeypatch.setenv("GEMM_EPI_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("GEMM_EPI_TEST_HOOKS", "1")
    monkeypatch.setenv("GEMM_EPI_INJECT_STALL", "1")
    _, db = _noalloc(inp, aux, dtype)
    torch.cuda.synchronize()
    assert torch.all(torch.isnan(db)), "the watchdog's expiry must reach the caller as NaN dbias"
    monkeypatch.delenv("GEMM_EPI_INJECT_STALL")
    dZ_n, db_n = _noalloc(inp, aux, dtype)
    torch.cuda.synchronize()
    _same_as_plan(inp, aux, dZ_n, db_n, dtype)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = binding.lib()
    T, N, K = 128 * 64, 16400, 64  # 64 row tiles x 16400 floats x 4 B > 4 MiB
    rc = L.drelu_bgrad_execute_noalloc(T, N, K, binding.BF16, 16, 16, 16, 16, 16, None)
    assert rc == binding.ERR_INVALID_ARG
    assert "scratch" in binding.gemm_epi_last_error()
