"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, and rejects bad arguments with error
codes before touching a device."""
import ctypes
import os
import re

import pytest
import torch

from gemm_epilogues_tcgen05_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^GEMM_EPI_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, re.M)
    return names


def test_header_declares_the_entry_points():
    names = _declared()
    for want in ("gemm_epi_plan", "gemm_epi_execute", "drelu_bgrad_execute", "gemm_epi_free"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    names = _declared()
    assert names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert sorted(names) == sorted(binding.EXPORTED)


@pytest.mark.parametrize("T,N,K", [(0, 64, 64), (-1, 64, 64), (64, 0, 64), (64, 12, 64), (64, 64, 4),
                                   (64, 64, 100), (1 << 31, 64, 64)])
def test_plan_rejects_bad_shapes(L, T, N, K):
    assert not L.gemm_epi_plan(T, N, K, 0, 0)
    assert "shape" in binding.gemm_epi_last_error()


def test_plan_rejects_bad_enums(L):
    assert not L.gemm_epi_plan(64, 64, 64, 7, 0)
    assert "dtype" in binding.gemm_epi_last_error()
    assert not L.gemm_epi_plan(64, 64, 64, 0, 9)
    assert "epilog" in binding.gemm_epi_last_error()


def test_plan_flags_are_checked_before_the_device(L):
    assert not L.gemm_epi_plan_ex(64, 64, 64, 0, 0, 8)  # no such flag
    assert "flags" in binding.gemm_epi_last_error()
    assert not L.gemm_epi_plan_ex(64, 64, 64, 0, binding.WGRAD, binding.FLAG_W_NK)
    assert "W_NK" in binding.gemm_epi_last_error()


def test_unknown_plan_handles_are_rejected_not_dereferenced(L):
    bogus = ctypes.c_void_p(0x12345678)
    rc = L.gemm_epi_execute(bogus, 16, 16, 16, 16, 16, None)
    assert rc == binding.ERR_INVALID_ARG
    rc = L.drelu_bgrad_execute(bogus, 16, 16, 16, 16, 16, None)
    assert rc == binding.ERR_INVALID_ARG
    assert L.gemm_epi_status(bogus) == binding.ERR_INVALID_ARG
    info = binding.Info()
    assert L.gemm_epi_query(bogus, ctypes.byref(info)) == binding.ERR_INVALID_ARG
    L.gemm_epi_free(bogus)  # ignored
    L.gemm_epi_free(None)   # NULL-safe


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_plan_without_a_device_fails_cleanly(L):
    assert not L.gemm_epi_plan(256, 256, 256, 0, 2)
    msg = binding.gemm_epi_last_error()
    assert msg  # a CUDA error message, no crash


def test_binding_checks_tensors_before_calling():
    with pytest.raises(ValueError):
        binding._ptr(torch.zeros(4, 4, dtype=torch.float16), (4, 4), torch.float16, "X")  # not on a GPU
    with pytest.raises(TypeError):
        binding._ptr([1, 2], (2,), torch.float16, "X")
