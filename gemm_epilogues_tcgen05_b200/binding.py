"""ctypes binding of ``libgemm_epi.so`` (the C ABI in include/gemm_epi.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their ``data_ptr()`` and the current CUDA stream are passed
to the C function of the same name. All arithmetic happens in the library's
kernels; if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

F16, BF16 = 0, 1
BIAS, RELU_BIAS, RELU_AUX_BIAS, DRELU_BGRAD, GELU_BIAS, WGRAD, NONE, GELU_AUX_BIAS = 0, 1, 2, 3, 4, 5, 6, 7
EPILOGS = {"BIAS": BIAS, "RELU_BIAS": RELU_BIAS, "RELU_AUX_BIAS": RELU_AUX_BIAS, "DRELU_BGRAD": DRELU_BGRAD,
           "GELU_BIAS": GELU_BIAS, "WGRAD": WGRAD, "NONE": NONE, "GELU_AUX_BIAS": GELU_AUX_BIAS}
DTYPES = {torch.float16: F16, torch.bfloat16: BF16}

OK = 0
ERR_INVALID_ARG = -1
ERR_MISALIGNED = -2
ERR_EPILOG_MISMATCH = -3
ERR_CUDA = -4
ERR_TIMEOUT = -5
ERR_UNSUPPORTED = -6

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgemm_epi.so")

EXPORTED = ["gemm_epi_plan", "gemm_epi_execute", "drelu_bgrad_execute", "gemm_epi_free", "gemm_epi_last_error",
            "gemm_epi_query", "gemm_epi_status", "gemm_epi_unfused_execute", "drelu_bgrad_unfused_execute",
            "drelu_bgrad_execute_noalloc", "gemm_epi_wgrad_execute", "gemm_epi_set_bias_f32", "gemm_epi_plan_ex"]
FLAG_W_NK = 1  # GEMM_EPI_FLAG_W_NK
FLAG_OUT_F32 = 2  # GEMM_EPI_FLAG_OUT_F32

NOALLOC_SCRATCH_BYTES = 4 << 20  # GEMM_EPI_NOALLOC_SCRATCH_BYTES


class GemmEpiError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"gemm_epi error {code}: {msg}")
        self.code = code


class Info(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("dtype", ctypes.c_int), ("epilog", ctypes.c_int), ("kernel", ctypes.c_int),
                ("tile_m", ctypes.c_int), ("tile_n", ctypes.c_int), ("tile_k", ctypes.c_int),
                ("stages", ctypes.c_int), ("split_k", ctypes.c_int), ("grid", ctypes.c_int),
                ("launches", ctypes.c_int), ("num_sms", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m gemm_epilogues_tcgen05_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.gemm_epi_plan.restype = vp
        L.gemm_epi_plan.argtypes = [i64, i64, i64, ci, ci]
        L.gemm_epi_plan_ex.restype = vp
        L.gemm_epi_plan_ex.argtypes = [i64, i64, i64, ci, ci, ctypes.c_uint32]
        L.gemm_epi_execute.restype = ci
        L.gemm_epi_execute.argtypes = [vp] * 7
        L.drelu_bgrad_execute.restype = ci
        L.drelu_bgrad_execute.argtypes = [vp] * 7
        L.gemm_epi_free.restype = None
        L.gemm_epi_free.argtypes = [vp]
        L.gemm_epi_last_error.restype = ctypes.c_char_p
        L.gemm_epi_last_error.argtypes = []
        L.gemm_epi_query.restype = ci
        L.gemm_epi_query.argtypes = [vp, ctypes.POINTER(Info)]
        L.gemm_epi_status.restype = ci
        L.gemm_epi_status.argtypes = [vp]
        L.gemm_epi_unfused_execute.restype = ci
        L.gemm_epi_unfused_execute.argtypes = [vp] * 9
        L.drelu_bgrad_unfused_execute.restype = ci
        L.drelu_bgrad_unfused_execute.argtypes = [vp] * 8
        L.drelu_bgrad_execute_noalloc.restype = ci
        L.drelu_bgrad_execute_noalloc.argtypes = [i64, i64, i64, ci] + [vp] * 6
        L.gemm_epi_set_bias_f32.restype = ci
        L.gemm_epi_set_bias_f32.argtypes = [vp, ci]
        L.gemm_epi_wgrad_execute.restype = ci
        L.gemm_epi_wgrad_execute.argtypes = [vp] * 6
        _lib = L
    return _lib


def gemm_epi_last_error() -> str:
    return lib().gemm_epi_last_error().decode()


def _check(rc: int):
    if rc != OK:
        raise GemmEpiError(rc, gemm_epi_last_error())


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t, shape, dtype, name) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def gemm_epi_plan(T: int, N: int, K: int, dtype, epilog, flags: int = 0) -> int:
    """Raw handle (int) from the C gemm_epi_plan_ex; raises on error."""
    if isinstance(dtype, torch.dtype):
        dtype = DTYPES[dtype]
    if isinstance(epilog, str):
        epilog = EPILOGS[epilog]
    h = lib().gemm_epi_plan_ex(T, N, K, dtype, epilog, flags)
    if not h:
        raise GemmEpiError(ERR_INVALID_ARG, gemm_epi_last_error())
    return h


def gemm_epi_free(handle) -> None:
    lib().gemm_epi_free(handle)


def drelu_bgrad_execute_noalloc(dY2, W2, aux, dZ, dbias, stream=None):
    """DRELU_BGRAD without a plan and without any device allocation.

    For callers that may not allocate device memory (a host framework that
    owns the device's memory, or an enqueue callback that must not call
    cudaMalloc because it can synchronise the device). The column partials
    live in the library's fixed 4 MiB static scratch, shared by every call:
    calls that overlap on the GPU race, so keep them on one stream. The first
    call on a device does a one-time set-up; make it before any stream
    capture. If the kernel's watchdog fires, dbias comes back as NaN.
    """
    T, K = dY2.shape
    N = W2.shape[1]
    dt = dY2.dtype
    args = (_ptr(dY2, (T, K), dt, "dY2"), _ptr(W2, (K, N), dt, "W2"),
            _ptr(aux, (T, (N + 31) // 32), torch.int32, "aux"), _ptr(dZ, (T, N), dt, "dZ"),
            _ptr(dbias, (N,), torch.float32, "dbias"))
    _check(lib().drelu_bgrad_execute_noalloc(T, N, K, DTYPES[dt], *args, _stream_ptr(stream)))


class Plan:
    """A plan for one (T, N, K, dtype, epilog); execute any number of times."""

    def __init__(self, T: int, N: int, K: int, dtype: torch.dtype, epilog: str | int, w_nk: bool = False,
                 out_f32: bool = False):
        """w_nk: the weight (W, or W2 of DRELU_BGRAD) is N x K, K contiguous.
        out_f32: the output (Y, dZ or dW) is fp32."""
        self.T, self.N, self.K = T, N, K
        self.out_dtype = torch.float32 if out_f32 else dtype
        self.w_shape = (N, K) if w_nk else (K, N)
        self.dtype = dtype
        self.epilog = EPILOGS[epilog] if isinstance(epilog, str) else epilog
        self.aux_words = (N + 31) // 32
        self.bias_dtype = dtype
        self.handle = gemm_epi_plan(T, N, K, dtype, self.epilog,
                                    (FLAG_W_NK if w_nk else 0) | (FLAG_OUT_F32 if out_f32 else 0))

    def aux_spec(self):
        """Shape and dtype of the forward's auxiliary output: the mask words
        (T x ceil(N/32) int32) for RELU_AUX_BIAS, the pre-activation (T x N,
        the plan's 16-bit type) for GELU_AUX_BIAS, None otherwise."""
        if self.epilog == RELU_AUX_BIAS:
            return (self.T, self.aux_words), torch.int32
        if self.epilog == GELU_AUX_BIAS:
            return (self.T, self.N), self.dtype
        return None

    def _aux(self, aux):
        spec = self.aux_spec() or ((self.T, self.aux_words), torch.int32)
        return _ptr(aux, spec[0], spec[1], "aux")

    def set_bias_f32(self, on: bool = True):
        """Read the forward bias as fp32 (True) or in the plan's 16-bit type (False)."""
        _check(lib().gemm_epi_set_bias_f32(self.handle, 1 if on else 0))
        self.bias_dtype = torch.float32 if on else self.dtype

    # life cycle ----------------------------------------------------------
    def free(self):
        if self.handle:
            gemm_epi_free(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.free()

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass

    def info(self) -> dict:
        inf = Info()
        _check(lib().gemm_epi_query(self.handle, ctypes.byref(inf)))
        return inf.as_dict()

    def status(self) -> int:
        """OK, or ERR_TIMEOUT if a kernel of this plan gave up a wait (after a sync)."""
        return lib().gemm_epi_status(self.handle)

    # calls -------------------------------------------------------------
    def gemm_epi_execute(self, X, W, bias, Y, aux=None, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (_ptr(X, (T, K), dt, "X"), _ptr(W, self.w_shape, dt, "W"), _ptr(bias, (N,), self.bias_dtype, "bias"),
                _ptr(Y, (T, N), self.out_dtype, "Y"), self._aux(aux))
        _check(lib().gemm_epi_execute(self.handle, *args, _stream_ptr(stream)))

    def drelu_bgrad_execute(self, dY2, W2, aux, dZ, dbias, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (_ptr(dY2, (T, K), dt, "dY2"), _ptr(W2, self.w_shape, dt, "W2"),
                _ptr(aux, (T, self.aux_words), torch.int32, "aux"), _ptr(dZ, (T, N), self.out_dtype, "dZ"),
                _ptr(dbias, (N,), torch.float32, "dbias"))
        _check(lib().drelu_bgrad_execute(self.handle, *args, _stream_ptr(stream)))

    def gemm_epi_wgrad_execute(self, X, dZ, dW, dbias=None, stream=None):
        """WGRAD plan: dW (K x N) = X^T . dZ; dbias (K floats, optional) = sum over t of X."""
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (_ptr(X, (T, K), dt, "X"), _ptr(dZ, (T, N), dt, "dZ"),
                _ptr(dW, (K, N), self.out_dtype, "dW"),
                _ptr(dbias, (K,), torch.float32, "dbias"))
        _check(lib().gemm_epi_wgrad_execute(self.handle, *args, _stream_ptr(stream)))

    def gemm_epi_unfused_execute(self, X, W, bias, T1, T2, Y, aux=None, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (_ptr(X, (T, K), dt, "X"), _ptr(W, self.w_shape, dt, "W"), _ptr(bias, (N,), self.bias_dtype, "bias"),
                _ptr(T1, (T, N), dt, "T1"), _ptr(T2, (T, N), dt, "T2"), _ptr(Y, (T, N), self.out_dtype, "Y"),
                self._aux(aux))
        _check(lib().gemm_epi_unfused_execute(self.handle, *args, _stream_ptr(stream)))

    def drelu_bgrad_unfused_execute(self, dY2, W2, aux, G, dZ, dbias, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (_ptr(dY2, (T, K), dt, "dY2"), _ptr(W2, self.w_shape, dt, "W2"),
                _ptr(aux, (T, self.aux_words), torch.int32, "aux"), _ptr(G, (T, N), dt, "G"),
                _ptr(dZ, (T, N), self.out_dtype, "dZ"), _ptr(dbias, (N,), torch.float32, "dbias"))
        _check(lib().drelu_bgrad_unfused_execute(self.handle, *args, _stream_ptr(stream)))

    # prebuilt calls: (fn, args) so that fn(*args) enqueues the C call with no
    # per-call argument checking (for tight launch loops; check rc yourself)
    def execute_call(self, X, W, bias, Y, aux=None, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (self.handle, _ptr(X, (T, K), dt, "X"), _ptr(W, self.w_shape, dt, "W"), _ptr(bias, (N,), self.bias_dtype, "bias"),
                _ptr(Y, (T, N), self.out_dtype, "Y"), self._aux(aux), _stream_ptr(stream))
        return lib().gemm_epi_execute, args

    def drelu_bgrad_call(self, dY2, W2, aux, dZ, dbias, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (self.handle, _ptr(dY2, (T, K), dt, "dY2"), _ptr(W2, self.w_shape, dt, "W2"),
                _ptr(aux, (T, self.aux_words), torch.int32, "aux"), _ptr(dZ, (T, N), self.out_dtype, "dZ"),
                _ptr(dbias, (N,), torch.float32, "dbias"), _stream_ptr(stream))
        return lib().drelu_bgrad_execute, args

    def wgrad_call(self, X, dZ, dW, dbias=None, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (self.handle, _ptr(X, (T, K), dt, "X"), _ptr(dZ, (T, N), dt, "dZ"),
                _ptr(dW, (K, N), self.out_dtype, "dW"),
                _ptr(dbias, (K,), torch.float32, "dbias"), _stream_ptr(stream))
        return lib().gemm_epi_wgrad_execute, args

    def unfused_call(self, X, W, bias, T1, T2, Y, aux=None, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (self.handle, _ptr(X, (T, K), dt, "X"), _ptr(W, self.w_shape, dt, "W"), _ptr(bias, (N,), self.bias_dtype, "bias"),
                _ptr(T1, (T, N), dt, "T1"), _ptr(T2, (T, N), dt, "T2"), _ptr(Y, (T, N), self.out_dtype, "Y"),
                self._aux(aux), _stream_ptr(stream))
        return lib().gemm_epi_unfused_execute, args

    def drelu_bgrad_unfused_call(self, dY2, W2, aux, G, dZ, dbias, stream=None):
        T, N, K, dt = self.T, self.N, self.K, self.dtype
        args = (self.handle, _ptr(dY2, (T, K), dt, "dY2"), _ptr(W2, self.w_shape, dt, "W2"),
                _ptr(aux, (T, self.aux_words), torch.int32, "aux"), _ptr(G, (T, N), dt, "G"),
                _ptr(dZ, (T, N), self.out_dtype, "dZ"), _ptr(dbias, (N,), torch.float32, "dbias"), _stream_ptr(stream))
        return lib().drelu_bgrad_unfused_execute, args

    # conveniences that allocate their outputs (allocation happens in torch,
    # outside the library; the library call itself allocates nothing)
    def forward(self, X, W, bias, stream=None):
        Y = torch.empty((self.T, self.N), dtype=self.out_dtype, device=X.device)
        spec = self.aux_spec()
        aux = torch.empty(spec[0], dtype=spec[1], device=X.device) if spec else None
        self.gemm_epi_execute(X, W, bias, Y, aux, stream)
        return Y, aux

    def backward(self, dY2, W2, aux, stream=None):
        dZ = torch.empty((self.T, self.N), dtype=self.out_dtype, device=dY2.device)
        dbias = torch.empty((self.N,), dtype=torch.float32, device=dY2.device)
        self.drelu_bgrad_execute(dY2, W2, aux, dZ, dbias, stream)
        return dZ, dbias

    def wgrad(self, X, dZ, with_dbias=False, stream=None):
        dW = torch.empty((self.K, self.N), dtype=self.out_dtype, device=X.device)
        dbias = torch.empty((self.K,), dtype=torch.float32, device=X.device) if with_dbias else None
        self.gemm_epi_wgrad_execute(X, dZ, dW, dbias, stream)
        return (dW, dbias) if with_dbias else dW
