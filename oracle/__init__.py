"""Plain fp64 CPU oracle for the fused linear-layer GEMM + epilogue.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. It shares no code with the CUDA library and never imports it; both
sides receive the same seeded 16-bit input bytes from the input generator.

The contraction ``sum_k a[r,k] * b[k,c] (+ bias[c])`` and its error scale
``S = sum_k |a[r,k] * b[k,c]| (+ |bias[c]|)`` are computed by ``oracle.c`` in
binary64, summed in ascending k. The epilogue steps below follow the pages in
their order and notation:

* ``linear_fwd`` -- epilogs BIAS, RELU_BIAS, RELU_AUX_BIAS.
  "Fusing bias addition into matrix multiplication with nvmath-python":
  BIAS adds the bias to the product, RELU_BIAS applies ReLU after it, and
  RELU_AUX_BIAS also returns the bit-encoded ReLU mask ``relu_aux``.
  "AI inference compiler optimisation: operator fusion", section 3.1: the
  fused kernel sums over K, adds ``bias[col]`` and takes ``max(sum, 0)``.
* ``gelu`` -- epilog GELU_BIAS, which "nvmath-python cuBLASLt bindings for
  PyTorch fusion" lists among the predefined epilogs as bias followed by
  GELU. The page does not say which GELU; the oracle takes the definition
  GELU(z) = z * Phi(z), Phi the standard normal CDF, i.e.
  z/2 * (1 + erf(z / sqrt 2)), with scipy's double-precision erf as the
  library primitive.
* GELU_AUX_BIAS -- GELU_BIAS that also returns an auxiliary output for the
  backward pass, as RELU_AUX_BIAS does for ReLU. The pages describe
  RELU_AUX_BIAS's auxiliary output (the mask, for the backward epilog) but
  not GELU's; the derivative of GELU depends on the pre-activation z itself,
  not only on its sign, so the auxiliary output is read as that
  pre-activation Z = X.W + bias (``pre``), which the library stores in its
  16-bit type.
* ``wgrad`` -- the weight gradient dW = X^T . dZ of the linear layer, the
  part of the backward pass that "nvmath-python fused epilogs for linear
  layers" (FAQ) says DRELU_BGRAD does not cover. The plain definition:
  dW[k, n] = sum_t X[t, k] * dZ[t, n], i.e. the contraction above applied to
  the transposed X.
* ``ffn_step`` -- one training step of a two-layer block (ReLU between
  the layers, weights in the [out, in] layout) chained from the calls
  above: forward through both layers, then the backward pass that
  DRELU_BGRAD plus the weight gradients make up. Intermediates the step
  stores in the 16-bit type (H, dZ1) are encoded exactly (``encode_exact``
  refuses values the type cannot hold), so the chain needs no rounding
  routine; tests feed it integer-valued inputs.
* ``relu_aux_words`` -- the mask's bit layout. The pages call it opaque and
  meant only for the dedicated backward epilog ("nvmath-python fused epilogs
  for linear layers", forward section), so its layout is this library's own
  choice: word ``aux[t, n // 32]`` holds bit ``n % 32`` = 1 iff Z[t, n] > 0,
  least significant bit first, bits past N zero.
* ``drelu_bgrad`` -- epilog DRELU_BGRAD ("nvmath-python fused epilogs for
  linear layers", section on the DRELU_BGRAD backward path): the mask from
  ``relu_aux`` is applied to the product G = dY2 . W2, and the column-wise sum
  of the masked result is returned as the bias gradient ``drelu_bgrad``.

Functions take numpy ``uint16`` arrays of bit patterns and return fp64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import scipy.special

F16 = 0
BF16 = 1

EPILOG_BIAS = "BIAS"
EPILOG_RELU_BIAS = "RELU_BIAS"
EPILOG_RELU_AUX_BIAS = "RELU_AUX_BIAS"
EPILOG_GELU_BIAS = "GELU_BIAS"
EPILOG_GELU_AUX_BIAS = "GELU_AUX_BIAS"
EPILOG_NONE = "NONE"

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (plain gcc, no CUDA).

    ``-ffp-contract=off`` keeps every multiply and add a separately rounded
    binary64 operation, exactly as written in the C source.
    """
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_matmul_bias.restype = ctypes.c_int
        lib.oracle_matmul_bias.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def decode(bits: np.ndarray, dtype: int) -> np.ndarray:
    """16-bit patterns -> fp64 values through the oracle's own decoder."""
    lib = _load()
    fn = lib.oracle_bf16_to_double if dtype == BF16 else lib.oracle_half_to_double
    flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    table = np.array([fn(i) for i in range(65536)], dtype=np.float64)
    return table[flat].reshape(np.shape(bits))


def _ptr(a):
    return None if a is None else a.ctypes.data


def matmul_bias(A: np.ndarray, B: np.ndarray, bias, dtype: int, rows=None, cols=None, threads=None):
    """C = A[rows] . B[:, cols] (+ bias[cols]) and its scale S, both fp64.

    ``A`` is R x K, ``B`` is K x C (row-major 16-bit patterns); ``bias`` is
    length C or None. ``rows`` / ``cols`` select output rows / columns
    (None = all). Returns (C, S) of shape len(rows) x len(cols).
    """
    A = np.ascontiguousarray(A, dtype=np.uint16)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    R, K = A.shape
    K2, Cn = B.shape
    if K2 != K:
        raise ValueError(f"inner dimensions differ: {K} vs {K2}")
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.uint16).ravel()
        if bias.shape[0] != Cn:
            raise ValueError("bias length must equal the column count")
    r_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c_arr = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nr = R if r_arr is None else r_arr.shape[0]
    nc = Cn if c_arr is None else c_arr.shape[0]
    C = np.empty((nr, nc), dtype=np.float64)
    S = np.empty((nr, nc), dtype=np.float64)
    rc = _load().oracle_matmul_bias(_ptr(A), _ptr(B), _ptr(bias), int(dtype), R, Cn, K,
                                    _ptr(r_arr), nr, _ptr(c_arr), nc, _ptr(C), _ptr(S),
                                    int(threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_matmul_bias rejected its arguments")
    return C, S


def relu_aux_words(bits: np.ndarray) -> np.ndarray:
    """Pack a T x N boolean mask into uint32 words, T x ceil(N/32).

    Bit ``n % 32`` of word ``[t, n // 32]`` is ``bits[t, n]``; bits past N are 0.
    """
    bits = np.asarray(bits, dtype=bool)
    T, N = bits.shape
    W = (N + 31) // 32
    padded = np.zeros((T, W * 32), dtype=np.uint64)
    padded[:, :N] = bits
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = (padded.reshape(T, W, 32) * weights).sum(axis=2)
    return words.astype(np.uint32)


def relu_aux_bits(words: np.ndarray, N: int) -> np.ndarray:
    """Inverse of ``relu_aux_words``: T x ceil(N/32) uint32 -> T x N bool."""
    words = np.asarray(words, dtype=np.uint32)
    shifts = np.arange(32, dtype=np.uint32)
    bits = ((words[:, :, None] >> shifts) & np.uint32(1)).astype(bool)
    return bits.reshape(words.shape[0], -1)[:, :N]


def gelu(Z):
    """GELU(z) = z * Phi(z) = z / 2 * (1 + erf(z / sqrt 2)) in binary64."""
    Z = np.asarray(Z, dtype=np.float64)
    return 0.5 * Z * (1.0 + scipy.special.erf(Z / np.sqrt(2.0)))


def linear_fwd(X, W, bias, dtype: int, epilog: str, rows=None, cols=None, threads=None):
    """Forward epilogs on X (T x K) and W (K x N) with bias (N): 16-bit
    patterns (uint16), or float32 values for an fp32 bias.

    Returns a dict with
      Z     the pre-activation X.W + bias (fp64, exact up to binary64 rounding)
      S     the error scale sum_k |x w| + |b|
      Y     Z for BIAS; max(Z, 0) for RELU_BIAS / RELU_AUX_BIAS; gelu(Z) for GELU_BIAS and
            GELU_AUX_BIAS
      bits  Z > 0 (strict: a zero pre-activation gives bit 0), for RELU_AUX_BIAS
      aux   the packed words (only when every column was computed)
      pre   GELU_AUX_BIAS's auxiliary output: the pre-activation Z
    """
    if epilog not in (EPILOG_BIAS, EPILOG_RELU_BIAS, EPILOG_RELU_AUX_BIAS, EPILOG_GELU_BIAS, EPILOG_GELU_AUX_BIAS,
                      EPILOG_NONE):
        raise ValueError(f"unknown forward epilog {epilog}")
    if epilog == EPILOG_NONE:
        bias = None  # the plain product
    if bias is not None and np.asarray(bias).dtype == np.float32:
        # an fp32 bias ("Fusing bias addition ...", engineering checklist: a
        # float32 bias with 16-bit operands): the product, then the bias added
        # in binary64 -- the same last step the C routine takes for a 16-bit bias
        Z, S = matmul_bias(X, W, None, dtype, rows=rows, cols=cols, threads=threads)
        b = np.asarray(bias, dtype=np.float64).ravel()
        if b.shape[0] != np.asarray(W).shape[1]:
            raise ValueError("bias length must equal the column count")
        b = b if cols is None else b[np.asarray(cols, dtype=np.int64)]
        Z = Z + b[None, :]
        S = S + np.abs(b)[None, :]
    else:
        Z, S = matmul_bias(X, W, bias, dtype, rows=rows, cols=cols, threads=threads)
    out = {"Z": Z, "S": S}
    if epilog in (EPILOG_BIAS, EPILOG_NONE):
        out["Y"] = Z.copy()
    elif epilog in (EPILOG_GELU_BIAS, EPILOG_GELU_AUX_BIAS):
        out["Y"] = gelu(Z)
        if epilog == EPILOG_GELU_AUX_BIAS:
            out["pre"] = Z.copy()
    else:
        out["Y"] = np.maximum(Z, 0.0)
    if epilog == EPILOG_RELU_AUX_BIAS:
        out["bits"] = Z > 0.0
        if cols is None:
            out["aux"] = relu_aux_words(out["bits"])
    return out


def encode_exact(values, dtype: int) -> np.ndarray:
    """fp64 values to 16-bit patterns of ``dtype``; ValueError unless every
    value is exactly representable (then the encoding needs no rounding)."""
    v = np.asarray(values, dtype=np.float64)
    if dtype == F16:
        bits = v.astype(np.float16).view(np.uint16)
    elif dtype == BF16:
        f32 = v.astype(np.float32)
        bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    else:
        raise ValueError(f"unknown dtype {dtype}")
    if not np.array_equal(decode(bits, dtype), v):
        raise ValueError("value not exactly representable in the 16-bit type")
    return bits


def ffn_step(X, W1, b1, W2, b2, dY, dtype: int):
    """One step of Y = relu(X W1^T + b1) W2^T + b2 and its backward for the
    loss gradient dY. X: T x D, W1: F x D, b1: F, W2: D x F, b2: D, dY: T x D
    (16-bit patterns; weights in the [out, in] layout). Returns fp64 H, bits,
    Y, dZ1, db1, dW2, db2, dW1, dX."""
    W1 = np.asarray(W1, dtype=np.uint16)
    W2 = np.asarray(W2, dtype=np.uint16)
    f1 = linear_fwd(X, np.ascontiguousarray(W1.T), b1, dtype, EPILOG_RELU_AUX_BIAS)
    H = encode_exact(f1["Y"], dtype)
    f2 = linear_fwd(H, np.ascontiguousarray(W2.T), b2, dtype, EPILOG_BIAS)
    F = W1.shape[0]
    bwd = drelu_bgrad(dY, W2, f1["aux"], dtype, F)     # G = dY . W2 (W2 read as D x F = K x N)
    dZ1 = encode_exact(bwd["dZ"], dtype)
    g2 = wgrad(dY, H, dtype)                           # dW2 = dY^T H, db2 = sum_t dY
    g1 = wgrad(dZ1, X, dtype)                          # dW1 = dZ1^T X
    dX = linear_fwd(dZ1, W1, None, dtype, EPILOG_NONE)  # dX = dZ1 . W1 (W1 read as F x D = K x N)
    return {"H": f1["Y"], "bits": f1["bits"], "Y": f2["Y"], "dZ1": bwd["dZ"], "db1": bwd["dbias"],
            "dW2": g2["dW"], "db2": g2["dbias"], "dW1": g1["dW"], "dX": dX["Y"]}


def wgrad(X, dZ, dtype: int, rows=None, cols=None, threads=None):
    """dW = X^T . dZ for X (T x K) and dZ (T x N): K x N, summed over t.

    Returns a dict with
      dW    the product (fp64)
      S     sum_t |x dz|, its error scale
      dbias sum over t of X[t, k] (the bias gradient when X is a layer's
            output gradient), and Sb = sum_t |X[t, k]|; both for the
            selected rows k
    ``rows`` / ``cols`` select rows k / columns n of dW.
    """
    X = np.asarray(X, dtype=np.uint16)
    dZ = np.asarray(dZ, dtype=np.uint16)
    if X.shape[0] != dZ.shape[0]:
        raise ValueError(f"X and dZ need the same row count: {X.shape[0]} vs {dZ.shape[0]}")
    dW, S = matmul_bias(np.ascontiguousarray(X.T), dZ, None, dtype, rows=rows, cols=cols, threads=threads)
    xv = decode(X, dtype)
    if rows is not None:
        xv = xv[:, np.asarray(rows, dtype=np.int64)]
    return {"dW": dW, "S": S, "dbias": xv.sum(axis=0), "Sb": np.abs(xv).sum(axis=0)}


def drelu_bgrad(dY2, W2, aux, dtype: int, N: int, rows=None, cols=None, threads=None):
    """DRELU_BGRAD on dY2 (T x D2), W2 (D2 x N) and the forward's relu_aux words.

    Returns a dict with
      G     dY2 . W2 (fp64)
      S     sum_d |dy w2|, the error scale of G and dZ
      dZ    G where the mask bit is set, else 0
      dbias (only when every row was computed) sum over rows of dZ per column
      Sb    sum over rows of |dZ|, the error scale of dbias
    """
    aux = np.ascontiguousarray(aux, dtype=np.uint32)
    G, S = matmul_bias(dY2, W2, None, dtype, rows=rows, cols=cols, threads=threads)
    bits_all = relu_aux_bits(aux, N)
    r_idx = np.arange(aux.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    c_idx = np.arange(N) if cols is None else np.asarray(cols, dtype=np.int64)
    bits = bits_all[np.ix_(r_idx, c_idx)]
    dZ = np.where(bits, G, 0.0)
    out = {"G": G, "S": S, "bits": bits, "dZ": dZ}
    if rows is None:
        out["dbias"] = dZ.sum(axis=0)
        out["Sb"] = np.abs(dZ).sum(axis=0)
    return out
