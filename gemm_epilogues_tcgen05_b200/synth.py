"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and distributions of the workloads below and rounds them to
the 16-bit type (round-to-nearest-even, torch's cast). Both the CUDA library
and the CPU oracle receive the same bytes from here.

Workloads (T rows, K contraction, N features; D2 = contraction of the
backward product G = dY2 . W2):

=============  ======  =====  =====  =====  =====
name           dtype   T      K      N      D2
=============  ======  =====  =====  =====  =====
pr1            fp16    1024   2048   512    512
square         fp16    4096   4096   4096   --
ffn            bf16    4096   4096   11008  4096
large          fp16    65536  16384  8192   --
skinny-<T>     bf16    T      4096   11008  4096   (T in 1, 8, 64, 256)
=============  ======  =====  =====  =====  =====

Distributions: X ~ N(0, 1); W ~ N(0, 1/K); bias ~ N(0, 0.1) read as a
variance (std = sqrt(0.1)); dY2 ~ N(0, 1); W2 ~ N(0, 1/512) for pr1 and
N(0, 1/11008) for ffn and skinny. The pr1 shape (m, n, k = 1024, 512, 2048)
is the worked call of "nvmath-python cuBLASLt bindings for PyTorch fusion";
the large shape is the H200 fp16 case of "nvmath-python fused epilogs for
linear layers" (performance-evidence section); ffn is the M=4096, N=11008
layer of "AI inference compiler optimisation: operator fusion", section 3.2.
"""
from __future__ import annotations

import dataclasses
import math

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    T: int
    K: int
    N: int
    D2: int | None = None
    w2_var: float | None = None
    seed: int = 1234

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def has_backward(self) -> bool:
        return self.D2 is not None


WORKLOADS = {
    "pr1": Workload("pr1", "fp16", 1024, 2048, 512, 512, 1.0 / 512, seed=1234),
    "square": Workload("square", "fp16", 4096, 4096, 4096, seed=1235),
    "ffn": Workload("ffn", "bf16", 4096, 4096, 11008, 4096, 1.0 / 11008, seed=1236),
    "large": Workload("large", "fp16", 65536, 16384, 8192, seed=1237),
}
# a same-K slice of the large shape (8192 of its 65536 rows, ~0.7 GB on the
# device), small enough for multi-pass profiler captures of the large
# shape's kernel
WORKLOADS["large-proxy"] = Workload("large-proxy", "fp16", 8192, 16384, 8192, seed=1237)
for _t in (1, 8, 64, 256):
    WORKLOADS[f"skinny-{_t}"] = Workload(f"skinny-{_t}", "bf16", _t, 4096, 11008, 4096, 1.0 / 11008,
                                         seed=1238)

BIAS_STD = math.sqrt(0.1)

# sub-seed per tensor, so that adding a tensor never shifts the others
_TENSOR_IDS = {"X": 1, "W": 2, "bias": 3, "dY2": 4, "W2": 5}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, dtype, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) draws in fp32, rounded to ``dtype``."""
    x = torch.randn(tuple(shape), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (x * std).to(dtype)


def integers(shape, lo: int, hi: int, dtype, seed: int, device="cpu") -> torch.Tensor:
    """Uniform integers in [lo, hi] stored exactly in ``dtype``."""
    x = torch.randint(lo, hi + 1, tuple(shape), generator=_gen(seed, device), device=device)
    return x.to(dtype)


def masked_grad(T: int, N: int, D2: int, dtype, seed: int, device="cpu") -> torch.Tensor:
    """A stand-in for the backward's dZ (T x N) with its value distribution:
    N(0, D2/N) draws (dY2 ~ N(0, 1) against W2 ~ N(0, 1/N), summed over D2),
    set to zero where a fair coin marks the unit inactive (the ReLU mask of a
    symmetric pre-activation)."""
    g = normal((T, N), (D2 / N) ** 0.5, torch.float32, seed, device)
    keep = torch.rand((T, N), generator=_gen(seed + 1, device), device=device) < 0.5
    return torch.where(keep, g, torch.zeros_like(g)).to(dtype)


def ffn_step_inputs(T: int, D: int, F: int, dtype: str, seed: int, kind: str = "normal", device="cpu") -> dict:
    """Inputs of one two-layer block step, weights in the [out, in] layout:
    X (T x D), W1 (F x D), b1 (F), W2 (D x F), b2 (D) and the loss gradient
    dY (T x D). "normal": X, dY ~ N(0, 1), W1 ~ N(0, 1/D), W2 ~ N(0, 1/F),
    biases ~ N(0, 0.1). "int": integers in [-1, 1] (biases [-2, 2]), so that
    every sum and product of the step is exact."""
    dt = DTYPES[dtype]
    shapes = {"X": (T, D), "W1": (F, D), "b1": (F,), "W2": (D, F), "b2": (D,), "dY": (T, D)}
    std = {"X": 1.0, "W1": D ** -0.5, "b1": BIAS_STD, "W2": F ** -0.5, "b2": BIAS_STD, "dY": 1.0}
    out = {}
    for i, (k, shp) in enumerate(shapes.items()):
        if kind == "int":
            r = 2 if k in ("b1", "b2") else 1
            out[k] = integers(shp, -r, r, dt, seed * 8 + i, device)
        else:
            out[k] = normal(shp, std[k], dt, seed * 8 + i, device)
    return out


def make_inputs(w: Workload, device="cpu", parts=("fwd", "bwd"), T: int | None = None) -> dict:
    """Inputs of one workload: X, W, bias (fwd) and dY2, W2 (bwd).

    ``T`` overrides the row count (for a smaller slice of the same recipe).
    """
    T = w.T if T is None else T
    dt = w.torch_dtype
    out = {}
    if "fwd" in parts:
        out["X"] = normal((T, w.K), 1.0, dt, w.seed * 16 + _TENSOR_IDS["X"], device)
        out["W"] = normal((w.K, w.N), 1.0 / math.sqrt(w.K), dt, w.seed * 16 + _TENSOR_IDS["W"], device)
        out["bias"] = normal((w.N,), BIAS_STD, dt, w.seed * 16 + _TENSOR_IDS["bias"], device)
    if "bwd" in parts and w.has_backward:
        out["dY2"] = normal((T, w.D2), 1.0, dt, w.seed * 16 + _TENSOR_IDS["dY2"], device)
        out["W2"] = normal((w.D2, w.N), math.sqrt(w.w2_var), dt, w.seed * 16 + _TENSOR_IDS["W2"], device)
    return out


def make_shape_inputs(T: int, N: int, K: int, dtype: str, seed: int, D2: int | None = None,
                      kind: str = "normal", device="cpu") -> dict:
    """Inputs for an arbitrary (T, N, K[, D2]) test shape.

    kind="normal": the workload recipe (X ~ N(0,1), W ~ N(0,1/K), bias ~
    N(0,0.1), dY2 ~ N(0,1), W2 ~ N(0,1/N)).
    kind="int": integers in [-3, 3] for every tensor, so that every product
    and partial sum is an exact small integer.
    """
    dt = DTYPES[dtype]
    out = {}
    if kind == "normal":
        out["X"] = normal((T, K), 1.0, dt, seed * 16 + 1, device)
        out["W"] = normal((K, N), 1.0 / math.sqrt(K), dt, seed * 16 + 2, device)
        out["bias"] = normal((N,), BIAS_STD, dt, seed * 16 + 3, device)
        if D2 is not None:
            out["dY2"] = normal((T, D2), 1.0, dt, seed * 16 + 4, device)
            out["W2"] = normal((D2, N), 1.0 / math.sqrt(N), dt, seed * 16 + 5, device)
    elif kind == "int":
        out["X"] = integers((T, K), -3, 3, dt, seed * 16 + 1, device)
        out["W"] = integers((K, N), -3, 3, dt, seed * 16 + 2, device)
        out["bias"] = integers((N,), -3, 3, dt, seed * 16 + 3, device)
        if D2 is not None:
            out["dY2"] = integers((T, D2), -3, 3, dt, seed * 16 + 4, device)
            out["W2"] = integers((D2, N), -3, 3, dt, seed * 16 + 5, device)
    else:
        raise ValueError(kind)
    return out


def sample_indices(n: int, count: int, seed: int) -> list[int]:
    """``count`` distinct sorted indices in [0, n), drawn with a fixed seed."""
    count = min(count, n)
    perm = torch.randperm(n, generator=_gen(seed, "cpu"))[:count]
    return sorted(int(i) for i in perm)


def bits_u16(t: torch.Tensor):
    """The raw 16-bit patterns of a CPU fp16/bf16 tensor as a numpy uint16 array."""
    import numpy as np

    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
