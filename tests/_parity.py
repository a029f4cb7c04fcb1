"""Helpers for the GPU parity tests: run the library through its C ABI and
compare with the CPU oracle under the acceptance bounds.

Bounds (per element): Y and dZ within 2e-3 * S + u * |ref|, where S is the
oracle's sum of |products| (+ |bias|) and u the unit roundoff of the 16-bit
output (2^-8 for bf16, 2^-11 for fp16): the 2e-3 * S term bounds the
computation, the u * |ref| term the one final rounding to the output type,
which 2e-3 * S alone cannot cover when |Y| is close to S (small K, bf16).

dbias (fp32) within the stated 1e-3 * sum_t |dZ_t| plus two fp32 terms:
  * each summed G[t, n] is an fp32 dot product of D2 exact products, so it
    carries the standard dot-product error bound gamma_D2 * S_t ~ D2 * u32 * S_t
    (recursive summation; u32 = 2^-23, the unit of a truncating adder, since
    the tensor cores' rounding mode is not documented): 2 * D2 * 2^-24 * S_t
    for every t whose mask bit is set;
  * the reduction over the T rows adds at most T * 2^-24 * sum_t |dZ_t|
    (round-to-nearest fp32 adds, any order).
Without the first term a column of one row (T = 1) would need 1e-3 relative
accuracy of a single fp32 dot product under cancellation. Every check records
the largest |err| / (1e-3 * sum_t |dZ_t|) it saw (``DBIAS_RATIOS``), so a run
shows how close the plain stated bound comes. relu_aux is bit-exact wherever
|Z_ref| > 2e-3 * S. For integer-valued inputs every result is exact, so the
comparison there is equality.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gemm_epilogues_tcgen05_b200 import Plan, synth

Y_REL = 2e-3
DBIAS_REL = 1e-3
DOT_C = 2.0  # gamma_D2 of a truncating fp32 adder, in units of D2 * 2^-24
DBIAS_RATIOS: dict[str, dict] = {}  # per check: worst |err| over the stated bound and over the full bound
GUARD = 4096  # sentinel elements before and after each output
SENTINEL16 = 0x7E5A  # a 16-bit pattern no result takes in these tests
SENTINEL32 = 0x5A5A5A5A


def odt(dtype: torch.dtype) -> int:
    return oracle.BF16 if dtype == torch.bfloat16 else oracle.F16


def guarded(shape, dtype, device):
    """An output tensor inside a larger buffer whose margins hold a sentinel."""
    n = int(np.prod(shape))
    if dtype in (torch.float16, torch.bfloat16):
        buf = torch.full((n + 2 * GUARD,), SENTINEL16, dtype=torch.int16, device=device).view(dtype)
    elif dtype == torch.int32:
        buf = torch.full((n + 2 * GUARD,), SENTINEL32, dtype=torch.int32, device=device)
    else:
        buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device=device)
    return buf, buf[GUARD:GUARD + n].view(shape)


def guards_intact(buf) -> bool:
    head, tail = buf[:GUARD], buf[-GUARD:]
    if buf.dtype in (torch.float16, torch.bfloat16):
        h, t = head.view(torch.int16), tail.view(torch.int16)
        return bool(torch.all(h == SENTINEL16)) and bool(torch.all(t == SENTINEL16))
    if buf.dtype == torch.int32:
        return bool(torch.all(head == SENTINEL32)) and bool(torch.all(tail == SENTINEL32))
    return bool(torch.all(torch.isnan(head))) and bool(torch.all(torch.isnan(tail)))


def run_forward(inp_cpu: dict, epilog: str, dtype, device="cuda", unfused=False, bias_f32=False, w_nk=False,
                out_f32=False):
    """One forward call; with bias_f32 the plan reads the fp32 bias under "bias32"; with
    w_nk the library gets W transposed to N x K (the oracle keeps the K x N original)."""
    X, W, b = (inp_cpu[k].to(device) for k in ("X", "W", "bias32" if bias_f32 else "bias"))
    T, K = X.shape
    N = W.shape[1]
    if w_nk:
        W = W.t().contiguous()
    with Plan(T, N, K, dtype, epilog, w_nk=w_nk, out_f32=out_f32) as plan:
        if bias_f32:
            plan.set_bias_f32(True)
        info = plan.info()
        ybuf, Y = guarded((T, N), plan.out_dtype, device)
        if epilog == "GELU_AUX_BIAS":  # the pre-activation, T x N in the plan's 16-bit type
            abuf, aux = guarded((T, N), dtype, device)
        else:
            abuf, aux = guarded((T, (N + 31) // 32), torch.int32, device)
        aux_arg = aux if epilog in ("RELU_AUX_BIAS", "GELU_AUX_BIAS") else None
        if unfused:
            T1 = torch.empty((T, N), dtype=dtype, device=device)
            T2 = (Y if epilog == "BIAS" else None if epilog == "GELU_AUX_BIAS"
                  else torch.empty((T, N), dtype=dtype, device=device))
            plan.gemm_epi_unfused_execute(X, W, b, T1, T2, Y, aux_arg)
        else:
            plan.gemm_epi_execute(X, W, b, Y, aux_arg)
        torch.cuda.synchronize()
        assert plan.status() == 0, "watchdog fired"
    assert guards_intact(ybuf), "Y guard region overwritten"
    if epilog in ("RELU_AUX_BIAS", "GELU_AUX_BIAS"):
        assert guards_intact(abuf), "aux guard region overwritten"
    out = {"Y": Y.cpu(), "info": info}
    if epilog == "RELU_AUX_BIAS":
        out["aux"] = aux.cpu().numpy().view(np.uint32)
    if epilog == "GELU_AUX_BIAS":
        out["pre"] = aux.cpu()
    return out


def run_backward(inp_cpu: dict, aux_words: np.ndarray, dtype, device="cuda", unfused=False, repeats=1, w_nk=False,
                 out_f32=False):
    dY2, W2 = inp_cpu["dY2"].to(device), inp_cpu["W2"].to(device)
    T, D2 = dY2.shape
    N = W2.shape[1]
    if w_nk:
        W2 = W2.t().contiguous()
    aux = torch.from_numpy(np.ascontiguousarray(aux_words).view(np.int32)).to(device)
    outs = []
    with Plan(T, N, D2, dtype, "DRELU_BGRAD", w_nk=w_nk, out_f32=out_f32) as plan:
        info = plan.info()
        for _ in range(repeats):
            zbuf, dZ = guarded((T, N), plan.out_dtype, device)
            bbuf, dbias = guarded((N,), torch.float32, device)
            if unfused:
                G = torch.empty((T, N), dtype=dtype, device=device)
                plan.drelu_bgrad_unfused_execute(dY2, W2, aux, G, dZ, dbias)
            else:
                plan.drelu_bgrad_execute(dY2, W2, aux, dZ, dbias)
            torch.cuda.synchronize()
            assert plan.status() == 0, "watchdog fired"
            assert guards_intact(zbuf), "dZ guard region overwritten"
            assert guards_intact(bbuf), "dbias guard region overwritten"
            outs.append({"dZ": dZ.cpu(), "dbias": dbias.cpu(), "info": info})
    return outs if repeats > 1 else outs[0]


def unit_roundoff(dtype) -> float:
    return {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 2.0 ** -24}.get(dtype, 0.0)


def assert_within(got: np.ndarray, ref: np.ndarray, scale: np.ndarray, rel: float, what: str, out_u: float = 0.0):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bound = rel * scale + out_u * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        worst = float(np.max(err / np.maximum(bound, 1e-300)))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside {rel}*S; worst ratio {worst:.3g}; "
                             f"first at {idx}")


# max over z of |d gelu / dz| = Phi(sqrt 2) + sqrt 2 * phi(sqrt 2) = 1.1289...: an error e in
# the pre-activation moves gelu(z) by at most 1.13 e
GELU_SLOPE = 1.13


def check_forward(inp_cpu, epilog, dtype, gpu, rows=None, cols=None, exact=False, stored_xw=False, bias_f32=False):
    """Y (and the mask) against the oracle.  ``stored_xw``: the path under test stored X·W in the
    16-bit output type before adding the bias (the unfused ablation), a second rounding that may
    add up to u·|X·W|, so the bound gains that term."""
    bits = synth.bits_u16
    bias = inp_cpu["bias32"].numpy() if bias_f32 else bits(inp_cpu["bias"])
    ref = oracle.linear_fwd(bits(inp_cpu["X"]), bits(inp_cpu["W"]), bias, odt(dtype), epilog, rows=rows, cols=cols)
    Y = gpu["Y"]
    r_idx = slice(None) if rows is None else torch.tensor(rows)
    c_idx = slice(None) if cols is None else torch.tensor(cols)
    Ys = Y[r_idx][:, c_idx].double().numpy()
    uo = unit_roundoff(Y.dtype)  # the output's own rounding (fp32 output: 2^-24)
    gelu = epilog in ("GELU_BIAS", "GELU_AUX_BIAS")
    if epilog == "GELU_AUX_BIAS":
        # the auxiliary output: Z rounded once to the plan's 16-bit type (twice on the unfused path)
        pre = gpu["pre"][r_idx][:, c_idx].double().numpy()
        if exact:
            expect = torch.from_numpy(ref["pre"]).to(dtype).double().numpy()
            assert np.array_equal(pre, expect), "GELU_AUX_BIAS aux (Z) not bit-exact on integer inputs"
        else:
            zscale = ref["S"]
            if stored_xw:
                b = inp_cpu["bias32" if bias_f32 else "bias"].double().numpy()
                b = b if cols is None else b[cols]
                zscale = zscale + (unit_roundoff(dtype) / Y_REL) * np.abs(ref["Z"] - b[None, :])
            assert_within(pre, ref["pre"], zscale, Y_REL, "GELU_AUX_BIAS aux (Z)", unit_roundoff(dtype))
    if exact and gelu:
        # Z is exact in fp32; only erff (a few fp32 ulps) and the final rounding remain
        err = np.abs(Ys - ref["Y"])
        bound = uo * np.abs(ref["Y"]) + 2e-7 * np.abs(ref["Z"]) + 1e-30
        assert np.all(err <= bound), f"GELU_BIAS on integer inputs: worst {np.max(err / bound):.3g} of the bound"
    elif exact:
        expect = torch.from_numpy(ref["Y"]).to(Y.dtype).double().numpy()  # exact Z rounded once
        assert np.array_equal(Ys, expect), f"{epilog}: Y not bit-exact on integer inputs"
    else:
        scale = ref["S"]
        if stored_xw:
            b = inp_cpu["bias32" if bias_f32 else "bias"].double().numpy()
            b = b if cols is None else b[cols]
            scale = scale + (unit_roundoff(dtype) / Y_REL) * np.abs(ref["Z"] - b[None, :])
            if gelu:  # the unfused path also stores X.W + b before the GELU kernel
                scale = scale + (unit_roundoff(dtype) / Y_REL) * np.abs(ref["Z"])
        if gelu:
            scale = GELU_SLOPE * scale
        assert_within(Ys, ref["Y"], scale, Y_REL, f"{epilog} Y", uo)
    if epilog in ("RELU_BIAS", "RELU_AUX_BIAS"):
        assert np.all(Ys >= 0), "ReLU output negative"
    if epilog == "RELU_AUX_BIAS":
        N = Y.shape[1]
        got_bits = oracle.relu_aux_bits(gpu["aux"], N)
        got_bits = got_bits[(slice(None) if rows is None else rows)][:, (slice(None) if cols is None else cols)]
        if exact:
            assert np.array_equal(got_bits, ref["bits"]), "relu_aux not bit-exact on integer inputs"
        else:
            sure = np.abs(ref["Z"]) > Y_REL * ref["S"]
            mism = (got_bits != ref["bits"]) & sure
            assert not mism.any(), f"relu_aux differs at {int(mism.sum())} decided positions"
        # pad bits past N are zero
        if N % 32:
            last = gpu["aux"][:, -1]
            assert np.all((last >> np.uint32(N % 32)) == 0), "pad bits set"
    return ref


def check_backward(inp_cpu, aux_words, dtype, gpu, rows=None, cols=None, exact=False, record=None, stored_dz=False):
    """dZ and dbias against the oracle. ``stored_dz``: the path under test summed
    dZ after rounding it to the 16-bit type (the unfused ablation) rather than
    the fp32 masked product, so each summed term may be off by its rounding,
    u * |dZ|: the dbias bound gains u * sum_t |dZ_t|."""
    bits = synth.bits_u16
    N = inp_cpu["W2"].shape[1]
    ref = oracle.drelu_bgrad(bits(inp_cpu["dY2"]), bits(inp_cpu["W2"]), aux_words, odt(dtype), N, rows=rows, cols=cols)
    r_idx = slice(None) if rows is None else torch.tensor(rows)
    c_idx = slice(None) if cols is None else torch.tensor(cols)
    dZ = gpu["dZ"][r_idx][:, c_idx].double().numpy()
    if exact:
        expect = torch.from_numpy(ref["dZ"]).to(gpu["dZ"].dtype).double().numpy()
        assert np.array_equal(dZ, expect), "dZ not bit-exact on integer inputs"
    else:
        assert_within(dZ, ref["dZ"], ref["S"], Y_REL, "dZ", unit_roundoff(gpu["dZ"].dtype))
    if rows is None:
        db = gpu["dbias"][c_idx].double().numpy()
        if exact:
            assert np.array_equal(db, ref["dbias"]), "dbias not exact on integer inputs"
        else:
            D2 = inp_cpu["dY2"].shape[1]
            kern = {0: "tile", 1: "few-row", 2: "pair"}.get((gpu.get("info") or {}).get("kernel"), "?")
            assert_dbias(db, ref, D2, record or f"T={inp_cpu['dY2'].shape[0]} N={N} D2={D2} {str(dtype)[6:]} {kern}"
                         + (" unfused" if stored_dz else ""), extra=unit_roundoff(dtype) * ref["Sb"] if stored_dz else 0.0)
            assert_dbias_is_column_sum(gpu["dbias"][c_idx], gpu["dZ"][:, c_idx], dtype)
    return ref


def dbias_scale(ref, D2: int) -> np.ndarray:
    """Bound on |dbias - dbias_ref| per column (see the module docstring):
    1e-3 * sum_t |dZ_t| + 2 * D2 * 2^-24 * sum_{t: bit} S_t + T * 2^-24 * sum_t |dZ_t|."""
    T = ref["bits"].shape[0]
    acc = DOT_C * D2 * 2.0 ** -24 * np.where(ref["bits"], ref["S"], 0.0).sum(axis=0)
    return DBIAS_REL * ref["Sb"] + acc + T * 2.0 ** -24 * ref["Sb"]


def assert_dbias(got: np.ndarray, ref, D2: int, what: str, extra=0.0):
    """dbias against the oracle under ``dbias_scale`` (+ ``extra``); records the worst ratios."""
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref["dbias"])
    scale = dbias_scale(ref, D2) + extra
    stated = np.max(err / np.maximum(DBIAS_REL * ref["Sb"], 1e-300)) if err.size else 0.0
    full = np.max(err / np.maximum(scale, 1e-300)) if err.size else 0.0
    prev = DBIAS_RATIOS.get(what, {"stated": 0.0, "bound": 0.0, "checks": 0})
    DBIAS_RATIOS[what] = {"stated": max(prev["stated"], float(stated)), "bound": max(prev["bound"], float(full)),
                          "checks": prev["checks"] + 1}
    assert_within(got, ref["dbias"], scale, 1.0, f"dbias ({what})")


def assert_dbias_is_column_sum(dbias, dZ, dtype):
    """Property at any size: dbias is the column sum of the masked gradient.
    dZ is that gradient rounded to the 16-bit type, so the two agree to the
    stated 1e-3 of sum |dZ| plus one rounding of each summed term."""
    dz = dZ.double()
    col = dz.sum(dim=0).numpy()
    mag = dz.abs().sum(dim=0).numpy()
    err = np.abs(dbias.double().numpy() - col)
    bound = (DBIAS_REL + unit_roundoff(dtype)) * mag
    assert np.all(err <= bound), f"dbias is not the column sum of dZ: worst {np.max(err / np.maximum(bound, 1e-300)):.3g}"


def run_wgrad(inp_cpu: dict, dtype, device="cuda", dz_key="dY2", out_f32=False):
    """dW = X^T dZ through the WGRAD plan; dZ is the T x N tensor under ``dz_key``."""
    X, dZ = inp_cpu["X"].to(device), inp_cpu[dz_key].to(device)
    T, K = X.shape
    N = dZ.shape[1]
    with Plan(T, N, K, dtype, "WGRAD", out_f32=out_f32) as plan:
        info = plan.info()
        wbuf, dW = guarded((K, N), plan.out_dtype, device)
        bbuf, dbias = guarded((K,), torch.float32, device)
        plan.gemm_epi_wgrad_execute(X, dZ, dW, dbias)
        torch.cuda.synchronize()
        assert plan.status() == 0, "watchdog fired"
    assert guards_intact(wbuf), "dW guard region overwritten"
    assert guards_intact(bbuf), "dbias guard region overwritten"
    return {"dW": dW.cpu(), "dbias": dbias.cpu(), "info": info}


def check_wgrad(inp_cpu, dtype, gpu, rows=None, cols=None, exact=False, dz_key="dY2"):
    bits = synth.bits_u16
    ref = oracle.wgrad(bits(inp_cpu["X"]), bits(inp_cpu[dz_key]), odt(dtype), rows=rows, cols=cols)
    r_idx = slice(None) if rows is None else torch.tensor(rows)
    c_idx = slice(None) if cols is None else torch.tensor(cols)
    got = gpu["dW"][r_idx][:, c_idx].double().numpy()
    if exact:
        expect = torch.from_numpy(ref["dW"]).to(gpu["dW"].dtype).double().numpy()
        assert np.array_equal(got, expect), "dW not bit-exact on integer inputs"
    else:
        assert_within(got, ref["dW"], ref["S"], Y_REL, "dW", unit_roundoff(gpu["dW"].dtype))
    db = gpu["dbias"].double().numpy()
    db = db if rows is None else db[rows]
    if exact:
        assert np.array_equal(db, ref["dbias"]), "wgrad dbias not exact on integer inputs"
    else:  # fp32 sums of 16-bit values in a fixed order
        assert_within(db, ref["dbias"], ref["Sb"], 1e-3, "wgrad dbias")
    return ref


def run_ffn_step(inp_cpu: dict, dtype, device="cuda"):
    """One two-layer block step through the public API (six plans, weights in
    the [out, in] layout): H, aux = layer 1 (RELU_AUX_BIAS); Y = layer 2
    (BIAS); dZ1, db1 = DRELU_BGRAD(dY, W2, aux); dW2, db2 = WGRAD(dY, H);
    dW1 = WGRAD(dZ1, X); dX = NONE(dZ1, W1)."""
    g = {k: v.to(device) for k, v in inp_cpu.items()}
    T, D = g["X"].shape
    F = g["W1"].shape[0]
    plans = [Plan(T, F, D, dtype, "RELU_AUX_BIAS", w_nk=True), Plan(T, D, F, dtype, "BIAS", w_nk=True),
             Plan(T, F, D, dtype, "DRELU_BGRAD"), Plan(T, F, D, dtype, "WGRAD"), Plan(T, D, F, dtype, "WGRAD"),
             Plan(T, D, F, dtype, "NONE")]
    try:
        H, aux = plans[0].forward(g["X"], g["W1"], g["b1"])
        Y, _ = plans[1].forward(H, g["W2"], g["b2"])
        dZ1, db1 = plans[2].backward(g["dY"], g["W2"], aux)
        dW2, db2 = plans[3].wgrad(g["dY"], H, with_dbias=True)
        dW1 = plans[4].wgrad(dZ1, g["X"])
        dX, _ = plans[5].forward(dZ1, g["W1"], None)
        torch.cuda.synchronize()
        assert all(p.status() == 0 for p in plans), "watchdog fired"
        kernels = [p.info()["kernel"] for p in plans]
    finally:
        for p in plans:
            p.free()
    out = {"H": H, "aux": aux, "Y": Y, "dZ1": dZ1, "db1": db1, "dW2": dW2, "db2": db2, "dW1": dW1, "dX": dX}
    out = {k: v.cpu() for k, v in out.items()}
    out["kernels"] = kernels
    return out
