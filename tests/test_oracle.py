"""Pins of the CPU oracle against facts fixed outside it (no GPU needed).

Each pin checks the oracle against something it does not compute itself:
hand-worked examples (tests/golden), an exact rational brute force, exact
integer arithmetic, a library matmul in float64, closed forms and
invariants. ``test_planted_mistakes_are_caught`` plants plausible mistakes
in wrappers around the oracle and checks that at least one pin fails for
each, so that the pins are known to have teeth.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from gemm_epilogues_tcgen05_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DT = {"fp16": 0, "bf16": 1}


def _bits(values, dtype):
    t = torch.tensor(values, dtype=torch.float64).to(synth.DTYPES[dtype])
    return synth.bits_u16(t)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- decoders

def test_decode_half_every_pattern(oracle_mod):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle_mod.decode(pats, oracle_mod.F16)
    ref = pats.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert np.array_equal(np.signbit(mine[ok]), np.signbit(ref[ok]))


def test_decode_bf16_every_pattern(oracle_mod):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle_mod.decode(pats, oracle_mod.BF16)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])


# ----------------------------------------------------------- pin functions
# Each pin takes (fwd, bwd) callables with the oracle's signatures and
# returns a list of failure strings (empty = pass).

def pin_golden_forward(fwd, bwd):
    g = _load("linear_fwd_hand.json")
    fails = []
    for dtype in ("fp16", "bf16"):
        X, W, b = _bits(g["X"], dtype), _bits(g["W"], dtype), _bits(g["bias"], dtype)
        for ep, ykey in (("BIAS", "Y_BIAS"), ("RELU_BIAS", "Y_RELU"), ("RELU_AUX_BIAS", "Y_RELU")):
            r = fwd(X, W, b, DT[dtype], ep)
            if not np.array_equal(r["Z"], np.array(g["Z"], dtype=float)):
                fails.append(f"golden fwd Z {dtype} {ep}")
            if not np.array_equal(r["S"], np.array(g["S"], dtype=float)):
                fails.append(f"golden fwd S {dtype} {ep}")
            if not np.array_equal(r["Y"], np.array(g[ykey], dtype=float)):
                fails.append(f"golden fwd Y {dtype} {ep}")
            if ep == "RELU_AUX_BIAS" and not np.array_equal(r["aux"], np.array(g["aux"], dtype=np.uint32)):
                fails.append(f"golden fwd aux {dtype}")
    return fails


def pin_golden_mask_layout(fwd, bwd):
    g = _load("relu_aux_layout_hand.json")
    N = g["N"]
    w = np.full((1, N), -1.0)
    w[0, g["positive"]] = 1.0
    w[0, g["zero"]] = 0.0
    fails = []
    for dtype in ("fp16", "bf16"):
        r = fwd(_bits([[1.0]], dtype), _bits(w, dtype), _bits(np.zeros(N), dtype), DT[dtype], "RELU_AUX_BIAS")
        if not np.array_equal(r["aux"], np.array(g["aux"], dtype=np.uint32)):
            fails.append(f"golden mask layout {dtype}: {r['aux']}")
    return fails


def pin_golden_backward(fwd, bwd):
    g = _load("drelu_bgrad_hand.json")
    fails = []
    for dtype in ("fp16", "bf16"):
        r = bwd(_bits(g["dY2"], dtype), _bits(g["W2"], dtype), np.array(g["aux"], dtype=np.uint32),
                DT[dtype], 3)
        for key in ("G", "S", "dZ", "dbias", "Sb"):
            if not np.array_equal(r[key], np.array(g[key], dtype=float)):
                fails.append(f"golden bwd {key} {dtype}: {r[key]}")
    return fails


def _exact_linear(Xf, Wf, bf):
    """Exact rational Z and S of small float matrices (brute force)."""
    T, K = len(Xf), len(Xf[0])
    N = len(Wf[0])
    Z = [[None] * N for _ in range(T)]
    S = [[None] * N for _ in range(T)]
    for t in range(T):
        for n in range(N):
            acc = Fraction(0)
            sc = Fraction(0)
            for k in range(K):
                p = Fraction(Xf[t][k]) * Fraction(Wf[k][n])
                acc += p
                sc += abs(p)
            if bf is not None:
                acc += Fraction(bf[n])
                sc += abs(Fraction(bf[n]))
            Z[t][n] = acc
            S[t][n] = sc
    return Z, S


def pin_bruteforce_rational(fwd, bwd):
    """Tiny random fp16/bf16 inputs: oracle within K * 2^-52 * S of the exact value."""
    fails = []
    shapes = [(1, 1, 1), (3, 5, 2), (5, 33, 7), (2, 17, 16), (4, 9, 33), (7, 40, 3)]
    for i, (T, N, K) in enumerate(shapes):
        for dtype in ("fp16", "bf16"):
            inp = synth.make_shape_inputs(T, N, K, dtype, seed=100 + i)
            X, W, b = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
            Xf = inp["X"].double().tolist()
            Wf = inp["W"].double().tolist()
            bf = inp["bias"].double().tolist()
            Zx, Sx = _exact_linear(Xf, Wf, bf)
            r = fwd(X, W, b, DT[dtype], "RELU_AUX_BIAS")
            for t in range(T):
                for n in range(N):
                    err = abs(Fraction(float(r["Z"][t, n])) - Zx[t][n])
                    bound = Fraction(K + 1) * Fraction(2) ** -52 * Sx[t][n]
                    if err > bound:
                        fails.append(f"bruteforce Z {dtype} {T}x{N}x{K} at {t},{n}")
                    if abs(Fraction(float(r["S"][t, n])) - Sx[t][n]) > bound:
                        fails.append(f"bruteforce S {dtype} {T}x{N}x{K} at {t},{n}")
                    if bool(r["bits"][t, n]) != (Zx[t][n] > 0):
                        fails.append(f"bruteforce bit {dtype} at {t},{n}")
            # backward: G = dY2 . W2 exactly, masked by bits from an independent source
            D2 = max(1, K - 1)
            inb = synth.make_shape_inputs(T, N, K, dtype, seed=200 + i, D2=D2)
            dY = inb["dY2"].double().tolist()
            W2 = inb["W2"].double().tolist()
            Gx, Gs = _exact_linear(dY, W2, None)
            rng = np.random.default_rng(7 + i)
            mask = rng.integers(0, 2, size=(T, N)).astype(bool)
            words = np.zeros((T, (N + 31) // 32), dtype=np.uint32)
            for t in range(T):
                for n in range(N):
                    if mask[t, n]:
                        words[t, n // 32] |= np.uint32(1 << (n % 32))
            rb = bwd(synth.bits_u16(inb["dY2"]), synth.bits_u16(inb["W2"]), words, DT[dtype], N)
            for n in range(N):
                col = Fraction(0)
                for t in range(T):
                    dz = Gx[t][n] if mask[t, n] else Fraction(0)
                    col += dz
                    bound = Fraction(D2 + 1) * Fraction(2) ** -52 * Gs[t][n]
                    if abs(Fraction(float(rb["dZ"][t, n])) - dz) > bound:
                        fails.append(f"bruteforce dZ {dtype} at {t},{n}")
                sb = sum((abs(Gx[t][n]) if mask[t, n] else 0) for t in range(T))
                bound = Fraction(2) ** -40 * (sb + sum(Gs[t][n] for t in range(T)))
                if abs(Fraction(float(rb["dbias"][n])) - col) > bound:
                    fails.append(f"bruteforce dbias {dtype} at {n}")
    return fails


def pin_integer_exact(fwd, bwd):
    """Integer inputs in [-3, 3]: Z, G, dZ, dbias equal exact int64 arithmetic."""
    fails = []
    for i, (T, N, K, D2) in enumerate([(17, 40, 24, 9), (33, 65, 16, 31), (8, 8, 8, 8), (1, 96, 64, 64)]):
        for dtype in ("fp16", "bf16"):
            inp = synth.make_shape_inputs(T, N, K, dtype, seed=300 + i, D2=D2, kind="int")
            Xi, Wi, bi = (inp[k].to(torch.int64).numpy() for k in ("X", "W", "bias"))
            Zi = Xi @ Wi + bi[None, :]
            Si = np.abs(Xi[:, :, None] * Wi[None, :, :]).sum(axis=1) + np.abs(bi)[None, :]
            r = fwd(*(synth.bits_u16(inp[k]) for k in ("X", "W", "bias")), DT[dtype], "RELU_AUX_BIAS")
            if not np.array_equal(r["Z"], Zi.astype(float)):
                fails.append(f"int Z {dtype} {T}x{N}x{K}")
            if not np.array_equal(r["S"], Si.astype(float)):
                fails.append(f"int S {dtype}")
            if not np.array_equal(r["Y"], np.maximum(Zi, 0).astype(float)):
                fails.append(f"int Y {dtype}")
            expect_words = np.zeros((T, (N + 31) // 32), dtype=np.uint64)
            for t in range(T):
                for n in range(N):
                    if Zi[t, n] > 0:
                        expect_words[t, n // 32] += 1 << (n % 32)
            if not np.array_equal(r["aux"], expect_words.astype(np.uint32)):
                fails.append(f"int aux {dtype}")
            dYi, W2i = inp["dY2"].to(torch.int64).numpy(), inp["W2"].to(torch.int64).numpy()
            Gi = dYi @ W2i
            dZi = np.where(Zi > 0, Gi, 0)
            rb = bwd(synth.bits_u16(inp["dY2"]), synth.bits_u16(inp["W2"]), r["aux"], DT[dtype], N)
            if not np.array_equal(rb["G"], Gi.astype(float)):
                fails.append(f"int G {dtype}")
            if not np.array_equal(rb["dZ"], dZi.astype(float)):
                fails.append(f"int dZ {dtype}")
            if not np.array_equal(rb["dbias"], dZi.sum(axis=0).astype(float)):
                fails.append(f"int dbias {dtype}")
    return fails


def pin_library_matmul(fwd, bwd):
    """Zero bias: Z equals torch.matmul in float64; S equals |X| @ |W|."""
    fails = []
    for i, (T, N, K) in enumerate([(37, 72, 130), (64, 40, 257)]):
        for dtype in ("fp16", "bf16"):
            inp = synth.make_shape_inputs(T, N, K, dtype, seed=400 + i)
            zero_b = torch.zeros(N, dtype=synth.DTYPES[dtype])
            r = fwd(synth.bits_u16(inp["X"]), synth.bits_u16(inp["W"]), synth.bits_u16(zero_b), DT[dtype], "BIAS")
            x, w = inp["X"].double(), inp["W"].double()
            ref = (x @ w).numpy()
            sref = (x.abs() @ w.abs()).numpy()
            if np.max(np.abs(r["Z"] - ref) / sref) > 1e-12:
                fails.append(f"library Z {dtype}")
            if np.max(np.abs(r["S"] - sref) / sref) > 1e-12:
                fails.append(f"library S {dtype}")
            rr = fwd(synth.bits_u16(inp["X"]), synth.bits_u16(inp["W"]), synth.bits_u16(zero_b), DT[dtype], "RELU_BIAS")
            if np.max(np.abs(rr["Y"] - np.maximum(ref, 0)) / sref) > 1e-12:
                fails.append(f"library relu {dtype}")
    return fails


def pin_identity_closed_form(fwd, bwd):
    """X = I (T = K): Z = W + b exactly, per element."""
    fails = []
    T = N = 24
    for dtype in ("fp16", "bf16"):
        inp = synth.make_shape_inputs(T, N, T, dtype, seed=500)
        eye = torch.eye(T, dtype=synth.DTYPES[dtype])
        r = fwd(synth.bits_u16(eye), synth.bits_u16(inp["W"]), synth.bits_u16(inp["bias"]), DT[dtype], "RELU_BIAS")
        exact = inp["W"].double().numpy() + inp["bias"].double().numpy()[None, :]
        if not np.array_equal(r["Z"], exact):
            fails.append(f"identity Z {dtype}")
        if not np.array_equal(r["Y"], np.maximum(exact, 0)):
            fails.append(f"identity Y {dtype}")
    return fails


def pin_backward_library(fwd, bwd):
    """G equals torch.matmul in float64; dbias equals ones^T . dZ; mask bits select G."""
    fails = []
    T, N, D2 = 45, 72, 100
    for dtype in ("fp16", "bf16"):
        inp = synth.make_shape_inputs(T, N, 64, dtype, seed=600, D2=D2)
        fw = fwd(*(synth.bits_u16(inp[k]) for k in ("X", "W", "bias")), DT[dtype], "RELU_AUX_BIAS")
        rb = bwd(synth.bits_u16(inp["dY2"]), synth.bits_u16(inp["W2"]), fw["aux"], DT[dtype], N)
        Gref = (inp["dY2"].double() @ inp["W2"].double()).numpy()
        Sref = (inp["dY2"].double().abs() @ inp["W2"].double().abs()).numpy()
        if np.max(np.abs(rb["G"] - Gref) / Sref) > 1e-12:
            fails.append(f"bwd G {dtype}")
        mask = fw["Z"] > 0
        if not np.array_equal(rb["dZ"][~mask], np.zeros(int((~mask).sum()))):
            fails.append(f"bwd dZ off-mask {dtype}")
        if np.max(np.abs(rb["dZ"][mask] - Gref[mask]) / Sref[mask]) > 1e-12:
            fails.append(f"bwd dZ on-mask {dtype}")
        ones = torch.ones(1, T, dtype=torch.float64)
        dref = (ones @ torch.from_numpy(np.where(mask, Gref, 0.0))).numpy()[0]
        if np.max(np.abs(rb["dbias"] - dref) / (rb["Sb"] + 1e-300)) > 1e-12:
            fails.append(f"bwd dbias {dtype}")
    return fails


PINS = [pin_golden_forward, pin_golden_mask_layout, pin_golden_backward, pin_bruteforce_rational,
        pin_integer_exact, pin_library_matmul, pin_identity_closed_form, pin_backward_library]


def _real(oracle_mod):
    return oracle_mod.linear_fwd, (lambda dY2, W2, aux, dt, N, **kw: oracle_mod.drelu_bgrad(dY2, W2, aux, dt, N, **kw))


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle_mod, pin):
    fwd, bwd = _real(oracle_mod)
    fails = pin(fwd, bwd)
    assert not fails, fails[:10]


# --------------------------------------------------------- planted mistakes

def _mutants(oracle_mod):
    o = oracle_mod

    def fwd_bias_per_row(X, W, b, dt, ep, **kw):
        r = o.linear_fwd(X, W, None if False else b, dt, ep, **kw)
        T = r["Z"].shape[0]
        bvals = o.decode(b, dt)
        Z = r["Z"] - bvals[None, :] + bvals[np.arange(T) % len(bvals)][:, None]
        return _refinish(o, Z, r["S"], ep)

    def fwd_transposed_w(X, W, b, dt, ep, **kw):
        if W.shape[0] != W.shape[1]:
            return o.linear_fwd(X, W, b, dt, ep, **kw)
        return o.linear_fwd(X, np.ascontiguousarray(W.T), b, dt, ep, **kw)

    def fwd_dropped_bias(X, W, b, dt, ep, **kw):
        return o.linear_fwd(X, W, np.zeros_like(b), dt, ep, **kw)

    def fwd_tie_inclusive(X, W, b, dt, ep, **kw):
        r = o.linear_fwd(X, W, b, dt, ep, **kw)
        if "bits" in r:
            r["bits"] = r["Z"] >= 0
            r["aux"] = o.relu_aux_words(r["bits"])
        return r

    def fwd_inverted_polarity(X, W, b, dt, ep, **kw):
        r = o.linear_fwd(X, W, b, dt, ep, **kw)
        if "bits" in r:
            r["bits"] = r["Z"] < 0
            r["aux"] = o.relu_aux_words(r["bits"])
        return r

    def fwd_msb_first(X, W, b, dt, ep, **kw):
        r = o.linear_fwd(X, W, b, dt, ep, **kw)
        if "aux" in r:
            rev = np.zeros_like(r["aux"])
            for j in range(32):
                rev |= ((r["aux"] >> np.uint32(j)) & np.uint32(1)) << np.uint32(31 - j)
            r["aux"] = rev
        return r

    def fwd_sign_flip_product(X, W, b, dt, ep, **kw):
        r = o.linear_fwd(X, W, b, dt, ep, **kw)
        bvals = o.decode(b, dt)
        Z = -(r["Z"] - bvals[None, :]) + bvals[None, :]
        return _refinish(o, Z, r["S"], ep)

    real_bwd = lambda dY2, W2, aux, dt, N, **kw: o.drelu_bgrad(dY2, W2, aux, dt, N, **kw)

    def bwd_dbias_over_cols(dY2, W2, aux, dt, N, **kw):
        r = o.drelu_bgrad(dY2, W2, aux, dt, N, **kw)
        if "dbias" in r:
            s = r["dZ"].sum(axis=1)
            r["dbias"] = np.resize(s, r["dbias"].shape)
        return r

    def bwd_mask_ignored(dY2, W2, aux, dt, N, **kw):
        r = o.drelu_bgrad(dY2, W2, aux, dt, N, **kw)
        r["dZ"] = r["G"].copy()
        r["dbias"] = r["dZ"].sum(axis=0)
        r["Sb"] = np.abs(r["dZ"]).sum(axis=0)
        return r

    def bwd_w2_transposed(dY2, W2, aux, dt, N, **kw):
        if W2.shape[0] != W2.shape[1]:
            return o.drelu_bgrad(dY2, W2, aux, dt, N, **kw)
        return o.drelu_bgrad(dY2, np.ascontiguousarray(W2.T), aux, dt, N, **kw)

    def bwd_dropped_last_term(dY2, W2, aux, dt, N, **kw):
        W2z = W2.copy()
        W2z[-1, :] = 0
        return o.drelu_bgrad(dY2, W2z, aux, dt, N, **kw)

    fwd = o.linear_fwd
    return {
        "bias per row": (fwd_bias_per_row, real_bwd),
        "W transposed": (fwd_transposed_w, real_bwd),
        "bias dropped": (fwd_dropped_bias, real_bwd),
        "tie Z==0 sets bit": (fwd_tie_inclusive, real_bwd),
        "mask polarity inverted": (fwd_inverted_polarity, real_bwd),
        "mask MSB first": (fwd_msb_first, real_bwd),
        "product sign flipped": (fwd_sign_flip_product, real_bwd),
        "dbias summed over columns": (fwd, bwd_dbias_over_cols),
        "mask ignored in backward": (fwd, bwd_mask_ignored),
        "W2 transposed": (fwd, bwd_w2_transposed),
        "last contraction term dropped": (fwd, bwd_dropped_last_term),
    }


def _refinish(o, Z, S, ep):
    out = {"Z": Z, "S": S, "Y": Z.copy() if ep == "BIAS" else np.maximum(Z, 0.0)}
    if ep == "RELU_AUX_BIAS":
        out["bits"] = Z > 0
        out["aux"] = o.relu_aux_words(out["bits"])
    return out


def test_planted_mistakes_are_caught(oracle_mod):
    caught = {}
    for name, (fwd, bwd) in _mutants(oracle_mod).items():
        n_fail = 0
        for pin in PINS:
            try:
                n_fail += len(pin(fwd, bwd))
            except Exception:  # a crash also counts as caught
                n_fail += 1
        caught[name] = n_fail
    missed = [k for k, v in caught.items() if v == 0]
    assert not missed, f"pins did not catch: {missed}"


# ------------------------------------------------------------ misc behaviour

def test_row_col_subsets_match_full(oracle_mod):
    inp = synth.make_shape_inputs(40, 70, 33, "bf16", seed=700)
    X, W, b = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
    full = oracle_mod.linear_fwd(X, W, b, 1, "RELU_AUX_BIAS")
    rows, cols = [0, 7, 39], [1, 32, 69]
    part = oracle_mod.linear_fwd(X, W, b, 1, "RELU_AUX_BIAS", rows=rows, cols=cols)
    assert np.array_equal(part["Z"], full["Z"][np.ix_(rows, cols)])
    assert np.array_equal(part["S"], full["S"][np.ix_(rows, cols)])
    single = oracle_mod.linear_fwd(X, W, b, 1, "RELU_AUX_BIAS", threads=1)
    assert np.array_equal(single["Z"], full["Z"])


def test_bad_arguments_rejected(oracle_mod):
    X = np.zeros((2, 3), np.uint16)
    W = np.zeros((3, 4), np.uint16)
    with pytest.raises(ValueError):
        oracle_mod.matmul_bias(X, np.zeros((2, 4), np.uint16), None, 0)
    with pytest.raises(ValueError):
        oracle_mod.matmul_bias(X, W, None, 0, rows=[5])
    with pytest.raises(ValueError):
        oracle_mod.matmul_bias(X, W, None, 0, cols=[-1])
    with pytest.raises(ValueError):
        oracle_mod.matmul_bias(X, W, None, 7)
    C, S = oracle_mod.matmul_bias(X, W, None, 0, rows=[])
    assert C.shape == (0, 4)


def test_mask_pack_roundtrip(oracle_mod):
    rng = np.random.default_rng(1)
    for N in (1, 31, 32, 33, 64, 100):
        bits = rng.integers(0, 2, size=(5, N)).astype(bool)
        words = oracle_mod.relu_aux_words(bits)
        assert words.shape == (5, math.ceil(N / 32))
        assert np.array_equal(oracle_mod.relu_aux_bits(words, N), bits)
        # pad bits past N are zero
        tail = N % 32
        if tail:
            assert np.all(words[:, -1] >> np.uint32(tail) == 0)


# ---------------------------------------------------------------- GELU_BIAS
# Standard normal CDF values from a printed normal table (closed-form
# constants, not computed by the oracle's own erf); GELU(x) = x * Phi(x).
PHI_TABLE = {0.5: 0.6914624612740131, 1.0: 0.8413447460685429, 1.5: 0.9331927987311419,
             2.0: 0.9772498680518208, 3.0: 0.9986501019683699, -1.0: 0.15865525393145707}


def pin_gelu(gelu, fwd):
    fails = []
    for x, phi in PHI_TABLE.items():
        if abs(gelu(np.array([x]))[0] - x * phi) > 1e-13 * abs(x):
            fails.append(f"table {x}")
    xs = np.array([0.25, 0.7, 1.3, 2.6, 4.0])
    if np.max(np.abs(gelu(xs) - gelu(-xs) - xs)) > 1e-14:  # z*Phi(z) - (-z)*Phi(-z) = z
        fails.append("odd part")
    if gelu(np.array([0.0]))[0] != 0.0 or abs(gelu(np.array([12.0]))[0] - 12.0) > 1e-12 \
            or not (-1e-20 <= gelu(np.array([-12.0]))[0] <= 0.0):
        fails.append("limits")
    # through the forward epilog: X a column of exact fp16 values, W = [[1]], bias 0; then bias 1 on x = 1
    col = [0.5, 1.0, 2.0, -1.0, 3.0]
    r = fwd(_bits([[v] for v in col], "fp16"), _bits([[1.0]], "fp16"), _bits([0.0], "fp16"), 0, "GELU_BIAS")
    want = np.array([[v * PHI_TABLE[v]] for v in col])
    if np.max(np.abs(r["Y"] - want)) > 1e-13:
        fails.append("epilog")
    r = fwd(_bits([[1.0]], "bf16"), _bits([[1.0]], "bf16"), _bits([1.0], "bf16"), 1, "GELU_BIAS")
    if abs(r["Y"][0, 0] - 2.0 * PHI_TABLE[2.0]) > 1e-13 or r["Z"][0, 0] != 2.0:
        fails.append("epilog with bias")
    return fails


def test_gelu_pins(oracle_mod):
    fails = pin_gelu(oracle_mod.gelu, oracle_mod.linear_fwd)
    assert not fails, fails


def test_gelu_planted_mistakes_are_caught(oracle_mod):
    o = oracle_mod
    mutants = {
        "tanh approximation": lambda z: 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3))),
        "erf without 1/sqrt2": lambda z: 0.5 * z * (1 + np.vectorize(math.erf)(z)),
        "no one half": lambda z: z * (1 + np.vectorize(math.erf)(z / math.sqrt(2))),
        "sign of erf": lambda z: 0.5 * z * (1 - np.vectorize(math.erf)(z / math.sqrt(2))),
    }
    for name, g in mutants.items():
        def fwd(X, W, b, dt, ep, g=g, **kw):
            r = o.linear_fwd(X, W, b, dt, "BIAS", **kw)
            r["Y"] = g(r["Z"])
            return r
        assert pin_gelu(g, fwd), f"pins did not catch: {name}"


def test_gelu_epilog_is_bias_then_gelu(oracle_mod):
    inp = synth.make_shape_inputs(9, 24, 40, "bf16", seed=41)
    X, W, b = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
    rb = oracle_mod.linear_fwd(X, W, b, 1, "BIAS")
    rg = oracle_mod.linear_fwd(X, W, b, 1, "GELU_BIAS")
    assert np.array_equal(rg["Z"], rb["Z"]) and np.array_equal(rg["S"], rb["S"])
    z = rb["Z"]
    assert np.max(np.abs(rg["Y"] - z * 0.5 * (1 + np.vectorize(math.erf)(z / math.sqrt(2))))) < 1e-15


# ------------------------------------------------------------ GELU_AUX_BIAS
def pin_gelu_aux(fwd, gelu):
    """GELU_AUX_BIAS's auxiliary output is the pre-activation Z = X.W + bias and
    Y = gelu(Z). Pinned to the hand-worked forward example (Z worked out by
    hand there), to the X = I closed form (Z = W + bias), and to GELU's own
    pins through ``gelu``."""
    fails = []
    g = _load("linear_fwd_hand.json")
    for dt in ("fp16", "bf16"):
        r = fwd(_bits(g["X"], dt), _bits(g["W"], dt), _bits(g["bias"], dt), DT[dt], "GELU_AUX_BIAS")
        if not np.array_equal(r["pre"], np.array(g["Z"], dtype=np.float64)):
            fails.append(f"hand-worked Z ({dt})")
        if np.max(np.abs(r["Y"] - gelu(np.array(g["Z"], dtype=np.float64)))) > 0.0:
            fails.append(f"hand-worked Y ({dt})")
    rng = np.random.default_rng(3)
    n = 6
    Wv = (rng.integers(-64, 64, size=(n, 10)) / 16.0)
    bv = (rng.integers(-64, 64, size=10) / 32.0)
    r = fwd(_bits(np.eye(n).tolist(), "bf16"), _bits(Wv.tolist(), "bf16"), _bits(bv.tolist(), "bf16"), 1,
            "GELU_AUX_BIAS")
    if not np.array_equal(r["pre"], Wv + bv[None, :]):
        fails.append("closed form X = I")
    return fails


def test_gelu_aux_pins(oracle_mod):
    fails = pin_gelu_aux(oracle_mod.linear_fwd, oracle_mod.gelu)
    assert not fails, fails


def test_gelu_aux_planted_mistakes_are_caught(oracle_mod):
    o = oracle_mod

    def mutant(change):
        def fwd(X, W, b, dt, ep, **kw):
            r = o.linear_fwd(X, W, b, dt, "GELU_AUX_BIAS", **kw)
            change(r, X, W, b, dt)
            return r
        return fwd

    def no_bias(r, X, W, b, dt):
        r["pre"] = o.linear_fwd(X, W, None, dt, "NONE")["Y"]

    mutants = {
        "aux holds gelu(Z)": lambda r, *a: r.__setitem__("pre", o.gelu(r["Z"])),
        "aux holds X.W without the bias": no_bias,
        "aux holds relu(Z)": lambda r, *a: r.__setitem__("pre", np.maximum(r["Z"], 0.0)),
        "Y is relu(Z)": lambda r, *a: r.__setitem__("Y", np.maximum(r["Z"], 0.0)),
        "aux transposed": lambda r, *a: r.__setitem__("pre", r["Z"].T.copy() if r["Z"].shape[0] == r["Z"].shape[1]
                                                        else r["Z"][::-1].copy()),
    }
    for name, change in mutants.items():
        assert pin_gelu_aux(mutant(change), o.gelu), f"pins did not catch: {name}"


def test_gelu_aux_is_gelu_bias_plus_its_pre_activation(oracle_mod):
    inp = synth.make_shape_inputs(9, 24, 40, "bf16", seed=43)
    X, W, b = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
    rg = oracle_mod.linear_fwd(X, W, b, 1, "GELU_BIAS")
    ra = oracle_mod.linear_fwd(X, W, b, 1, "GELU_AUX_BIAS")
    assert np.array_equal(ra["Y"], rg["Y"]) and np.array_equal(ra["pre"], rg["Z"]) and "pre" not in rg


# ------------------------------------------------------------------ WGRAD
def pin_wgrad(wg):
    fails = []
    # worked by hand: X (T=3 x K=2), dZ (T=3 x N=3)
    #   dW[0] = 1*[1,0,2] + 3*[0,1,0] + 5*[1,1,1] = [6, 8, 7]
    #   dW[1] = 2*[1,0,2] + 4*[0,1,0] + 6*[1,1,1] = [8, 10, 10]
    X = _bits([[1, 2], [3, 4], [5, 6]], "fp16")
    dZ = _bits([[1, 0, 2], [0, 1, 0], [1, 1, 1]], "fp16")
    r = wg(X, dZ, 0)
    if not np.array_equal(r["dW"], np.array([[6.0, 8.0, 7.0], [8.0, 10.0, 10.0]])):
        fails.append("hand-worked")
    if not np.array_equal(r["dbias"], np.array([9.0, 12.0])):  # 1+3+5, 2+4+6
        fails.append("hand-worked column sums")
    # closed form: X = 1, dZ = 2 -> dW = 2T everywhere; S = 2T
    T = 37
    r = wg(_bits(np.ones((T, 5)).tolist(), "bf16"), _bits((2 * np.ones((T, 9))).tolist(), "bf16"), 1)
    if not (np.all(r["dW"] == 2.0 * T) and np.all(r["S"] == 2.0 * T) and r["dW"].shape == (5, 9)):
        fails.append("closed form")
    # brute force in exact rationals on a random tiny case
    rng = np.random.default_rng(5)
    Xv = (rng.integers(-40, 40, size=(6, 3)) / 8.0).tolist()
    Dv = (rng.integers(-40, 40, size=(6, 4)) / 16.0).tolist()
    r = wg(_bits(Xv, "fp16"), _bits(Dv, "fp16"), 0)
    for k in range(3):
        for n in range(4):
            exact = sum(Fraction(Xv[t][k]) * Fraction(Dv[t][n]) for t in range(6))
            if Fraction(r["dW"][k, n]) != exact:
                fails.append(f"rational {k},{n}")
    return fails


def test_wgrad_pins(oracle_mod):
    fails = pin_wgrad(oracle_mod.wgrad)
    assert not fails, fails


def test_wgrad_planted_mistakes_are_caught(oracle_mod):
    o = oracle_mod

    def no_transpose_rows_flipped(X, dZ, dt, **kw):  # pairs X row t with dZ row T-1-t
        return o.wgrad(np.ascontiguousarray(np.asarray(X)[::-1]), dZ, dt, **kw)

    def last_row_dropped(X, dZ, dt, **kw):
        return o.wgrad(np.asarray(X)[:-1], np.asarray(dZ)[:-1], dt, **kw)

    def sign(X, dZ, dt, **kw):
        r = o.wgrad(X, dZ, dt, **kw)
        return dict(r, dW=-r["dW"])

    def dz_transposed_product(X, dZ, dt, **kw):  # (dZ^T X)^T computed with X and dZ swapped roles
        r = o.wgrad(dZ, X, dt, **kw)
        ref = o.wgrad(X, dZ, dt, **kw)
        return dict(ref, dW=r["dW"].T.copy(), S=r["S"].T.copy())

    for name, m in {"rows flipped": no_transpose_rows_flipped, "last row dropped": last_row_dropped,
                    "sign": sign}.items():
        assert pin_wgrad(m), f"pins did not catch: {name}"
    # the swapped-role product is the same matrix (a correct identity), so the pins must pass it
    assert not pin_wgrad(dz_transposed_product)


def test_wgrad_subsets_match_full(oracle_mod):
    inp = synth.make_shape_inputs(33, 40, 24, "bf16", seed=8, D2=40)
    X, dZ = synth.bits_u16(inp["X"]), synth.bits_u16(inp["dY2"])
    full = oracle_mod.wgrad(X, dZ, 1)
    part = oracle_mod.wgrad(X, dZ, 1, rows=[0, 5, 23], cols=[1, 39])
    assert np.array_equal(part["dW"], full["dW"][np.ix_([0, 5, 23], [1, 39])])
    assert np.array_equal(part["dbias"], full["dbias"][[0, 5, 23]])
    with pytest.raises(ValueError):
        oracle_mod.wgrad(X, dZ[:-1], 1)


# ------------------------------------------------------------- fp32 bias
def test_fp32_bias_equal_to_16bit_bias_gives_the_same_result(oracle_mod):
    inp = synth.make_shape_inputs(7, 40, 24, "fp16", seed=12)
    X, W, b16 = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
    b32 = inp["bias"].float().numpy()  # the same values, held as fp32
    for ep in ("BIAS", "RELU_AUX_BIAS", "GELU_BIAS"):
        r16 = oracle_mod.linear_fwd(X, W, b16, 0, ep)
        r32 = oracle_mod.linear_fwd(X, W, b32, 0, ep)
        for key in ("Z", "S", "Y"):
            assert np.array_equal(r16[key], r32[key]), (ep, key)
    part = oracle_mod.linear_fwd(X, W, b32, 0, "BIAS", cols=[3, 39])
    assert np.array_equal(part["Z"], oracle_mod.linear_fwd(X, W, b32, 0, "BIAS")["Z"][:, [3, 39]])


def test_fp32_bias_values_are_taken_exactly(oracle_mod):
    # X = 0: Z is the fp32 bias itself (values no 16-bit type holds), S = |bias|
    b32 = np.array([0.1, -1e-3, 3.14159274, 65519.0, -7.0e-8, 0.0, 1.0, 2.5], dtype=np.float32)
    X = _bits(np.zeros((3, 16)).tolist(), "bf16")
    W = _bits(np.ones((16, 8)).tolist(), "bf16")
    r = oracle_mod.linear_fwd(X, W, b32, 1, "RELU_BIAS")
    assert np.array_equal(r["Z"], np.tile(b32.astype(np.float64), (3, 1)))
    assert np.array_equal(r["S"], np.tile(np.abs(b32.astype(np.float64)), (3, 1)))
    assert np.array_equal(r["Y"], np.maximum(r["Z"], 0.0))
    with pytest.raises(ValueError):
        oracle_mod.linear_fwd(X, W, b32[:5], 1, "BIAS")


# ------------------------------------------------------- NONE and the FFN step
def test_none_epilog_is_the_plain_product(oracle_mod):
    inp = synth.make_shape_inputs(6, 16, 24, "bf16", seed=44)
    X, W, b = (synth.bits_u16(inp[k]) for k in ("X", "W", "bias"))
    r = oracle_mod.linear_fwd(X, W, b, 1, "NONE")   # the bias is not used
    zero = _bits([0.0] * 16, "bf16")
    rz = oracle_mod.linear_fwd(X, W, zero, 1, "BIAS")
    assert np.array_equal(r["Y"], rz["Y"]) and np.array_equal(r["S"], rz["S"])


def test_encode_exact(oracle_mod):
    v = np.array([0.0, -3.0, 256.0, 0.5, -65504.0])
    assert np.array_equal(oracle_mod.decode(oracle_mod.encode_exact(v, 0), 0), v)
    assert np.array_equal(oracle_mod.decode(oracle_mod.encode_exact(v[:4], 1), 1), v[:4])
    with pytest.raises(ValueError):
        oracle_mod.encode_exact(np.array([257.0]), 1)   # bf16 holds 8 significant bits
    with pytest.raises(ValueError):
        oracle_mod.encode_exact(np.array([2049.0]), 0)  # fp16 holds 11


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_ffn_step_matches_float64_autograd(oracle_mod, dtype):
    """The chained step against torch's float64 autograd of the same block
    (exact on integer inputs): pins every transpose and orientation."""
    T, D, F = 12, 16, 24
    inp = synth.ffn_step_inputs(T, D, F, dtype, seed=3, kind="int")
    bits = {k: synth.bits_u16(v) for k, v in inp.items()}
    dt = DT[dtype]
    r = oracle_mod.ffn_step(bits["X"], bits["W1"], bits["b1"], bits["W2"], bits["b2"], bits["dY"], dt)
    t = {k: v.double().requires_grad_(k != "dY") for k, v in inp.items()}
    h = torch.relu(t["X"] @ t["W1"].T + t["b1"])
    y = h @ t["W2"].T + t["b2"]
    y.backward(t["dY"])
    assert np.array_equal(r["H"], h.detach().numpy()) and np.array_equal(r["Y"], y.detach().numpy())
    for ours, theirs in (("dX", "X"), ("dW1", "W1"), ("db1", "b1"), ("dW2", "W2"), ("db2", "b2")):
        assert np.array_equal(r[ours], t[theirs].grad.numpy()), ours
    assert np.array_equal(r["bits"], h.detach().numpy() > 0)


def test_ffn_step_refuses_inexact_intermediates(oracle_mod):
    T, D, F = 4, 8, 8
    inp = synth.ffn_step_inputs(T, D, F, "bf16", seed=1, kind="normal")
    bits = {k: synth.bits_u16(v) for k, v in inp.items()}
    with pytest.raises(ValueError):
        oracle_mod.ffn_step(bits["X"], bits["W1"], bits["b1"], bits["W2"], bits["b2"], bits["dY"], 1)
