"""Pins for the CPU oracle: what the pages and the mathematics fix, checked
against the oracle without trusting it.

* the IEEE binary16 format (exhaustive decode, correctly rounded encode);
* a hand-derived worked example (``tests/golden/worked_example_2x4x3.json``);
* an independent brute force in exact rational arithmetic on tiny matrices;
* closed forms and invariants: +-absmax -> +-127, threshold = inf reduces to
  the pure vector-wise product, integer inputs quantise losslessly, all-outlier
  inputs reduce to the fp16 matmul, the per-element quantisation error is at
  most absmax/254, and the result stays within the method's error bound of the
  exact product.

Method: "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale",
abstract (vector-wise quantisation + mixed-precision decomposition); axolotl
"llama3-model-quantization", "Understanding Outliers in Transformer Models"
(outliers are feature columns) and "Key Points" (max normalisation); scite
report for nuQmm (round to nearest).
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int8_quantized_matmul_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# exact IEEE rounding, written from the format definition (independent of C)
# --------------------------------------------------------------------------

def _round_format(q: Fraction, frac_bits: int, emin: int, emax: int) -> float:
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - frac_bits)
    n = round(a / ulp)  # Fraction.__round__ is round-half-even
    r = n * ulp
    max_finite = (2 - Fraction(2) ** (-frac_bits)) * Fraction(2) ** emax
    if r > max_finite:
        return sign * math.inf
    return sign * float(r)


def rn32(q) -> Fraction:
    return Fraction(_round_format(Fraction(q), 23, -126, 127))


def rn16(q) -> float:
    return _round_format(Fraction(q), 10, -14, 15)


# --------------------------------------------------------------------------
# literal brute force of the method on tiny inputs, in exact rationals
# --------------------------------------------------------------------------

def brute_force(X: np.ndarray, W: np.ndarray, thr: float, keep):
    M, K = X.shape
    N = W.shape[1]
    xs = [[Fraction(float(v)) for v in row] for row in X.astype(np.float64)]
    ws = [[Fraction(float(v)) for v in row] for row in W.astype(np.float64)]
    outl = [k for k in range(K) if any(abs(xs[m][k]) >= thr for m in range(M))]
    oset = set(outl)

    def quant(vals):
        amax = max((abs(v) for v in vals), default=Fraction(0))
        if amax == 0:
            return [0] * len(vals), amax
        s = rn32(Fraction(127) / amax)
        return [max(-127, min(127, round(rn32(v * s)))) for v in vals], amax

    xq, ra = [], []
    for m in range(M):
        inl = [xs[m][k] for k in range(K) if k not in oset]
        amax = max((abs(v) for v in inl), default=Fraction(0))
        if amax == 0:
            q = [0] * K
        else:
            s = rn32(Fraction(127) / amax)
            q = [0 if k in oset else max(-127, min(127, round(rn32(xs[m][k] * s)))) for k in range(K)]
        xq.append(q)
        ra.append(amax)
    wq, ca = [], []
    for n in range(N):
        q, amax = quant([ws[k][n] for k in range(K)])
        wq.append(q)
        ca.append(amax)
    acc = [[sum(xq[m][k] * wq[n][k] for k in range(K)) for n in range(N)] for m in range(M)]
    wo = []
    for k in outl:
        if k in keep:
            wo.append([ws[k][n] for n in range(N)])
        else:
            wo.append([Fraction(rn16(rn32(rn32(Fraction(wq[n][k]) * ca[n]) / 127))) for n in range(N)])
    y = []
    for m in range(M):
        row = []
        for n in range(N):
            o = Fraction(0)
            for j, k in enumerate(outl):
                o = rn32(o + rn32(xs[m][k] * wo[j][n]))
            v = rn32(acc[m][n])
            v = rn32(v * ra[m])
            v = rn32(v * ca[n])
            v = rn32(v / 16129)
            v = rn32(v + o)
            row.append(rn16(v))
        y.append(row)
    return {
        "idx": outl, "xq": xq, "ra": [float(v) for v in ra], "wq": wq, "ca": [float(v) for v in ca],
        "acc": acc, "y": y,
    }


# --------------------------------------------------------------------------
# the fp16 format
# --------------------------------------------------------------------------

def test_half_to_float_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_round_half_even():
    rng = np.random.default_rng(1)
    vals = [0.0, -0.0, 1.0, 65504.0, 65519.996, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 6e-8, float("inf"), float("-inf")]
    # exact midpoints between neighbouring fp16 values: ties must go to the even code
    h = np.arange(0x0001, 0x7bff, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    h_next = (np.arange(0x0001, 0x7bff, 7, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    vals += list(((h + h_next) / 2).astype(np.float32))
    vals += list(rng.standard_normal(3000).astype(np.float32) * np.float32(100.0))
    vals += list((rng.standard_normal(2000) * 1e-5).astype(np.float32))
    for v in vals:
        v32 = np.float32(v)
        with np.errstate(over="ignore"):
            want = int(np.array(v32, dtype=np.float32).astype(np.float16).view(np.uint16))
        assert oracle.float_to_half(float(v32)) == want, (float(v32), hex(want))
        # and the independent rational rounding agrees on finite values
        if np.isfinite(v32):
            r = rn16(Fraction(float(v32)))
            assert np.float16(r).view(np.uint16) == want or (r == 0 and (want & 0x7FFF) == 0)


# --------------------------------------------------------------------------
# the hand-derived worked example
# --------------------------------------------------------------------------

def test_worked_example_golden():
    with open(os.path.join(GOLDEN, "worked_example_2x4x3.json")) as f:
        g = json.load(f)
    X = np.array(g["X"], dtype=np.float16)
    W = np.array(g["W"], dtype=np.float16)
    prep = oracle.prepare_weight(W, g["keep_idx"])
    r = oracle.forward(X, prep, g["threshold"], threads=1)
    e = g["expected"]
    assert r["idx"].tolist() == e["outlier_idx"]
    assert r["ra"].tolist() == e["row_absmax"]
    assert r["xq"].tolist() == e["xq"]
    assert prep["ca"].tolist() == e["col_absmax"]
    assert prep["wq"].tolist() == e["wq"]
    assert r["acc"].tolist() == e["acc"]
    assert r["xo"].astype(np.float64).tolist() == e["xo"]
    assert r["o"].astype(np.float64).tolist() == e["o"]
    assert r["y"].astype(np.float64).tolist() == e["y"]
    # the brute force reproduces the same hand-derived values
    bf = brute_force(X, W, g["threshold"], set(g["keep_idx"]))
    assert bf["acc"] == e["acc"] and bf["y"] == e["y"] and bf["xq"] == e["xq"]


# --------------------------------------------------------------------------
# brute force on tiny matrices
# --------------------------------------------------------------------------

def _tiny_case(seed):
    rng = np.random.default_rng(seed)
    M, K, N = (int(v) for v in rng.integers(1, 9, size=3))
    X = (rng.standard_normal((M, K)) * rng.choice([0.5, 2.0, 4.0])).astype(np.float16)
    # plant outlier columns and special rows / columns
    for k in rng.choice(K, size=int(rng.integers(0, K + 1)), replace=False)[: max(0, K // 3)]:
        X[int(rng.integers(0, M)), k] = np.float16(rng.choice([-1, 1]) * rng.uniform(6, 60))
    if rng.random() < 0.2:
        X[int(rng.integers(0, M)), :] = 0
    W = (rng.standard_normal((K, N)) * 0.05).astype(np.float16)
    if rng.random() < 0.2:
        W[:, int(rng.integers(0, N))] = 0
    thr = float(rng.choice([6.0, 3.0, math.inf, 0.5]))
    keep = set(int(k) for k in rng.choice(K, size=int(rng.integers(0, K + 1)), replace=False))
    return X, W, thr, keep


@pytest.mark.parametrize("seed", range(120))
def test_brute_force_tiny(seed):
    X, W, thr, keep = _tiny_case(seed)
    bf = brute_force(X, W, thr, keep)
    prep = oracle.prepare_weight(W, sorted(keep))
    r = oracle.forward(X, prep, thr, threads=1)
    assert r["idx"].tolist() == bf["idx"]
    assert r["xq"].tolist() == bf["xq"]
    assert r["ra"].tolist() == bf["ra"]
    assert prep["wq"].tolist() == bf["wq"]
    assert prep["ca"].tolist() == bf["ca"]
    assert r["acc"].tolist() == bf["acc"]
    assert np.array_equal(r["y"].astype(np.float64), np.array(bf["y"], dtype=np.float64).reshape(r["y"].shape))


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------

def test_absmax_maps_to_127():
    X, W, _ = synth.make_case(64, 512, 96, n_seed=5, seed=3)
    X = X.numpy()
    W = W.numpy()
    idx = oracle.detect_outliers(X, 6.0)
    Xq, ra, _ = oracle.quantize_rows(X, idx)
    inl = np.setdiff1d(np.arange(X.shape[1]), idx)
    xf = X.astype(np.float32)
    for m in range(X.shape[0]):
        k = inl[np.argmax(np.abs(xf[m, inl]))]
        assert abs(xf[m, k]) == ra[m]
        assert Xq[m, k] == (127 if xf[m, k] > 0 else -127)
    assert np.all(Xq[:, idx] == 0)
    assert np.abs(Xq.astype(np.int32)).max() <= 127
    Wq, ca = oracle.quantize_weight(W)
    wf = W.astype(np.float32)
    for n in range(W.shape[1]):
        k = int(np.argmax(np.abs(wf[:, n])))
        assert abs(wf[k, n]) == ca[n]
        assert Wq[n, k] == (127 if wf[k, n] > 0 else -127)
    assert np.abs(Wq.astype(np.int32)).max() <= 127


def test_threshold_inf_is_pure_vectorwise():
    X, W, keep = synth.make_case(48, 384, 80, n_seed=3, seed=4)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight(W, keep)
    r = oracle.forward(X, prep, math.inf)
    assert r["idx"].size == 0
    ref = (r["xq"].astype(np.int64) @ prep["wq"].astype(np.int64).T).astype(np.float64)
    assert np.array_equal(r["acc"].astype(np.int64), ref.astype(np.int64))
    y64 = ref * r["ra"].astype(np.float64)[:, None] * prep["ca"].astype(np.float64)[None, :] / 16129.0
    y = r["y"].astype(np.float64)
    # fp16 half-ulp plus a few fp32 roundings
    assert np.all(np.abs(y - y64) <= np.abs(y64) * (2.0 ** -11 + 2.0 ** -20) + 2.0 ** -25)


def test_lossless_integer_inputs():
    rng = np.random.default_rng(5)
    M, K, N = 7, 8, 9
    X = rng.integers(-127, 128, size=(M, K)).astype(np.float16)
    W = rng.integers(-127, 128, size=(K, N)).astype(np.float16)
    X[np.arange(M), rng.integers(0, K, M)] = 127 * rng.choice([-1, 1], M)
    W[rng.integers(0, K, N), np.arange(N)] = 127 * rng.choice([-1, 1], N)
    prep = oracle.prepare_weight(W, [])
    r = oracle.forward(X, prep, 1000.0)
    assert r["idx"].size == 0
    assert np.all(r["ra"] == 127) and np.all(prep["ca"] == 127)
    assert np.array_equal(r["xq"].astype(np.int64), X.astype(np.int64))
    assert np.array_equal(prep["wq"].astype(np.int64), W.astype(np.int64).T)
    exact = X.astype(np.int64) @ W.astype(np.int64)
    assert np.array_equal(r["acc"].astype(np.int64), exact)
    y = r["y"].astype(np.float64)
    assert np.all(np.abs(y - exact) <= np.abs(exact) * 2.0 ** -10)


def test_all_outlier_reduces_to_fp16_matmul():
    rng = np.random.default_rng(6)
    # small integers: every fp32 partial sum is exact, so Y is fp16(exact product)
    X = rng.integers(-8, 9, size=(5, 12)).astype(np.float16)
    X[X == 0] = 1
    W = rng.integers(-8, 9, size=(12, 7)).astype(np.float16)
    prep = oracle.prepare_weight(W, list(range(12)))
    r = oracle.forward(X, prep, 0.5)
    assert r["idx"].tolist() == list(range(12))
    assert np.all(r["xq"] == 0) and np.all(r["ra"] == 0) and np.all(r["acc"] == 0)
    exact = X.astype(np.int64) @ W.astype(np.int64)
    assert np.array_equal(r["y"].astype(np.float64), exact.astype(np.float16).astype(np.float64))
    # general values: within fp32 summation error of the float64 product
    X, W, _ = synth.make_case(20, 64, 33, seed=7)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight(W, list(range(64)))
    r = oracle.forward(X, prep, 0.0)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    bound = (np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64))) * 64 * 2.0 ** -24
    assert np.all(np.abs(r["y"].astype(np.float64) - ref) <= bound + np.abs(ref) * 2.0 ** -11 + 2.0 ** -24)


def test_quantisation_error_within_half_step():
    X, W, _ = synth.make_case(96, 640, 130, n_seed=4, seed=8)
    X = X.numpy()
    W = W.numpy()
    idx = oracle.detect_outliers(X, 6.0)
    Xq, ra, _ = oracle.quantize_rows(X, idx)
    inl = np.setdiff1d(np.arange(X.shape[1]), idx)
    xf = X.astype(np.float64)[:, inl]
    deq = Xq[:, inl].astype(np.float64) * ra.astype(np.float64)[:, None] / 127.0
    assert np.all(np.abs(xf - deq) <= ra.astype(np.float64)[:, None] / 254.0 * (1 + 2.0 ** -20))
    Wq, ca = oracle.quantize_weight(W)
    deq = Wq.T.astype(np.float64) * ca.astype(np.float64)[None, :] / 127.0
    assert np.all(np.abs(W.astype(np.float64) - deq) <= ca.astype(np.float64)[None, :] / 254.0 * (1 + 2.0 ** -20))


def test_result_within_method_error_bound():
    """Y against the exact float64 X W: the only errors are the int8 half-steps
    of the non-outlier part, fp32 roundings and the final fp16 rounding."""
    X, W, keep = synth.make_case(40, 768, 72, n_seed=6, seed=9)
    X = X.numpy().astype(np.float64)
    W = W.numpy().astype(np.float64)
    prep = oracle.prepare_weight(W.astype(np.float16), keep)
    r = oracle.forward(X.astype(np.float16), prep, 6.0)
    assert set(keep.tolist()) <= set(r["idx"].tolist())
    exact = X @ W
    inl = np.setdiff1d(np.arange(X.shape[1]), r["idx"])
    ra = r["ra"].astype(np.float64)[:, None]
    ca = prep["ca"].astype(np.float64)[None, :]
    ex = ra / 254.0
    ew = ca / 254.0
    bound = (ex * np.abs(W[inl, :]).sum(0)[None, :] + np.abs(X[:, inl]).sum(1)[:, None] * ew
             + len(inl) * ex * ew)
    bound += (np.abs(X) @ np.abs(W)) * 2.0 ** -20 + np.abs(exact) * 2.0 ** -11 + 2.0 ** -24
    assert np.all(np.abs(r["y"].astype(np.float64) - exact) <= bound)
    # the same bound is violated once a term is dropped: drop the outlier part
    y_no_o = oracle.epilogue(r["acc"], r["ra"], prep["ca"], None).astype(np.float64)
    assert np.any(np.abs(y_no_o - exact) > bound)


def test_dequantised_outlier_rows_when_not_kept():
    X, W, keep = synth.make_case(16, 256, 40, n_seed=3, seed=10)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight(W, [])
    r = oracle.forward(X, prep, 6.0)
    assert r["idx"].size >= 3
    wo64 = prep["wq"].T[r["idx"], :].astype(np.float64) * prep["ca"].astype(np.float64)[None, :] / 127.0
    assert np.all(np.abs(r["wo"].astype(np.float64) - wo64) <= np.abs(wo64) * 2.0 ** -11 + 2.0 ** -25)


def test_points_match_full_forward():
    X, W, keep = synth.make_case(130, 272, 260, n_seed=4, seed=11)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight(W, keep)
    r = oracle.forward(X, prep, 6.0)
    steps = oracle.forward_steps_abc(X, prep, 6.0)
    pm, pn = synth.sample_points(130, 260, 200, seed=1, tiles=((128, 256),))
    acc, y = oracle.forward_points(steps, prep, pm, pn)
    assert np.array_equal(acc, r["acc"][pm, pn])
    assert np.array_equal(y.view(np.uint16), r["y"][pm, pn].view(np.uint16))
    assert np.array_equal(oracle.int8_gemm(r["xq"], prep["wq"], threads=1), oracle.int8_gemm(r["xq"], prep["wq"], threads=5))


def test_eight_bit_share_on_decode_recipe():
    """The abstract's claim that over 99.9 % of the values go through the 8-bit product: with
    the decode recipe's 6 seeded columns out of 4096 the share is 99.85%."""
    wl = synth.WORKLOADS["decode"]
    gen = __import__("torch").Generator().manual_seed(wl.seed)
    X, cols = synth.make_activations(wl.M, wl.K, wl.n_seed, wl.lo, wl.hi, wl.mode, gen)
    idx = oracle.detect_outliers(X.numpy(), wl.threshold)
    assert set(cols.tolist()) <= set(idx.tolist())
    share = 1.0 - idx.size / wl.K
    assert abs(share - (1 - 6 / 4096)) < 1e-3


def test_value_exactly_at_threshold_is_outlier():
    """The criterion is |x| >= threshold: a value exactly at 6.0 makes its column an outlier."""
    X = np.zeros((3, 32), dtype=np.float16)
    X[:, :] = 1.0
    X[1, 5] = -6.0
    X[2, 9] = np.float16(5.99609375)  # the fp16 value just below 6
    assert oracle.detect_outliers(X, 6.0).tolist() == [5]


def _all_halves_within(amax: float) -> np.ndarray:
    h = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16)
    pos = h[(h.astype(np.float64) <= amax)]
    return np.concatenate([pos, -pos]).astype(np.float16)


@pytest.mark.parametrize("amax", [5.99609375, 1.0, 3.140625, 0.01229095458984375, 254.0, 40.96875,
                                  0.46044921875, 1.5947265625])
def test_quantisation_rule_exhaustive(amax):
    """Every fp16 value in [-absmax, absmax] is quantised as
    round-half-even(RN32(x * RN32(127 / absmax))), checked in exact rationals."""
    vals = _all_halves_within(amax)
    vals = vals[::max(1, vals.size // 20000)]
    row = np.concatenate([np.array([amax], dtype=np.float16), vals])
    K = (row.size + 15) // 16 * 16
    X = np.zeros((1, K), dtype=np.float16)
    X[0, : row.size] = row
    Xq, ra, _ = oracle.quantize_rows(X, np.zeros(0, dtype=np.int32))
    assert ra[0] == np.float32(amax)
    s = rn32(Fraction(127) / Fraction(float(amax)))
    want = [max(-127, min(127, round(rn32(Fraction(float(v)) * s)))) for v in X[0].astype(np.float64)]
    assert Xq[0].tolist() == want
