"""Pins for the oracle's variants beyond the vector-wise matmul, checked
without trusting the oracle:

* the block-wise linear 8-bit codec (axolotl "llama3-model-quantization",
  "8-Bit Optimizers": blocks normalised by their own maximum, an 8-bit index
  per value) -- a hand-derived worked example
  (``tests/golden/blockwise_codec_14x4.json``), a brute force in exact
  rationals, +-absmax -> +-127, the half-step error bound, isolation of an
  outlier to its own block, integer inputs that round-trip exactly, and the
  single-block case against the vector-wise row rule;
* the group-wise matmul (scite report for nuQmm: nuQmm and ZeroQuant use one
  constant per group, finer than vector-wise) -- G = K is the vector-wise
  method bit for bit, a brute force in exact rationals, integer inputs that
  give the exact integer product, G = 1 reproduces the fp32 product, the
  method's error bound per group, and finer groups lowering the error on
  weights with large entries;
* the 4-bit weight-only product (the talk's "4-Bit Inference"; axolotl page,
  "Impact of Precision and Parameter Count") -- correctly rounded double to
  fp16, a brute force in exact rationals, a sum that must be rounded to fp16
  once, +-absmax -> +-7 with the half-step bound, and integer weights that
  give the exact product.
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
from tests.test_oracle_pins import rn16, rn32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# block-wise codec
# --------------------------------------------------------------------------

def block_brute_force(x: np.ndarray, B: int):
    """Codes, absmax and dequantised values in exact rationals."""
    xs = [Fraction(float(v)) for v in np.asarray(x, dtype=np.float32)]
    codes, amaxes, deq = [], [], []
    for lo in range(0, len(xs), B):
        blk = xs[lo:lo + B]
        a = max(abs(v) for v in blk)
        amaxes.append(float(a))
        if a == 0:
            codes += [0] * len(blk)
            deq += [0.0] * len(blk)
            continue
        s = rn32(Fraction(127) / a)
        for v in blk:
            q = max(-127, min(127, round(rn32(v * s))))
            codes.append(q)
            deq.append(float(rn32(rn32(q * a) / 127)))
    return codes, amaxes, deq


def test_block_worked_example_golden():
    with open(os.path.join(GOLDEN, "blockwise_codec_14x4.json")) as f:
        g = json.load(f)
    x = np.array(g["x"], dtype=np.float32)
    q, a = oracle.block_quantize(x, g["B"])
    e = g["expected"]
    assert q.tolist() == e["codes"]
    assert a.astype(np.float64).tolist() == e["absmax"]
    d = oracle.block_dequantize(q, a, g["B"])
    assert d.astype(np.float64).tolist() == e["dequantised"]
    # the rational brute force reproduces the hand-derived values
    bq, ba, bd = block_brute_force(x, g["B"])
    assert bq == e["codes"] and ba == e["absmax"] and bd == e["dequantised"]


def _block_case(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 41))
    B = int(rng.integers(1, n + 4))
    kind = seed % 3
    if kind == 0:
        x = rng.standard_normal(n) * rng.choice([1e-3, 1.0, 50.0])
    elif kind == 1:
        # dyadic values: many products land on exact ties
        x = rng.integers(-64, 65, n) / rng.choice([1.0, 4.0, 16.0])
    else:
        x = rng.standard_normal(n)
        x[rng.random(n) < 0.15] *= 40.0  # sparse large entries
        x[rng.random(n) < 0.2] = 0.0
    return x.astype(np.float32), B


@pytest.mark.parametrize("seed", range(60))
def test_block_brute_force(seed):
    x, B = _block_case(seed)
    q, a = oracle.block_quantize(x, B)
    bq, ba, bd = block_brute_force(x, B)
    assert q.tolist() == bq
    assert a.astype(np.float64).tolist() == ba
    assert oracle.block_dequantize(q, a, B).astype(np.float64).tolist() == bd


def test_block_absmax_maps_to_127_and_error_within_half_step():
    rng = np.random.default_rng(21)
    n, B = 100_003, 2048  # ragged tail block
    x = (rng.standard_normal(n) * np.exp(rng.standard_normal(n))).astype(np.float32)
    q, a = oracle.block_quantize(x, B)
    assert a.size == (n + B - 1) // B
    assert np.abs(q.astype(np.int32)).max() <= 127
    for b in range(a.size):
        blk = x[b * B:(b + 1) * B]
        i = int(np.argmax(np.abs(blk)))
        assert abs(blk[i]) == a[b]
        assert q[b * B + i] == (127 if blk[i] > 0 else -127)
    d = oracle.block_dequantize(q, a, B).astype(np.float64)
    step = np.repeat(a.astype(np.float64), B)[:n] / 127.0
    # half a quantisation step, plus the fp32 roundings of scale, product and dequantisation
    assert np.all(np.abs(x.astype(np.float64) - d) <= step / 2 * (1 + 2.0 ** -20) + np.abs(d) * 2.0 ** -22)


def test_block_outlier_stays_in_its_block():
    rng = np.random.default_rng(22)
    B = 64
    x = rng.standard_normal(10 * B + 17).astype(np.float32)
    q0, a0 = oracle.block_quantize(x, B)
    y = x.copy()
    y[3 * B + 5] = 500.0
    q1, a1 = oracle.block_quantize(y, B)
    changed = np.nonzero(a0 != a1)[0].tolist()
    assert changed == [3]
    diff = np.nonzero(q0 != q1)[0]
    assert diff.size > 0 and diff.min() >= 3 * B and diff.max() < 4 * B


def test_block_integers_round_trip_exactly():
    rng = np.random.default_rng(23)
    B = 16
    x = rng.integers(-127, 128, 5 * B + 3).astype(np.float32)
    for lo in range(0, x.size, B):
        x[lo] = 127.0 * rng.choice([-1, 1])  # every block reaches 127: scale 1
    q, a = oracle.block_quantize(x, B)
    assert np.all(a == 127.0)
    assert np.array_equal(q.astype(np.float32), x)
    assert np.array_equal(oracle.block_dequantize(q, a, B), x)


def test_block_single_block_follows_the_row_rule():
    """With one block the codec is the vector-wise rule of a single row
    without outliers: same codes, same absmax (fp16-representable inputs)."""
    X, _, _ = synth.make_case(1, 4096, 16, seed=24)
    row = X.numpy()
    q, a = oracle.block_quantize(row.astype(np.float32)[0], 4096)
    Xq, ra, _ = oracle.quantize_rows(row, np.zeros(0, dtype=np.int32))
    assert np.array_equal(q, Xq[0]) and a[0] == ra[0]


def test_block_zero_and_one_element_blocks():
    q, a = oracle.block_quantize(np.zeros(9, dtype=np.float32), 4)
    assert np.all(q == 0) and np.all(a == 0)
    assert np.all(oracle.block_dequantize(q, a, 4) == 0)
    x = np.array([-3.5, 0.25, 1e-20, -7.0], dtype=np.float32)
    q, a = oracle.block_quantize(x, 1)
    assert q.tolist() == [-127, 127, 127, -127]
    assert np.array_equal(a, np.abs(x))


# --------------------------------------------------------------------------
# group-wise matmul
# --------------------------------------------------------------------------

def grouped_brute_force(X: np.ndarray, W: np.ndarray, thr: float, keep, G: int):
    M, K = X.shape
    N = W.shape[1]
    ng = K // G
    xs = [[Fraction(float(v)) for v in row] for row in X.astype(np.float64)]
    ws = [[Fraction(float(v)) for v in row] for row in W.astype(np.float64)]
    outl = [k for k in range(K) if any(abs(xs[m][k]) >= thr for m in range(M))]
    oset = set(outl)

    def quant(vals, skip):
        amax = max((abs(v) for i, v in enumerate(vals) if i not in skip), default=Fraction(0))
        if amax == 0:
            return [0] * len(vals), amax
        s = rn32(Fraction(127) / amax)
        return [0 if i in skip else max(-127, min(127, round(rn32(v * s)))) for i, v in enumerate(vals)], amax

    xq = [[0] * K for _ in range(M)]
    ra = [[Fraction(0)] * ng for _ in range(M)]
    for m in range(M):
        for g in range(ng):
            cols = range(g * G, (g + 1) * G)
            q, a = quant([xs[m][k] for k in cols], {i for i, k in enumerate(cols) if k in oset})
            for i, k in enumerate(cols):
                xq[m][k] = q[i]
            ra[m][g] = a
    wq = [[0] * K for _ in range(N)]
    ca = [[Fraction(0)] * ng for _ in range(N)]
    for n in range(N):
        for g in range(ng):
            cols = range(g * G, (g + 1) * G)
            q, a = quant([ws[k][n] for k in cols], set())
            for i, k in enumerate(cols):
                wq[n][k] = q[i]
            ca[n][g] = a
    acc = [[[sum(xq[m][k] * wq[n][k] for k in range(g * G, (g + 1) * G)) for g in range(ng)]
            for n in range(N)] for m in range(M)]
    wo = []
    for k in outl:
        if k in keep:
            wo.append([ws[k][n] for n in range(N)])
        else:
            wo.append([Fraction(rn16(rn32(rn32(Fraction(wq[n][k]) * ca[n][k // G]) / 127))) for n in range(N)])
    y = []
    for m in range(M):
        row = []
        for n in range(N):
            o = Fraction(0)
            for j, k in enumerate(outl):
                o = rn32(o + rn32(xs[m][k] * wo[j][n]))
            v = Fraction(0)
            for g in range(ng):
                t = rn32(acc[m][n][g])
                t = rn32(t * ra[m][g])
                t = rn32(t * ca[n][g])
                t = rn32(t / 16129)
                v = rn32(v + t)
            v = rn32(v + o)
            row.append(rn16(v))
        y.append(row)
    return {"idx": outl, "xq": xq, "ra": [[float(v) for v in r] for r in ra], "wq": wq,
            "ca": [[float(v) for v in r] for r in ca], "acc": acc, "y": y}


def _grouped_tiny_case(seed):
    rng = np.random.default_rng(1000 + seed)
    G = int(rng.choice([1, 2, 3, 4]))
    ng = int(rng.integers(1, 4))
    K = G * ng
    M, N = (int(v) for v in rng.integers(1, 7, size=2))
    X = (rng.standard_normal((M, K)) * rng.choice([0.5, 2.0])).astype(np.float16)
    for k in rng.choice(K, size=int(rng.integers(0, K + 1)), replace=False)[: max(0, K // 3)]:
        X[int(rng.integers(0, M)), k] = np.float16(rng.choice([-1, 1]) * rng.uniform(6, 60))
    W = (rng.standard_normal((K, N)) * 0.05).astype(np.float16)
    if rng.random() < 0.3:
        W[int(rng.integers(0, K)), :] *= 30  # a large weight row: group constants differ
    thr = float(rng.choice([6.0, 3.0, math.inf]))
    keep = set(int(k) for k in rng.choice(K, size=int(rng.integers(0, K + 1)), replace=False))
    return X, W, thr, keep, G


@pytest.mark.parametrize("seed", range(60))
def test_grouped_brute_force_tiny(seed):
    X, W, thr, keep, G = _grouped_tiny_case(seed)
    bf = grouped_brute_force(X, W, thr, keep, G)
    prep = oracle.prepare_weight_grouped(W, sorted(keep), G)
    r = oracle.forward_grouped(X, prep, thr)
    assert r["idx"].tolist() == bf["idx"]
    assert r["xq"].tolist() == bf["xq"]
    assert r["ra"].astype(np.float64).tolist() == bf["ra"]
    assert prep["wq"].tolist() == bf["wq"]
    assert prep["ca"].astype(np.float64).tolist() == bf["ca"]
    assert r["acc"].tolist() == bf["acc"]
    assert np.array_equal(r["y"].astype(np.float64), np.array(bf["y"], dtype=np.float64).reshape(r["y"].shape))


@pytest.mark.parametrize("keep_all", [False, True])
def test_grouped_with_one_group_is_the_vectorwise_method(keep_all):
    X, W, keep = synth.make_case(24, 320, 48, n_seed=4, seed=25)
    X = X.numpy()
    W = W.numpy()
    keep = list(range(320)) if keep_all else keep
    v = oracle.forward(X, oracle.prepare_weight(W, keep), 6.0, threads=1)
    prep = oracle.prepare_weight_grouped(W, keep, 320)
    g = oracle.forward_grouped(X, prep, 6.0)
    vp = oracle.prepare_weight(W, keep)
    assert np.array_equal(g["idx"], v["idx"])
    assert np.array_equal(g["xq"], v["xq"]) and np.array_equal(g["ra"][:, 0], v["ra"])
    assert np.array_equal(prep["wq"], vp["wq"]) and np.array_equal(prep["ca"][:, 0], vp["ca"])
    assert np.array_equal(g["acc"][:, :, 0], v["acc"])
    assert np.array_equal(g["wo"].view(np.uint16), v["wo"].view(np.uint16))
    assert np.array_equal(g["y"].view(np.uint16), v["y"].view(np.uint16))


def test_grouped_integer_inputs_give_the_exact_product():
    rng = np.random.default_rng(26)
    M, K, N, G = 6, 24, 7, 8
    X = rng.integers(-127, 128, size=(M, K)).astype(np.float16)
    W = rng.integers(-127, 128, size=(K, N)).astype(np.float16)
    for g in range(K // G):
        X[np.arange(M), g * G + rng.integers(0, G, M)] = 127 * rng.choice([-1, 1], M)
        W[g * G + rng.integers(0, G, N), np.arange(N)] = 127 * rng.choice([-1, 1], N)
    prep = oracle.prepare_weight_grouped(W, [], G)
    r = oracle.forward_grouped(X, prep, 1000.0)
    assert np.all(r["ra"] == 127) and np.all(prep["ca"] == 127)
    assert np.array_equal(r["xq"].astype(np.int64), X.astype(np.int64))
    exact = X.astype(np.int64) @ W.astype(np.int64)
    assert np.array_equal(r["acc"].astype(np.int64).sum(axis=2), exact)
    # every partial sum is an integer below 2^24: the fp32 sums are exact, and
    # Y is the exact product rounded to fp16 (infinite beyond 65504)
    with np.errstate(over="ignore"):
        want = exact.astype(np.float16)
    assert np.isfinite(want).mean() > 0.5
    assert np.array_equal(r["y"].astype(np.float64), want.astype(np.float64))


def test_grouped_with_unit_groups_is_the_fp32_product():
    """G = 1: every non-zero code is +-127 and the constants are |x| and |w|,
    so each term is x*w up to fp32 rounding."""
    X, W, _ = synth.make_case(12, 96, 20, seed=27)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight_grouped(W, [], 1)
    r = oracle.forward_grouped(X, prep, math.inf)
    nz = X != 0
    assert np.all(np.abs(r["xq"][nz].astype(np.int32)) == 127) and np.all(r["xq"][~nz] == 0)
    assert np.array_equal(r["ra"], np.abs(X.astype(np.float32)))
    ref = X.astype(np.float64) @ W.astype(np.float64)
    bound = (np.abs(X.astype(np.float64)) @ np.abs(W.astype(np.float64))) * 96 * 2.0 ** -21
    assert np.all(np.abs(r["y"].astype(np.float64) - ref) <= bound + np.abs(ref) * 2.0 ** -11 + 2.0 ** -24)


def _grouped_error_bound(X, W, r, prep, G):
    K = X.shape[1]
    ng = K // G
    inl = np.ones(K, dtype=bool)
    inl[r["idx"]] = False
    exact = X @ W
    bound = np.zeros_like(exact)
    for g in range(ng):
        cols = np.arange(g * G, (g + 1) * G)
        cols = cols[inl[cols]]
        ex = r["ra"][:, g].astype(np.float64)[:, None] / 254.0
        ew = prep["ca"][:, g].astype(np.float64)[None, :] / 254.0
        bound += ex * np.abs(W[cols, :]).sum(0)[None, :] + np.abs(X[:, cols]).sum(1)[:, None] * ew + len(cols) * ex * ew
    bound += (np.abs(X) @ np.abs(W)) * 2.0 ** -19 + np.abs(exact) * 2.0 ** -11 + 2.0 ** -24
    return exact, bound


def test_grouped_result_within_method_error_bound():
    X, W, keep = synth.make_case(32, 512, 40, n_seed=5, seed=28)
    X = X.numpy().astype(np.float64)
    W = W.numpy().astype(np.float64)
    G = 64
    prep = oracle.prepare_weight_grouped(W.astype(np.float16), keep, G)
    r = oracle.forward_grouped(X.astype(np.float16), prep, 6.0)
    exact, bound = _grouped_error_bound(X, W, r, prep, G)
    y = r["y"].astype(np.float64)
    assert np.all(np.abs(y - exact) <= bound)
    # dropping the outlier term breaks the bound
    _, y_no_o = oracle.grouped_product(r["xq"], r["ra"], prep["wq"], prep["ca"], G, None)
    assert np.any(np.abs(y_no_o.astype(np.float64) - exact) > bound)


def test_finer_groups_lower_the_error_on_uneven_weights():
    """The reason for groups: a large weight entry coarsens only its own group."""
    rng = np.random.default_rng(29)
    X, W, _ = synth.make_case(32, 1024, 64, seed=29)
    W = W.numpy().astype(np.float32)
    rows = rng.choice(1024, 8, replace=False)
    W[rows, :] *= 50.0
    W = W.astype(np.float16)
    X = X.numpy()
    exact = X.astype(np.float64) @ W.astype(np.float64)
    err = {}
    for G in (1024, 128, 32):
        prep = oracle.prepare_weight_grouped(W, [], G)
        y = oracle.forward_grouped(X, prep, math.inf)["y"].astype(np.float64)
        err[G] = float(np.sqrt(np.mean((y - exact) ** 2)))
    assert err[32] < err[128] < err[1024]


# --------------------------------------------------------------------------
# 4-bit weight-only product
# --------------------------------------------------------------------------

def test_double_to_half_rounds_once():
    rng = np.random.default_rng(30)
    h = np.arange(0x0001, 0x7bff, 5, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2
    vals = list(mid) + list(mid * (1 + 2.0 ** -40)) + list(mid * (1 - 2.0 ** -40))
    vals += list(rng.standard_normal(3000) * 300.0) + [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e300, 2.0 ** -25,
                                                        2.0 ** -25 * (1 + 2.0 ** -40), 3 * 2.0 ** -26]
    for v in vals:
        with np.errstate(over="ignore"):
            want = int(np.array(v, dtype=np.float64).astype(np.float16).view(np.uint16))
        assert oracle.double_to_half(v) == want, (v, hex(want))
        if np.isfinite(v) and abs(v) < 65520:
            r = rn16(Fraction(v))
            assert np.float16(r).view(np.uint16) == want or (r == 0 and (want & 0x7FFF) == 0)


def int4_brute_force(X: np.ndarray, W: np.ndarray, G: int):
    M, K = X.shape
    N = W.shape[1]
    xs = [[Fraction(float(v)) for v in row] for row in X.astype(np.float64)]
    ws = [[Fraction(float(v)) for v in row] for row in W.astype(np.float64)]
    q = [[0] * K for _ in range(N)]
    ca = [[Fraction(0)] * (K // G) for _ in range(N)]
    for n in range(N):
        for g in range(K // G):
            cols = range(g * G, (g + 1) * G)
            a = max(abs(ws[k][n]) for k in cols)
            ca[n][g] = a
            if a == 0:
                continue
            s = rn32(Fraction(7) / a)
            for k in cols:
                q[n][k] = max(-7, min(7, round(rn32(ws[k][n] * s))))
    wd = [[rn32(rn32(q[n][k] * ca[n][k // G]) / 7) for k in range(K)] for n in range(N)]
    y = [[rn16(sum(xs[m][k] * wd[n][k] for k in range(K))) for n in range(N)] for m in range(M)]
    return q, [[float(v) for v in r] for r in ca], y


@pytest.mark.parametrize("seed", range(40))
def test_int4_brute_force_tiny(seed):
    rng = np.random.default_rng(2000 + seed)
    G = int(rng.choice([1, 2, 4, 5]))
    K = G * int(rng.integers(1, 4))
    M, N = (int(v) for v in rng.integers(1, 7, size=2))
    X = (rng.standard_normal((M, K)) * rng.choice([0.5, 4.0])).astype(np.float16)
    W = (rng.standard_normal((K, N)) * rng.choice([0.02, 1.0])).astype(np.float16)
    if rng.random() < 0.3:
        W[:, int(rng.integers(0, N))] = 0
    q, ca = oracle.quantize_weight_int4(W, G)
    bq, bca, by = int4_brute_force(X, W, G)
    assert q.tolist() == bq
    assert ca.astype(np.float64).tolist() == bca
    y = oracle.int4_product(X, q, ca, G)
    assert np.array_equal(y.astype(np.float64), np.array(by, dtype=np.float64).reshape(y.shape))


def test_int4_rounds_the_sum_once():
    """1 + 2^-11 + 2^-24 lies just above the midpoint of 1 and 1 + 2^-10: one
    rounding to fp16 gives 1 + 2^-10 (a detour through fp32 would make it a tie
    and give 1)."""
    X = np.array([[1.0, 2.0 ** -11, 2.0 ** -24, 0.0]], dtype=np.float16)
    W = np.array([[1.0], [1.0], [1.0], [7.0]], dtype=np.float16)
    q, ca = oracle.quantize_weight_int4(W, 4)
    assert q[:, :].tolist() == [[1, 1, 1, 7]] and ca.tolist() == [[7.0]]
    assert float(oracle.int4_product(X, q, ca, 4)[0, 0]) == 1.0 + 2.0 ** -10


def test_int4_absmax_maps_to_7_and_error_within_half_step():
    X, W, _ = synth.make_case(8, 1024, 96, seed=31)
    W = W.numpy()
    G = 128
    q, ca = oracle.quantize_weight_int4(W, G)
    assert np.abs(q.astype(np.int32)).max() <= 7
    wf = W.astype(np.float64)
    for n in range(0, 96, 7):
        for g in range(1024 // G):
            blk = wf[g * G:(g + 1) * G, n]
            i = int(np.argmax(np.abs(blk)))
            assert abs(blk[i]) == ca[n, g]
            assert q[n, g * G + i] == (7 if blk[i] > 0 else -7)
    step = np.repeat(ca.astype(np.float64), G, axis=1).T / 7.0  # K x N
    wd = q.T.astype(np.float64) * np.repeat(ca.astype(np.float64), G, axis=1).T / 7.0
    assert np.all(np.abs(wf - wd) <= step / 2 * (1 + 2.0 ** -20))
    # Y against the exact product: the weight half-steps plus the fp16 rounding
    X = X.numpy().astype(np.float64)
    y = oracle.int4_product(X.astype(np.float16), q, ca, G).astype(np.float64)
    exact = X @ wf
    # weight half-steps, the fp32 roundings of w', the final fp16 rounding
    bound = (np.abs(X) @ (step / 2 * (1 + 2.0 ** -20)) + (np.abs(X) @ np.abs(wd)) * 2.0 ** -22
             + np.abs(y) * 2.0 ** -11 + 2.0 ** -25)
    assert np.all(np.abs(y - exact) <= bound)


def test_int4_integer_weights_are_exact():
    rng = np.random.default_rng(32)
    K, N, G = 32, 9, 8
    W = rng.integers(-7, 8, size=(K, N)).astype(np.float16)
    for g in range(K // G):
        W[g * G + rng.integers(0, G, N), np.arange(N)] = 7 * rng.choice([-1, 1], N)
    q, ca = oracle.quantize_weight_int4(W, G)
    assert np.all(ca == 7.0)
    assert np.array_equal(q.T.astype(np.float16), W)
    X = rng.integers(-16, 17, size=(3, K)).astype(np.float16)
    exact = X.astype(np.int64) @ W.astype(np.int64)
    assert np.array_equal(oracle.int4_product(X, q, ca, G).astype(np.float64),
                          exact.astype(np.float16).astype(np.float64))


# --------------------------------------------------------------------------
# sampled points (the form the full-size parity checks use)
# --------------------------------------------------------------------------

def test_grouped_points_match_the_full_product():
    X, W, keep = synth.make_case(70, 384, 90, n_seed=3, seed=33)
    X = X.numpy()
    W = W.numpy()
    prep = oracle.prepare_weight_grouped(W, keep[:1], 64)
    r = oracle.forward_grouped(X, prep, 6.0)
    pm, pn = synth.sample_points(70, 90, 150, seed=3, tiles=((32, 32),))
    acc, y = oracle.forward_grouped_points(r, prep, pm, pn)
    assert np.array_equal(acc, r["acc"][pm, pn])
    assert np.array_equal(y.view(np.uint16), r["y"][pm, pn].view(np.uint16))


def test_int4_points_match_the_full_product():
    X, W, _ = synth.make_case(9, 512, 80, seed=34)
    X = X.numpy()
    q, ca = oracle.quantize_weight_int4(W.numpy(), 128)
    y_full = oracle.int4_product(X, q, ca, 128)
    pm, pn = synth.sample_points(9, 80, 100, seed=4, tiles=((8, 16),))
    y = oracle.int4_points(X, q, ca, 128, pm, pn)
    assert np.array_equal(y.view(np.uint16), y_full[pm, pn].view(np.uint16))
