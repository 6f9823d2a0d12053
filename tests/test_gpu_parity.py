"""GPU parity: the CUDA path through the C-ABI against the CPU oracle on the
same seeded inputs (outlier list, int8 codes, scales and int32 sums
bit-exact; fp16 Y within 2^-9 |y| + 1e-3 rms)."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import int8_quantized_matmul_02_b200 as i8
from int8_quantized_matmul_02_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    torch.manual_seed(0)
    yield


def _run_case(M, K, N, n_seed, thr=6.0, path="auto", keep="seeded", cap=None, seed=0, mode="element",
              lo=10.0, hi=60.0, with_acc=True):
    """One case against the oracle.  with_acc=False runs the kernels that
    production calls run (no int32 debug output: the GEMM's instantiation
    without the accumulator stores) and checks every intermediate it leaves
    plus Y; with_acc=True also checks the int32 sums."""
    X, W, cols = synth.make_case(M, K, N, n_seed=n_seed, lo=lo, hi=hi, mode=mode, seed=seed)
    keep_idx = {"seeded": cols, "none": [], "all": list(range(K))}[keep]
    w = parity.gpu_prepare(W, keep_idx)
    prep, r = parity.oracle_full(X, W, keep_idx, thr)
    parity.check_weight(w, prep)
    g = parity.gpu_forward(X, w, thr, path=path, cap=cap, with_acc=with_acc)
    return parity.check_forward_full(g, r), r


def _both_instantiations(M, K, N, n_seed, path, seed, thr=6.0):
    """The forward with and without the int32 debug output: each against the
    oracle, and Y bit-identical between the two (the stores of the sums are
    the only difference between the two kernels)."""
    X, W, cols = synth.make_case(M, K, N, n_seed=n_seed, seed=seed)
    w = parity.gpu_prepare(W, cols)
    prep, r = parity.oracle_full(X, W, cols, thr)
    g1 = parity.gpu_forward(X, w, thr, path=path, with_acc=True)
    parity.check_forward_full(g1, r)
    g0 = parity.gpu_forward(X, w, thr, path=path, with_acc=False)
    parity.check_forward_full(g0, r)
    assert torch.equal(g0["Y_dev"].view(torch.int16), g1["Y_dev"].view(torch.int16)), \
        "Y differs between the kernels with and without the int32 output"
    return r


# ------------------------------------------------------------------ tiled GEMM path

@pytest.mark.parametrize("M,K,N,n_seed", [
    (16, 256, 384, 2),        # the tiny configuration's shape
    (300, 1040, 784, 4),      # several tiles, ragged M, N and K
    (129, 512, 528, 3),
    (256, 2048, 512, 7),
    (700, 1024, 1040, 5),     # several SM-pair tiles with a ragged pair
])
@pytest.mark.parametrize("path", ["gemm", "gemm1sm"])
@pytest.mark.parametrize("with_acc", [True, False])
def test_gemm_path_matches_oracle(M, K, N, n_seed, path, with_acc):
    """"gemm" uses SM-pair 256 x 256 tiles for M > 128; "gemm1sm" the single-SM
    kernel.  with_acc=False is the instantiation every production call runs."""
    _run_case(M, K, N, n_seed, path=path, with_acc=with_acc)


@pytest.mark.parametrize("path", ["gemm", "gemm1sm", "decode"])
@pytest.mark.parametrize("M,K,N,n_seed", [(8, 2048, 1040, 5), (300, 1040, 784, 4), (700, 1024, 1040, 65)])
def test_production_kernels_match_debug_kernels(M, K, N, n_seed, path):
    if path == "decode" and M > 16:
        pytest.skip("the decode kernel takes M <= 16")
    _both_instantiations(M, K, N, n_seed, path, seed=500 + M + n_seed)


@pytest.mark.parametrize("M", [1, 8, 17, 64, 65, 129])
def test_gemm_path_row_counts(M):
    _run_case(M, 512, 272, 3, path="gemm", seed=M)


@pytest.mark.parametrize("n_seed", [0, 1, 15, 16, 17, 64, 65])
def test_gemm_path_outlier_counts(n_seed):
    _, r = _run_case(160, 1024, 512, n_seed, path="gemm", seed=100 + n_seed)
    assert r["idx"].size >= n_seed


@pytest.mark.parametrize("n_seed", [0, 1, 64, 65])
@pytest.mark.parametrize("path", ["gemm", "gemm1sm"])
def test_gemm_path_outlier_counts_production_kernel(n_seed, path):
    _, r = _run_case(300, 1024, 528, n_seed, path=path, seed=200 + n_seed, with_acc=False)
    assert r["idx"].size >= n_seed


@pytest.mark.parametrize("with_acc", [True, False])
def test_gemm_path_long_rows(with_acc):
    """K above what the row quantiser holds in registers (256 threads x 8
    chunks of 8 columns): the two-pass row quantiser runs instead."""
    _run_case(40, 16400, 272, 3, path="gemm", seed=61, with_acc=with_acc)


@pytest.mark.parametrize("keep", ["none", "all"])
def test_gemm_path_kept_and_dequantised_rows(keep):
    _run_case(130, 768, 528, 5, path="gemm", keep=keep, seed=7)


def test_gemm_path_threshold_inf():
    _, r = _run_case(200, 1024, 512, 6, thr=math.inf, path="gemm", seed=3)
    assert r["idx"].size == 0


def test_gemm_path_all_outliers():
    # threshold below every |x|: every column is an outlier, the int8 part is empty
    _, r = _run_case(96, 256, 272, 0, thr=1e-30, path="gemm", keep="all", seed=5)
    assert r["idx"].size == 256


def test_gemm_path_zero_rows_and_columns():
    X, W, cols = synth.make_case(140, 512, 528, n_seed=3, seed=9)
    X[5, :] = 0
    X[:, 17] = 0
    W[:, 33] = 0
    w = parity.gpu_prepare(W, cols)
    prep, r = parity.oracle_full(X, W, cols, 6.0)
    parity.check_weight(w, prep)
    parity.check_forward_full(parity.gpu_forward(X, w, 6.0, path="gemm"), r)


# ------------------------------------------------------------------ fused decode path

@pytest.mark.parametrize("M,K,N,n_seed", [
    (1, 256, 384, 2),
    (8, 4096, 1024, 6),
    (9, 1024, 528, 3),
    (16, 4112, 400, 5),       # K not a multiple of 128, N not a multiple of 128
    (3, 2048, 11008, 1),
    (4, 16, 272, 1),          # one 16-column K block: a cluster of one CTA
    (5, 128, 1040, 2),        # one full K block
    (16, 20480, 272, 7),      # the longest K the decode kernel takes (clusters of 8, one CTA per SM)
    (8, 11008, 4096, 6),      # FFN down-projection shape: clusters of 8, two CTAs per SM, 2-3 tiles each
    (8, 16384, 1040, 5),      # M <= 8 on the one-CTA-per-SM shape
    (16, 12288, 2048, 4),     # M > 8 on the one-CTA-per-SM shape, clusters of 8
])
@pytest.mark.parametrize("with_acc", [True, False])
def test_decode_path_matches_oracle(M, K, N, n_seed, with_acc):
    _run_case(M, K, N, n_seed, path="decode", seed=M * 31 + K, with_acc=with_acc)


@pytest.mark.parametrize("keep", ["none", "all"])
def test_decode_path_kept_and_dequantised_rows(keep):
    _run_case(8, 1024, 528, 4, path="decode", keep=keep, seed=11)


def test_decode_path_threshold_inf_and_all_outliers():
    _run_case(8, 1024, 272, 4, thr=math.inf, path="decode", seed=12)
    _run_case(4, 256, 272, 0, thr=1e-30, path="decode", keep="all", seed=13)


@pytest.mark.parametrize("thr", [6.0, 5.998, 5.99609375, 65504.0, 70000.0])
@pytest.mark.parametrize("path", ["decode", "gemm"])
def test_threshold_boundaries(thr, path):
    """Values exactly at, just below and just above the threshold (which may
    fall between two fp16 values) are classified like the oracle does."""
    M, K, N = 8, 512, 272
    X, W, cols = synth.make_case(M, K, N, n_seed=0, seed=41)
    X[1, 10] = 6.0
    X[2, 20] = -5.99609375          # the fp16 value just below 6
    X[3, 30] = 6.00390625           # the fp16 value just above 6
    X[4, 40] = 65504.0
    X[5, 50] = 60000.0
    w = parity.gpu_prepare(W, [10, 20])
    prep, r = parity.oracle_full(X, W, [10, 20], thr)
    parity.check_forward_full(parity.gpu_forward(X, w, thr, path=path), r)


@pytest.mark.parametrize("amax", [5.99609375, 3.140625, 0.46044921875, 1.5947265625, 0.01229095458984375])
@pytest.mark.parametrize("path", ["decode", "gemm"])
def test_quantisation_rule_every_fp16_value(amax, path):
    """Every fp16 value in [-absmax, absmax] (including those where x * scale
    falls exactly half-way between two integers) gets the oracle's code."""
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)
    pos = h[h.astype(np.float64) <= amax]
    vals = np.concatenate([pos, -pos]).astype(np.float16)
    M, N = 16, 64  # the values spread over 16 rows, each row also holding absmax
    per = (vals.size + M - 1) // M
    K = (per + 1 + 15) // 16 * 16
    X = np.zeros((M, K), dtype=np.float16)
    for m in range(M):
        part = vals[m * per:(m + 1) * per]
        X[m, 0] = amax if m % 2 == 0 else -amax
        X[m, 1:1 + part.size] = part
    X = torch.from_numpy(X)
    W = torch.from_numpy((np.random.default_rng(0).standard_normal((K, N)) * 0.02).astype(np.float16))
    w = parity.gpu_prepare(W, [])
    g = parity.gpu_forward(X, w, 6.0, path=path)
    Xq, ra, _ = oracle.quantize_rows(X.numpy(), oracle.detect_outliers(X.numpy(), 6.0))
    assert np.array_equal(g["ra"].view(np.uint32), ra.view(np.uint32))
    assert np.array_equal(g["xq_dev"].cpu().numpy(), Xq)


def test_decode_workspace_is_reusable():
    """Repeated calls on one workspace give the oracle's result every time."""
    M, K, N = 8, 4096, 2048
    _, W, cols = synth.make_case(M, K, N, n_seed=4, seed=21)
    w = parity.gpu_prepare(W, cols)
    prep = oracle.prepare_weight(W.numpy(), cols)
    ws = i8.Workspace(M, K, N)
    for s in range(3):
        X, _, _ = synth.make_case(M, K, N, n_seed=4, seed=21)  # same columns, new draws below
        X = (X.float() * (1.0 + 0.1 * s)).half()
        r = oracle.forward(X.numpy(), prep, 6.0)
        parity.check_forward_full(parity.gpu_forward(X, w, 6.0, path="decode", ws=ws), r)


def test_gemm_workspace_is_reusable():
    M, K, N = 200, 1024, 528
    X, W, cols = synth.make_case(M, K, N, n_seed=4, seed=22)
    w = parity.gpu_prepare(W, cols)
    prep = oracle.prepare_weight(W.numpy(), cols)
    ws = i8.Workspace(M, K, N)
    for s in range(3):
        Xs = X.clone()
        Xs[:, (s * 37) % K] = 30.0  # a different extra outlier column each call
        r = oracle.forward(Xs.numpy(), prep, 6.0)
        parity.check_forward_full(parity.gpu_forward(Xs, w, 6.0, path="gemm", ws=ws), r)


def test_paths_agree():
    X, W, cols = synth.make_case(12, 2048, 1040, n_seed=5, seed=23)
    w = parity.gpu_prepare(W, cols)
    a = parity.gpu_forward(X, w, 6.0, path="decode")
    b = parity.gpu_forward(X, w, 6.0, path="gemm")
    assert torch.equal(a["acc_dev"], b["acc_dev"])
    parity.assert_y_close(a["Y_dev"].float().cpu().numpy(), b["Y_dev"].float().cpu().numpy())


# ------------------------------------------------------------------ device-side errors

@pytest.mark.parametrize("path", ["gemm", "decode"])
def test_outlier_overflow_is_reported(path):
    X, W, cols = synth.make_case(8, 1024, 512, n_seed=6, seed=30)
    w = parity.gpu_prepare(W, cols)
    ws = i8.Workspace(8, 1024, 512, max_outliers=2)
    i8.forward(X.cuda(), w, 6.0, workspace=ws, path=path)
    st, n = i8.device_status(ws)
    assert st == 7 and n >= 6


@pytest.mark.parametrize("path", ["gemm", "decode"])
def test_wait_limit_reports_timeout_and_recovers(path):
    """The main kernel withholds one internal signal, so a wait runs out after
    its 50 ms limit: the kernel records a timeout and returns, and the context
    stays usable for the next call."""
    from int8_quantized_matmul_02_b200 import _abi

    M = 8 if path == "decode" else 200
    X, W, cols = synth.make_case(M, 2048, 1024, n_seed=3, seed=31)
    w = parity.gpu_prepare(W, cols)
    ws = i8.Workspace(M, 2048, 1024)
    i8.forward(X.cuda(), w, 6.0, workspace=ws, path=path, wait_limit_ns=50_000_000,
               test_flags=_abi.TEST_WITHHOLD_SIGNAL)
    st, _ = i8.device_status(ws)
    assert st == 6
    ws.reset()
    prep, r = parity.oracle_full(X, W, cols, 6.0)
    parity.check_forward_full(parity.gpu_forward(X, w, 6.0, path=path, ws=ws), r)


# ------------------------------------------------------------------ full-size workloads

def _full_size(name, cap=1024, full_oracle=False):
    """The workload at full size, in the launch configuration the benchmark
    times (workspace capacity 1024 outlier columns), run twice: without the
    int32 debug output (the kernels the benchmark runs) and with it.  Both
    against the oracle; Y bit-identical between the two."""
    wl = synth.WORKLOADS[name]
    X, W, cols = synth.make_inputs(wl)
    w = parity.gpu_prepare(W, cols)
    prep = oracle.prepare_weight(W.numpy(), cols)
    parity.check_weight(w, prep)
    del W
    cap = min(cap, wl.K)
    if full_oracle:
        r = oracle.forward(X.numpy(), prep, wl.threshold)
    else:
        steps = oracle.forward_steps_abc(X.numpy(), prep, wl.threshold)
        pm, pn = synth.sample_points(wl.M, wl.N, 4096, seed=wl.seed, tiles=((128, 256), (128, 256)))
    ys = []
    for with_acc in (False, True):
        g = parity.gpu_forward(X, w, wl.threshold, path="auto", cap=cap, with_acc=with_acc)
        if full_oracle:
            parity.check_forward_full(g, r)
        else:
            parity.check_forward_sampled(g, steps, prep, pm, pn)
        ys.append(g["Y_dev"])
        del g
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16)), \
        "Y differs between the kernels with and without the int32 output"
    return r["idx"].size if full_oracle else steps["idx"].size


def test_full_size_decode():
    n_o = _full_size("decode", full_oracle=True)
    assert n_o >= 6


@pytest.mark.parametrize("name", ["prefill", "175b", "qkv_o0", "qkv_o12", "qkv_o48", "qkv_o123", "qkv_inf"])
def test_full_size_sampled(name):
    n_o = _full_size(name)
    assert n_o >= synth.WORKLOADS[name].n_seed
