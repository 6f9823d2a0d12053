"""GPU parity of the group-wise variant (one constant per row of X and group
of G consecutive k, and per output column and group: the granularity the
scite report for nuQmm attributes to nuQmm and ZeroQuant) against the CPU
oracle on the same seeded inputs: weight codes and group constants, outlier
list, X codes and row constants, and the per-group int32 sums bit-exact; fp16
Y within 2^-9 |y| + 1e-3 rms(y) (the fp16 outlier product is summed in
another order; before it the running fp32 sum uses the definition's
operations in its order)."""
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


def _check_weight(w, prep):
    assert np.array_equal(w.wq.cpu().numpy(), prep["wq"]), "Wq differs"
    ca = w.col_absmax.cpu().numpy().T  # the library keeps (K/G) x N
    assert np.array_equal(np.ascontiguousarray(ca).view(np.uint32), prep["ca"].view(np.uint32)), "ca differs"


def _run(X, W, keep, G, thr=6.0, with_acc=True, cap=None):
    M, K = X.shape
    N = W.shape[1]
    w = i8.prepare_weight_grouped(W.cuda(), G, keep)
    prep = oracle.prepare_weight_grouped(W.numpy(), keep, G)
    _check_weight(w, prep)
    r = oracle.forward_grouped(X.numpy(), prep, thr)
    ws = i8.Workspace(M, K, N, cap, G=G)
    acc = torch.empty(M, N, K // G, dtype=torch.int32, device="cuda") if with_acc else None
    Y = i8.forward_grouped(X.cuda(), w, thr, workspace=ws, acc_out=acc)
    st, n_o = i8.device_status(ws)
    assert st == 0, st
    v = ws.view()
    assert n_o == r["idx"].size
    assert np.array_equal(v["outlier_idx"][:n_o].cpu().numpy(), r["idx"]), "outlier list differs"
    assert np.array_equal(v["row_absmax"].cpu().numpy().view(np.uint32), r["ra"].view(np.uint32)), "row constants differ"
    assert np.array_equal(v["xq"].cpu().numpy(), r["xq"]), "Xq differs"
    if with_acc:
        assert np.array_equal(acc.cpu().numpy(), r["acc"]), "per-group int32 sums differ"
    parity.assert_y_close(Y.float().cpu().numpy(), r["y"].astype(np.float64))
    return Y, r, w


@pytest.mark.parametrize("M,K,N,G,n_seed", [
    (16, 256, 384, 128, 2),
    (300, 1024, 784, 256, 4),     # ragged M and N, several pair tiles
    (129, 512, 528, 128, 3),
    (256, 2048, 512, 1024, 7),
    (700, 1024, 1040, 512, 65),   # two outlier slices
    (64, 1536, 272, 1536, 1),     # G = K: one group
])
def test_grouped_matches_oracle(cuda_ok, M, K, N, G, n_seed):
    X, W, cols = synth.make_case(M, K, N, n_seed=n_seed, seed=900 + M + G)
    Y1, _, _ = _run(X, W, cols, G, with_acc=True)
    Y0, _, _ = _run(X, W, cols, G, with_acc=False)
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16)), "Y differs with and without the int32 output"


@pytest.mark.parametrize("keep", ["none", "all"])
def test_grouped_kept_and_dequantised_rows(cuda_ok, keep):
    X, W, cols = synth.make_case(200, 1024, 528, n_seed=5, seed=77)
    _run(X, W, {"none": [], "all": list(range(1024))}[keep], 256)


def test_grouped_threshold_inf_and_all_outliers(cuda_ok):
    X, W, cols = synth.make_case(160, 512, 272, n_seed=4, seed=78)
    _, r, _ = _run(X, W, cols, 128, thr=math.inf)
    assert r["idx"].size == 0
    X, W, _ = synth.make_case(96, 256, 272, n_seed=0, seed=79)
    _, r, _ = _run(X, W, list(range(256)), 128, thr=1e-30)
    assert r["idx"].size == 256


def test_grouped_with_one_group_matches_vector_wise_intermediates(cuda_ok):
    """G = K: the group-wise forward computes the vector-wise method; every
    intermediate equals the vector-wise path's bit for bit."""
    M, K, N = 300, 1024, 528
    X, W, cols = synth.make_case(M, K, N, n_seed=4, seed=80)
    Yg, r, _ = _run(X, W, cols, K)
    wv = i8.prepare_weight(W.cuda(), cols)
    g = parity.gpu_forward(X, wv, 6.0, path="gemm")
    assert np.array_equal(g["acc_dev"].cpu().numpy(), r["acc"][:, :, 0])
    parity.assert_y_close(g["Y_dev"].float().cpu().numpy(), Yg.float().cpu().numpy())


def test_grouped_timeout_is_reported_and_recovers(cuda_ok):
    from int8_quantized_matmul_02_b200 import _abi

    M, K, N, G = 300, 1024, 528, 256
    X, W, cols = synth.make_case(M, K, N, n_seed=3, seed=81)
    w = i8.prepare_weight_grouped(W.cuda(), G, cols)
    ws = i8.Workspace(M, K, N, G=G)
    i8.forward_grouped(X.cuda(), w, 6.0, workspace=ws, wait_limit_ns=50_000_000, test_flags=_abi.TEST_WITHHOLD_SIGNAL)
    st, _ = i8.device_status(ws)
    assert st == 6
    ws.reset()
    _run(X, W, cols, G)


def test_grouped_full_size_sampled(cuda_ok):
    """The benchmark's group-wise workload: the 175B-scale FFN shape with
    groups of 1024, in the launch configuration the benchmark times
    (workspace capacity 1024 outlier columns).  Weight codes and constants,
    the X-side steps in full; sums and Y at sampled points plus two whole
    tiles."""
    wl = synth.WORKLOADS["175b"]
    G = 1024
    X, W, cols = synth.make_inputs(wl)
    w = i8.prepare_weight_grouped(W.cuda(), G, cols)
    prep = oracle.prepare_weight_grouped(W.numpy(), cols, G)
    _check_weight(w, prep)
    del W
    idx = oracle.detect_outliers(X.numpy(), wl.threshold)
    xq, ra, xo = oracle.quantize_rows_grouped(X.numpy(), idx, G)
    wo = oracle.gather_w_outlier_grouped(prep, idx)
    ws = i8.Workspace(wl.M, wl.K, wl.N, 1024, G=G)
    Y = i8.forward_grouped(X.cuda(), w, wl.threshold, workspace=ws)
    st, n_o = i8.device_status(ws)
    assert st == 0 and n_o == idx.size
    v = ws.view()
    assert np.array_equal(v["outlier_idx"][:n_o].cpu().numpy(), idx)
    assert np.array_equal(v["row_absmax"].cpu().numpy().view(np.uint32), ra.view(np.uint32))
    assert np.array_equal(v["xq"].cpu().numpy(), xq)
    pm, pn = synth.sample_points(wl.M, wl.N, 4096, seed=wl.seed, tiles=((128, 128), (128, 128)))
    _, y_ref = oracle.forward_grouped_points({"xq": xq, "ra": ra, "xo": xo, "wo": wo}, prep, pm, pn)
    y = Y[torch.from_numpy(pm.astype(np.int64)).cuda(), torch.from_numpy(pn.astype(np.int64)).cuda()]
    parity.assert_y_close(y.float().cpu().numpy(), y_ref.astype(np.float64))
