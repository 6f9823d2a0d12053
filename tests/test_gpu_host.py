"""GPU parity of the host-buffer forward (int8mm_forward_host): X read from and
Y written to pinned host memory, the product run in row bands with each
band's copy-back overlapping the next band.  Y against the oracle within the
forward's tolerance, and bit-identical to the device-buffer forward on the
same inputs (same kernels; a band changes which tile an output belongs to,
not the order of its sums)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import int8_quantized_matmul_02_b200 as i8
from int8_quantized_matmul_02_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    yield


@pytest.mark.parametrize("M,K,N,n_seed", [
    (8, 1024, 768, 3),        # decode path: one kernel, one copy back
    (300, 1024, 2048, 5),     # two bands: 256 rows (SM pairs) and 44 rows (single-SM kernel)
    (1000, 2048, 1024, 7),    # four bands of 256 rows, ragged last band of 232
    (4096, 1024, 512, 2),     # eight bands of 512 rows
    (2100, 512, 4096, 0),     # no outliers; bands of 512 and a last one of 52
])
def test_host_forward_matches_oracle_and_device_path(M, K, N, n_seed):
    X, W, cols = synth.make_case(M, K, N, n_seed=n_seed, seed=M + N)
    w = parity.gpu_prepare(W, cols)
    prep, r = parity.oracle_full(X, W, cols, 6.0)
    ws = i8.Workspace(M, K, N)
    Xh = X.contiguous().pin_memory()
    Yh = torch.empty(M, N, dtype=torch.float16, pin_memory=True)
    out = i8.forward(Xh, w, 6.0, workspace=ws, out=Yh)
    assert out.data_ptr() == Yh.data_ptr() and not out.is_cuda
    status, n_o = i8.device_status(ws)
    assert status == 0 and n_o == r["idx"].size
    parity.assert_y_close(Yh.numpy().astype(np.float64), r["y"].astype(np.float64), "host Y")
    Yd = i8.forward(X.cuda(), w, 6.0, workspace=ws)
    assert np.array_equal(Yh.numpy().view(np.uint16), Yd.cpu().numpy().view(np.uint16)), \
        "host and device paths differ"


def test_host_forward_pageable_and_repeated():
    """Pageable host buffers work too (the driver stages them), and repeated
    calls reuse the library's copy stream and events."""
    M, K, N = 520, 512, 1024
    X, W, cols = synth.make_case(M, K, N, n_seed=4, seed=11)
    w = parity.gpu_prepare(W, cols)
    _, r = parity.oracle_full(X, W, cols, 6.0)
    ws = i8.Workspace(M, K, N)
    first = None
    for _ in range(3):
        Y = i8.forward(X.contiguous(), w, 6.0, workspace=ws)
        parity.assert_y_close(Y.numpy().astype(np.float64), r["y"].astype(np.float64), "pageable host Y")
        if first is None:
            first = Y.clone()
        assert torch.equal(Y.view(torch.int16), first.view(torch.int16))


def test_host_forward_rejects_bad_arguments():
    M, K, N = 64, 256, 256
    X, W, cols = synth.make_case(M, K, N, n_seed=1, seed=3)
    w = parity.gpu_prepare(W, cols)
    with pytest.raises(ValueError):
        i8.forward(X, w, 6.0, path="gemm")       # options are device-path only
    with pytest.raises(ValueError):
        i8.forward(X, w, 6.0, out=torch.empty(M, N + 16, dtype=torch.float16))
    with pytest.raises(i8.Int8mmError):
        i8.forward(X, w, float("nan"))            # the library rejects the threshold
