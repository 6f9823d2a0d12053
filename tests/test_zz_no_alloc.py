"""The decode-sized forward that allocates nothing.

Some callers cannot allocate device memory: code that only receives input
and output buffers from a host framework that owns all device memory, and
latency-critical paths where cudaMalloc's cost and device-wide
synchronisation are not acceptable.  int8mm_forward_decode_noalloc serves
them with scratch memory in a fixed-size array inside the library.  This test
calls it through the C-ABI on two calls in a row with different inputs and
checks each against the CPU oracle (within the tolerance of the parity tests)
and against the regular entry point (int8mm_forward with a caller workspace,
on the same kernel: bit-identical).

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import int8_quantized_matmul_02_b200 as i8
from int8_quantized_matmul_02_b200 import _abi, synth
from tests import parity

pytestmark = pytest.mark.gpu


def _noalloc(lib, X: torch.Tensor, w: i8.PreparedWeight, thr: float) -> torch.Tensor:
    Y = torch.empty(X.shape[0], w.N, dtype=torch.float16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.int8mm_forward_decode_noalloc(ctypes.c_void_p(X.data_ptr()), X.shape[0], ctypes.byref(w.struct),
                                           float(thr), ctypes.c_void_p(Y.data_ptr()), stream)
    assert st == 0, _abi.STATUS_NAMES.get(st, st)
    n = ctypes.c_int32(0)
    st = lib.int8mm_noalloc_device_status(stream, ctypes.byref(n))
    assert st == 0, _abi.STATUS_NAMES.get(st, st)
    return Y, int(n.value)


@pytest.mark.parametrize("M,K,N,n_seed", [(8, 4096, 11008, 6), (16, 2048, 1040, 3), (1, 256, 384, 1)])
def test_noalloc_matches_regular_entry_point_twice(cuda_ok, M, K, N, n_seed):
    """Two calls in a row with different inputs.  Each call is checked against
    the oracle (outlier count exact, Y within the parity tolerance) and against
    int8mm_forward on the same fused decode kernel (Y bit-identical: only the
    place of the scratch memory differs)."""
    lib = _abi.load()
    _, W, cols = synth.make_case(M, K, N, n_seed=n_seed, seed=7000 + M)
    w = i8.prepare_weight(W.cuda(), cols)
    prep = oracle.prepare_weight(W.numpy(), cols)
    for call in range(2):  # the second call must not see the first call's scratch
        X, _, _ = synth.make_case(M, K, N, n_seed=n_seed, seed=7000 + M)
        X = (X.float() * (1.0 + 0.25 * call)).half()
        if call == 1:
            X[:, (37 * M) % K] = 25.0  # one more outlier column on the second call
        ref = oracle.forward(X.numpy(), prep, 6.0)
        Xd = X.cuda()
        ws = i8.Workspace(M, K, N)
        Y_ref = i8.forward(Xd, w, 6.0, workspace=ws, path="decode")
        st_ref, n_ref = i8.device_status(ws)
        assert st_ref == 0
        Y, n = _noalloc(lib, Xd, w, 6.0)
        assert n == n_ref == ref["idx"].size
        parity.assert_y_close(Y.float().cpu().numpy(), ref["y"].astype(np.float64), what=f"call {call} vs oracle")
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), f"call {call}: Y differs from int8mm_forward"


def test_noalloc_rejects_sizes_beyond_its_limit(cuda_ok):
    lib = _abi.load()
    _, W, cols = synth.make_case(8, 16400, 64, n_seed=0, seed=1)
    w = i8.prepare_weight(W.cuda(), cols)  # K = 16400 > 16384
    X = torch.zeros(8, 16400, dtype=torch.float16, device="cuda")
    Y = torch.empty(8, 64, dtype=torch.float16, device="cuda")
    st = lib.int8mm_forward_decode_noalloc(ctypes.c_void_p(X.data_ptr()), 8, ctypes.byref(w.struct), 6.0,
                                           ctypes.c_void_p(Y.data_ptr()), None)
    assert st == 1
    _, W, cols = synth.make_case(17, 256, 64, n_seed=0, seed=2)
    w = i8.prepare_weight(W.cuda(), cols)
    X = torch.zeros(17, 256, dtype=torch.float16, device="cuda")
    Y = torch.empty(17, 64, dtype=torch.float16, device="cuda")
    st = lib.int8mm_forward_decode_noalloc(ctypes.c_void_p(X.data_ptr()), 17, ctypes.byref(w.struct), 6.0,
                                           ctypes.c_void_p(Y.data_ptr()), None)
    assert st == 1
