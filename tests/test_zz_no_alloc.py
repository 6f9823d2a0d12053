"""The decode-sized forward that allocates nothing.

Some callers cannot allocate device memory: code that only receives input
and output buffers from a host framework that owns all device memory, and
latency-critical paths where cudaMalloc's cost and device-wide
synchronisation are not acceptable.  int8mm_forward_decode_noalloc serves
them with scratch memory in a fixed-size array inside the library.  This test
calls it through the C-ABI and checks that it gives the same output as the
regular entry point (int8mm_forward with a caller workspace), within the
tolerance of the parity tests, on two calls in a row with different inputs.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

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
    lib = _abi.load()
    _, W, cols = synth.make_case(M, K, N, n_seed=n_seed, seed=7000 + M)
    w = i8.prepare_weight(W.cuda(), cols)
    for call in range(2):  # the second call must not see the first call's scratch
        X, _, _ = synth.make_case(M, K, N, n_seed=n_seed, seed=7000 + M)
        X = (X.float() * (1.0 + 0.25 * call)).half().cuda()
        ws = i8.Workspace(M, K, N)
        Y_ref = i8.forward(X, w, 6.0, workspace=ws)
        st_ref, n_ref = i8.device_status(ws)
        assert st_ref == 0
        Y, n = _noalloc(lib, X, w, 6.0)
        assert n == n_ref
        parity.assert_y_close(Y.float().cpu().numpy(), Y_ref.float().cpu().numpy(), what=f"call {call}")


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
