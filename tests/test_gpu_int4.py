"""GPU parity of the 4-bit weight-only decode product against the CPU oracle
(video page "8-bit Methods for Efficient Deep Learning with Tim Dettmers",
"4-Bit Inference"): codes and group constants bit-exact, Y within
2^-9 |y| + 1e-3 rms(y) (the kernel scales fp32 tensor-core sums per group of
128 k; the oracle sums the products with fp32 dequantised weights in double
and rounds once)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import int8_quantized_matmul_02_b200 as i8
from tests import parity

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, seed, sigma=0.02):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(M, K, generator=g).half()
    W = (torch.randn(K, N, generator=g) * sigma).half()
    # a few large weights, so that group constants differ from group to group
    idx = torch.randint(0, K * N, (max(1, K * N // 5000),), generator=g)
    W.view(-1)[idx] = (torch.randn(idx.numel(), generator=g) * 0.5).half()
    return X, W


def _check_weight(w, W, G):
    q_ref, ca_ref = oracle.quantize_weight_int4(W.numpy(), G)
    q = i8.unpack_int4_codes(w.codes.cpu().numpy())
    assert np.array_equal(q, q_ref), "codes differ"
    assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), ca_ref.view(np.uint32)), "constants differ"
    return q_ref, ca_ref


@pytest.mark.parametrize("M,K,N,G", [
    (1, 256, 384, 128),
    (8, 1024, 528, 256),
    (3, 2048, 1040, 2048),     # one group per column
    (16, 2048, 1040, 128),     # 16 rows
    (9, 1152, 400, 128),       # K % 256 == 128: the last half box lies past K
    (5, 128, 16, 128),         # one 128-k block, a tile of 16 columns
    (8, 11008, 4096, 128),     # FFN down-projection shape, clusters over 43 boxes
    (16, 28672, 144, 256),     # the longest K for 16 rows (clusters of 8, 3 ring stages)
    (8, 73728, 48, 1024),      # the longest K for 8 rows
])
def test_int4_matches_oracle(cuda_ok, M, K, N, G):
    X, W = _inputs(M, K, N, seed=M * 1000 + K + N + G)
    w = i8.prepare_weight_int4(W.cuda(), G)
    q_ref, ca_ref = _check_weight(w, W, G)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = i8.forward_int4(X.cuda(), w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    y_ref = oracle.int4_product(X.numpy(), q_ref, ca_ref, G)
    parity.assert_y_close(Y.float().cpu().numpy(), y_ref.astype(np.float64))


@pytest.mark.parametrize("G", [128, 1024])
def test_int4_decode_shape(cuda_ok, G):
    """The decode-shaped FFN up-projection (X 8 x 4096, W 4096 x 11008), in
    full, twice in a row (the second call reuses every buffer)."""
    M, K, N = 8, 4096, 11008
    X, W = _inputs(M, K, N, seed=4242 + G)
    w = i8.prepare_weight_int4(W.cuda(), G)
    q_ref, ca_ref = _check_weight(w, W, G)
    Xd = X.cuda()
    Y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_ref = oracle.int4_product(X.numpy(), q_ref, ca_ref, G).astype(np.float64)
    for _ in range(2):
        i8.forward_int4(Xd, w, out=Y, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        parity.assert_y_close(Y.float().cpu().numpy(), y_ref)


def test_int4_rejects_bad_shapes(cuda_ok):
    W = torch.zeros(256, 384, dtype=torch.float16, device="cuda")
    with pytest.raises(i8.Int8mmError):
        i8.prepare_weight_int4(W, 96)         # G not a multiple of 128
    with pytest.raises(i8.Int8mmError):
        i8.prepare_weight_int4(W, 512)        # G does not divide K
    w = i8.prepare_weight_int4(W, 128)
    with pytest.raises(i8.Int8mmError):
        i8.forward_int4(torch.zeros(17, 256, dtype=torch.float16, device="cuda"), w)  # M > 16
    W2 = torch.zeros(28928, 16, dtype=torch.float16, device="cuda")
    w2 = i8.prepare_weight_int4(W2, 128)
    i8.forward_int4(torch.zeros(8, 28928, dtype=torch.float16, device="cuda"), w2)  # fits with 8 rows
    with pytest.raises(i8.Int8mmError):
        i8.forward_int4(torch.zeros(9, 28928, dtype=torch.float16, device="cuda"), w2)  # X share too long
