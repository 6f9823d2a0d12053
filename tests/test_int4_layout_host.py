"""Host checks of the 4-bit code layout helper (no GPU): a word built bit by
bit from the documented nibble order unpacks to the codes it was built from."""
from __future__ import annotations

import numpy as np

import int8_quantized_matmul_02_b200 as i8


def test_unpack_follows_the_documented_nibble_order():
    rng = np.random.default_rng(0)
    N, K = 5, 64
    q = rng.integers(-7, 8, (N, K)).astype(np.int8)
    order = [0, 16, 4, 20, 8, 24, 12, 28]  # bit position of k0 + i, from the header
    words = np.zeros((N, K // 8), dtype=np.uint32)
    for n in range(N):
        for w in range(K // 8):
            v = 0
            for i in range(8):
                v |= (int(q[n, 8 * w + i]) + 8) << order[i]
            words[n, w] = v
    packed = words.view(np.uint8).reshape(N, K // 2)
    assert np.array_equal(i8.unpack_int4_codes(packed), q)


def test_unpack_of_zero_bytes_is_minus_eight():
    # a byte of zeros is not a valid code (codes are q + 8 with q >= -7)
    assert np.all(i8.unpack_int4_codes(np.zeros((1, 4), dtype=np.uint8)) == -8)
