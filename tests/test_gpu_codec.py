"""GPU parity of the block-wise 8-bit codec (axolotl "llama3-model-quantization",
"8-Bit Optimizers" paragraphs: blocks normalised by their own maximum, an 8-bit
index per value) against the CPU oracle: codes, block absmax and dequantised
values bit for bit, on the same seeded inputs."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
import int8_quantized_matmul_02_b200 as i8

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _vector(n: int, seed: int) -> torch.Tensor:
    """Heavy-tailed values (N(0,1) * exp(N(0,1))), 5 % exact zeros, one block
    of zeros, dyadic values that land on rounding ties, and a few x50 outliers."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, generator=g) * torch.exp(torch.randn(n, generator=g))
    x[torch.rand(n, generator=g) < 0.05] = 0.0
    x[torch.rand(n, generator=g) < 0.001] *= 50.0
    ties = torch.rand(n, generator=g) < 0.1
    x[ties] = torch.randint(-64, 65, (int(ties.sum()),), generator=g).float() / 4.0
    if n >= 64:
        x[16:48] = 0.0
    return x.contiguous()


def _check(x: torch.Tensor, B: int) -> None:
    q_ref, a_ref = oracle.block_quantize(x.numpy(), B)
    q, a = i8.block_quantize(x.cuda(), B)
    assert np.array_equal(q.cpu().numpy(), q_ref), "codes differ"
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32)), "absmax differs"
    d_ref = oracle.block_dequantize(q_ref, a_ref, B)
    d = i8.block_dequantize(q, a, B)
    assert np.array_equal(d.cpu().numpy().view(np.uint32), d_ref.view(np.uint32)), "dequantised values differ"


def test_block_codec_golden(cuda_ok):
    with open(os.path.join(GOLDEN, "blockwise_codec_14x4.json")) as f:
        g = json.load(f)
    x = torch.tensor(g["x"], dtype=torch.float32)
    q, a = i8.block_quantize(x.cuda(), g["B"])
    assert q.cpu().tolist() == g["expected"]["codes"]
    assert a.cpu().double().tolist() == g["expected"]["absmax"]
    assert i8.block_dequantize(q, a, g["B"]).cpu().double().tolist() == g["expected"]["dequantised"]


@pytest.mark.parametrize("n,B", [
    (1, 4), (13, 4), (14, 8),                 # shorter than a block, ragged tails
    (4096, 128), (65_537, 64), (777, 1000),
    (100_003, 2048), (10_000, 4096),          # blocks held in registers (up to 16 float4 per lane)
    (50_001, 8192), (123_457, 2052),          # blocks longer than the registers hold: a second read
    (1 << 20, 2048),
])
def test_block_codec_matches_oracle(cuda_ok, n, B):
    _check(_vector(n, seed=n * 7 + B), B)


def test_block_codec_full_size_sampled(cuda_ok):
    """The benchmark's workload (n = 4096 * 12288 fp32, B = 2048): every code,
    absmax and dequantised value against the oracle."""
    n, B = 4096 * 12288, 2048
    _check(_vector(n, seed=1234), B)


def test_block_codec_rejects_bad_arguments(cuda_ok):
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(i8.Int8mmError):
        i8.block_quantize(x, 6)       # B not a multiple of 4
    with pytest.raises(i8.Int8mmError):
        i8.block_quantize(x[1:], 8)   # x not 16-byte aligned
