"""Seeded synthetic inputs for the LLM.int8() matmul workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CPU oracle and the CUDA path can take their inputs from
it.  Everything is drawn with a ``torch.Generator`` on the CPU, so any two
consumers see identical bits.

Workload recipe (shapes are X: M x K, W: K x N, Y = X W):

* background activations X ~ N(0, 1), weights W ~ N(0, sigma), both rounded
  to fp16;
* ``n_seed`` outlier feature columns drawn as ``randperm(K)[:n_seed]``,
  sorted -- outliers concentrate in a few feature dimensions (axolotl
  "llama3-model-quantization", "Understanding Outliers in Transformer
  Models");
* outlier values, per ``mode``:
  - ``"scale"``: the column is multiplied by ``lo`` (tiny case, x40);
  - ``"element"``: sign of the background value times U(lo, hi);
  - ``"row"``: one random sign per row, shared by the row's outlier columns,
    times U(lo, hi);
* ``keep_idx`` (the fp16 weight rows kept at preparation time) is the seeded
  outlier column list.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    n_seed: int
    lo: float
    hi: float
    mode: str          # "scale" | "element" | "row"
    sigma_w: float
    threshold: float
    seed: int

    @property
    def ops(self) -> float:
        """int8 multiply-adds counted as 2 ops over all K."""
        return 2.0 * self.M * self.N * self.K


def _wl(name, idx, M, K, N, n_seed, lo, hi, mode, sigma, thr=6.0, sweep=0):
    return Workload(name, M, K, N, n_seed, lo, hi, mode, sigma, thr, idx * 1000 + sweep)


WORKLOADS = {
    "tiny": _wl("tiny", 0, 16, 256, 384, 2, 40.0, 40.0, "scale", 0.02),
    "decode": _wl("decode", 1, 8, 4096, 11008, 6, 20.0, 60.0, "element", 0.02),
    "prefill": _wl("prefill", 2, 2048, 8192, 28672, 8, 20.0, 60.0, "row", 0.015),
    "175b": _wl("175b", 3, 4096, 12288, 49152, 24, 10.0, 60.0, "element", 0.01),
}
for _n in (0, 12, 48, 123):
    WORKLOADS[f"qkv_o{_n}"] = _wl(f"qkv_o{_n}", 4, 16384, 12288, 36864, _n, 10.0, 60.0, "element", 0.01, sweep=_n)
WORKLOADS["qkv_inf"] = replace(WORKLOADS["qkv_o0"], name="qkv_inf", threshold=math.inf, seed=4 * 1000 + 999)


def make_activations(M: int, K: int, n_seed: int, lo: float, hi: float, mode: str,
                     gen: torch.Generator) -> tuple[torch.Tensor, np.ndarray]:
    """X (M x K fp16, CPU) and its sorted seeded outlier columns."""
    x = torch.randn(M, K, generator=gen, dtype=torch.float32)
    cols = torch.randperm(K, generator=gen)[:n_seed].sort().values
    if n_seed:
        if mode == "scale":
            x[:, cols] *= lo
        else:
            mag = torch.empty(M, n_seed, dtype=torch.float32).uniform_(lo, hi, generator=gen)
            if mode == "element":
                sign = torch.where(x[:, cols] >= 0, 1.0, -1.0)
            elif mode == "row":
                sign = torch.where(torch.rand(M, 1, generator=gen) < 0.5, -1.0, 1.0)
            else:
                raise ValueError(f"unknown outlier mode {mode!r}")
            x[:, cols] = sign * mag
    return x.to(torch.float16), cols.numpy().astype(np.int32)


def make_weight(K: int, N: int, sigma: float, gen: torch.Generator) -> torch.Tensor:
    """W (K x N fp16, CPU) ~ N(0, sigma)."""
    w = torch.randn(K, N, generator=gen, dtype=torch.float32)
    w.mul_(sigma)
    return w.to(torch.float16)


def make_inputs(wl: Workload):
    """(X, W, keep_idx) for a workload, all on the CPU."""
    gen = torch.Generator().manual_seed(wl.seed)
    X, cols = make_activations(wl.M, wl.K, wl.n_seed, wl.lo, wl.hi, wl.mode, gen)
    W = make_weight(wl.K, wl.N, wl.sigma_w, gen)
    return X, W, cols


def make_case(M: int, K: int, N: int, n_seed: int = 0, lo: float = 10.0, hi: float = 60.0,
              mode: str = "element", sigma_w: float = 0.02, seed: int = 0):
    """A free-form seeded case for tests: (X, W, keep_idx)."""
    wl = Workload("case", M, K, N, n_seed, lo, hi, mode, sigma_w, 6.0, seed)
    return make_inputs(wl)


def sample_points(M: int, N: int, count: int, seed: int, tiles=((128, 256),)):
    """Seeded output coordinates: whole tiles at random positions plus points.

    Returns (pm, pn) int32 arrays.  Tiles are clipped to the matrix.
    """
    g = np.random.default_rng(seed)
    pm, pn = [], []
    for th, tw in tiles:
        m0 = int(g.integers(0, max(1, M - th + 1))) // th * th if M > th else 0
        n0 = int(g.integers(0, max(1, N - tw + 1))) // tw * tw if N > tw else 0
        mm, nn = np.meshgrid(np.arange(m0, min(M, m0 + th)), np.arange(n0, min(N, n0 + tw)), indexing="ij")
        pm.append(mm.ravel())
        pn.append(nn.ravel())
    pm.append(g.integers(0, M, count))
    pn.append(g.integers(0, N, count))
    # the last row / column, so the ragged edge is always sampled
    pm.append(np.array([M - 1, M - 1, 0]))
    pn.append(np.array([N - 1, 0, N - 1]))
    return np.concatenate(pm).astype(np.int32), np.concatenate(pn).astype(np.int32)


# ----------------------------------------------------------------------------- variants of the path

# The 4-bit weight-only product runs on the decode workload's X and W; its
# group size is the one the scite report for nuQmm quotes from GPTQ (1024),
# with 128 as the finer setting.
INT4_GROUPS = (1024, 128)

# Group-wise variant: the 175B-scale FFN shape with groups of 1024 (the group
# size of the scite report's GPTQ snippet) and of 128 (a finer setting).
GROUP_SIZES = (1024, 128)

# Block-wise codec workload: the fp32 state of one weight of the 175B-scale FFN
# (4096 x 12288 values), blocks of 2048.
CODEC_N = 4096 * 12288
CODEC_BLOCK = 2048
CODEC_SEED = 5000


def make_codec_vector(n: int = CODEC_N, seed: int = CODEC_SEED) -> torch.Tensor:
    """A heavy-tailed fp32 vector, N(0,1) * exp(N(0,1)), with 0.1 % of the
    values multiplied by 50: an optimizer state whose outliers would waste the
    bits of a single global constant (axolotl "llama3-model-quantization",
    "8-Bit Optimizers" paragraphs)."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(n, generator=gen) * torch.exp(torch.randn(n, generator=gen))
    pick = torch.rand(n, generator=gen) < 0.001
    x[pick] *= 50.0
    return x.contiguous()
