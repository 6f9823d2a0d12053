"""CPU oracle for the LLM.int8() matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path never does: the GPU library
has no CPU fallback.

The arithmetic lives in ``int8mm_oracle.c`` (plain C, ``-O2
-ffp-contract=off``, no fast-math); this module compiles it on first use and
wraps each step with numpy arrays.  fp16 arrays cross the boundary as their
raw 16-bit patterns.  Each wrapper names the passage it follows:

* outlier detection -- axolotl "llama3-model-quantization", "Understanding
  Outliers in Transformer Models": outliers sit in specific feature columns;
* row / column quantisation -- "LLM.int8(): 8-bit Matrix Multiplication for
  Transformers at Scale", abstract (vector-wise quantisation: every inner
  product gets its own normalisation constants), max normalisation from the
  axolotl page's "Key Points", round-to-nearest from the nuQmm scite report;
* 16-bit outlier product -- the same abstract (the mixed-precision
  decomposition moves the outlier feature dimensions into a matmul in 16 bit);
* weight conversion once at load -- the same abstract (a 16-bit checkpoint is
  turned into int8 when it is loaded and used from then on);
* block-wise 8-bit codec -- the axolotl page's "8-Bit Optimizers" paragraphs
  (blocks normalised by their own maximum, an 8-bit index per value);
* group-wise matmul -- the scite report for nuQmm (nuQmm / ZeroQuant use one
  constant per group, finer than vector-wise; GPTQ's grouping of consecutive
  weights);
* 4-bit weight-only product -- the talk's "4-Bit Inference" and the axolotl
  page's "Impact of Precision and Parameter Count" (weight loading dominates
  inference, so bits per weight set its time).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "int8mm_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared", "-pthread"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_build/liboracle.so``; return its path."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _setup(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    F = ctypes.c_float
    lib.orc_half_to_float.argtypes = [ctypes.c_uint16]
    lib.orc_half_to_float.restype = F
    lib.orc_float_to_half.argtypes = [F]
    lib.orc_float_to_half.restype = ctypes.c_uint16
    lib.orc_detect_outliers.argtypes = [P, I, I, F, P]
    lib.orc_detect_outliers.restype = I
    lib.orc_quantize_rows.argtypes = [P, I, I, P, I, P, P, P]
    lib.orc_quantize_rows.restype = None
    lib.orc_quantize_weight.argtypes = [P, I, I, P, P]
    lib.orc_quantize_weight.restype = None
    lib.orc_int8_gemm.argtypes = [P, P, I, I, I, P, I]
    lib.orc_int8_gemm.restype = I
    lib.orc_int8_gemm_points.argtypes = [P, P, I, P, P, I, P]
    lib.orc_int8_gemm_points.restype = I
    lib.orc_gather_w_outlier.argtypes = [P, P, I, P, P, I, I, P, I, P]
    lib.orc_gather_w_outlier.restype = None
    lib.orc_outlier_gemm.argtypes = [P, P, I, I, I, P]
    lib.orc_outlier_gemm.restype = None
    lib.orc_epilogue.argtypes = [P, P, P, P, I, I, P]
    lib.orc_epilogue.restype = None
    lib.orc_forward_points.argtypes = [P, P, P, P, P, P, I, I, I, P, P, I, P, P]
    lib.orc_forward_points.restype = I
    L = ctypes.c_long
    lib.orc_block_quantize.argtypes = [P, L, I, P, P]
    lib.orc_block_quantize.restype = None
    lib.orc_block_dequantize.argtypes = [P, P, L, I, P]
    lib.orc_block_dequantize.restype = None
    lib.orc_quantize_rows_grouped.argtypes = [P, I, I, I, P, I, P, P, P]
    lib.orc_quantize_rows_grouped.restype = None
    lib.orc_quantize_weight_grouped.argtypes = [P, I, I, I, P, P]
    lib.orc_quantize_weight_grouped.restype = None
    lib.orc_gather_w_outlier_grouped.argtypes = [P, P, I, P, P, I, I, I, P, I, P]
    lib.orc_gather_w_outlier_grouped.restype = None
    lib.orc_grouped_forward.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
    lib.orc_grouped_forward.restype = I
    lib.orc_double_to_half.argtypes = [ctypes.c_double]
    lib.orc_double_to_half.restype = ctypes.c_uint16
    lib.orc_quantize_weight_int4.argtypes = [P, I, I, I, P, P]
    lib.orc_quantize_weight_int4.restype = None
    lib.orc_int4_product.argtypes = [P, P, P, I, I, I, I, P]
    lib.orc_int4_product.restype = None
    lib.orc_grouped_points.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P, I, P, P]
    lib.orc_grouped_points.restype = I
    lib.orc_int4_points.argtypes = [P, P, P, I, I, P, P, I, P]
    lib.orc_int4_points.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _setup(ctypes.CDLL(build()))
    return _lib


def _swap_library(path):
    """Test hook: route every wrapper through another build of the oracle
    source (``None`` restores the default build).  Only the pin-strength test
    uses it, to show that deliberately broken copies fail the pins."""
    global _lib
    with _lock:
        _lib = None if path is None else _setup(ctypes.CDLL(path))


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(0)


def _bits(h: np.ndarray) -> np.ndarray:
    """fp16 array -> contiguous uint16 bit patterns."""
    return np.ascontiguousarray(h, dtype=np.float16).view(np.uint16)


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------
# scalar fp16 conversions
# --------------------------------------------------------------------------

def half_to_float(bits: int) -> float:
    return float(_load().orc_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(_load().orc_float_to_half(float(x)))


# --------------------------------------------------------------------------
# the steps of the forward pass
# --------------------------------------------------------------------------

def detect_outliers(X: np.ndarray, threshold: float) -> np.ndarray:
    """(a) ascending int32 list of columns k with |X[m,k]| >= threshold for some m."""
    xb = _bits(X)
    M, K = xb.shape
    idx = np.zeros(max(K, 1), dtype=np.int32)
    n = _load().orc_detect_outliers(_ptr(xb), M, K, float(threshold), _ptr(idx))
    return idx[:n].copy()


def quantize_rows(X: np.ndarray, idx: np.ndarray):
    """(b) -> (Xq int8 MxK, ra float32 M, Xo float16 M x n_o)."""
    xb = _bits(X)
    M, K = xb.shape
    idx = _c(idx, np.int32)
    n_o = int(idx.size)
    Xq = np.zeros((M, K), dtype=np.int8)
    ra = np.zeros(M, dtype=np.float32)
    Xo = np.zeros((M, n_o), dtype=np.uint16)
    _load().orc_quantize_rows(_ptr(xb), M, K, _ptr(idx), n_o, _ptr(Xq), _ptr(ra), _ptr(Xo))
    return Xq, ra, Xo.view(np.float16)


def quantize_weight(W: np.ndarray):
    """(c) W (K x N fp16) -> (Wq int8 N x K, ca float32 N)."""
    wb = _bits(W)
    K, N = wb.shape
    Wq = np.zeros((N, K), dtype=np.int8)
    ca = np.zeros(N, dtype=np.float32)
    _load().orc_quantize_weight(_ptr(wb), K, N, _ptr(Wq), _ptr(ca))
    return Wq, ca


def prepare_weight(W: np.ndarray, keep_idx) -> dict:
    """One-time conversion of a 16-bit weight: int8 codes, scales and kept fp16 rows."""
    Wq, ca = quantize_weight(W)
    keep = np.asarray(sorted(set(int(k) for k in np.asarray(keep_idx).ravel())), dtype=np.int32)
    w_keep = np.ascontiguousarray(np.asarray(W, dtype=np.float16)[keep, :])
    return {"K": W.shape[0], "N": W.shape[1], "wq": Wq, "ca": ca, "keep_idx": keep, "w_keep": w_keep}


def int8_gemm(Xq: np.ndarray, Wq: np.ndarray, threads: int | None = None) -> np.ndarray:
    """(d1) exact int32 acc = Xq (M x K) . Wq (N x K)^T."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    assert Wq.shape[1] == K
    acc = np.zeros((M, N), dtype=np.int32)
    rc = _load().orc_int8_gemm(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), int(threads or default_threads()))
    if rc != 0:
        raise OverflowError("int8 product does not fit int32")
    return acc


def int8_gemm_points(Xq, Wq, pm, pn) -> np.ndarray:
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    pm = _c(pm, np.int32)
    pn = _c(pn, np.int32)
    acc = np.zeros(pm.size, dtype=np.int32)
    rc = _load().orc_int8_gemm_points(_ptr(Xq), _ptr(Wq), Xq.shape[1], _ptr(pm), _ptr(pn), pm.size, _ptr(acc))
    if rc != 0:
        raise OverflowError("int8 product does not fit int32")
    return acc


def gather_w_outlier(prep: dict, idx: np.ndarray) -> np.ndarray:
    """fp16 weight rows of the outlier dims: Wo (n_o x N)."""
    idx = _c(idx, np.int32)
    keep = _c(prep["keep_idx"], np.int32)
    wk = _bits(prep["w_keep"]) if keep.size else np.zeros((0, prep["N"]), dtype=np.uint16)
    Wo = np.zeros((idx.size, prep["N"]), dtype=np.uint16)
    _load().orc_gather_w_outlier(_ptr(wk), _ptr(keep), keep.size, _ptr(_c(prep["wq"], np.int8)),
                                 _ptr(_c(prep["ca"], np.float32)), prep["K"], prep["N"], _ptr(idx),
                                 idx.size, _ptr(Wo))
    return Wo.view(np.float16)


def outlier_gemm(Xo: np.ndarray, Wo: np.ndarray) -> np.ndarray:
    """(d2) fp32 o = Xo (M x n_o) . Wo (n_o x N), ascending outlier order."""
    xb = _bits(Xo)
    wb = _bits(Wo)
    M, n_o = xb.shape
    N = wb.shape[1]
    o = np.zeros((M, N), dtype=np.float32)
    _load().orc_outlier_gemm(_ptr(xb), _ptr(wb), M, N, n_o, _ptr(o))
    return o


def epilogue(acc, ra, ca, o=None) -> np.ndarray:
    """(d3) Y = fp16(acc * ra[m] * ca[n] / 16129 + o)."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    ra = _c(ra, np.float32)
    ca = _c(ca, np.float32)
    op = ctypes.c_void_p(0)
    if o is not None:
        o = _c(o, np.float32)
        op = _ptr(o)
    Y = np.zeros((M, N), dtype=np.uint16)
    _load().orc_epilogue(_ptr(acc), _ptr(ra), _ptr(ca), op, M, N, _ptr(Y))
    return Y.view(np.float16)


def forward(X: np.ndarray, prep: dict, threshold: float, threads: int | None = None) -> dict:
    """The whole forward pass; returns every intermediate and Y."""
    idx = detect_outliers(X, threshold)
    Xq, ra, Xo = quantize_rows(X, idx)
    acc = int8_gemm(Xq, prep["wq"], threads)
    Wo = gather_w_outlier(prep, idx)
    o = outlier_gemm(Xo, Wo)
    Y = epilogue(acc, ra, prep["ca"], o)
    return {"idx": idx, "xq": Xq, "ra": ra, "xo": Xo, "acc": acc, "wo": Wo, "o": o, "y": Y}


def forward_points(X_steps: dict, prep: dict, pm, pn):
    """acc and Y at the sampled points (pm[i], pn[i]) from the (a)-(c) results."""
    pm = _c(pm, np.int32)
    pn = _c(pn, np.int32)
    Xq = _c(X_steps["xq"], np.int8)
    ra = _c(X_steps["ra"], np.float32)
    xo = _bits(X_steps["xo"])
    wo = _bits(X_steps["wo"])
    n_o = xo.shape[1]
    acc = np.zeros(pm.size, dtype=np.int32)
    y = np.zeros(pm.size, dtype=np.uint16)
    rc = _load().orc_forward_points(_ptr(Xq), _ptr(ra), _ptr(_c(prep["wq"], np.int8)),
                                    _ptr(_c(prep["ca"], np.float32)), _ptr(xo), _ptr(wo),
                                    Xq.shape[1], prep["N"], n_o, _ptr(pm), _ptr(pn), pm.size,
                                    _ptr(acc), _ptr(y))
    if rc != 0:
        raise OverflowError("int8 product does not fit int32")
    return acc, y.view(np.float16)


def forward_steps_abc(X: np.ndarray, prep: dict, threshold: float) -> dict:
    """Steps (a), (b) and the outlier weight rows in full, without the int8 product."""
    idx = detect_outliers(X, threshold)
    Xq, ra, Xo = quantize_rows(X, idx)
    Wo = gather_w_outlier(prep, idx)
    return {"idx": idx, "xq": Xq, "ra": ra, "xo": Xo, "wo": Wo}



# --------------------------------------------------------------------------
# block-wise 8-bit codec
# --------------------------------------------------------------------------

def block_quantize(x: np.ndarray, B: int):
    """fp32 vector -> (codes int8 n, absmax float32 ceil(n/B)); block b covers
    [b*B, min(n, (b+1)*B)), each normalised by its own maximum."""
    x = _c(np.ravel(x), np.float32)
    n = int(x.size)
    assert B >= 1
    q = np.zeros(n, dtype=np.int8)
    amax = np.zeros((n + B - 1) // B, dtype=np.float32)
    _load().orc_block_quantize(_ptr(x), n, int(B), _ptr(q), _ptr(amax))
    return q, amax


def block_dequantize(q: np.ndarray, absmax: np.ndarray, B: int) -> np.ndarray:
    """x' = (q * absmax[block]) / 127 in fp32."""
    q = _c(np.ravel(q), np.int8)
    absmax = _c(absmax, np.float32)
    n = int(q.size)
    assert absmax.size == (n + B - 1) // B
    out = np.zeros(n, dtype=np.float32)
    _load().orc_block_dequantize(_ptr(q), _ptr(absmax), n, int(B), _ptr(out))
    return out


# --------------------------------------------------------------------------
# group-wise matmul (one constant per G consecutive inner-product indices)
# --------------------------------------------------------------------------

def quantize_rows_grouped(X: np.ndarray, idx: np.ndarray, G: int):
    """-> (Xq int8 MxK, ra float32 M x K/G, Xo float16 M x n_o)."""
    xb = _bits(X)
    M, K = xb.shape
    assert G >= 1 and K % G == 0
    idx = _c(idx, np.int32)
    Xq = np.zeros((M, K), dtype=np.int8)
    ra = np.zeros((M, K // G), dtype=np.float32)
    Xo = np.zeros((M, idx.size), dtype=np.uint16)
    _load().orc_quantize_rows_grouped(_ptr(xb), M, K, int(G), _ptr(idx), idx.size, _ptr(Xq), _ptr(ra), _ptr(Xo))
    return Xq, ra, Xo.view(np.float16)


def quantize_weight_grouped(W: np.ndarray, G: int):
    """W (K x N fp16) -> (Wq int8 N x K, ca float32 N x K/G)."""
    wb = _bits(W)
    K, N = wb.shape
    assert G >= 1 and K % G == 0
    Wq = np.zeros((N, K), dtype=np.int8)
    ca = np.zeros((N, K // G), dtype=np.float32)
    _load().orc_quantize_weight_grouped(_ptr(wb), K, N, int(G), _ptr(Wq), _ptr(ca))
    return Wq, ca


def prepare_weight_grouped(W: np.ndarray, keep_idx, G: int) -> dict:
    Wq, ca = quantize_weight_grouped(W, G)
    keep = np.asarray(sorted(set(int(k) for k in np.asarray(keep_idx).ravel())), dtype=np.int32)
    w_keep = np.ascontiguousarray(np.asarray(W, dtype=np.float16)[keep, :])
    return {"K": W.shape[0], "N": W.shape[1], "G": int(G), "wq": Wq, "ca": ca, "keep_idx": keep, "w_keep": w_keep}


def gather_w_outlier_grouped(prep: dict, idx: np.ndarray) -> np.ndarray:
    idx = _c(idx, np.int32)
    keep = _c(prep["keep_idx"], np.int32)
    wk = _bits(prep["w_keep"]) if keep.size else np.zeros((0, prep["N"]), dtype=np.uint16)
    Wo = np.zeros((idx.size, prep["N"]), dtype=np.uint16)
    _load().orc_gather_w_outlier_grouped(_ptr(wk), _ptr(keep), keep.size, _ptr(_c(prep["wq"], np.int8)),
                                         _ptr(_c(prep["ca"], np.float32)), prep["K"], prep["N"], prep["G"],
                                         _ptr(idx), idx.size, _ptr(Wo))
    return Wo.view(np.float16)


def grouped_product(Xq, ra, Wq, ca, G: int, o=None):
    """-> (acc int32 M x N x K/G, Y float16 M x N)."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    assert Wq.shape[1] == K and K % G == 0
    ng = K // G
    ra = _c(ra, np.float32)
    ca = _c(ca, np.float32)
    assert ra.shape == (M, ng) and ca.shape == (N, ng)
    op = ctypes.c_void_p(0)
    if o is not None:
        o = _c(o, np.float32)
        op = _ptr(o)
    acc = np.zeros((M, N, ng), dtype=np.int32)
    Y = np.zeros((M, N), dtype=np.uint16)
    rc = _load().orc_grouped_forward(_ptr(Xq), _ptr(ra), _ptr(Wq), _ptr(ca), op, M, N, K, int(G), _ptr(acc), _ptr(Y))
    if rc != 0:
        raise OverflowError("a group sum does not fit int32")
    return acc, Y.view(np.float16)


def forward_grouped_points(steps: dict, prep: dict, pm, pn):
    """acc_g (npts x K/G) and Y at the points (pm[i], pn[i]) from the X-side
    results of the group-wise forward (xq, ra, xo, wo)."""
    G = prep["G"]
    pm = _c(pm, np.int32)
    pn = _c(pn, np.int32)
    Xq = _c(steps["xq"], np.int8)
    K = Xq.shape[1]
    xo = _bits(steps["xo"])
    wo = _bits(steps["wo"])
    acc = np.zeros((pm.size, K // G), dtype=np.int32)
    y = np.zeros(pm.size, dtype=np.uint16)
    rc = _load().orc_grouped_points(_ptr(Xq), _ptr(_c(steps["ra"], np.float32)), _ptr(_c(prep["wq"], np.int8)),
                                    _ptr(_c(prep["ca"], np.float32)), _ptr(xo), _ptr(wo), K, prep["N"], G,
                                    xo.shape[1], _ptr(pm), _ptr(pn), pm.size, _ptr(acc), _ptr(y))
    if rc != 0:
        raise OverflowError("a group sum does not fit int32")
    return acc, y.view(np.float16)


def forward_grouped(X: np.ndarray, prep: dict, threshold: float) -> dict:
    """The group-wise forward pass; returns every intermediate and Y."""
    G = prep["G"]
    idx = detect_outliers(X, threshold)
    Xq, ra, Xo = quantize_rows_grouped(X, idx, G)
    Wo = gather_w_outlier_grouped(prep, idx)
    o = outlier_gemm(Xo, Wo)
    acc, Y = grouped_product(Xq, ra, prep["wq"], prep["ca"], G, o)
    return {"idx": idx, "xq": Xq, "ra": ra, "xo": Xo, "acc": acc, "wo": Wo, "o": o, "y": Y}


# --------------------------------------------------------------------------
# 4-bit weight-only product
# --------------------------------------------------------------------------

def double_to_half(x: float) -> int:
    return int(_load().orc_double_to_half(float(x)))


def quantize_weight_int4(W: np.ndarray, G: int):
    """W (K x N fp16) -> (codes int8 N x K in [-7, 7], ca float32 N x K/G)."""
    wb = _bits(W)
    K, N = wb.shape
    assert G >= 1 and K % G == 0
    q = np.zeros((N, K), dtype=np.int8)
    ca = np.zeros((N, K // G), dtype=np.float32)
    _load().orc_quantize_weight_int4(_ptr(wb), K, N, int(G), _ptr(q), _ptr(ca))
    return q, ca


def int4_product(X: np.ndarray, q: np.ndarray, ca: np.ndarray, G: int) -> np.ndarray:
    """Y (M x N fp16) = X (M x K fp16) times the dequantised 4-bit weight."""
    xb = _bits(X)
    M, K = xb.shape
    q = _c(q, np.int8)
    N = q.shape[0]
    assert q.shape[1] == K and K % G == 0
    ca = _c(ca, np.float32)
    assert ca.shape == (N, K // G)
    Y = np.zeros((M, N), dtype=np.uint16)
    _load().orc_int4_product(_ptr(xb), _ptr(q), _ptr(ca), M, N, K, int(G), _ptr(Y))
    return Y.view(np.float16)


def int4_points(X: np.ndarray, q: np.ndarray, ca: np.ndarray, G: int, pm, pn) -> np.ndarray:
    """Y of the 4-bit weight-only product at the points (pm[i], pn[i])."""
    xb = _bits(X)
    K = xb.shape[1]
    q = _c(q, np.int8)
    pm = _c(pm, np.int32)
    pn = _c(pn, np.int32)
    y = np.zeros(pm.size, dtype=np.uint16)
    _load().orc_int4_points(_ptr(xb), _ptr(q), _ptr(_c(ca, np.float32)), K, int(G), _ptr(pm), _ptr(pn), pm.size, _ptr(y))
    return y.view(np.float16)
