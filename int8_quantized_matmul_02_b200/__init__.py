"""LLM.int8() matrix multiplication for NVIDIA B200 (sm_100a).

Python face of ``libint8mm`` (C-ABI in ``include/int8mm.h``).  PyTorch is used
for device memory and streams only; every step of the product runs in the
library's CUDA kernels, and there is no CPU fallback.

Method: "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale"
(Dettmers et al., 2022), abstract -- vector-wise int8 quantisation plus a
16-bit matmul over the outlier feature dimensions, for the feed-forward and
attention-projection layers of a transformer.

    w  = prepare_weight(W_fp16_KxN, keep_idx)      # once, at load
    ws = Workspace(M, K, N)                         # reusable scratch
    Y  = forward(X_fp16_MxK, w, threshold=6.0, workspace=ws)
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _abi
from ._abi import PATH_AUTO, PATH_DECODE, PATH_GEMM, PATH_GEMM_1SM, Int8mmError

__all__ = [
    "PreparedWeight", "Workspace", "prepare_weight", "forward", "device_status", "library",
    "block_quantize", "block_dequantize",
    "Int4Weight", "prepare_weight_int4", "forward_int4", "unpack_int4_codes",
    "GroupedWeight", "prepare_weight_grouped", "forward_grouped",
    "Int8mmError", "PATH_AUTO", "PATH_GEMM", "PATH_DECODE",
]

_PATHS = {"auto": PATH_AUTO, "gemm": PATH_GEMM, "decode": PATH_DECODE, "gemm1sm": PATH_GEMM_1SM}


def library():
    """The loaded ctypes handle of libint8mm.so (raises if it is missing)."""
    return _abi.load()


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _view(buf: torch.Tensor, ptr: int, count: int, dtype: torch.dtype, shape=None) -> torch.Tensor:
    off = int(ptr) - buf.data_ptr()
    nbytes = count * torch.empty(0, dtype=dtype).element_size()
    t = buf[off: off + nbytes].view(dtype)
    return t.view(*shape) if shape is not None else t


class PreparedWeight:
    """An int8 weight in one device buffer (see ``int8mm_weight`` in the header)."""

    def __init__(self, buf: torch.Tensor, st: _abi.Weight):
        self.buf = buf
        self.struct = st
        self.K, self.N, self.n_keep = st.K, st.N, st.n_keep

    @property
    def wq(self) -> torch.Tensor:           # N x K int8
        return _view(self.buf, self.struct.wq, self.N * self.K, torch.int8, (self.N, self.K))

    @property
    def col_absmax(self) -> torch.Tensor:   # N float32
        return _view(self.buf, self.struct.col_absmax, self.N, torch.float32)

    @property
    def w_keep(self) -> torch.Tensor:       # n_keep x N fp16
        return _view(self.buf, self.struct.w_keep, self.n_keep * self.N, torch.float16, (self.n_keep, self.N))

    @property
    def keep_idx(self) -> torch.Tensor:
        return _view(self.buf, self.struct.keep_idx, self.n_keep, torch.int32)


def prepare_weight(W: torch.Tensor, keep_idx=(), stream=None) -> PreparedWeight:
    """Convert a K x N fp16 CUDA weight to int8 once (at load, per the LLM.int8() abstract)."""
    lib = _abi.load()
    if not (W.is_cuda and W.dtype == torch.float16 and W.dim() == 2 and W.is_contiguous()):
        raise ValueError("W must be a contiguous 2-D float16 CUDA tensor (K x N)")
    K, N = W.shape
    keep = np.unique(np.asarray(keep_idx, dtype=np.int64).ravel()).astype(np.int32)
    nbytes = lib.int8mm_weight_bytes(K, N, int(keep.size))
    if nbytes == 0:
        raise Int8mmError(1, f"int8mm_weight_bytes(K={K}, N={N}, n_keep={keep.size})")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    st = _abi.Weight()
    kp = keep.ctypes.data_as(ctypes.c_void_p) if keep.size else None
    with torch.cuda.device(W.device):
        _abi.check(lib.int8mm_prepare_weight(ctypes.c_void_p(W.data_ptr()), K, N, kp, int(keep.size),
                                             ctypes.c_void_p(buf.data_ptr()), nbytes, ctypes.byref(st),
                                             _stream(stream)), "int8mm_prepare_weight")
    return PreparedWeight(buf, st)


class Workspace:
    """Device scratch of one forward shape; zero-filled at creation."""

    def __init__(self, M: int, K: int, N: int, max_outliers: int | None = None, device=None, G: int | None = None):
        """G: group size of a group-wise forward (None: vector-wise)."""
        lib = _abi.load()
        self.M, self.K, self.N, self.G = M, K, N, G
        self.max_outliers = K if max_outliers is None else int(max_outliers)
        if G is None:
            self.nbytes = lib.int8mm_workspace_bytes(M, K, N, self.max_outliers)
        else:
            self.nbytes = lib.int8mm_grouped_workspace_bytes(M, K, N, int(G), self.max_outliers)
        if self.nbytes == 0:
            raise Int8mmError(1, f"workspace bytes (M={M}, K={K}, N={N}, max_outliers={self.max_outliers}, G={G})")
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device or "cuda")

    def reset(self, stream=None) -> None:
        """Zero the workspace again (needed after a forward reported a device error)."""
        with torch.cuda.device(self.buf.device):
            _abi.check(_abi.load().int8mm_workspace_init(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes,
                                                         _stream(stream)), "int8mm_workspace_init")

    def view(self) -> dict:
        """Torch views of the intermediates the last forward left in the workspace."""
        v = _abi.WorkspaceView()
        lib = _abi.load()
        if self.G is None:
            _abi.check(lib.int8mm_workspace_view_get(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes, self.M,
                                                     self.K, self.N, self.max_outliers, ctypes.byref(v)),
                       "int8mm_workspace_view_get")
        else:
            _abi.check(lib.int8mm_grouped_workspace_view_get(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes, self.M,
                                                             self.K, self.N, int(self.G), self.max_outliers,
                                                             ctypes.byref(v)), "int8mm_grouped_workspace_view_get")
        nr = 1 if self.G is None else self.K // self.G
        b = self.buf
        return {
            "status": _view(b, v.status, 1, torch.int32),
            "n_outliers": _view(b, v.n_outliers, 1, torch.int32),
            "outlier_idx": _view(b, v.outlier_idx, self.K, torch.int32),
            "row_absmax": (_view(b, v.row_absmax, self.M, torch.float32) if self.G is None else
                           _view(b, v.row_absmax, self.M * nr, torch.float32, (self.M, nr))),
            "xq": _view(b, v.xq, self.M * self.K, torch.int8, (self.M, self.K)),
            "xo": _view(b, v.xo, self.M * v.kp, torch.float16, (self.M, v.kp)) if v.kp else None,
            "kp": v.kp,
        }


def forward(X: torch.Tensor, w: PreparedWeight, threshold: float = 6.0, *, max_outliers: int | None = None,
            out: torch.Tensor | None = None, workspace: Workspace | None = None, path: str = "auto",
            acc_out: torch.Tensor | None = None, wait_limit_ns: int = 0, test_flags: int = 0,
            stream=None) -> torch.Tensor:
    """Y = X W by LLM.int8().  X: M x K fp16.  A CPU X goes through
    int8mm_forward_host (copy in, product, copy back in row bands that overlap
    the product) and a CPU Y (``out``, pinned if given, else a new pinned
    tensor) is returned once it is complete; a CUDA X stays on its device."""
    lib = _abi.load()
    on_host = not X.is_cuda
    dev = w.buf.device
    if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != w.K:
        raise ValueError(f"X must be float16 of shape (M, {w.K})")
    if not X.is_contiguous():
        raise ValueError("X must be contiguous")
    M = X.shape[0]
    if on_host:
        if acc_out is not None or path != "auto" or wait_limit_ns or test_flags:
            raise ValueError("a host X takes the default path and options")
        if workspace is None:
            workspace = Workspace(M, w.K, w.N, max_outliers, device=dev)
        if (workspace.M, workspace.K, workspace.N) != (M, w.K, w.N):
            raise ValueError("workspace was made for another shape")
        host = out if out is not None else torch.empty(M, w.N, dtype=torch.float16, pin_memory=True)
        if host.is_cuda or host.shape != (M, w.N) or host.dtype != torch.float16 or not host.is_contiguous():
            raise ValueError("out must be a contiguous CPU float16 tensor of shape (M, N) for a host X")
        Xd = torch.empty(M, w.K, dtype=torch.float16, device=dev)
        Yd = torch.empty(M, w.N, dtype=torch.float16, device=dev)
        with torch.cuda.device(dev):
            st = stream or torch.cuda.current_stream()
            _abi.check(lib.int8mm_forward_host(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(w.struct),
                                               float(threshold), workspace.max_outliers,
                                               ctypes.c_void_p(host.data_ptr()), ctypes.c_void_p(Xd.data_ptr()),
                                               ctypes.c_void_p(Yd.data_ptr()),
                                               ctypes.c_void_p(workspace.buf.data_ptr()), workspace.nbytes,
                                               _stream(stream)), "int8mm_forward_host")
            st.synchronize()
        return host
    Xd = X
    if workspace is None:
        workspace = Workspace(M, w.K, w.N, max_outliers, device=dev)
    if (workspace.M, workspace.K, workspace.N) != (M, w.K, w.N):
        raise ValueError("workspace was made for another shape")
    Y = out if out is not None else torch.empty(M, w.N, dtype=torch.float16, device=dev)
    opts = _abi.ForwardOpts(_PATHS[path], ctypes.c_void_p(acc_out.data_ptr()) if acc_out is not None else None,
                            int(wait_limit_ns), None, None, int(test_flags))
    with torch.cuda.device(dev):
        _abi.check(lib.int8mm_forward_ex(ctypes.c_void_p(Xd.data_ptr()), M, ctypes.byref(w.struct), float(threshold),
                                         workspace.max_outliers, ctypes.c_void_p(Y.data_ptr()),
                                         ctypes.c_void_p(workspace.buf.data_ptr()), workspace.nbytes,
                                         ctypes.byref(opts), _stream(stream)), "int8mm_forward")
    return Y


def device_status(workspace: Workspace, stream=None) -> tuple[int, int]:
    """(status code, detected outlier count) of the last forward; syncs the stream."""
    n = ctypes.c_int32(0)
    with torch.cuda.device(workspace.buf.device):
        st = _abi.load().int8mm_get_device_status(ctypes.c_void_p(workspace.buf.data_ptr()), _stream(stream),
                                                  ctypes.byref(n))
    return int(st), int(n.value)


# ---------------------------------------------------------------------------- block-wise 8-bit codec

def block_quantize(x: torch.Tensor, B: int, q: torch.Tensor | None = None, absmax: torch.Tensor | None = None,
                   stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Block-wise linear 8-bit codes of a float32 CUDA vector: block b covers
    [b*B, min(n, (b+1)*B)) and is normalised by its own absolute maximum
    (axolotl "llama3-model-quantization", "8-Bit Optimizers" paragraphs).
    Returns (codes int8 of n, absmax float32 of ceil(n/B))."""
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    n = x.numel()
    nb = (n + B - 1) // B
    q = torch.empty(n, dtype=torch.int8, device=x.device) if q is None else q
    absmax = torch.empty(nb, dtype=torch.float32, device=x.device) if absmax is None else absmax
    with torch.cuda.device(x.device):
        _abi.check(_abi.load().int8mm_block_quantize(ctypes.c_void_p(x.data_ptr()), n, int(B),
                                                     ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(absmax.data_ptr()),
                                                     _stream(stream)), "int8mm_block_quantize")
    return q, absmax


def block_dequantize(q: torch.Tensor, absmax: torch.Tensor, B: int, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """float32 values (q * absmax[block]) / 127 of block-wise codes."""
    if not (q.is_cuda and q.dtype == torch.int8 and q.is_contiguous()):
        raise ValueError("q must be a contiguous int8 CUDA tensor")
    n = q.numel()
    out = torch.empty(n, dtype=torch.float32, device=q.device) if out is None else out
    with torch.cuda.device(q.device):
        _abi.check(_abi.load().int8mm_block_dequantize(ctypes.c_void_p(q.data_ptr()),
                                                       ctypes.c_void_p(absmax.data_ptr()), n, int(B),
                                                       ctypes.c_void_p(out.data_ptr()), _stream(stream)),
                   "int8mm_block_dequantize")
    return out


# ---------------------------------------------------------------------------- 4-bit weight-only decode product

class Int4Weight:
    """A 4-bit weight in one device buffer (see ``int8mm_int4_weight``)."""

    def __init__(self, buf: torch.Tensor, st: _abi.Int4Weight):
        self.buf = buf
        self.struct = st
        self.K, self.N, self.G = st.K, st.N, st.G

    @property
    def codes(self) -> torch.Tensor:        # N x K/2 packed nibbles
        return _view(self.buf, self.struct.codes, self.N * self.K // 2, torch.uint8, (self.N, self.K // 2))

    @property
    def absmax(self) -> torch.Tensor:       # N x K/G float32
        return _view(self.buf, self.struct.absmax, self.N * (self.K // self.G), torch.float32,
                      (self.N, self.K // self.G))


def prepare_weight_int4(W: torch.Tensor, G: int, stream=None) -> Int4Weight:
    """Convert a K x N fp16 CUDA weight to 4-bit codes with one constant per
    output column and group of G consecutive k (once, at load)."""
    lib = _abi.load()
    if not (W.is_cuda and W.dtype == torch.float16 and W.dim() == 2 and W.is_contiguous()):
        raise ValueError("W must be a contiguous 2-D float16 CUDA tensor (K x N)")
    K, N = W.shape
    nbytes = lib.int8mm_int4_weight_bytes(K, N, int(G))
    if nbytes == 0:
        raise Int8mmError(1, f"int8mm_int4_weight_bytes(K={K}, N={N}, G={G})")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    st = _abi.Int4Weight()
    with torch.cuda.device(W.device):
        _abi.check(lib.int8mm_prepare_weight_int4(ctypes.c_void_p(W.data_ptr()), K, N, int(G),
                                                  ctypes.c_void_p(buf.data_ptr()), nbytes, ctypes.byref(st),
                                                  _stream(stream)), "int8mm_prepare_weight_int4")
    return Int4Weight(buf, st)


def forward_int4(X: torch.Tensor, w: Int4Weight, out: torch.Tensor | None = None,
                 status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X W' with the 4-bit weight (X: M x K fp16 on the weight's device,
    M <= 16).  ``status`` (int32 CUDA tensor of one zero word) receives
    device-side errors; a fresh one is used when it is None."""
    lib = _abi.load()
    if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != w.K or not X.is_cuda or not X.is_contiguous():
        raise ValueError(f"X must be a contiguous float16 CUDA tensor of shape (M, {w.K})")
    M = X.shape[0]
    Y = out if out is not None else torch.empty(M, w.N, dtype=torch.float16, device=X.device)
    status = status if status is not None else torch.zeros(1, dtype=torch.int32, device=X.device)
    with torch.cuda.device(X.device):
        _abi.check(lib.int8mm_forward_int4(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(w.struct),
                                           ctypes.c_void_p(Y.data_ptr()), ctypes.c_void_p(status.data_ptr()),
                                           _stream(stream)), "int8mm_forward_int4")
    return Y


def unpack_int4_codes(packed: np.ndarray) -> np.ndarray:
    """Codes q (N x K int8) from the packed layout (N x K/2 uint8) that
    ``int8mm_int4_weight`` documents; a layout helper, no arithmetic."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N, half = packed.shape
    words = packed.view("<u4").reshape(N, half // 4)
    q = np.empty((N, half * 2), dtype=np.int8)
    for i in range(8):
        shift = (i & 1) * 16 + (i >> 1) * 4
        q[:, i::8] = (((words >> shift) & 0xF).astype(np.int16) - 8).astype(np.int8)
    return q


# ---------------------------------------------------------------------------- group-wise variant

class GroupedWeight:
    """A group-wise int8 weight (see ``int8mm_grouped_weight``)."""

    def __init__(self, buf: torch.Tensor, st: _abi.GroupedWeight):
        self.buf = buf
        self.struct = st
        self.K, self.N, self.G, self.n_keep = st.K, st.N, st.G, st.n_keep

    @property
    def wq(self) -> torch.Tensor:           # N x K int8
        return _view(self.buf, self.struct.wq, self.N * self.K, torch.int8, (self.N, self.K))

    @property
    def col_absmax(self) -> torch.Tensor:   # (K/G) x N float32
        ng = self.K // self.G
        return _view(self.buf, self.struct.col_absmax, ng * self.N, torch.float32, (ng, self.N))

    @property
    def w_keep(self) -> torch.Tensor:
        return _view(self.buf, self.struct.w_keep, self.n_keep * self.N, torch.float16, (self.n_keep, self.N))

    @property
    def keep_idx(self) -> torch.Tensor:
        return _view(self.buf, self.struct.keep_idx, self.n_keep, torch.int32)


def prepare_weight_grouped(W: torch.Tensor, G: int, keep_idx=(), stream=None) -> GroupedWeight:
    """Convert a K x N fp16 CUDA weight to int8 with one constant per output
    column and group of G consecutive k (once, at load)."""
    lib = _abi.load()
    if not (W.is_cuda and W.dtype == torch.float16 and W.dim() == 2 and W.is_contiguous()):
        raise ValueError("W must be a contiguous 2-D float16 CUDA tensor (K x N)")
    K, N = W.shape
    keep = np.unique(np.asarray(keep_idx, dtype=np.int64).ravel()).astype(np.int32)
    nbytes = lib.int8mm_grouped_weight_bytes(K, N, int(G), int(keep.size))
    if nbytes == 0:
        raise Int8mmError(1, f"int8mm_grouped_weight_bytes(K={K}, N={N}, G={G}, n_keep={keep.size})")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    st = _abi.GroupedWeight()
    kp = keep.ctypes.data_as(ctypes.c_void_p) if keep.size else None
    with torch.cuda.device(W.device):
        _abi.check(lib.int8mm_prepare_weight_grouped(ctypes.c_void_p(W.data_ptr()), K, N, int(G), kp, int(keep.size),
                                                     ctypes.c_void_p(buf.data_ptr()), nbytes, ctypes.byref(st),
                                                     _stream(stream)), "int8mm_prepare_weight_grouped")
    return GroupedWeight(buf, st)


def forward_grouped(X: torch.Tensor, w: GroupedWeight, threshold: float = 6.0, *, max_outliers: int | None = None,
                    out: torch.Tensor | None = None, workspace: Workspace | None = None,
                    acc_out: torch.Tensor | None = None, wait_limit_ns: int = 0, test_flags: int = 0,
                    stream=None) -> torch.Tensor:
    """Y = X W by the group-wise method (X: M x K fp16 on the weight's device).
    acc_out (M x N x K/G int32), if given, receives the per-group int32 sums."""
    lib = _abi.load()
    if X.dtype != torch.float16 or X.dim() != 2 or X.shape[1] != w.K or not X.is_cuda or not X.is_contiguous():
        raise ValueError(f"X must be a contiguous float16 CUDA tensor of shape (M, {w.K})")
    M = X.shape[0]
    if workspace is None:
        workspace = Workspace(M, w.K, w.N, max_outliers, device=X.device, G=w.G)
    if (workspace.M, workspace.K, workspace.N, workspace.G) != (M, w.K, w.N, w.G):
        raise ValueError("workspace was made for another shape or group size")
    Y = out if out is not None else torch.empty(M, w.N, dtype=torch.float16, device=X.device)
    opts = _abi.ForwardOpts(0, ctypes.c_void_p(acc_out.data_ptr()) if acc_out is not None else None,
                            int(wait_limit_ns), None, None, int(test_flags))
    with torch.cuda.device(X.device):
        _abi.check(lib.int8mm_forward_grouped(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(w.struct),
                                              float(threshold), workspace.max_outliers, ctypes.c_void_p(Y.data_ptr()),
                                              ctypes.c_void_p(workspace.buf.data_ptr()), workspace.nbytes,
                                              ctypes.byref(opts), _stream(stream)), "int8mm_forward_grouped")
    return Y
