"""Host-only checks of the C-ABI: the library loads, exports every function
include/int8mm.h declares, and rejects bad arguments before it touches the
GPU (no compute call runs here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from int8_quantized_matmul_02_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int8mm.h")


def declared_functions() -> list[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(int8mm_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from int8_quantized_matmul_02_b200 import build

    build.build()
    return _abi.load()


def test_header_declares_the_binding_list():
    assert declared_functions() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in _abi.STATUS_NAMES.items():
        assert lib.int8mm_status_string(code).decode() == name
    assert lib.int8mm_status_string(99).decode() == "INT8MM_UNKNOWN_STATUS"
    assert lib.int8mm_version() >= 100


def test_weight_bytes_rules(lib):
    assert lib.int8mm_weight_bytes(256, 384, 2) >= 256 * 384 + 384 * 4 + 2 * 384 * 2 + 256 * 4
    assert lib.int8mm_weight_bytes(250, 384, 0) == 0      # K % 16
    assert lib.int8mm_weight_bytes(256, 100, 0) == 0      # N % 16
    assert lib.int8mm_weight_bytes(256, 384, 257) == 0    # n_keep > K
    assert lib.int8mm_weight_bytes(262144, 16, 0) == 0    # K too large for exact int32 sums


def test_workspace_bytes_rules(lib):
    small = lib.int8mm_workspace_bytes(16, 256, 384, 0)
    big = lib.int8mm_workspace_bytes(16, 256, 384, 256)
    assert 0 < small < big
    assert lib.int8mm_workspace_bytes(0, 256, 384, 0) == 0
    assert lib.int8mm_workspace_bytes(16, 256, 384, 257) == 0
    assert lib.int8mm_workspace_bytes(16, 256, 384, -1) == 0
    # the row-sized parts (codes, scales, fp16 outlier rows) grow with M
    assert lib.int8mm_workspace_bytes(4096, 256, 384, 64) > lib.int8mm_workspace_bytes(16, 256, 384, 64)


FAKE = 0x7F0000000000  # never dereferenced: every call below fails its argument checks first


def _weight(K=256, N=384, wq=FAKE):
    st = _abi.Weight()
    st.K, st.N, st.n_keep = K, N, 0
    st.wq = wq
    st.col_absmax = FAKE
    st.w_keep = FAKE
    st.keep_idx = FAKE
    st.keep_slot = FAKE
    return st


def _fwd(lib, X=FAKE, M=16, w=None, thr=6.0, cap=0, Y=FAKE, ws=FAKE, nbytes=1 << 30, opts=None):
    w = w or _weight()
    return lib.int8mm_forward_ex(ctypes.c_void_p(X), M, ctypes.byref(w), thr, cap, ctypes.c_void_p(Y),
                                 ctypes.c_void_p(ws), nbytes, ctypes.byref(opts) if opts else None, None)


def test_forward_rejects_bad_arguments(lib):
    assert _fwd(lib, X=0) == 1
    assert _fwd(lib, Y=0) == 1
    assert _fwd(lib, M=0) == 1
    assert _fwd(lib, thr=0.0) == 1
    assert _fwd(lib, thr=-1.0) == 1
    assert _fwd(lib, thr=float("nan")) == 1
    assert _fwd(lib, cap=257) == 1
    assert _fwd(lib, w=_weight(K=250)) == 1
    assert _fwd(lib, opts=_abi.ForwardOpts(7, None, 0)) == 1


def _fwd_host(lib, Xh=FAKE, M=16, w=None, thr=6.0, cap=0, Yh=FAKE, Xd=FAKE, Yd=FAKE, ws=FAKE, nbytes=1 << 30):
    w = w or _weight()
    return lib.int8mm_forward_host(ctypes.c_void_p(Xh), M, ctypes.byref(w), thr, cap, ctypes.c_void_p(Yh),
                                   ctypes.c_void_p(Xd), ctypes.c_void_p(Yd), ctypes.c_void_p(ws), nbytes, None)


def test_host_forward_rejects_bad_arguments_before_the_device(lib):
    """int8mm_forward_host checks every argument before it touches the
    device (so these calls return the same codes on a machine without one)."""
    assert _fwd_host(lib, Xh=0) == 1
    assert _fwd_host(lib, Yh=0) == 1
    assert _fwd_host(lib, Xd=0) == 1
    assert _fwd_host(lib, Yd=0) == 1
    assert _fwd_host(lib, ws=0) == 1
    assert _fwd_host(lib, M=0) == 1
    assert _fwd_host(lib, thr=float("nan")) == 1
    assert _fwd_host(lib, cap=257) == 1
    assert _fwd_host(lib, w=_weight(K=250)) == 1
    assert _fwd_host(lib, Xd=FAKE + 2) == 2       # device staging buffers: 16-byte aligned
    assert _fwd_host(lib, Yd=FAKE + 8) == 2
    assert _fwd_host(lib, ws=FAKE + 16) == 2
    need = lib.int8mm_workspace_bytes(16, 256, 384, 0)
    assert _fwd_host(lib, nbytes=need - 1) == 3


def test_forward_rejects_misaligned_pointers(lib):
    assert _fwd(lib, X=FAKE + 2) == 2
    assert _fwd(lib, Y=FAKE + 8) == 2
    assert _fwd(lib, ws=FAKE + 16) == 2
    assert _fwd(lib, w=_weight(wq=FAKE + 64)) == 2
    assert _fwd(lib, opts=_abi.ForwardOpts(0, FAKE + 4, 0)) == 2


def test_forward_rejects_small_workspace(lib):
    need = lib.int8mm_workspace_bytes(16, 256, 384, 0)
    assert _fwd(lib, nbytes=need - 1) == 3


def test_forced_decode_path_needs_small_m(lib):
    assert _fwd(lib, M=17, opts=_abi.ForwardOpts(_abi.PATH_DECODE, None, 0)) == 1


def test_forced_decode_path_needs_k_within_its_limit(lib):
    # a cluster of 8 CTAs splits K; each CTA's range must fit its X-side threads (K <= 20480)
    assert _fwd(lib, M=8, w=_weight(K=20608), opts=_abi.ForwardOpts(_abi.PATH_DECODE, None, 0)) == 1


def test_prepare_rejects_bad_keep_lists(lib):
    out = _abi.Weight()
    keep = (ctypes.c_int32 * 3)(5, 3, 9)  # not ascending
    assert lib.int8mm_prepare_weight(ctypes.c_void_p(FAKE), 256, 384, keep, 3, ctypes.c_void_p(FAKE), 1 << 30,
                                     ctypes.byref(out), None) == 1
    keep = (ctypes.c_int32 * 2)(5, 256)  # out of range
    assert lib.int8mm_prepare_weight(ctypes.c_void_p(FAKE), 256, 384, keep, 2, ctypes.c_void_p(FAKE), 1 << 30,
                                     ctypes.byref(out), None) == 1
    assert lib.int8mm_prepare_weight(ctypes.c_void_p(FAKE), 256, 384, None, 1, ctypes.c_void_p(FAKE), 1 << 30,
                                     ctypes.byref(out), None) == 1
    assert lib.int8mm_prepare_weight(ctypes.c_void_p(FAKE + 4), 256, 384, None, 0, ctypes.c_void_p(FAKE), 1 << 30,
                                     ctypes.byref(out), None) == 2
    assert lib.int8mm_prepare_weight(ctypes.c_void_p(FAKE), 256, 384, None, 0, ctypes.c_void_p(FAKE), 16,
                                     ctypes.byref(out), None) == 3


def test_view_and_init_argument_checks(lib):
    v = _abi.WorkspaceView()
    assert lib.int8mm_workspace_view_get(None, 1 << 20, 16, 256, 384, 0, ctypes.byref(v)) == 1
    assert lib.int8mm_workspace_view_get(ctypes.c_void_p(FAKE), 16, 16, 256, 384, 0, ctypes.byref(v)) == 3
    assert lib.int8mm_workspace_view_get(ctypes.c_void_p(FAKE), 1 << 30, 16, 256, 384, 64, ctypes.byref(v)) == 0
    assert v.kp == 64 and v.status == FAKE and v.n_outliers == FAKE + 4
    assert lib.int8mm_workspace_init(None, 16, None) == 1
    assert lib.int8mm_workspace_init(ctypes.c_void_p(FAKE + 8), 16, None) == 2
    assert lib.int8mm_get_device_status(None, None, None) == 1


def test_product_path_has_no_oracle_dependency():
    """The package never imports the oracle: no CPU fallback exists."""
    pkg = os.path.join(ROOT, "int8_quantized_matmul_02_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
