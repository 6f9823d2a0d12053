"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI
and the CPU oracle on the same seeded inputs, and compare.

Bar (LLM.int8() forward): outlier list, outlier count, int8 codes, scales and
int32 sums bit-exact; fp16 Y within
    |y - y_ref| <= 2^-9 |y_ref| + 1e-3 rms(y_ref)
since the fp16 outlier product may be summed in another order, and the GPU
applies ra * ca / 127^2 in another order than the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import int8_quantized_matmul_02_b200 as i8

REL_TOL = 2.0 ** -9
RMS_TOL = 1e-3


def assert_y_close(y: np.ndarray, y_ref: np.ndarray, what: str = "Y") -> float:
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + RMS_TOL * rms
    bad = err > bound
    if bad.any():
        i = np.unravel_index(int(np.argmax(err - bound)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {y.size} outside tolerance; worst at {i}: "
                             f"got {y[i]}, want {y_ref[i]}, bound {bound[i]}")
    return float((err / np.maximum(bound, 1e-30)).max()) if err.size else 0.0


def gpu_prepare(W: torch.Tensor, keep) -> i8.PreparedWeight:
    return i8.prepare_weight(W.cuda(), keep)


def gpu_forward(X: torch.Tensor, w: i8.PreparedWeight, thr: float, path: str = "auto", cap: int | None = None,
                with_acc: bool = True, ws: i8.Workspace | None = None) -> dict:
    M, K = X.shape
    ws = ws or i8.Workspace(M, K, w.N, cap)
    Xd = X.cuda()
    acc = torch.empty(M, w.N, dtype=torch.int32, device="cuda") if with_acc else None
    Y = i8.forward(Xd, w, thr, workspace=ws, path=path, acc_out=acc)
    status, n_o = i8.device_status(ws)
    v = ws.view()
    n_eff = min(n_o, ws.max_outliers)
    return {
        "status": status, "n_o": n_o, "ws": ws, "Y_dev": Y, "acc_dev": acc,
        "idx": v["outlier_idx"][:n_eff].cpu().numpy(),
        "xq_dev": v["xq"], "ra": v["row_absmax"].cpu().numpy(),
    }


def oracle_full(X: torch.Tensor, W: torch.Tensor, keep, thr: float) -> tuple[dict, dict]:
    prep = oracle.prepare_weight(W.numpy(), keep)
    return prep, oracle.forward(X.numpy(), prep, thr)


def check_weight(w: i8.PreparedWeight, prep: dict) -> None:
    assert np.array_equal(w.wq.cpu().numpy(), prep["wq"]), "Wq differs"
    assert np.array_equal(w.col_absmax.cpu().numpy().view(np.uint32), prep["ca"].view(np.uint32)), "ca differs"
    if prep["keep_idx"].size:
        assert np.array_equal(w.keep_idx.cpu().numpy(), prep["keep_idx"])
        assert np.array_equal(w.w_keep.cpu().numpy().view(np.uint16), prep["w_keep"].view(np.uint16))


def check_forward_full(g: dict, r: dict) -> float:
    """Every intermediate bit-exact, Y within tolerance (whole matrices)."""
    assert g["status"] == 0, f"device status {g['status']}"
    assert g["n_o"] == r["idx"].size
    assert np.array_equal(g["idx"], r["idx"]), "outlier list differs"
    assert np.array_equal(g["ra"].view(np.uint32), r["ra"].view(np.uint32)), "row absmax differs"
    assert np.array_equal(g["xq_dev"].cpu().numpy(), r["xq"]), "Xq differs"
    if g["acc_dev"] is not None:
        assert np.array_equal(g["acc_dev"].cpu().numpy(), r["acc"]), "int32 sums differ"
    return assert_y_close(g["Y_dev"].float().cpu().numpy(), r["y"].astype(np.float64))


def check_forward_sampled(g: dict, steps: dict, prep: dict, pm: np.ndarray, pn: np.ndarray) -> float:
    """Full-size check: X-side steps exact in full, sums and Y at sampled points."""
    assert g["status"] == 0, f"device status {g['status']}"
    assert g["n_o"] == steps["idx"].size
    assert np.array_equal(g["idx"], steps["idx"]), "outlier list differs"
    assert np.array_equal(g["ra"].view(np.uint32), steps["ra"].view(np.uint32)), "row absmax differs"
    assert np.array_equal(g["xq_dev"].cpu().numpy(), steps["xq"]), "Xq differs"
    acc_ref, y_ref = oracle.forward_points(steps, prep, pm, pn)
    tpm = torch.from_numpy(pm.astype(np.int64)).cuda()
    tpn = torch.from_numpy(pn.astype(np.int64)).cuda()
    if g["acc_dev"] is not None:
        acc = g["acc_dev"][tpm, tpn].cpu().numpy()
        assert np.array_equal(acc, acc_ref), f"int32 sums differ at {int((acc != acc_ref).sum())} points"
    y = g["Y_dev"][tpm, tpn].float().cpu().numpy()
    return assert_y_close(y, y_ref.astype(np.float64))
