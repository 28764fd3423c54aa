"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them with the tolerance of the input type.

Error metric (per output tensor, per (b, h) slice, worst slice reported):
normwise max relative error max|x - y| / max|y|; for the stabiliser m,
max|dm| / max(1, max|m|).  Tolerances: 2e-2 for bf16 inputs with fp32
accumulation, 1e-4 for fp32 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (None if v is None else v.to(device)) for k, v in x.items()}


def slice_heads(x: dict, heads) -> dict:
    """Restrict every input to the listed (b, h) pairs, as a [1, len(heads)] batch."""
    out = {}
    for k, v in x.items():
        if v is None:
            out[k] = None
            continue
        out[k] = torch.stack([v[b, h] for b, h in heads], dim=0).unsqueeze(0)
    return out


def oracle_run(x: dict, gate_mode: str, heads=None, snap_every=0) -> dict:
    if heads is not None:
        x = slice_heads(x, heads)
    return oracle.mlstm_recurrent(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"],
                                  x["C0"], x["n0"], x["m0"], gate_mode=gate_mode,
                                  snap_every=snap_every)


def pick(t: torch.Tensor, heads) -> np.ndarray:
    """GPU output -> fp64 numpy restricted to the listed heads ([1, n, ...])."""
    if heads is None:
        return t.detach().double().cpu().numpy()
    return torch.stack([t[b, h] for b, h in heads], 0).unsqueeze(0).double().cpu().numpy()


def worst_rel(x: np.ndarray, y: np.ndarray) -> float:
    """Worst per-(b,h) normwise relative error of x against y ([B, NH, ...])."""
    B, NH = y.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(NH):
            d = np.abs(x[b, h] - y[b, h])
            if d.size == 0:
                continue
            s = np.max(np.abs(y[b, h]))
            e = float(np.max(d) / s) if s > 0 else float(np.max(d))
            worst = max(worst, e)
    return worst


def m_err(x: np.ndarray, y: np.ndarray) -> float:
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(1.0, float(np.max(np.abs(y)))))


def compare(H, final, ref: dict, tol: float, heads=None, label="") -> dict:
    errs = {"H": worst_rel(pick(H, heads), ref["H"])}
    if final is not None:
        C_T, n_T, m_T = final
        errs["C_T"] = worst_rel(pick(C_T, heads), ref["C_T"])
        errs["n_T"] = worst_rel(pick(n_T, heads), ref["n_T"])
        errs["m_T"] = m_err(pick(m_T, heads), ref["m_T"])
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, f"{label}: errors above {tol}: {bad} (all: {errs})"
    return errs


def worst_row_rel(x: np.ndarray, y: np.ndarray, floor: float = 1e-3) -> float:
    """Worst per-token-row relative error of x against y ([B, NH, T, D]).

    Each output row h_t is compared with its own size: max_j |x - y| divided by
    max(max_j |y|, floor * max|y| of its (b, h) slice), so that rows whose exact
    value is near zero do not divide by (almost) nothing.  This shows errors on
    individual rows that the normwise slice metric averages away."""
    d = np.abs(x - y).max(axis=-1)
    rmax = np.abs(y).max(axis=-1)
    smax = np.abs(y).max(axis=(-1, -2), keepdims=True)[..., 0]
    den = np.maximum(rmax, floor * smax)
    den = np.where(den > 0, den, 1.0)
    return float((d / den).max()) if d.size else 0.0
