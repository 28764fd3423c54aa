"""fp64 CPU oracle for the mLSTM forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  The product path (the CUDA library in
``mlstm_chunkwise_b200``) never imports it, and the two share no code.

The arithmetic lives in ``mlstm_oracle.c`` (plain C, fp64, token-by-token
recurrence; see its header for the formula and the passages it follows).  This
module only compiles that file with gcc and marshals numpy arrays into it.

The sigmoid-input-gate variant with reduced computation (no stabiliser, no
normaliser) is a separate function written from its plain definition.

Parity pins (all in ``tests/test_oracle_pins.py``): the quadratic parallel form,
chunk-size invariance of an independent chunkwise derivation, the single-token
closed form, memory hold, the reduction to causal normalised linear attention,
hand-derived golden sequences, and invariants (linearity in V, oddness in q,
causality, head independence, stabiliser-frame shift, segment resume).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlstm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GATE_EXP = 0
GATE_SIGMOID = 1


def build(force: bool = False) -> str:
    """Compile ``mlstm_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def open_library(path: str):
    """Load a compiled oracle library at ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.mlstm_oracle_recurrent.restype = ctypes.c_int
    lib.mlstm_oracle_recurrent.argtypes = (
        [dp] * 8 + [ctypes.c_int] * 6 + [dp] * 6 + [ctypes.c_int] + [dp] * 3
    )
    lib.mlstm_oracle_num_threads.restype = ctypes.c_int
    lib.mlstm_oracle_sigmoid_plain.restype = ctypes.c_int
    lib.mlstm_oracle_sigmoid_plain.argtypes = [dp] * 8 + [ctypes.c_int] * 5 + [dp] * 3
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = open_library(_LIB)
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().mlstm_oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact up-cast of bf16/fp32 values
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def mlstm_recurrent(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None,
                    gate_mode: str = "exp", snap_every: int = 0, lib=None) -> dict:
    """Token-by-token fp64 mLSTM forward.

    Q, K: [B, NH, T, DK]; V: [B, NH, T, DV]; i_pre, f_pre: [B, NH, T];
    C0: [B, NH, DK, DV], n0: [B, NH, DK], m0: [B, NH] (all or none).
    Returns a dict with H [B,NH,T,DV], C_T, n_T, m_T (final state, C as
    [DK, DV]), den [B,NH,T] = max(|n^T q|, e^{-m}), m [B,NH,T], and, when
    ``snap_every`` > 0, C_snap/n_snap/m_snap: the state after every
    ``snap_every`` tokens (index j holds the state entering token
    j*snap_every).  ``lib`` selects another compiled copy of the oracle
    (the pin-sensitivity test uses this); by default the built one is used.
    """
    lib = _load() if lib is None else lib
    Q, K, V, i_pre, f_pre = (_f64(a) for a in (Q, K, V, i_pre, f_pre))
    C0, n0, m0 = _f64(C0), _f64(n0), _f64(m0)
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    assert K.shape == (B, NH, T, DK) and V.shape == (B, NH, T, DV)
    assert i_pre.shape == (B, NH, T) and f_pre.shape == (B, NH, T)
    if C0 is not None and n0 is not None and m0 is not None:
        assert C0.shape == (B, NH, DK, DV) and n0.shape == (B, NH, DK) and m0.shape == (B, NH)
    mode = {"exp": GATE_EXP, "sigmoid": GATE_SIGMOID}[gate_mode]
    H = np.zeros((B, NH, T, DV))
    C_T = np.zeros((B, NH, DK, DV))
    n_T = np.zeros((B, NH, DK))
    m_T = np.zeros((B, NH))
    den = np.zeros((B, NH, T))
    m = np.zeros((B, NH, T))
    out = dict(H=H, C_T=C_T, n_T=n_T, m_T=m_T, den=den, m=m)
    C_snap = n_snap = m_snap = None
    if snap_every > 0:
        ns = T // snap_every
        C_snap = np.zeros((B, NH, ns, DK, DV))
        n_snap = np.zeros((B, NH, ns, DK))
        m_snap = np.zeros((B, NH, ns))
        out.update(C_snap=C_snap, n_snap=n_snap, m_snap=m_snap)
    rc = lib.mlstm_oracle_recurrent(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        B, NH, T, DK, DV, mode,
        _ptr(H), _ptr(C_T), _ptr(n_T), _ptr(m_T), _ptr(den), _ptr(m),
        int(snap_every), _ptr(C_snap), _ptr(n_snap), _ptr(m_snap))
    if rc != 0:
        raise ValueError("mlstm_oracle_recurrent rejected its arguments")
    return out


def mlstm_sigmoid_plain(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, lib=None) -> dict:
    """The sigmoid-input-gate variant with reduced computation, from its plain
    definition (unstabilised, no normaliser; see ``mlstm_oracle_sigmoid_plain``
    in ``mlstm_oracle.c``): h_t = C_t^T q_t with
    C_t = sigmoid(f~_t) C_{t-1} + sigmoid(i~_t) (s k_t) v_t^T.

    Returns H [B,NH,T,DV] and the unstabilised final state C_T [B,NH,DK,DV],
    n_T [B,NH,DK] (frame m = 0)."""
    lib = _load() if lib is None else lib
    Q, K, V, i_pre, f_pre = (_f64(a) for a in (Q, K, V, i_pre, f_pre))
    C0, n0, m0 = _f64(C0), _f64(n0), _f64(m0)
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    H = np.zeros((B, NH, T, DV))
    C_T = np.zeros((B, NH, DK, DV))
    n_T = np.zeros((B, NH, DK))
    rc = lib.mlstm_oracle_sigmoid_plain(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        B, NH, T, DK, DV, _ptr(H), _ptr(C_T), _ptr(n_T))
    if rc != 0:
        raise RuntimeError("mlstm_oracle_sigmoid_plain failed")
    return dict(H=H, C_T=C_T, n_T=n_T)
