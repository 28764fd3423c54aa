"""Python binding of the C ABI (argument marshalling only).

Every computation runs in the CUDA kernels of ``libmlstm_fw.so``; this module
allocates outputs and workspace with PyTorch on the inputs' device, passes raw
pointers and torch's current stream, and raises ``MlstmError`` on a non-OK
status.  Inputs must be CUDA tensors: there is no CPU path.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import MlstmError  # noqa: F401  (re-export)

_DT = {torch.float32: _lib.DT_F32, torch.bfloat16: _lib.DT_BF16}
_GATE = {"exp": _lib.GATE_EXP, "sigmoid": _lib.GATE_SIGMOID,
         "sigmoid_plain": _lib.GATE_SIGMOID_PLAIN}
_ALGO = {"auto": _lib.ALGO_AUTO, "simt": _lib.ALGO_SIMT, "tc": _lib.ALGO_TC,
         "tc_fused": _lib.ALGO_TC_FUSED}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_tensor(name, t, dtype, shape, device):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(B, NH, T, DK, DV, chunk_size, dtype=torch.bfloat16, algo="auto") -> int:
    n = ctypes.c_size_t(0)
    _lib.check(_lib.lib().mlstm_fw_workspace_size(B, NH, T, DK, DV, chunk_size, _DT[dtype],
                                                  _ALGO[algo], ctypes.byref(n)),
               "mlstm_fw_workspace_size")
    return int(n.value)


def substep_workspace_size(B, NH, T, DK, DV, chunk_size, dtype=torch.bfloat16,
                           algo="auto") -> int:
    n = ctypes.c_size_t(0)
    _lib.check(_lib.lib().mlstm_fw_substep_workspace_size(B, NH, T, DK, DV, chunk_size, _DT[dtype],
                                                          _ALGO[algo], ctypes.byref(n)),
               "mlstm_fw_substep_workspace_size")
    return int(n.value)


def _shapes(Q, V):
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    return B, NH, T, DK, DV


def _check_common(Q, K, V, i_pre, f_pre):
    if Q.dim() != 4:
        raise ValueError("Q must be [B, NH, T, DK]")
    B, NH, T, DK, DV = _shapes(Q, V)
    dev = Q.device
    dt = Q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt} (float32 or bfloat16)")
    _check_tensor("Q", Q, dt, (B, NH, T, DK), dev)
    _check_tensor("K", K, dt, (B, NH, T, DK), dev)
    _check_tensor("V", V, dt, (B, NH, T, DV), dev)
    _check_tensor("i_pre", i_pre, torch.float32, (B, NH, T), dev)
    _check_tensor("f_pre", f_pre, torch.float32, (B, NH, T), dev)
    return B, NH, T, DK, DV, dev, dt


def _check_state(C0, n0, m0, B, NH, DK, DV, dev):
    if (C0 is None) != (n0 is None) or (C0 is None) != (m0 is None):
        raise ValueError("C0, n0 and m0 must be given together")
    _check_tensor("C0", C0, torch.float32, (B, NH, DK, DV), dev)
    _check_tensor("n0", n0, torch.float32, (B, NH, DK), dev)
    _check_tensor("m0", m0, torch.float32, (B, NH), dev)


def mlstm_fw(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, *, chunk_size: int = 64,
             gate_mode: str = "exp", algo: str = "auto", return_last_states: bool = True,
             workspace: torch.Tensor | None = None, out: dict | None = None):
    """mLSTM forward pass on the GPU.

    Q, K [B,NH,T,DK] and V [B,NH,T,DV] (float32 or bfloat16, same dtype);
    i_pre, f_pre [B,NH,T] float32; optional initial state C0 [B,NH,DK,DV],
    n0 [B,NH,DK], m0 [B,NH] float32.  Returns ``H`` or ``(H, (C_T, n_T, m_T))``.
    ``out`` may hold preallocated ``H``/``C_T``/``n_T``/``m_T``; ``workspace``
    a uint8 CUDA tensor of at least ``workspace_size(...)`` bytes.
    """
    B, NH, T, DK, DV, dev, dt = _check_common(Q, K, V, i_pre, f_pre)
    _check_state(C0, n0, m0, B, NH, DK, DV, dev)
    out = {} if out is None else out
    H = out.get("H")
    if H is None:
        H = torch.empty((B, NH, T, DV), dtype=dt, device=dev)
    _check_tensor("H", H, dt, (B, NH, T, DV), dev)
    C_T = n_T = m_T = None
    if return_last_states:
        C_T = out.get("C_T")
        n_T = out.get("n_T")
        m_T = out.get("m_T")
        if C_T is None:
            C_T = torch.empty((B, NH, DK, DV), dtype=torch.float32, device=dev)
        if n_T is None:
            n_T = torch.empty((B, NH, DK), dtype=torch.float32, device=dev)
        if m_T is None:
            m_T = torch.empty((B, NH), dtype=torch.float32, device=dev)
    ws_bytes = workspace_size(B, NH, T, DK, DV, chunk_size, dt, algo)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    elif workspace.numel() < ws_bytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA uint8 tensor of >= {ws_bytes} bytes")
    st = _lib.lib().mlstm_fw(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        _ptr(H), _ptr(C_T), _ptr(n_T), _ptr(m_T), B, NH, T, DK, DV, chunk_size, _DT[dt],
        _GATE[gate_mode], _ALGO[algo], _ptr(workspace), workspace.numel(), _stream(dev))
    _lib.check(st, "mlstm_fw")
    if return_last_states:
        return H, (C_T, n_T, m_T)
    return H


def mlstm_bw(Q, K, V, i_pre, f_pre, dH, C0=None, n0=None, m0=None, *, chunk_size: int = 64,
             gate_mode: str = "exp"):
    """Gradients of a loss L(H) of the forward output, given dH = dL/dH.

    Inputs as ``mlstm_fw``.  Returns a dict with dQ, dK, dV (input dtype),
    di_pre, df_pre [B,NH,T] and, when an initial state is given, dC0, dn0,
    dm0 (float32).  bf16 inputs with d_qk of 128 or 256 (a d_v the tensor-core
    forward takes, T >= 128) run on the tensor cores in 128-token chunks,
    whatever ``chunk_size`` is; everything else on fp32 CUDA-core kernels.
    """
    B, NH, T, DK, DV, dev, dt = _check_common(Q, K, V, i_pre, f_pre)
    _check_state(C0, n0, m0, B, NH, DK, DV, dev)
    _check_tensor("dH", dH, dt, (B, NH, T, DV), dev)
    out = {"dQ": torch.empty_like(Q), "dK": torch.empty_like(K), "dV": torch.empty_like(V),
           "di_pre": torch.empty_like(i_pre), "df_pre": torch.empty_like(f_pre)}
    if C0 is not None:
        out.update(dC0=torch.empty_like(C0), dn0=torch.empty_like(n0), dm0=torch.empty_like(m0))
    n = ctypes.c_size_t(0)
    _lib.check(_lib.lib().mlstm_bw_workspace_size(B, NH, T, DK, DV, chunk_size, _DT[dt],
                                                  ctypes.byref(n)), "mlstm_bw_workspace_size")
    ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=dev)
    st = _lib.lib().mlstm_bw(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        _ptr(dH), _ptr(out["dQ"]), _ptr(out["dK"]), _ptr(out["dV"]), _ptr(out["di_pre"]),
        _ptr(out["df_pre"]), _ptr(out.get("dC0")), _ptr(out.get("dn0")), _ptr(out.get("dm0")),
        B, NH, T, DK, DV, chunk_size, _DT[dt], _GATE[gate_mode], _ptr(ws), ws.numel(),
        _stream(dev))
    _lib.check(st, "mlstm_bw")
    return out


def train_sizes(B, NH, T, DK, DV, dtype=torch.bfloat16):
    """Bytes of the saved buffer and of the two calls' workspaces of the
    training pair, or None when the shape has no training path (it needs the
    tensor-core backward: bf16, d_qk 128 or 256, d_v 128 or a multiple of 256
    up to 1024, T >= 128)."""
    sv, fw, bw = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = _lib.lib().mlstm_train_sizes(B, NH, T, DK, DV, _DT[dtype], ctypes.byref(sv),
                                      ctypes.byref(fw), ctypes.byref(bw))
    if st == _lib.ERR_UNSUPPORTED:
        return None
    _lib.check(st, "mlstm_train_sizes")
    return int(sv.value), int(fw.value), int(bw.value)


def mlstm_fw_train(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, *, gate_mode: str = "exp"):
    """The forward pass of ``mlstm_fw`` (128-token chunks on the tensor cores)
    that also keeps what ``mlstm_bw_saved`` needs.  Returns ``(H, (C_T, n_T,
    m_T), saved)``; ``saved`` is an opaque uint8 tensor.  Raises
    ``MlstmError`` (unsupported) outside the shapes of ``train_sizes``."""
    B, NH, T, DK, DV, dev, dt = _check_common(Q, K, V, i_pre, f_pre)
    _check_state(C0, n0, m0, B, NH, DK, DV, dev)
    sizes = train_sizes(B, NH, T, DK, DV, dt)
    if sizes is None:
        raise MlstmError(_lib.ERR_UNSUPPORTED, "mlstm_fw_train")
    sv_bytes, fw_bytes, _ = sizes
    H = torch.empty((B, NH, T, DV), dtype=dt, device=dev)
    C_T = torch.empty((B, NH, DK, DV), dtype=torch.float32, device=dev)
    n_T = torch.empty((B, NH, DK), dtype=torch.float32, device=dev)
    m_T = torch.empty((B, NH), dtype=torch.float32, device=dev)
    saved = torch.empty(sv_bytes, dtype=torch.uint8, device=dev)
    ws = torch.empty(max(fw_bytes, 1), dtype=torch.uint8, device=dev)
    _lib.check(_lib.lib().mlstm_fw_train(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        _ptr(H), _ptr(C_T), _ptr(n_T), _ptr(m_T), _ptr(saved), saved.numel(), B, NH, T, DK, DV,
        _DT[dt], _GATE[gate_mode], _ptr(ws), ws.numel(), _stream(dev)), "mlstm_fw_train")
    return H, (C_T, n_T, m_T), saved


def mlstm_bw_saved(Q, K, V, i_pre, f_pre, H, saved, dH, C0=None, n0=None, m0=None, *,
                   gate_mode: str = "exp"):
    """``mlstm_bw`` from the output and the saved buffer of ``mlstm_fw_train``
    (same inputs) instead of a recomputed forward.  Returns the same dict."""
    B, NH, T, DK, DV, dev, dt = _check_common(Q, K, V, i_pre, f_pre)
    _check_state(C0, n0, m0, B, NH, DK, DV, dev)
    _check_tensor("H", H, dt, (B, NH, T, DV), dev)
    _check_tensor("dH", dH, dt, (B, NH, T, DV), dev)
    sizes = train_sizes(B, NH, T, DK, DV, dt)
    if sizes is None:
        raise MlstmError(_lib.ERR_UNSUPPORTED, "mlstm_bw_saved")
    _, _, bw_bytes = sizes
    out = {"dQ": torch.empty_like(Q), "dK": torch.empty_like(K), "dV": torch.empty_like(V),
           "di_pre": torch.empty_like(i_pre), "df_pre": torch.empty_like(f_pre)}
    if C0 is not None:
        out.update(dC0=torch.empty_like(C0), dn0=torch.empty_like(n0), dm0=torch.empty_like(m0))
    ws = torch.empty(max(bw_bytes, 1), dtype=torch.uint8, device=dev)
    _lib.check(_lib.lib().mlstm_bw_saved(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0),
        _ptr(H), _ptr(saved), saved.numel(), _ptr(dH), _ptr(out["dQ"]), _ptr(out["dK"]),
        _ptr(out["dV"]), _ptr(out["di_pre"]), _ptr(out["df_pre"]), _ptr(out.get("dC0")),
        _ptr(out.get("dn0")), _ptr(out.get("dm0")), B, NH, T, DK, DV, _DT[dt],
        _GATE[gate_mode], _ptr(ws), ws.numel(), _stream(dev)), "mlstm_bw_saved")
    return out


def mlstm_step(q, k, v, i_pre, f_pre, C, n, m, *, gate_mode: str = "exp", h=None):
    """One token of the recurrence for every (b, h), in place on the state.

    q, k [B,NH,DK] and v [B,NH,DV] (float32 or bfloat16, same dtype); i_pre,
    f_pre [B,NH] float32; C [B,NH,DK,DV], n [B,NH,DK], m [B,NH] float32 CUDA
    tensors holding the state before the token, overwritten with the state
    after it.  Returns h [B,NH,DV] in the input dtype (``h`` may be given).
    """
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("q, k must be [B,NH,DK] and v [B,NH,DV] with the same B, NH")
    B, NH, DK = q.shape
    DV = v.shape[2]
    dt, dev = q.dtype, q.device
    if dt not in _DT or k.dtype != dt or v.dtype != dt:
        raise ValueError("q, k, v must share a dtype of float32 or bfloat16")
    for name, t in (("i_pre", i_pre), ("f_pre", f_pre), ("m", m)):
        _check_tensor(name, t, torch.float32, (B, NH), dev)
    _check_tensor("C", C, torch.float32, (B, NH, DK, DV), dev)
    _check_tensor("n", n, torch.float32, (B, NH, DK), dev)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(name, t, dt, tuple(t.shape), dev)
    if h is None:
        h = torch.empty((B, NH, DV), dtype=dt, device=dev)
    _check_tensor("h", h, dt, (B, NH, DV), dev)
    st = _lib.lib().mlstm_step(_ptr(q), _ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(C),
                               _ptr(n), _ptr(m), _ptr(h), B, NH, DK, DV, _DT[dt],
                               _GATE[gate_mode], _stream(dev))
    _lib.check(st, "mlstm_step")
    return h


def mlstm_fw_chunk_states(K, V, i_pre, f_pre, C0=None, n0=None, m0=None, *, chunk_size: int = 64,
                          gate_mode: str = "exp", algo: str = "auto"):
    """Recurrent half: states entering every chunk and the final state.

    Returns (C_states [B,NH,NC,DK,DV], n_states [B,NH,NC,DK], m_states
    [B,NH,NC+1], (C_T, n_T, m_T)).
    """
    B, NH, T, DK, DV, dev, dt = _check_common(K, K, V, i_pre, f_pre)
    _check_state(C0, n0, m0, B, NH, DK, DV, dev)
    NC = (T + chunk_size - 1) // chunk_size
    C_states = torch.empty((B, NH, NC, DK, DV), dtype=torch.float32, device=dev)
    n_states = torch.empty((B, NH, NC, DK), dtype=torch.float32, device=dev)
    m_states = torch.empty((B, NH, NC + 1), dtype=torch.float32, device=dev)
    C_T = torch.empty((B, NH, DK, DV), dtype=torch.float32, device=dev)
    n_T = torch.empty((B, NH, DK), dtype=torch.float32, device=dev)
    m_T = torch.empty((B, NH), dtype=torch.float32, device=dev)
    ws = torch.empty(max(substep_workspace_size(B, NH, T, DK, DV, chunk_size, dt, algo), 1),
                     dtype=torch.uint8, device=dev)
    st = _lib.lib().mlstm_fw_chunk_states(
        _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(C0), _ptr(n0), _ptr(m0), _ptr(C_states),
        _ptr(n_states), _ptr(m_states), _ptr(C_T), _ptr(n_T), _ptr(m_T), B, NH, T, DK, DV,
        chunk_size, _DT[dt], _GATE[gate_mode], _ALGO[algo], _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "mlstm_fw_chunk_states")
    return C_states, n_states, m_states, (C_T, n_T, m_T)


def mlstm_fw_parallel(Q, K, V, i_pre, f_pre, C_states, n_states, m0=None, *,
                      chunk_size: int = 64, gate_mode: str = "exp", algo: str = "auto"):
    """Parallel half: (H, n_out, m_out) from the chunk states."""
    B, NH, T, DK, DV, dev, dt = _check_common(Q, K, V, i_pre, f_pre)
    NC = (T + chunk_size - 1) // chunk_size
    _check_tensor("C_states", C_states, torch.float32, (B, NH, NC, DK, DV), dev)
    _check_tensor("n_states", n_states, torch.float32, (B, NH, NC, DK), dev)
    _check_tensor("m0", m0, torch.float32, (B, NH), dev)
    H = torch.empty((B, NH, T, DV), dtype=dt, device=dev)
    n_out = torch.empty((B, NH, T), dtype=torch.float32, device=dev)
    m_out = torch.empty((B, NH, T), dtype=torch.float32, device=dev)
    ws = torch.empty(max(substep_workspace_size(B, NH, T, DK, DV, chunk_size, dt, algo), 1),
                     dtype=torch.uint8, device=dev)
    st = _lib.lib().mlstm_fw_parallel(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(i_pre), _ptr(f_pre), _ptr(m0), _ptr(C_states),
        _ptr(n_states), _ptr(H), _ptr(n_out), _ptr(m_out), B, NH, T, DK, DV, chunk_size, _DT[dt],
        _GATE[gate_mode], _ALGO[algo], _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "mlstm_fw_parallel")
    return H, n_out, m_out


def last_device_error(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device
    error status (``_lib.OK``, ``_lib.ERR_TIMEOUT``, ...)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(_lib.lib().mlstm_last_device_error(_stream(dev)))


def set_watchdog(max_polls: int) -> None:
    _lib.lib().mlstm_set_watchdog(int(max_polls))


def watchdog_selftest(device=None) -> None:
    """Enqueues the failure-detection self-test (one bounded wait that nothing
    satisfies) on the current stream; the next ``last_device_error`` returns
    ``_lib.ERR_TIMEOUT``."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _lib.check(_lib.lib().mlstm_watchdog_selftest(_stream(dev)), "mlstm_watchdog_selftest")


class _MlstmChunkwise(torch.autograd.Function):
    """Differentiable mLSTM.  Where the training pair exists (``train_sizes``)
    and ``recompute`` is off, the forward is ``mlstm_fw_train`` and the
    backward ``mlstm_bw_saved`` (about 1 GB kept per 7B-shaped call, no
    recomputation); otherwise the forward is ``mlstm_fw`` and the backward
    ``mlstm_bw``, which recomputes what it needs from the inputs.  Gradients
    flow from H only; the returned final state carries none."""

    @staticmethod
    def forward(ctx, Q, K, V, i_pre, f_pre, C0, n0, m0, chunk_size, gate_mode, algo, recompute):
        saved = None
        if not recompute and algo == "auto" and Q.is_cuda and Q.dtype in _DT and \
                train_sizes(Q.shape[0], Q.shape[1], Q.shape[2], Q.shape[3], V.shape[-1],
                            Q.dtype) is not None:
            H, (C_T, n_T, m_T), saved = mlstm_fw_train(Q, K, V, i_pre, f_pre, C0, n0, m0,
                                                       gate_mode=gate_mode)
        else:
            H, (C_T, n_T, m_T) = mlstm_fw(Q, K, V, i_pre, f_pre, C0, n0, m0,
                                          chunk_size=chunk_size, gate_mode=gate_mode, algo=algo)
        if saved is not None:
            ctx.save_for_backward(Q, K, V, i_pre, f_pre, C0, n0, m0, H, saved)
        else:
            ctx.save_for_backward(Q, K, V, i_pre, f_pre, C0, n0, m0)
        ctx.cfg = (chunk_size, gate_mode, saved is not None)
        ctx.mark_non_differentiable(C_T, n_T, m_T)
        return H, C_T, n_T, m_T

    @staticmethod
    def backward(ctx, dH, dC_T, dn_T, dm_T):
        chunk_size, gate_mode, kept = ctx.cfg
        if kept:
            Q, K, V, i_pre, f_pre, C0, n0, m0, H, saved = ctx.saved_tensors
            g = mlstm_bw_saved(Q, K, V, i_pre, f_pre, H, saved, dH.contiguous(), C0, n0, m0,
                               gate_mode=gate_mode)
        else:
            Q, K, V, i_pre, f_pre, C0, n0, m0 = ctx.saved_tensors
            g = mlstm_bw(Q, K, V, i_pre, f_pre, dH.contiguous(), C0, n0, m0,
                         chunk_size=chunk_size, gate_mode=gate_mode)
        return (g["dQ"], g["dK"], g["dV"], g["di_pre"], g["df_pre"], g.get("dC0"), g.get("dn0"),
                g.get("dm0"), None, None, None, None)


def mlstm_chunkwise(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, *, chunk_size: int = 64,
                    gate_mode: str = "exp", algo: str = "auto", recompute: bool = False):
    """mLSTM forward pass that autograd can differentiate.

    Same arguments and shapes as ``mlstm_fw``; returns ``(H, (C_T, n_T, m_T))``.
    The gradient of a loss on H reaches Q, K, V, both gate pre-activations and
    the initial state; the final state is returned without a gradient path.
    Where the training pair exists (bf16, d_qk 128 or 256, T >= 128; see
    ``train_sizes``) the forward keeps the chunk states and per-token
    normalisers for the backward (128-token chunks, whatever ``chunk_size``
    says); ``recompute=True`` keeps nothing and recomputes them in the
    backward instead (less memory, a slower backward).
    """
    H, C_T, n_T, m_T = _MlstmChunkwise.apply(Q, K, V, i_pre, f_pre, C0, n0, m0, chunk_size,
                                             gate_mode, algo, recompute)
    return H, (C_T, n_T, m_T)
