"""fp64 CPU oracle for the gradients of the mLSTM forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` (and nothing in the product path) may import this module; it
shares no code with the CUDA library.

The forward is the token-by-token recurrence that the tensor-product
formulation of the mLSTM defines ("Tiled Flash Linear Attention: More
Efficient Linear RNN and xLSTM Kernels", abstract: the mLSTM, the xLSTM with
matrix memory; the recurrence with exponential gating, normalisation and
stabilisation is the one the ``xLSTM: the NX-AI repository behind the extended
LSTM architecture`` page describes in "Exponential gating, matrix memory, and
why the kernels decide everything"), written out with plain torch fp64 ops:

    lf = logsigmoid(f~_t),  li = i~_t (exp) | logsigmoid(i~_t) (sigmoid)
    m_t = max(lf + m_{t-1}, li)
    C_t = e^{lf + m_{t-1} - m_t} C_{t-1} + e^{li - m_t} (s k_t) v_t^T
    n_t = e^{lf + m_{t-1} - m_t} n_{t-1} + e^{li - m_t} (s k_t)
    h_t = C_t^T q_t / max(|n_t^T q_t|, e^{-m_t}),   s = 1/sqrt(d_qk)

The gradients are torch autograd of that program, in fp64.  Pins
(``tests/test_oracle_backward.py``): the forward equals the C oracle's, and
the gradients equal central finite differences on tiny inputs.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F


def forward(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, gate_mode: str = "exp"):
    """fp64 recurrence.  Shapes as the library's: Q, K [B,NH,T,DK], V [B,NH,T,DV],
    i_pre, f_pre [B,NH,T], optional C0 [B,NH,DK,DV], n0 [B,NH,DK], m0 [B,NH].
    Returns H [B,NH,T,DV] and the final (C, n, m)."""
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    s = 1.0 / math.sqrt(DK)
    C = C0 if C0 is not None else Q.new_zeros((B, NH, DK, DV))
    n = n0 if n0 is not None else Q.new_zeros((B, NH, DK))
    m = m0 if m0 is not None else Q.new_zeros((B, NH))
    H = []
    for t in range(T):
        lf = F.logsigmoid(f_pre[:, :, t])
        li = i_pre[:, :, t] if gate_mode == "exp" else F.logsigmoid(i_pre[:, :, t])
        m_new = torch.maximum(lf + m, li)
        fa = torch.exp(lf + m - m_new)
        ia = torch.exp(li - m_new)
        k = s * K[:, :, t]
        v = V[:, :, t]
        q = Q[:, :, t]
        C = fa[..., None, None] * C + ia[..., None, None] * k[..., :, None] * v[..., None, :]
        n = fa[..., None] * n + ia[..., None] * k
        m = m_new
        num = torch.einsum("bhkv,bhk->bhv", C, q)
        den = torch.maximum((n * q).sum(-1).abs(), torch.exp(-m))
        H.append(num / den[..., None])
    return torch.stack(H, dim=2), (C, n, m)


def gradients(x: dict, dH, gate_mode: str = "exp") -> dict:
    """Gradients of L = sum(dH * H) with respect to every input of ``x`` (keys
    Q, K, V, i_pre, f_pre and, when present, C0, n0, m0), all in fp64.  Also
    returns H and the final state of the same forward."""
    names = [k for k in ("Q", "K", "V", "i_pre", "f_pre", "C0", "n0", "m0") if x.get(k) is not None]
    leaves = {k: x[k].detach().double().clone().requires_grad_(True) for k in names}
    H, (C, n, m) = forward(leaves["Q"], leaves["K"], leaves["V"], leaves["i_pre"], leaves["f_pre"],
                           leaves.get("C0"), leaves.get("n0"), leaves.get("m0"), gate_mode)
    L = (H * dH.double()).sum()
    grads = torch.autograd.grad(L, [leaves[k] for k in names])
    out = {"d" + k: g.detach() for k, g in zip(names, grads)}
    out.update(H=H.detach(), C_T=C.detach(), n_T=n.detach(), m_T=m.detach())
    return out
