"""Pins of the gradient oracle (oracle/backward.py), on the CPU.

1. Its forward is the same function as the C oracle's (H and final states).
2. Its autograd gradients equal central finite differences on tiny inputs,
   for every input, in both gate modes and with an initial state.
3. The identities the CUDA backward is built on hold for it: for a loss on H
   alone, dL/d(log i_s) = k_s . dk_s and
   dL/d(log f_l) = sum_{t >= l} (q_t . dq_t - k_t . dk_t).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob

pytestmark = pytest.mark.filterwarnings("ignore")


def _inputs(B=1, NH=2, T=7, DK=3, DV=2, init=True, seed=3, i_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = dict(Q=torch.randn(B, NH, T, DK, generator=g, dtype=torch.float64),
             K=torch.randn(B, NH, T, DK, generator=g, dtype=torch.float64),
             V=torch.randn(B, NH, T, DV, generator=g, dtype=torch.float64),
             i_pre=torch.randn(B, NH, T, generator=g, dtype=torch.float64) * i_scale,
             f_pre=torch.rand(B, NH, T, generator=g, dtype=torch.float64) * 3 + 1,
             C0=None, n0=None, m0=None)
    if init:
        x["C0"] = torch.randn(B, NH, DK, DV, generator=g, dtype=torch.float64) * 0.3
        x["n0"] = torch.randn(B, NH, DK, generator=g, dtype=torch.float64) * 0.3
        x["m0"] = torch.randn(B, NH, generator=g, dtype=torch.float64) * 0.5
    dH = torch.randn(B, NH, T, DV, generator=g, dtype=torch.float64)
    return x, dH


@pytest.mark.parametrize("gate_mode", ["exp", "sigmoid"])
@pytest.mark.parametrize("init", [False, True])
def test_forward_matches_the_c_oracle(gate_mode, init):
    x, _ = _inputs(B=2, NH=2, T=40, DK=5, DV=4, init=init)
    H, (C, n, m) = ob.forward(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"], x["C0"], x["n0"],
                              x["m0"], gate_mode)
    ref = oracle.mlstm_recurrent(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"], x["C0"],
                                 x["n0"], x["m0"], gate_mode=gate_mode)
    np.testing.assert_allclose(H.numpy(), ref["H"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(C.numpy(), ref["C_T"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(n.numpy(), ref["n_T"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(m.numpy(), ref["m_T"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("gate_mode", ["exp", "sigmoid"])
def test_gradients_match_finite_differences(gate_mode):
    x, dH = _inputs()
    g = ob.gradients(x, dH, gate_mode)

    def loss(xx):
        H, _ = ob.forward(xx["Q"], xx["K"], xx["V"], xx["i_pre"], xx["f_pre"], xx["C0"],
                          xx["n0"], xx["m0"], gate_mode)
        return float((H * dH).sum())

    eps = 1e-6
    for name in ("Q", "K", "V", "i_pre", "f_pre", "C0", "n0", "m0"):
        base = x[name]
        fd = torch.zeros_like(base)
        flat = base.reshape(-1)
        for j in range(flat.numel()):
            xp = dict(x)
            xm = dict(x)
            tp = flat.clone()
            tm = flat.clone()
            tp[j] += eps
            tm[j] -= eps
            xp[name] = tp.reshape(base.shape)
            xm[name] = tm.reshape(base.shape)
            fd.reshape(-1)[j] = (loss(xp) - loss(xm)) / (2 * eps)
        got = g["d" + name]
        scale = max(1.0, float(fd.abs().max()))
        assert float((got - fd).abs().max()) / scale < 1e-7, name


@pytest.mark.parametrize("gate_mode", ["exp", "sigmoid"])
def test_gate_gradient_identities(gate_mode):
    """The identities the CUDA backward computes its gate gradients from."""
    x, dH = _inputs(B=1, NH=2, T=33, DK=4, DV=3, init=True, seed=5)
    g = ob.gradients(x, dH, gate_mode)
    qdq = (x["Q"] * g["dQ"]).sum(-1)
    kdk = (x["K"] * g["dK"]).sum(-1)
    # d/d(log i) = k . dk; chain rule to i~ (exp: 1; sigmoid: 1 - sigmoid)
    dli = kdk
    di = dli if gate_mode == "exp" else dli * (1 - torch.sigmoid(x["i_pre"]))
    np.testing.assert_allclose(g["di_pre"].numpy(), di.numpy(), rtol=1e-9, atol=1e-11)
    # d/d(log f_l) = sum_{t >= l} (q.dq - k.dk); d(log f)/df~ = 1 - sigmoid(f~)
    suffix = torch.flip(torch.cumsum(torch.flip(qdq - kdk, [-1]), -1), [-1])
    df = suffix * (1 - torch.sigmoid(x["f_pre"]))
    np.testing.assert_allclose(g["df_pre"].numpy(), df.numpy(), rtol=1e-9, atol=1e-11)
    # the initial state: dm0 = <C0, dC0> + n0 . dn0 (C0, n0 are given in frame m0)
    dm0 = (x["C0"] * g["dC0"]).sum((-1, -2)) + (x["n0"] * g["dn0"]).sum(-1)
    np.testing.assert_allclose(g["dm0"].numpy(), dm0.numpy(), rtol=1e-9, atol=1e-11)
