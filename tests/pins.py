"""Independent fp64 references and the pins that hold the oracle in place.

Nothing here calls the CUDA path.  Each ``pin_*`` function takes ``run``, a
callable with the signature of ``oracle.mlstm_recurrent``, and raises
``AssertionError`` when the oracle disagrees with something the mathematics
fixes independently of it:

* the quadratic (fully parallel) form of the recurrence: a T x T gated,
  causal, stabilised matrix, evaluated with matrix products;
* a chunkwise derivation (inter-chunk state recurrence plus intra-chunk
  parallel part, the structure that "Tiled Flash Linear Attention" (abstract)
  builds on), at several chunk sizes;
* the single-token closed form h = v (s k.q) / max(|s k.q|, e^{-li});
* memory hold: a saturated forget gate with a closed input gate leaves
  (C, n, m) unchanged;
* the reduction to causal normalised linear attention when both gates are
  fully open;
* hand-derived sequences in ``golden/hand_derived_sequences.json``;
* invariants: linearity in V, oddness in q, causality, (b, h) independence,
  a shift of the stabiliser frame of the initial state, and segment resume.

The pin-sensitivity test (``test_oracle_mutants.py``) plants plausible
mistakes in a copy of the oracle and checks that each one fails a pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "hand_derived_sequences.json")


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def logsigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return np.where(x >= 0, -np.log1p(np.exp(-np.abs(x))), x - np.log1p(np.exp(-np.abs(x))))


def gate_logs(i_pre, f_pre, gate_mode):
    lf = logsigmoid(f_pre)
    li = np.asarray(i_pre, dtype=np.float64) if gate_mode == "exp" else logsigmoid(i_pre)
    return li, lf


def rel_err(x, y):
    """Normwise-max relative error max|x-y| / max|y| (0/0 counts as 0)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    d = np.max(np.abs(x - y)) if x.size else 0.0
    s = np.max(np.abs(y)) if y.size else 0.0
    if s == 0.0:
        return float(d)
    return float(d / s)


def rand_case(seed, B=1, NH=2, T=32, DK=8, DV=6, init_state=False, i_mean=0.0,
              f_low=-1.0, f_high=4.0):
    """Small fp64 inputs; the forget range reaches negative pre-activations so
    that the stabiliser and the decay both matter."""
    rng = np.random.default_rng(seed)
    c = dict(
        Q=rng.standard_normal((B, NH, T, DK)),
        K=rng.standard_normal((B, NH, T, DK)),
        V=rng.standard_normal((B, NH, T, DV)),
        i_pre=rng.standard_normal((B, NH, T)) * 2.0 + i_mean,
        f_pre=rng.uniform(f_low, f_high, (B, NH, T)),
        C0=None, n0=None, m0=None,
    )
    if init_state:
        c["C0"] = rng.standard_normal((B, NH, DK, DV)) * 0.5
        c["n0"] = rng.standard_normal((B, NH, DK)) * 0.5
        c["m0"] = rng.standard_normal((B, NH))
    return c


# ----------------------------------------------------------------------------
# independent references
# ----------------------------------------------------------------------------

def quadratic_form(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, gate_mode="exp"):
    """Fully parallel form, per (b, h).

    With F_t = sum_{l<=t} lf_l, the unstabilised weight of token j in the
    memory read at t is exp(F_t - F_j + li_j) (j <= t), and the initial state
    enters with exp(F_t + m0).  The stabiliser is the largest log-weight,
    m_t = max(F_t + m0, max_{j<=t} F_t - F_j + li_j); everything is evaluated
    as one T x T matrix.
    """
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    s = 1.0 / math.sqrt(DK)
    H = np.zeros((B, NH, T, DV))
    M = np.zeros((B, NH, T))
    DEN = np.zeros((B, NH, T))
    for b in range(B):
        for h in range(NH):
            li, lf = gate_logs(i_pre[b, h], f_pre[b, h], gate_mode)
            F = np.cumsum(lf)
            logW = F[:, None] - F[None, :] + li[None, :]
            causal = np.tril(np.ones((T, T), dtype=bool))
            logW = np.where(causal, logW, -np.inf)
            mm0 = 0.0 if m0 is None else float(m0[b, h])
            log_init = F + mm0
            m = np.maximum(log_init, logW.max(axis=1))
            W = np.exp(logW - m[:, None])
            Sqk = s * Q[b, h] @ K[b, h].T
            A = W * Sqk
            num = A @ V[b, h]
            den = A.sum(axis=1)
            if C0 is not None:
                ginit = np.exp(log_init - m)
                num = num + ginit[:, None] * (Q[b, h] @ C0[b, h])
                den = den + ginit * (Q[b, h] @ n0[b, h])
            denom = np.maximum(np.abs(den), np.exp(-m))
            H[b, h] = num / denom[:, None]
            M[b, h] = m
            DEN[b, h] = denom
    return dict(H=H, m=M, den=DEN)


def chunkwise(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None, gate_mode="exp", L=16):
    """Chunkwise form: inter-chunk state recurrence + intra-chunk parallel part.

    Inside chunk k (local index r), b_r is the inclusive cumulative log forget
    gate, g = b_{L-1}, and the column log-weight is a_s = li_s - b_s.  The
    per-token stabiliser is m_r = b_r + max(m_prev, max_{s<=r} a_s); the
    state leaving the chunk has m_k = max(g + m_prev, g + max_s a_s).
    """
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    assert T % L == 0
    s = 1.0 / math.sqrt(DK)
    H = np.zeros((B, NH, T, DV))
    M = np.zeros((B, NH, T))
    DEN = np.zeros((B, NH, T))
    CT = np.zeros((B, NH, DK, DV))
    NT = np.zeros((B, NH, DK))
    MT = np.zeros((B, NH))
    for b in range(B):
        for h in range(NH):
            li, lf = gate_logs(i_pre[b, h], f_pre[b, h], gate_mode)
            C = np.zeros((DK, DV)) if C0 is None else C0[b, h].copy()
            n = np.zeros(DK) if n0 is None else n0[b, h].copy()
            mp = 0.0 if m0 is None else float(m0[b, h])
            for k0 in range(0, T, L):
                sl = slice(k0, k0 + L)
                q, kk, v = Q[b, h, sl], K[b, h, sl] * s, V[b, h, sl]
                bcum = np.cumsum(lf[sl])
                g = bcum[-1]
                a = li[sl] - bcum
                m_tok = bcum + np.maximum(mp, np.maximum.accumulate(a))
                logD = bcum[:, None] + a[None, :]
                logD = np.where(np.tril(np.ones((L, L), dtype=bool)), logD, -np.inf)
                Wt = np.exp(logD - m_tok[:, None])
                A = Wt * (q @ kk.T)
                inter = np.exp(bcum + mp - m_tok)
                num = A @ v + inter[:, None] * (q @ C)
                den = A.sum(axis=1) + inter * (q @ n)
                denom = np.maximum(np.abs(den), np.exp(-m_tok))
                H[b, h, sl] = num / denom[:, None]
                M[b, h, sl] = m_tok
                DEN[b, h, sl] = denom
                m_new = max(g + mp, g + a.max())
                decay = math.exp(g + mp - m_new)
                w = np.exp(g + a - m_new)
                C = decay * C + (kk * w[:, None]).T @ v
                n = decay * n + (kk * w[:, None]).sum(axis=0)
                mp = m_new
            CT[b, h], NT[b, h], MT[b, h] = C, n, mp
    return dict(H=H, m=M, den=DEN, C_T=CT, n_T=NT, m_T=MT)


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

TOL = 1e-10


def pin_quadratic(run):
    for seed, gm, init in [(1, "exp", False), (2, "sigmoid", False), (3, "exp", True),
                           (4, "sigmoid", True)]:
        c = rand_case(seed, T=40, init_state=init)
        o = run(**c, gate_mode=gm)
        r = quadratic_form(**c, gate_mode=gm)
        assert rel_err(o["H"], r["H"]) < TOL, ("H vs quadratic form", seed, gm, init)
        assert np.max(np.abs(o["m"] - r["m"])) < TOL * 10, ("m vs quadratic form", seed)
        assert rel_err(o["den"], r["den"]) < TOL, ("den vs quadratic form", seed)


def pin_chunkwise(run):
    c = rand_case(5, B=2, NH=2, T=64, DK=8, DV=5, init_state=True)
    for gm in ("exp", "sigmoid"):
        o = run(**c, gate_mode=gm)
        for L in (1, 4, 16, 64):
            r = chunkwise(**c, gate_mode=gm, L=L)
            for key in ("H", "den", "C_T", "n_T"):
                assert rel_err(o[key], r[key]) < TOL, (key, "vs chunkwise", gm, L)
            assert np.max(np.abs(o["m_T"] - r["m_T"])) < TOL, ("m_T vs chunkwise", gm, L)
            assert np.max(np.abs(o["m"] - r["m"])) < TOL, ("m vs chunkwise", gm, L)


def pin_single_token(run):
    rng = np.random.default_rng(6)
    for gm in ("exp", "sigmoid"):
        for _ in range(4):
            DK, DV = 7, 3
            q, k, v = rng.standard_normal(DK), rng.standard_normal(DK), rng.standard_normal(DV)
            ip = rng.standard_normal() * 3
            fp = rng.standard_normal() * 3
            o = run(q.reshape(1, 1, 1, DK), k.reshape(1, 1, 1, DK), v.reshape(1, 1, 1, DV),
                    np.array([[[ip]]]), np.array([[[fp]]]), gate_mode=gm)
            li = ip if gm == "exp" else float(logsigmoid(ip))
            kq = float(k @ q) / math.sqrt(DK)
            want = v * kq / max(abs(kq), math.exp(-li))
            assert rel_err(o["H"][0, 0, 0], want) < TOL, ("single-token closed form", gm)


def pin_memory_hold(run):
    c = rand_case(7, T=24, init_state=True)
    c["f_pre"] = np.full_like(c["f_pre"], 1e4)
    c["i_pre"] = np.full_like(c["i_pre"], -1e4)
    o = run(**c, gate_mode="exp")
    num = np.einsum("bhtk,bhkv->bhtv", c["Q"], c["C0"])
    den = np.einsum("bhtk,bhk->bht", c["Q"], c["n0"])
    want = num / np.maximum(np.abs(den), np.exp(-c["m0"])[:, :, None])[..., None]
    assert rel_err(o["H"], want) < TOL, "memory hold: H"
    assert rel_err(o["C_T"], c["C0"]) < TOL, "memory hold: C"
    assert rel_err(o["n_T"], c["n0"]) < TOL, "memory hold: n"
    assert np.max(np.abs(o["m_T"] - c["m0"])) < TOL, "memory hold: m"


def pin_linear_attention(run):
    c = rand_case(8, T=30)
    c["f_pre"] = np.full_like(c["f_pre"], 1e4)
    c["i_pre"] = np.zeros_like(c["i_pre"])
    o = run(**c, gate_mode="exp")
    DK = c["Q"].shape[-1]
    A = np.einsum("bhtk,bhjk->bhtj", c["Q"], c["K"]) / math.sqrt(DK)
    A = A * np.tril(np.ones(A.shape[-2:]))
    num = A @ c["V"]
    den = A.sum(-1)
    want = num / np.maximum(np.abs(den), 1.0)[..., None]
    assert rel_err(o["H"], want) < TOL, "causal normalised linear attention"
    assert np.max(np.abs(o["m"])) < TOL, "stabiliser stays 0"


def pin_golden(run):
    with open(GOLDEN) as fh:
        g = json.load(fh)
    for case in g["cases"]:
        T = len(case["i_pre"])
        DK, DV = case["DK"], case["DV"]
        q = np.array(case["q"]).reshape(1, 1, T, DK)
        k = np.array(case["k"]).reshape(1, 1, T, DK)
        v = np.array(case["v"]).reshape(1, 1, T, DV)
        o = run(q, k, v, np.array(case["i_pre"]).reshape(1, 1, T),
                np.array(case["f_pre"]).reshape(1, 1, T), gate_mode=case["gate_mode"])
        nm = case["name"]
        assert np.allclose(o["H"][0, 0], np.array(case["H"]), rtol=1e-12, atol=1e-12), (nm, "H")
        assert np.allclose(o["den"][0, 0], case["den"], rtol=1e-12, atol=1e-12), (nm, "den")
        assert np.allclose(o["m"][0, 0], case["m"], rtol=1e-12, atol=1e-12), (nm, "m")
        assert np.allclose(o["C_T"][0, 0], np.array(case["C_T"]), rtol=1e-12), (nm, "C_T")
        assert np.allclose(o["n_T"][0, 0], case["n_T"], rtol=1e-12), (nm, "n_T")
        assert abs(o["m_T"][0, 0] - case["m_T"]) < 1e-12, (nm, "m_T")


def pin_invariants(run):
    c = rand_case(9, B=2, NH=3, T=36, init_state=True)
    base = run(**c, gate_mode="exp")
    # linearity in V (H and C; n and m do not depend on V)
    c2 = dict(c, V=c["V"] * 2.5, C0=c["C0"] * 2.5)
    o = run(**c2, gate_mode="exp")
    assert rel_err(o["H"], 2.5 * base["H"]) < TOL, "linearity in V"
    assert rel_err(o["C_T"], 2.5 * base["C_T"]) < TOL, "linearity in V (state)"
    # oddness in q
    o = run(**dict(c, Q=-c["Q"]), gate_mode="exp")
    assert rel_err(o["H"], -base["H"]) < TOL, "oddness in q"
    # causality: perturbing token t' leaves h_t (t < t') unchanged, and changes h_{t'}
    tp = 20
    c3 = {k_: (None if v_ is None else v_.copy()) for k_, v_ in c.items()}
    c3["K"][:, :, tp:] += 1.0
    c3["V"][:, :, tp:] -= 0.5
    c3["i_pre"][:, :, tp:] += 0.3
    c3["f_pre"][:, :, tp:] -= 0.3
    o = run(**c3, gate_mode="exp")
    assert np.array_equal(o["H"][:, :, :tp], base["H"][:, :, :tp]), "causality"
    assert rel_err(o["H"][:, :, tp:], base["H"][:, :, tp:]) > 1e-3, "later tokens respond"
    # (b, h) independence: permuting heads permutes outputs
    perm = [2, 0, 1]
    cp = {k_: (None if v_ is None else v_[:, perm]) for k_, v_ in c.items()}
    o = run(**cp, gate_mode="exp")
    assert np.array_equal(o["H"], base["H"][:, perm]), "head independence"
    # frame shift of the initial state leaves H unchanged
    delta = 1.7
    cs = dict(c, m0=c["m0"] + delta, C0=c["C0"] * math.exp(-delta), n0=c["n0"] * math.exp(-delta))
    o = run(**cs, gate_mode="exp")
    assert rel_err(o["H"], base["H"]) < 1e-9, "stabiliser frame shift"
    # segment resume: T/2 + T/2 with the carried state equals one call
    T = c["Q"].shape[2]
    h1 = {k_: (v_[:, :, : T // 2] if k_ in ("Q", "K", "V", "i_pre", "f_pre") else v_)
          for k_, v_ in c.items()}
    o1 = run(**h1, gate_mode="exp")
    h2 = {k_: v_[:, :, T // 2:] for k_, v_ in c.items() if k_ in ("Q", "K", "V", "i_pre", "f_pre")}
    o2 = run(**h2, C0=o1["C_T"], n0=o1["n_T"], m0=o1["m_T"], gate_mode="exp")
    assert rel_err(np.concatenate([o1["H"], o2["H"]], axis=2), base["H"]) < TOL, "segment resume H"
    assert rel_err(o2["C_T"], base["C_T"]) < TOL, "segment resume C"
    assert np.max(np.abs(o2["m_T"] - base["m_T"])) < TOL, "segment resume m"


def pin_snapshots(run):
    c = rand_case(10, T=48, init_state=True)
    o = run(**c, gate_mode="sigmoid", snap_every=16)
    for j in range(3):
        t = 16 * j
        if t == 0:
            assert np.array_equal(o["C_snap"][:, :, 0], c["C0"]), "snapshot 0 is the initial state"
            continue
        part = {k_: (v_[:, :, :t] if k_ in ("Q", "K", "V", "i_pre", "f_pre") else v_)
                for k_, v_ in c.items()}
        p = run(**part, gate_mode="sigmoid")
        assert rel_err(o["C_snap"][:, :, j], p["C_T"]) < TOL, "snapshot C"
        assert rel_err(o["n_snap"][:, :, j], p["n_T"]) < TOL, "snapshot n"
        assert np.max(np.abs(o["m_snap"][:, :, j] - p["m_T"])) < TOL, "snapshot m"


ALL_PINS = [pin_quadratic, pin_chunkwise, pin_single_token, pin_memory_hold,
            pin_linear_attention, pin_golden, pin_invariants, pin_snapshots]


# ----------------------------------------------------------------------------
# the sigmoid-input-gate variant with reduced computation (no stabiliser, no
# normaliser): h_t = C_t^T q_t, C_t = sig(f~_t) C_{t-1} + sig(i~_t) (s k_t) v_t^T
# ----------------------------------------------------------------------------

def quadratic_form_sigmoid_plain(Q, K, V, i_pre, f_pre, C0=None, n0=None, m0=None):
    """Fully parallel form of the variant, per (b, h): with F_t = sum_{l<=t}
    log sig(f~_l), token j enters the read-out at t with weight
    sig(i~_j) exp(F_t - F_j) (j <= t) and the initial state with
    exp(F_t + m0); H = ((s Q K^T) o W) V + exp(F + m0) (Q C0).  The final state
    is the same sum at t = T."""
    B, NH, T, DK = Q.shape
    DV = V.shape[-1]
    s = 1.0 / math.sqrt(DK)
    H = np.zeros((B, NH, T, DV))
    C_T = np.zeros((B, NH, DK, DV))
    n_T = np.zeros((B, NH, DK))
    for b in range(B):
        for h in range(NH):
            lf = logsigmoid(f_pre[b, h])
            li = logsigmoid(i_pre[b, h])
            F = np.cumsum(lf)
            causal = np.tril(np.ones((T, T), dtype=bool))
            W = np.where(causal, np.exp(F[:, None] - F[None, :] + li[None, :]), 0.0)
            H[b, h] = (W * (s * Q[b, h] @ K[b, h].T)) @ V[b, h]
            wT = np.exp(F[-1] - F + li) if T else np.zeros(0)
            C_T[b, h] = (K[b, h] * (s * wT)[:, None]).T @ V[b, h]
            n_T[b, h] = (K[b, h] * (s * wT)[:, None]).sum(axis=0)
            if C0 is not None:
                g = np.exp(F + float(m0[b, h]))
                H[b, h] += g[:, None] * (Q[b, h] @ C0[b, h])
                gT = math.exp((F[-1] if T else 0.0) + float(m0[b, h]))
                C_T[b, h] += gT * C0[b, h]
                n_T[b, h] += gT * n0[b, h]
    return dict(H=H, C_T=C_T, n_T=n_T)


def pin_sig_quadratic(run_plain):
    for init in (False, True):
        c = rand_case(31, T=40, init_state=init)
        o = run_plain(**c)
        r = quadratic_form_sigmoid_plain(**c)
        assert rel_err(o["H"], r["H"]) < TOL, "plain sigmoid H vs quadratic form"
        assert rel_err(o["C_T"], r["C_T"]) < TOL, "plain sigmoid C_T vs quadratic form"
        assert rel_err(o["n_T"], r["n_T"]) < TOL, "plain sigmoid n_T vs quadratic form"


def pin_sig_single_token(run_plain):
    """T = 1 from a zero state: h = sig(i~) s (k.q) v."""
    c = rand_case(32, T=1, DK=5, DV=3)
    o = run_plain(**c)
    q, k, v = c["Q"][0, :, 0], c["K"][0, :, 0], c["V"][0, :, 0]
    ig = 1.0 / (1.0 + np.exp(-c["i_pre"][0, :, 0]))
    want = (ig * (q * k).sum(-1) / math.sqrt(5))[:, None] * v
    assert rel_err(o["H"][0, :, 0], want) < TOL, "plain sigmoid single token"


def pin_sig_memory_hold(run_plain):
    """sig(f~) = 1 and sig(i~) = 0 (f~ = +1e4, i~ = -1e4): h_t = e^{m0} C0^T q_t."""
    c = rand_case(33, T=12, init_state=True)
    c["f_pre"] = np.full_like(c["f_pre"], 1e4)
    c["i_pre"] = np.full_like(c["i_pre"], -1e4)
    o = run_plain(**c)
    want = np.exp(c["m0"])[:, :, None, None] * np.einsum("bhtk,bhkv->bhtv", c["Q"], c["C0"])
    assert rel_err(o["H"], want) < TOL, "plain sigmoid memory hold"


def pin_sig_against_stabilised(run_plain):
    """The variant's state is the sigmoid mode's state in the frame m = 0, and
    its output is that mode's h times its denominator and e^{m}: the two oracle
    functions (different code) must agree on both."""
    c = rand_case(34, T=36, init_state=True)
    o = run_plain(**c)
    st = oracle.mlstm_recurrent(**c, gate_mode="sigmoid")
    e = np.exp(st["m_T"])
    assert rel_err(o["C_T"], e[:, :, None, None] * st["C_T"]) < TOL, "plain vs stabilised C_T"
    assert rel_err(o["n_T"], e[:, :, None] * st["n_T"]) < TOL, "plain vs stabilised n_T"
    scale = np.exp(st["m"]) * st["den"]
    assert rel_err(o["H"], st["H"] * scale[..., None]) < TOL, "plain vs stabilised H"


SIG_PLAIN_PINS = [pin_sig_quadratic, pin_sig_single_token, pin_sig_memory_hold,
                  pin_sig_against_stabilised]
