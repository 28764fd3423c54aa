"""Backward pass (mlstm_bw) against the fp64 autograd oracle.

Same seeded inputs on both sides; the upstream gradient dH is drawn in the
input dtype.  Metric as the forward's: per (b, h) slice, max|x - y| / max|y|.
"""
import pytest
import torch

import parity
from oracle import backward as ob
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# tolerance of the gradients: as the forward's for bf16 inputs; fp32 inputs
# accumulate the suffix sums of the forget-gate gradient over T tokens in fp32
TOL = {"f32": 1e-4, "bf16": 2e-2}

CASES = [
    # B, NH, T, DK, DV, chunk, dtype, gate, initial state
    (1, 2, 256, 64, 64, 64, "f32", "exp", False),
    (1, 2, 256, 64, 64, 64, "bf16", "exp", False),
    (2, 1, 200, 64, 64, 64, "f32", "exp", True),        # ragged tail, initial state
    (1, 2, 512, 128, 128, 128, "bf16", "exp", False),
    (1, 2, 512, 128, 128, 256, "f32", "sigmoid", True),
    (1, 1, 130, 100, 72, 64, "f32", "exp", True),       # dims that are not tile multiples
    (1, 2, 1, 64, 64, 64, "f32", "exp", True),          # single token
    (1, 2, 640, 256, 512, 256, "bf16", "exp", True),    # 7B head shape: forward recomputed on TC
    (1, 2, 384, 128, 128, 64, "bf16", "sigmoid", False),  # chunk 64 on TC (pair mode)
    # bf16 with d_qk 128 or 256: tensor-core gradients on 128-token chunks
    (2, 2, 200, 128, 256, 64, "bf16", "exp", True),     # ragged last chunk, 2 value tiles
    (1, 1, 2048, 128, 128, 256, "bf16", "sigmoid", True),  # one head: segmented recurrences
    (1, 2, 130, 128, 128, 128, "bf16", "exp", True),    # a 2-token last chunk
    (2, 1, 100, 128, 128, 128, "bf16", "exp", True),    # shorter than a chunk: fp32 kernels
    (1, 2, 300, 256, 256, 512, "bf16", "sigmoid", True),  # d_qk 256 x d_v 256, ragged
    (1, 1, 256, 128, 1024, 256, "bf16", "exp", True),   # widest d_v: 16 column blocks per row
    (1, 2, 260, 256, 128, 128, "bf16", "exp", False),   # d_qk 256 x d_v 128
]


def _grad_case(B, NH, T, DK, DV, L, dtype, gate, init, seed=11):
    w = WORKLOADS["mid"].replace(name="bw", B=B, NH=NH, T=T, DK=DK, DV=DV, chunk_size=L,
                                 dtype=dtype, gate_mode=gate, init_state=init, i_mean=0.0)
    x = make_inputs(w, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    dH = torch.randn((B, NH, T, DV), generator=g).to(w.torch_dtype)
    ref = ob.gradients(x, dH, gate)
    d = parity.to_dev(x)
    got = api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH.cuda(), d["C0"],
                       d["n0"], d["m0"], chunk_size=L, gate_mode=gate)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    return w, ref, got


def _errors(ref, got):
    names = [("dQ", "dQ"), ("dK", "dK"), ("dV", "dV"), ("di_pre", "di_pre"), ("df_pre", "df_pre")]
    if "dC0" in got:
        names += [("dC0", "dC0"), ("dn0", "dn0")]
    errs = {k: parity.worst_rel(got[g].double().cpu().numpy(), ref[k].numpy()) for g, k in names}
    if "dm0" in got:
        errs["dm0"] = float((got["dm0"].double().cpu() - ref["dm0"]).abs().max()
                            / max(1.0, float(ref["dm0"].abs().max())))
    return errs


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_autograd_oracle(case):
    w, ref, got = _grad_case(*case)
    errs = _errors(ref, got)
    bad = {k: v for k, v in errs.items() if not v <= TOL[w.dtype]}
    assert not bad, f"{case}: {errs}"


@pytest.mark.parametrize("gates", [(4.0, -3.0, 6.0), (-6.0, 0.0, 2.0)],
                         ids=["big-input-strong-forget", "small-input-fast-forget"])
def test_tensor_core_backward_extreme_gates(gates):
    """Tensor-core backward (bf16, 128-token chunks) with gate statistics far
    from the workloads': i_pre ~ N(mu, 1) with mu = 4 (inputs that dominate the
    stabiliser inside a chunk) or -6, f_pre ~ U(lo, hi) reaching strong
    forgetting (f~ = -3: f = 0.05 per token)."""
    mu, lo, hi = gates
    w = WORKLOADS["mid"].replace(name="bw_gates", B=1, NH=3, T=384, DK=128, DV=256,
                                 chunk_size=128, dtype="bf16", gate_mode="exp",
                                 init_state=True, i_mean=mu, f_low=lo, f_high=hi)
    x = make_inputs(w, seed=31)
    g = torch.Generator().manual_seed(32)
    dH = torch.randn((w.B, w.NH, w.T, w.DV), generator=g).to(w.torch_dtype)
    ref = ob.gradients(x, dH, w.gate_mode)
    d = parity.to_dev(x)
    got = api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH.cuda(), d["C0"],
                       d["n0"], d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    errs = _errors(ref, got)
    bad = {k: v for k, v in errs.items() if not v <= TOL["bf16"]}
    assert not bad, f"{gates}: {errs}"


@pytest.mark.parametrize("name", ["xlstm7b", "sigmoid_long"])
def test_backward_full_size_sampled_heads(name):
    """The full workload shape through mlstm_bw (the launch configuration
    `bench.py --op bw` times), with the upstream gradient nonzero only on the
    first T1 tokens of two heads (the first and the last).  The loss then sees
    nothing else, so those heads' gradients on their first T1 tokens (and of
    their initial state) equal the oracle's on the truncated sequences, and
    every other gradient is exactly zero: later tokens, and every other head."""
    w = WORKLOADS[name]
    T1 = 384
    x = make_inputs(w)
    heads = [(0, 0), (w.B - 1, w.NH - 1)]
    g = torch.Generator().manual_seed(41)
    dH = torch.zeros((w.B, w.NH, w.T, w.DV), dtype=w.torch_dtype)
    for b, h in heads:
        dH[b, h, :T1] = torch.randn((T1, w.DV), generator=g).to(w.torch_dtype)
    d = parity.to_dev(x)
    got = api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH.cuda(), d["C0"],
                       d["n0"], d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    del d
    # the oracle on the sampled heads' first T1 tokens
    xs = parity.slice_heads(x, heads)
    per_token = ("Q", "K", "V", "i_pre", "f_pre")
    xt = {k: (None if v is None else (v[:, :, :T1].contiguous() if k in per_token else v))
          for k, v in xs.items()}
    dHt = torch.stack([dH[b, h, :T1] for b, h in heads], 0).unsqueeze(0)
    ref = ob.gradients(xt, dHt, w.gate_mode)
    errs = {}
    for k in ("dQ", "dK", "dV", "di_pre", "df_pre"):
        t = got[k]
        sampled = torch.stack([t[b, h, :T1] for b, h in heads], 0).unsqueeze(0)
        errs[k] = parity.worst_rel(sampled.double().cpu().numpy(), ref[k].numpy())
        for b, h in heads:
            assert not t[b, h, T1:].any(), f"{k}: gradient after the last token of the loss"
        assert not t[0, 1].any() and not t[w.B - 1, 0].any(), f"{k}: gradient on a head outside the loss"
    if "dC0" in got:
        for k in ("dC0", "dn0"):
            sampled = torch.stack([got[k][b, h] for b, h in heads], 0).unsqueeze(0)
            errs[k] = parity.worst_rel(sampled.double().cpu().numpy(), ref[k].numpy())
    bad = {k: v for k, v in errs.items() if not v <= TOL[w.dtype]}
    assert not bad, f"{name}: {errs}"


def test_backward_chunk_size_invariance():
    """The gradients do not depend on the chunk size (64, 128, 256)."""
    outs = []
    for L in (64, 128, 256):
        _, _, got = _grad_case(1, 2, 512, 64, 64, L, "f32", "exp", True)
        outs.append(got)
    for o in outs[1:]:
        for k in ("dQ", "dK", "dV", "di_pre", "df_pre", "dC0"):
            assert parity.worst_rel(o[k].double().cpu().numpy(),
                                    outs[0][k].double().cpu().numpy()) < 1e-4, k


def test_autograd_function_matches_the_oracle():
    """mlstm_chunkwise under torch.autograd: loss.backward() fills the inputs'
    .grad with the oracle's gradients (bf16 inputs, initial state)."""
    w = WORKLOADS["mid"].replace(name="ag", B=1, NH=2, T=384, chunk_size=128, init_state=True)
    x = make_inputs(w, seed=21)
    g = torch.Generator().manual_seed(22)
    dH = torch.randn((w.B, w.NH, w.T, w.DV), generator=g).to(w.torch_dtype)
    ref = ob.gradients(x, dH, w.gate_mode)
    leaves = {k: v.cuda().requires_grad_(True) for k, v in x.items() if v is not None}
    H, _ = api.mlstm_chunkwise(leaves["Q"], leaves["K"], leaves["V"], leaves["i_pre"],
                               leaves["f_pre"], leaves["C0"], leaves["n0"], leaves["m0"],
                               chunk_size=w.chunk_size)
    (H.float() * dH.cuda().float()).sum().backward()
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    for name in ("Q", "K", "V", "i_pre", "f_pre", "C0", "n0"):
        err = parity.worst_rel(leaves[name].grad.double().cpu().numpy(), ref["d" + name].numpy())
        assert err < TOL[w.dtype], (name, err)
