"""Single-token step kernel (mlstm_step) against the fp64 oracle.

The oracle's token-by-token recurrence with a given initial state is, for one
token, exactly the step; over T tokens from a zero state it is T steps.  The
step must also continue a sequence that mlstm_fw has processed: T tokens by
mlstm_fw, then one step, equal T + 1 tokens by the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# d_v 1024: 8 tiles per cluster; 262: two launches; 97 x 33 two 32-column
# tiles (4-byte accesses), the last one ragged; 300 and 200 rows are not a
# multiple of the eight rows a batch keeps in flight per warp.
SHAPES = [(2, 3, 64, 64), (1, 4, 128, 128), (2, 2, 256, 512), (1, 2, 100, 72), (1, 1, 1, 1),
          (1, 2, 64, 1024), (1, 2, 32, 262), (1, 2, 300, 96), (1, 1, 200, 40), (3, 1, 97, 33)]


def _state(B, NH, DK, DV, seed):
    g = torch.Generator().manual_seed(seed)
    C = torch.randn((B, NH, DK, DV), generator=g) * 0.1
    n = torch.randn((B, NH, DK), generator=g) * 0.1
    m = torch.randn((B, NH), generator=g)
    return C, n, m


def _token(B, NH, DK, DV, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, NH, DK), generator=g).to(dtype)
    k = torch.randn((B, NH, DK), generator=g).to(dtype)
    v = torch.randn((B, NH, DV), generator=g).to(dtype)
    i_pre = torch.randn((B, NH), generator=g)
    f_pre = torch.rand((B, NH), generator=g) * 3 + 3
    return q, k, v, i_pre, f_pre


def _check_ok():
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK


@pytest.mark.parametrize("gate_mode", ["exp", "sigmoid"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_one_step_from_a_given_state(shape, dtype, gate_mode):
    B, NH, DK, DV = shape
    C, n, m = _state(B, NH, DK, DV, 7)
    q, k, v, i_pre, f_pre = _token(B, NH, DK, DV, dtype, 8)
    ref = oracle.mlstm_recurrent(q[:, :, None], k[:, :, None], v[:, :, None], i_pre[:, :, None],
                                 f_pre[:, :, None], C, n, m, gate_mode=gate_mode)
    Cd, nd, md = C.cuda(), n.cuda(), m.cuda()
    h = api.mlstm_step(q.cuda(), k.cuda(), v.cuda(), i_pre.cuda(), f_pre.cuda(), Cd, nd, md,
                       gate_mode=gate_mode)
    _check_ok()
    tol = parity.TOL["bf16" if dtype == torch.bfloat16 else "f32"]
    assert parity.worst_rel(h.double().cpu().numpy(), ref["H"][:, :, 0]) < tol
    assert parity.worst_rel(Cd.double().cpu().numpy(), ref["C_T"]) < tol
    assert parity.worst_rel(nd.double().cpu().numpy(), ref["n_T"]) < tol
    assert parity.m_err(md.double().cpu().numpy(), ref["m_T"]) < 1e-5


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_steps_from_zero_equal_the_sequence(dtype):
    """40 steps from the zero state = the oracle over the 40 tokens."""
    B, NH, DK, DV, T = 2, 2, 128, 64, 40
    w = WORKLOADS["mid"].replace(name="steps", B=B, NH=NH, T=T, DK=DK, DV=DV,
                                 dtype="bf16" if dtype == torch.bfloat16 else "f32")
    x = make_inputs(w)
    ref = parity.oracle_run(x, w.gate_mode)
    d = parity.to_dev(x)
    C = torch.zeros((B, NH, DK, DV), device="cuda")
    n = torch.zeros((B, NH, DK), device="cuda")
    m = torch.zeros((B, NH), device="cuda")
    hs = []
    for t in range(T):
        hs.append(api.mlstm_step(d["Q"][:, :, t].contiguous(), d["K"][:, :, t].contiguous(),
                                 d["V"][:, :, t].contiguous(), d["i_pre"][:, :, t].contiguous(),
                                 d["f_pre"][:, :, t].contiguous(), C, n, m))
    _check_ok()
    H = torch.stack(hs, dim=2)
    tol = parity.TOL[w.dtype]
    parity.compare(H, (C, n, m), ref, tol, label=f"{T} steps {w.dtype}")


@pytest.mark.parametrize("algo", ["auto", "tc", "simt"])
def test_step_continues_a_forward_pass(algo):
    """mlstm_fw over T tokens, then one step == the oracle over T + 1 tokens."""
    w = WORKLOADS["mid"].replace(name="cont", B=1, NH=2, T=513, chunk_size=128)
    x = make_inputs(w)
    ref = parity.oracle_run(x, w.gate_mode)
    d = parity.to_dev(x)
    T = w.T - 1
    head = {k: d[k][:, :, :T].contiguous() for k in ("Q", "K", "V", "i_pre", "f_pre")}
    try:
        _, (C, n, m) = api.mlstm_fw(head["Q"], head["K"], head["V"], head["i_pre"],
                                    head["f_pre"], chunk_size=w.chunk_size, algo=algo)
    except api.MlstmError as e:
        assert e.status == _lib.ERR_UNSUPPORTED
        pytest.skip(f"{algo} unsupported")
    h = api.mlstm_step(d["Q"][:, :, T].contiguous(), d["K"][:, :, T].contiguous(),
                       d["V"][:, :, T].contiguous(), d["i_pre"][:, :, T].contiguous(),
                       d["f_pre"][:, :, T].contiguous(), C, n, m)
    _check_ok()
    tol = parity.TOL[w.dtype]
    assert parity.worst_rel(h.double().cpu().numpy(), ref["H"][:, :, T]) < tol
    assert parity.worst_rel(C.double().cpu().numpy(), ref["C_T"]) < tol
    assert parity.worst_rel(n.double().cpu().numpy(), ref["n_T"]) < tol
    assert parity.m_err(m.double().cpu().numpy(), ref["m_T"]) < 1e-5


def test_step_rejects_bad_arguments_before_launching():
    B, NH, DK, DV = 1, 1, 64, 64
    q = torch.zeros((B, NH, DK), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((B, NH, DV), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((B, NH), device="cuda")
    C = torch.zeros((B, NH, DK, DV), device="cuda")
    n = torch.zeros((B, NH, DK), device="cuda")
    with pytest.raises(ValueError):
        api.mlstm_step(q, q, v, g, g, C, n, torch.zeros((B, NH, 2), device="cuda"))
    lib = _lib.lib()
    st = lib.mlstm_step(q.data_ptr(), q.data_ptr(), v.data_ptr(), g.data_ptr(), g.data_ptr(),
                        C.data_ptr(), n.data_ptr(), None, v.data_ptr(), B, NH, DK, DV,
                        _lib.DT_BF16, _lib.GATE_EXP, None)
    assert st == _lib.ERR_INVALID_ARG
    st = lib.mlstm_step(q.data_ptr(), q.data_ptr(), v.data_ptr(), g.data_ptr(), g.data_ptr(),
                        C.data_ptr(), n.data_ptr(), g.data_ptr(), v.data_ptr(), B, NH, 2048, DV,
                        _lib.DT_BF16, _lib.GATE_EXP, None)
    assert st == _lib.ERR_UNSUPPORTED


def test_step_full_size_sampled_heads():
    """The 7B-shaped decode batch that `bench.py --op step` times (B=8, NH=8,
    256 x 512 states, bf16 tokens): one step from a random state, two heads
    (the first and the last) recomputed by the oracle."""
    B, NH, DK, DV = 8, 8, 256, 512
    C, n, m = _state(B, NH, DK, DV, 51)
    q, k, v, i_pre, f_pre = _token(B, NH, DK, DV, torch.bfloat16, 52)
    Cd, nd, md = C.cuda(), n.cuda(), m.cuda()
    h = api.mlstm_step(q.cuda(), k.cuda(), v.cuda(), i_pre.cuda(), f_pre.cuda(), Cd, nd, md)
    _check_ok()
    heads = [(0, 0), (B - 1, NH - 1)]
    x = {"Q": q[:, :, None], "K": k[:, :, None], "V": v[:, :, None],
         "i_pre": i_pre[:, :, None], "f_pre": f_pre[:, :, None], "C0": C, "n0": n, "m0": m}
    ref = parity.oracle_run(x, "exp", heads=heads)
    tol = parity.TOL["bf16"]
    assert parity.worst_rel(parity.pick(h, heads), ref["H"][:, :, 0]) < tol
    assert parity.worst_rel(parity.pick(Cd, heads), ref["C_T"]) < tol
    assert parity.worst_rel(parity.pick(nd, heads), ref["n_T"]) < tol
    assert parity.m_err(parity.pick(md, heads), ref["m_T"]) < 1e-5
