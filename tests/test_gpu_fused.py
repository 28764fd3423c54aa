"""The fused kernel (chunk state carried on chip) against the fp64 oracle
(needs a B200).  It covers d_qk = 128, d_v of 64 or 128 and chunks of 128
tokens; the cases include several heads per CTA (the state and the n vector
handed over between heads), ragged and sub-chunk sequences, a given initial
state and the sigmoid input gate."""
import pytest
import torch

import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    dict(B=1, NH=2, T=1024, DV=128),
    dict(B=2, NH=3, T=1000, DV=64),    # ragged tail, d_v 64 (double-buffered V)
    dict(B=4, NH=80, T=256, DV=128),   # 320 heads: several heads per CTA
    dict(B=1, NH=1, T=128, DV=128),    # one chunk
    dict(B=1, NH=1, T=5, DV=64),       # shorter than a chunk
]


def _case(c, **over):
    return WORKLOADS["mid"].replace(name="fused", DK=128, chunk_size=128, **c, **over)


def _run(w, x, algo):
    d = parity.to_dev(x)
    H, fin = api.mlstm_fw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"], d["n0"],
                          d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode, algo=algo)
    torch.cuda.synchronize()
    st = api.last_device_error()
    assert st == _lib.OK, \
        f"device status {st}, error word 0x{_lib.lib().mlstm_last_device_error_word():08x}"
    return H, fin


@pytest.mark.parametrize("c", CASES, ids=lambda c: "x".join(str(v) for v in c.values()))
def test_fused_matches_oracle(c):
    w = _case(c)
    x = make_inputs(w)
    H, fin = _run(w, x, "tc_fused")
    ref = parity.oracle_run(x, w.gate_mode)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"fused {c}")


def test_fused_initial_state_and_sigmoid_gate():
    w = _case(dict(B=2, NH=4, T=640, DV=128), gate_mode="sigmoid", init_state=True)
    x = make_inputs(w)
    x["m0"] = torch.tensor([[0.5, -1.0, 2.0, 0.0], [1.5, -0.5, 0.25, 3.0]])
    H, fin = _run(w, x, "tc_fused")
    ref = parity.oracle_run(x, w.gate_mode)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], label="fused init/sigmoid")


def test_fused_agrees_with_the_unfused_path():
    w = _case(dict(B=2, NH=8, T=2048, DV=128))
    x = make_inputs(w)
    Hf, (Cf, nf, mf) = _run(w, x, "tc_fused")
    Hu, (Cu, nu, mu) = _run(w, x, "tc")
    assert parity.worst_rel(Hf.double().cpu().numpy(), Hu.double().cpu().numpy()) < 2e-2
    assert parity.worst_rel(Cf.double().cpu().numpy(), Cu.double().cpu().numpy()) < 2e-2
    assert torch.equal(mf.cpu(), mu.cpu())
