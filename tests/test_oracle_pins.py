"""The fp64 oracle against everything that fixes it independently (CPU only)."""
import numpy as np
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.mlstm_recurrent)


def test_independent_references_agree():
    """The quadratic and chunkwise references agree with each other too."""
    c = pins.rand_case(11, T=32, init_state=True)
    q = pins.quadratic_form(**c, gate_mode="sigmoid")
    for L in (2, 8, 32):
        r = pins.chunkwise(**c, gate_mode="sigmoid", L=L)
        assert pins.rel_err(r["H"], q["H"]) < 1e-10
        assert np.max(np.abs(r["m"] - q["m"])) < 1e-9


def test_rejects_bad_arguments():
    c = pins.rand_case(12, T=8, init_state=True)
    with pytest.raises(ValueError):
        oracle.mlstm_recurrent(**dict(c, n0=None), gate_mode="exp")  # partial state
    with pytest.raises(ValueError):
        oracle.mlstm_recurrent(**c, gate_mode="exp", snap_every=3)   # 3 does not divide 8


def test_empty_sequence():
    c = pins.rand_case(13, T=8, init_state=True)
    c = {k: (v[:, :, :0] if k in ("Q", "K", "V", "i_pre", "f_pre") else v) for k, v in c.items()}
    o = oracle.mlstm_recurrent(**c, gate_mode="exp")
    assert o["H"].shape[2] == 0
    assert np.array_equal(o["C_T"], c["C0"]) and np.array_equal(o["m_T"], c["m0"])


def test_bf16_inputs_up_cast_exactly():
    """Workload inputs reach the oracle as their exact fp64 values."""
    import torch
    from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled
    w = scaled(WORKLOADS["mid"], B=1, NH=1, T=16, DK=8, DV=8)
    x = make_inputs(w)
    assert x["Q"].dtype == torch.bfloat16
    o = oracle.mlstm_recurrent(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"])
    c = {k: x[k].double().numpy() for k in ("Q", "K", "V", "i_pre", "f_pre")}
    r = pins.quadratic_form(**c)
    assert pins.rel_err(o["H"], r["H"]) < 1e-10


@pytest.mark.parametrize("pin", pins.SIG_PLAIN_PINS, ids=lambda p: p.__name__)
def test_sigmoid_plain_oracle_pin(pin):
    pin(oracle.mlstm_sigmoid_plain)
