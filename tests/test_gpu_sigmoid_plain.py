"""The sigmoid-input-gate variant with reduced computation on the GPU (needs a
B200), against its plain-definition oracle (unstabilised, no normaliser):
h_t = C_t^T q_t, C_t = sig(f~_t) C_{t-1} + sig(i~_t) (s k_t) v_t^T.

Every algorithm that takes the shape, the workload draws and the gate regimes
(strong forgetting, memory hold, constant gates), the parallel call, the
single-token step and the full-size long-context workload on sampled heads.
The returned final state is the sigmoid mode's, in the frame m_T: it is
compared as e^{m_T} C_T with the oracle's unstabilised state."""
import numpy as np
import pytest
import torch

import oracle
import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu

ALGOS = ("simt", "tc", "tc_fused")
SHAPES = {
    "d128_L128": dict(DK=128, DV=128, chunk_size=128, T=1024),
    "d128_L64": dict(DK=128, DV=128, chunk_size=64, T=1000),
    "d256x512_L256": dict(DK=256, DV=512, chunk_size=256, T=1024),
    "d256x512_L512": dict(DK=256, DV=512, chunk_size=512, T=1536),
}
CASES = ("draws", "strong_forget", "hold", "constant")


def workload(shape, case):
    return WORKLOADS["sigmoid_long_plain"].replace(name=f"plain_{case}_{shape}", B=1, NH=2,
                                                   **SHAPES[shape])


def inputs(shape, case):
    w = workload(shape, case)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(91)
    if case == "strong_forget":
        x["f_pre"] = torch.rand(x["f_pre"].shape, generator=g) * 5.0 - 4.0
    elif case == "hold":
        x["f_pre"] = torch.full_like(x["f_pre"], 1e4)
        x["i_pre"] = torch.full_like(x["i_pre"], -1e4)
    elif case == "constant":  # sig(f~) = 1, sig(i~) = 1/2: unnormalised linear attention
        x["f_pre"] = torch.full_like(x["f_pre"], 1e4)
        x["i_pre"] = torch.zeros_like(x["i_pre"])
    return w, x


def supported(w, algo):
    try:
        api.workspace_size(w.B, w.NH, w.T, w.DK, w.DV, w.chunk_size, w.torch_dtype, algo)
        return True
    except api.MlstmError as e:
        assert e.status == _lib.ERR_UNSUPPORTED
        return False


def plain_oracle(x, heads=None):
    if heads is not None:
        x = parity.slice_heads(x, heads)
    return oracle.mlstm_sigmoid_plain(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"], x["C0"],
                                      x["n0"], x["m0"])


def check(w, x, algo, heads=None):
    d = parity.to_dev(x)
    H, (C_T, n_T, m_T) = api.mlstm_fw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"],
                                      d["n0"], d["m0"], chunk_size=w.chunk_size,
                                      gate_mode="sigmoid_plain", algo=algo)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    ref = plain_oracle(x, heads)
    tol = parity.TOL[w.dtype]
    Hn = parity.pick(H, heads)
    e = np.exp(parity.pick(m_T, heads))
    errs = {"H": parity.worst_rel(Hn, ref["H"]),
            "C_T": parity.worst_rel(e[..., None, None] * parity.pick(C_T, heads), ref["C_T"]),
            "n_T": parity.worst_rel(e[..., None] * parity.pick(n_T, heads), ref["n_T"])}
    assert all(v <= tol for v in errs.values()), \
        f"{w.name}/{algo}: {errs}, worst row {parity.worst_row_rel(Hn, ref['H']):.2e}"


def combos():
    out = []
    for c in CASES:
        for s in SHAPES:
            for a in ALGOS:
                try:
                    ok = supported(workload(s, c), a)
                except Exception:  # library not loadable here: keep every pair
                    ok = True
                if ok:
                    out.append((c, s, a))
    return out


@pytest.mark.parametrize("case,shape,algo", combos())
def test_sigmoid_plain(case, shape, algo):
    w, x = inputs(shape, case)
    check(w, x, algo)


def test_sigmoid_plain_full_size_sampled_heads():
    """The long-context workload in the launch configuration the bench times."""
    w = WORKLOADS["sigmoid_long_plain"]
    x = make_inputs(w)
    check(w, x, "auto", heads=[(0, 0), (w.B - 1, w.NH - 1)])


def test_sigmoid_plain_parallel_call_and_step():
    """mlstm_fw_chunk_states + mlstm_fw_parallel give the variant's H, and one
    mlstm_step continues the sequence by a token (oracle over T + 1 tokens)."""
    w, x = inputs("d128_L128", "draws")
    d = parity.to_dev(x)
    T = w.T
    ref = plain_oracle(x)
    C_s, n_s, m_s, _ = api.mlstm_fw_chunk_states(d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"],
                                                 d["n0"], d["m0"], chunk_size=w.chunk_size,
                                                 gate_mode="sigmoid_plain", algo="tc")
    H, n_out, m_out = api.mlstm_fw_parallel(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], C_s,
                                            n_s, d["m0"], chunk_size=w.chunk_size,
                                            gate_mode="sigmoid_plain", algo="tc")
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    assert parity.worst_rel(H.double().cpu().numpy(), ref["H"]) <= parity.TOL[w.dtype]
    # the step: the first T - 1 tokens through mlstm_fw, then token T - 1
    sl = lambda a: a[:, :, :T - 1].contiguous()  # noqa: E731
    _, (C, n, m) = api.mlstm_fw(sl(d["Q"]), sl(d["K"]), sl(d["V"]), sl(d["i_pre"]),
                                sl(d["f_pre"]), d["C0"], d["n0"], d["m0"],
                                chunk_size=w.chunk_size, gate_mode="sigmoid_plain")
    h = api.mlstm_step(d["Q"][:, :, -1].contiguous(), d["K"][:, :, -1].contiguous(),
                       d["V"][:, :, -1].contiguous(), d["i_pre"][:, :, -1].contiguous(),
                       d["f_pre"][:, :, -1].contiguous(), C, n, m, gate_mode="sigmoid_plain")
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    want = ref["H"][:, :, -1]
    err = float(np.max(np.abs(h.double().cpu().numpy() - want)) / np.max(np.abs(want)))
    assert err <= parity.TOL[w.dtype], err


def test_sigmoid_plain_has_no_backward():
    w, x = inputs("d128_L128", "draws")
    d = parity.to_dev(x)
    with pytest.raises(api.MlstmError) as e:
        api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], torch.zeros_like(d["V"]),
                     d["C0"], d["n0"], d["m0"], chunk_size=128, gate_mode="sigmoid_plain")
    assert e.value.status == _lib.ERR_UNSUPPORTED
