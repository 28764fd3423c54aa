"""Training pair (mlstm_fw_train + mlstm_bw_saved) against the oracles and
against the recomputing backward.

The pair runs the same kernels as the tensor-core backward's recomputation,
on the same 128-token chunking, so the saved buffer holds exactly what
mlstm_bw recomputes: the gradients must equal mlstm_bw's bit for bit, except
the gate gradients, whose per-token dot products are summed with atomics in
a run-dependent order.
"""
import pytest
import torch

import parity
from oracle import backward as ob
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, NH, T, DK, DV, gate, initial state
    (1, 2, 384, 128, 128, "exp", True),
    (1, 2, 300, 256, 512, "sigmoid", True),   # ragged last chunk, 7B head dims
    (2, 1, 200, 128, 256, "exp", False),
]


def _inputs(B, NH, T, DK, DV, gate, init, seed=61):
    w = WORKLOADS["mid"].replace(name="train", B=B, NH=NH, T=T, DK=DK, DV=DV, chunk_size=128,
                                 dtype="bf16", gate_mode=gate, init_state=init, i_mean=0.0)
    x = make_inputs(w, seed=seed)
    dH = torch.randn((B, NH, T, DV), generator=torch.Generator().manual_seed(seed + 1)).to(
        torch.bfloat16)
    return w, x, dH


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_train_pair(case):
    w, x, dH = _inputs(*case)
    d = parity.to_dev(x)
    H, fin, saved = api.mlstm_fw_train(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"],
                                       d["n0"], d["m0"], gate_mode=w.gate_mode)
    g_saved = api.mlstm_bw_saved(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], H, saved,
                                 dH.cuda(), d["C0"], d["n0"], d["m0"], gate_mode=w.gate_mode)
    g_rec = api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH.cuda(), d["C0"],
                         d["n0"], d["m0"], chunk_size=128, gate_mode=w.gate_mode)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    # forward: H and the final state against the recurrence
    ref_fw = parity.oracle_run(x, w.gate_mode)
    parity.compare(H, fin, ref_fw, parity.TOL["bf16"], label="fw_train")
    # the saved buffer is what the backward would recompute
    for k in ("dQ", "dK", "dV", "dC0", "dn0"):
        if k in g_rec:
            assert torch.equal(g_saved[k], g_rec[k]), k
    for k in ("di_pre", "df_pre", "dm0"):
        if k in g_rec:
            torch.testing.assert_close(g_saved[k], g_rec[k], rtol=1e-5, atol=1e-6)
    # and the gradients against the fp64 autograd oracle
    ref = ob.gradients(x, dH, w.gate_mode)
    names = ["dQ", "dK", "dV", "di_pre", "df_pre"] + (["dC0", "dn0"] if "dC0" in g_saved else [])
    errs = {k: parity.worst_rel(g_saved[k].double().cpu().numpy(), ref[k].numpy()) for k in names}
    bad = {k: v for k, v in errs.items() if not v <= parity.TOL["bf16"]}
    assert not bad, f"{case}: {errs}"


def test_autograd_keeps_or_recomputes():
    """mlstm_chunkwise with the training pair (default) and with recompute=True
    give the same gradients (the pair's gate gradients up to summation order)."""
    w, x, dH = _inputs(1, 2, 256, 128, 128, "exp", True, seed=71)
    grads = []
    for recompute in (False, True):
        leaves = {k: v.cuda().requires_grad_(True) for k, v in x.items() if v is not None}
        H, _ = api.mlstm_chunkwise(leaves["Q"], leaves["K"], leaves["V"], leaves["i_pre"],
                                   leaves["f_pre"], leaves["C0"], leaves["n0"], leaves["m0"],
                                   chunk_size=128, recompute=recompute)
        H.backward(dH.cuda())
        torch.cuda.synchronize()
        assert api.last_device_error() == _lib.OK
        grads.append({k: v.grad for k, v in leaves.items()})
    for k in ("Q", "K", "V", "C0", "n0"):
        assert torch.equal(grads[0][k], grads[1][k]), k
    for k in ("i_pre", "f_pre", "m0"):
        torch.testing.assert_close(grads[0][k], grads[1][k], rtol=1e-5, atol=1e-6)


def test_train_pair_unsupported_shapes():
    """fp32 inputs and d_qk of 64 have no training pair: mlstm_fw_train refuses
    and mlstm_chunkwise falls back to the recomputing backward."""
    assert api.train_sizes(1, 2, 256, 64, 64, torch.bfloat16) is None
    assert api.train_sizes(1, 2, 256, 128, 128, torch.float32) is None
    w, x, dH = _inputs(1, 2, 256, 128, 128, "exp", False)
    d = parity.to_dev(x)
    with pytest.raises(api.MlstmError) as e:
        api.mlstm_fw_train(d["Q"].float(), d["K"].float(), d["V"].float(), d["i_pre"],
                           d["f_pre"])
    assert e.value.status == _lib.ERR_UNSUPPORTED


def test_train_pair_full_size():
    """The 7B-shaped batch (B=8, NH=8, T=8192, 256 x 512 heads) through the pair:
    H and the final state of two heads against the oracle, and the saved
    backward against the recomputing one over the whole batch (bit for bit on
    dQ, dK, dV; the gate gradients up to summation order)."""
    w = WORKLOADS["xlstm7b"]
    x = make_inputs(w)
    d = parity.to_dev(x)
    dH = torch.randn((w.B, w.NH, w.T, w.DV), generator=torch.Generator().manual_seed(81),
                     dtype=torch.float32).to(torch.bfloat16).cuda()
    H, fin, saved = api.mlstm_fw_train(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"],
                                       gate_mode=w.gate_mode)
    g_saved = api.mlstm_bw_saved(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], H, saved, dH,
                                 gate_mode=w.gate_mode)
    del saved
    g_rec = api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH,
                         chunk_size=w.chunk_size, gate_mode=w.gate_mode)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    for k in ("dQ", "dK", "dV"):
        assert torch.equal(g_saved[k], g_rec[k]), k
    for k in ("di_pre", "df_pre"):
        torch.testing.assert_close(g_saved[k], g_rec[k], rtol=1e-4, atol=1e-5)
    heads = [(0, 0), (w.B - 1, w.NH - 1)]
    ref = parity.oracle_run(x, w.gate_mode, heads=heads)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], heads=heads, label="fw_train/full")
