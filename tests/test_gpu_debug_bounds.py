"""The bounds-checked build (``libmlstm_fw_debug.so``, built with
-DMLSTM_DEBUG_BOUNDS=1) on every forward path, through the C ABI (needs a
B200).

Its tensor-core kernels check the offset of every state / output store and
every bulk copy of the chunk-state operand against the extents the problem
implies; a violation would set bit 1 of the device error word (reported as
MLSTM_ERR_DEVICE) and skip or redirect the access.  A clean run leaves the
word at 0 and gives the same outputs as the normal build, bit for bit (the
checks change no arithmetic)."""
import ctypes

import pytest
import torch

import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200 import build as libbuild
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

_DT = {torch.float32: _lib.DT_F32, torch.bfloat16: _lib.DT_BF16}
_GATE = {"exp": _lib.GATE_EXP, "sigmoid": _lib.GATE_SIGMOID}
_ALGO = {"simt": _lib.ALGO_SIMT, "tc": _lib.ALGO_TC, "tc_fused": _lib.ALGO_TC_FUSED}


@pytest.fixture(scope="module")
def dbg():
    path = libbuild.build(debug_bounds=True)
    return _lib.open_library(path)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_fw(lib, w, d, algo):
    B, NH, T, DK, DV = w.B, w.NH, w.T, w.DK, w.DV
    dev = d["Q"].device
    H = torch.zeros((B, NH, T, DV), dtype=w.torch_dtype, device=dev)
    C_T = torch.zeros((B, NH, DK, DV), device=dev)
    n_T = torch.zeros((B, NH, DK), device=dev)
    m_T = torch.zeros((B, NH), device=dev)
    nb = api.workspace_size(B, NH, T, DK, DV, w.chunk_size, w.torch_dtype, algo)
    ws = torch.zeros(max(1, nb), dtype=torch.uint8, device=dev)
    st = lib.mlstm_fw(_p(d["Q"]), _p(d["K"]), _p(d["V"]), _p(d["i_pre"]), _p(d["f_pre"]),
                      _p(d["C0"]), _p(d["n0"]), _p(d["m0"]), _p(H), _p(C_T), _p(n_T), _p(m_T),
                      B, NH, T, DK, DV, w.chunk_size, _DT[w.torch_dtype], _GATE[w.gate_mode],
                      _ALGO[algo], _p(ws), ws.numel(),
                      ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == _lib.OK, _lib.status_string(st)
    return H, C_T, n_T, m_T


def base(**kw):
    kw = dict(dict(B=1, NH=2), **kw)
    return WORKLOADS["mid"].replace(name="bounds", **kw)


CASES = {
    "wide_7b_head": (base(T=1024, DK=256, DV=512, chunk_size=256), "tc"),
    "wide_7b_head_unsegmented": (base(B=5, NH=8, T=512, DK=256, DV=512, chunk_size=256), "tc"),
    "pair_chunk64": (base(T=1000, chunk_size=64), "tc"),
    "long_chunk512": (base(T=1536, DK=256, DV=512, chunk_size=512), "tc"),
    "long_chunk1024_ragged": (base(T=2000, chunk_size=1024), "tc"),
    "segmented_d128": (base(T=1024, chunk_size=128, init_state=True), "tc"),
    "fused": (base(NH=4, T=640, chunk_size=128), "tc_fused"),
    "simt": (base(T=300, DK=64, DV=64, chunk_size=128), "simt"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_bounds_checked_build_is_clean_and_identical(dbg, name):
    w, algo = CASES[name]
    x = make_inputs(w)
    d = parity.to_dev(x)
    ref = call_fw(_lib.lib(), w, d, algo)
    got = call_fw(dbg, w, d, algo)
    torch.cuda.synchronize()
    assert dbg.mlstm_last_device_error(None) == _lib.OK
    assert dbg.mlstm_last_device_error_word() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_bounds_checked_build_dominated_states(dbg):
    """An early input-gate spike: the deflated stores of the state kernel and
    of its segment fix-up run under the checks."""
    w = base(T=1024, chunk_size=128)
    x = make_inputs(w)
    x["i_pre"][0, 0, 170] = 70.0
    x["i_pre"][0, 1, 261] = 70.0
    d = parity.to_dev(x)
    ref = call_fw(_lib.lib(), w, d, "tc")
    got = call_fw(dbg, w, d, "tc")
    torch.cuda.synchronize()
    assert dbg.mlstm_last_device_error(None) == _lib.OK
    assert dbg.mlstm_last_device_error_word() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_bounds_checked_build_fp32_chunk_states(dbg):
    """The fp32 chunk-state output (tensor-map stores of the state kernel)."""
    w = base(T=1024, DK=256, DV=512, chunk_size=256)
    x = make_inputs(w)
    d = parity.to_dev(x)
    B, NH, NC = w.B, w.NH, w.T // w.chunk_size
    outs = []
    for lib in (_lib.lib(), dbg):
        C_s = torch.zeros((B, NH, NC, w.DK, w.DV), device="cuda")
        n_s = torch.zeros((B, NH, NC, w.DK), device="cuda")
        m_s = torch.zeros((B, NH, NC + 1), device="cuda")
        nb = api.substep_workspace_size(B, NH, w.T, w.DK, w.DV, w.chunk_size, w.torch_dtype, "tc")
        ws = torch.zeros(max(1, nb), dtype=torch.uint8, device="cuda")
        st = lib.mlstm_fw_chunk_states(
            _p(d["K"]), _p(d["V"]), _p(d["i_pre"]), _p(d["f_pre"]), None, None, None, _p(C_s),
            _p(n_s), _p(m_s), None, None, None, B, NH, w.T, w.DK, w.DV, w.chunk_size,
            _lib.DT_BF16, _lib.GATE_EXP, _lib.ALGO_TC, _p(ws), ws.numel(), None)
        assert st == _lib.OK
        outs.append((C_s, n_s, m_s))
    torch.cuda.synchronize()
    assert dbg.mlstm_last_device_error(None) == _lib.OK
    assert dbg.mlstm_last_device_error_word() == 0
    for a, b in zip(*outs):
        assert torch.equal(a, b)
