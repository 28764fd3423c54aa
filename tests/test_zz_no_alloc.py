"""mlstm_fw_static_scratch: the forward pass for callers that cannot allocate.

Some callers hold their inputs and outputs but have no allocator to give the
library a workspace (a plugin hook that only hands over tensors, or a loop that
forbids cudaMalloc because it can synchronise the device).  The static-scratch
entry point takes no workspace and uses an array inside the library's device
image.  These tests call it through the C ABI and check that it reproduces
mlstm_fw() (the entry point with a caller-provided workspace) on two calls in a
row, and that a problem too large for the array is refused before any launch.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu

_DT = {torch.float32: _lib.DT_F32, torch.bfloat16: _lib.DT_BF16}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def static_call(w, d, algo=_lib.ALGO_AUTO):
    B, NH, T, DK, DV = w.B, w.NH, w.T, w.DK, w.DV
    dev = d["Q"].device
    H = torch.full((B, NH, T, DV), float("nan"), dtype=w.torch_dtype, device=dev)
    C_T = torch.full((B, NH, DK, DV), float("nan"), device=dev)
    n_T = torch.full((B, NH, DK), float("nan"), device=dev)
    m_T = torch.full((B, NH), float("nan"), device=dev)
    st = _lib.lib().mlstm_fw_static_scratch(
        _p(d["Q"]), _p(d["K"]), _p(d["V"]), _p(d["i_pre"]), _p(d["f_pre"]), _p(d["C0"]),
        _p(d["n0"]), _p(d["m0"]), _p(H), _p(C_T), _p(n_T), _p(m_T), B, NH, T, DK, DV,
        w.chunk_size, _DT[w.torch_dtype], 0 if w.gate_mode == "exp" else 1, algo,
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    return st, H, (C_T, n_T, m_T)


def profiled_families(fn):
    """Runs fn() with the library's per-family launch record on; returns the
    number of launches of each kernel family it made."""
    lib = _lib.lib()
    n = _lib.KERNEL_COUNT
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_uint64 * n)()
    lib.mlstm_profile_read(ms, cnt, n)  # drop anything recorded earlier
    lib.mlstm_profile_enable(1)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        lib.mlstm_profile_enable(0)
    assert lib.mlstm_profile_read(ms, cnt, n) == _lib.OK
    return out, list(cnt)


CASES = [
    # fp32 CUDA-core path
    (WORKLOADS["tiny"], None),
    # tensor-core path, 2 chunks of 512
    (scaled(WORKLOADS["sigmoid_long"], B=1, NH=2, T=1024, DK=128, DV=128), None),
    # tensor-core path with the chunk-state sequences cut into 4 segments: the
    # segments' end states and the fix-up launch use the scratch array too
    (scaled(WORKLOADS["mid"], B=1, NH=2, T=1024), "tc_states_segmented"),
    # 608 heads: AUTO picks the fused kernel
    (scaled(WORKLOADS["mid"], B=8, NH=76, T=256), "fused"),
]


@pytest.mark.parametrize("w,kind", CASES, ids=["tiny_f32", "sigmoid_bf16", "segmented", "fused"])
def test_static_scratch_matches_workspace_entry_point_twice(w, kind):
    """Same kernels, same inputs: the outputs must equal mlstm_fw's bit for bit
    (the forward kernels use no atomics), on two calls in a row, the second
    of which finds the first call's leftovers in the array."""
    assert torch.cuda.is_available()
    x = make_inputs(w)
    d = parity.to_dev(x)
    (H_ref, (C_ref, n_ref, m_ref)), fams = profiled_families(
        lambda: api.mlstm_fw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"], d["n0"],
                             d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode))
    if kind == "tc_states_segmented":
        # more than one launch of the state family: the segmented recurrence and
        # its fix-up
        assert fams[3] > 1, fams
    if kind == "fused":
        assert fams[5] == 1, fams
    for call in range(2):
        st, H, (C_T, n_T, m_T) = static_call(w, d)
        assert st == _lib.OK, _lib.status_string(st)
        torch.cuda.synchronize()
        assert api.last_device_error() == _lib.OK
        for name, got, ref in (("H", H, H_ref), ("C_T", C_T, C_ref), ("n_T", n_T, n_ref),
                               ("m_T", m_T, m_ref)):
            assert torch.isfinite(got).all(), (call, name)
            assert torch.equal(got, ref), (call, name)


def test_static_scratch_refuses_problems_that_do_not_fit():
    cap = _lib.lib().mlstm_fw_static_scratch_capacity()
    assert cap == 16 << 20
    # 2M tokens: even the gate arrays alone (12 bytes per token) exceed 16 MiB
    w = WORKLOADS["mid"].replace(B=4, NH=16, T=32768, DK=64, DV=64, chunk_size=256)
    assert api.workspace_size(w.B, w.NH, w.T, w.DK, w.DV, w.chunk_size, w.torch_dtype) > cap
    dev = torch.device("cuda", torch.cuda.current_device())
    dummy = torch.zeros(16, device=dev)
    p = ctypes.c_void_p(dummy.data_ptr())
    before = _lib.lib().mlstm_kernel_launches()
    st = _lib.lib().mlstm_fw_static_scratch(
        p, p, p, p, p, None, None, None, p, None, None, None, w.B, w.NH, w.T, w.DK, w.DV,
        w.chunk_size, _lib.DT_BF16, _lib.GATE_EXP, _lib.ALGO_AUTO, None)
    assert st == _lib.ERR_SCRATCH_TOO_SMALL
    assert "static" in _lib.status_string(st)
    assert _lib.lib().mlstm_kernel_launches() == before  # nothing was enqueued
    torch.cuda.synchronize()
    assert not dummy.any()
