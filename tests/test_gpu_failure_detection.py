"""Failure detection on the GPU without a GPU fault (needs a B200).

Every wait in the library's kernels is bounded by a watchdog on the global
timer; when it runs out the kernel records the watchdog bit and the site of
the wait in the device error word and returns.  The self-test entry point runs
one such wait that nothing ever satisfies.  Nothing traps, faults or hangs: the
wait ends after the (here ~1 ms) limit and the context stays usable.
"""
import pytest
import torch

import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu

SELFTEST_SITE = 0xF7


def _forward(w, x):
    d = parity.to_dev(x)
    return api.mlstm_fw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"], d["n0"],
                        d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode)


def test_expired_wait_reports_timeout_and_the_context_survives():
    api.set_watchdog(1 << 16)  # about 1 ms per wait
    try:
        api.watchdog_selftest()
        st = api.last_device_error()
        word = _lib.lib().mlstm_last_device_error_word()
    finally:
        api.set_watchdog(1 << 22)
    assert st == _lib.ERR_TIMEOUT
    assert word & 1, hex(word)
    assert (word >> 8) & 0xFF == SELFTEST_SITE, hex(word)
    # the word was cleared by the read
    assert api.last_device_error() == _lib.OK

    # The same context still runs the forward pass correctly (tensor-core path).
    w = scaled(WORKLOADS["xlstm7b"], B=1, NH=2, T=512)
    x = make_inputs(w)
    H, fin = _forward(w, x)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.OK
    ref = parity.oracle_run(x, w.gate_mode)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], label="after watchdog self-test")


def test_repeated_expiries_each_report_once():
    api.set_watchdog(1 << 14)
    try:
        for _ in range(3):
            api.watchdog_selftest()
            assert api.last_device_error() == _lib.ERR_TIMEOUT
            assert api.last_device_error() == _lib.OK
    finally:
        api.set_watchdog(1 << 22)
