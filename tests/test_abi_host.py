"""C ABI checks that need no GPU: exported symbols, argument validation,
workspace sizes and status strings.  Calls here either fail validation (which
happens before any CUDA call) or only query sizes."""
import ctypes
import os
import re

import pytest

from mlstm_chunkwise_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "mlstm_fw.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mlstm_\w+)\s*\(", text)))


def test_every_declared_function_is_exported(L):
    names = declared_functions()
    assert "mlstm_fw" in names and len(names) >= 8
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/mlstm_fw.h but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature in the binding"


def test_exports_match_nm():
    """The shared object exports exactly the C names (no C++ mangling)."""
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    for n in declared_functions():
        assert re.search(rf"\bT {n}\b", out), n


def test_status_strings(L):
    for s in range(7):
        assert _lib.status_string(s)
    assert _lib.status_string(99) == "unknown status"
    assert L.mlstm_abi_version() == 100


def ws(B=2, NH=3, T=256, DK=64, DV=64, L=64, dt=_lib.DT_BF16, algo=_lib.ALGO_SIMT):
    n = ctypes.c_size_t(0)
    st = _lib.lib().mlstm_fw_workspace_size(B, NH, T, DK, DV, L, dt, algo, ctypes.byref(n))
    return st, n.value


def test_workspace_size_formula(L):
    st, n = ws()
    assert st == _lib.OK
    B, NH, T, DK, DV, Lc = 2, 3, 256, 64, 64, 64
    NC = T // Lc
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # per-token bcum/acol/amax, per-chunk g, m (NC + 1), and per-chunk weight
    # sum, argmax, dominant token and its log-weight, and a per-head flag
    gates = 3 * r(B * NH * NC * Lc * 4) + r(B * NH * NC * 4) + r(B * NH * (NC + 1) * 4) + \
        4 * r(B * NH * NC * 4) + r(B * NH * 4)
    states = r(B * NH * NC * DK * DV * 4) + r(B * NH * NC * DK * 4)
    assert n == gates + states
    # ragged T rounds the chunk count up
    st, n2 = ws(T=200)
    assert st == _lib.OK and n2 == n
    # empty sequence needs only the stabiliser slot and the flag per head
    st, n0 = ws(T=0)
    assert st == _lib.OK and n0 == 2 * r(B * NH * 4)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), _lib.ERR_INVALID_ARG),
    (dict(NH=-1), _lib.ERR_INVALID_ARG),
    (dict(T=-5), _lib.ERR_INVALID_ARG),
    (dict(DK=0), _lib.ERR_INVALID_ARG),
    (dict(L=96), _lib.ERR_INVALID_ARG),     # not a multiple of 64
    (dict(L=0), _lib.ERR_INVALID_ARG),
    (dict(L=8192), _lib.ERR_UNSUPPORTED),   # above the largest chunk
    (dict(DV=2048), _lib.ERR_UNSUPPORTED),
    (dict(B=256, NH=512), _lib.ERR_UNSUPPORTED),
    (dict(dt=7), _lib.ERR_INVALID_ARG),
    (dict(algo=9), _lib.ERR_INVALID_ARG),
    (dict(dt=_lib.DT_F32, algo=_lib.ALGO_TC), _lib.ERR_UNSUPPORTED),
    (dict(dt=_lib.DT_F32, algo=_lib.ALGO_TC_FUSED), _lib.ERR_UNSUPPORTED),
])
def test_workspace_size_rejects(L, kw, expect):
    st, _ = ws(**kw)
    assert st == expect


def _fw(**over):
    """mlstm_fw with fake (never dereferenced) aligned pointers; every case
    below must be rejected by validation before any CUDA call."""
    p = ctypes.c_void_p(0x10000)
    a = dict(Q=p, K=p, V=p, i=p, f=p, C0=None, n0=None, m0=None, H=p, CT=None, nT=None, mT=None,
             B=1, NH=1, T=128, DK=64, DV=64, L=64, dt=_lib.DT_BF16, gm=_lib.GATE_EXP,
             algo=_lib.ALGO_SIMT, ws=p, wsb=1 << 40, st=None)
    a.update(over)
    return _lib.lib().mlstm_fw(a["Q"], a["K"], a["V"], a["i"], a["f"], a["C0"], a["n0"], a["m0"],
                               a["H"], a["CT"], a["nT"], a["mT"], a["B"], a["NH"], a["T"], a["DK"],
                               a["DV"], a["L"], a["dt"], a["gm"], a["algo"], a["ws"], a["wsb"],
                               a["st"])


@pytest.mark.parametrize("over", [
    dict(Q=None), dict(V=None), dict(f=None), dict(H=None),
    dict(C0=ctypes.c_void_p(0x10000)),                       # partial initial state
    dict(C0=ctypes.c_void_p(0x10000), n0=ctypes.c_void_p(0x10000)),
    dict(K=ctypes.c_void_p(0x10004)),                        # misaligned
    dict(ws=ctypes.c_void_p(0x10008)),
    dict(wsb=16),                                            # workspace too small
    dict(ws=None),
    dict(gm=5), dict(dt=-1), dict(algo=17),
    dict(L=100), dict(T=-1), dict(DK=0),
])
def test_fw_rejects_before_launch(L, over):
    assert _fw(**over) == _lib.ERR_INVALID_ARG


def test_fw_unsupported_combinations(L):
    assert _fw(dt=_lib.DT_F32, algo=_lib.ALGO_TC) == _lib.ERR_UNSUPPORTED
    assert _fw(dt=_lib.DT_F32, algo=_lib.ALGO_TC_FUSED) == _lib.ERR_UNSUPPORTED
    assert _fw(DK=4096) == _lib.ERR_UNSUPPORTED


def test_substeps_reject(L):
    p = ctypes.c_void_p(0x10000)
    lib = _lib.lib()
    st = lib.mlstm_fw_chunk_states(p, p, p, p, None, None, None, p, p, None, None, None, None,
                                   1, 1, 128, 64, 64, 64, 1, 0, 1, p, 1 << 30, None)
    assert st == _lib.ERR_INVALID_ARG  # m_states is required
    st = lib.mlstm_fw_parallel(p, p, p, p, p, None, None, p, p, None, None,
                               1, 1, 128, 64, 64, 64, 1, 0, 1, p, 1 << 30, None)
    assert st == _lib.ERR_INVALID_ARG  # C_states missing
    st = lib.mlstm_fw_chunk_states(p, p, p, p, None, None, None, p, p, p, None, None, None,
                                   1, 1, 128, 64, 64, 64, 1, 0, _lib.ALGO_TC_FUSED, p, 1 << 30,
                                   None)
    assert st == _lib.ERR_UNSUPPORTED  # the fused kernel has no chunk-state output


def test_python_binding_refuses_cpu_tensors():
    import torch

    from mlstm_chunkwise_b200 import mlstm_fw
    x = torch.zeros(1, 1, 64, 64)
    g = torch.zeros(1, 1, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mlstm_fw(x, x, x, g, g)


def train_sizes_raw(B=1, NH=2, T=256, DK=128, DV=128, dt=_lib.DT_BF16):
    sv, fw, bw = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = _lib.lib().mlstm_train_sizes(B, NH, T, DK, DV, dt, ctypes.byref(sv), ctypes.byref(fw),
                                      ctypes.byref(bw))
    return st, sv.value, fw.value, bw.value


def test_train_sizes(L):
    """The saved buffer holds the bf16 chunk states and fp32 n states of every
    128-token chunk plus two floats per token (256-byte aligned pieces)."""
    st, sv, fw, bw = train_sizes_raw(B=2, NH=3, T=300, DK=256, DV=512)
    assert st == _lib.OK
    BH, NC, T = 6, 3, 300
    al = lambda b: (b + 255) // 256 * 256  # noqa: E731
    assert sv == al(BH * NC * 256 * 512 * 2) + al(BH * NC * 256 * 4) + 2 * al(BH * T * 4)
    assert fw > 0 and bw > 0
    # no training path: fp32, d_qk 64, fewer than 128 tokens
    assert train_sizes_raw(dt=_lib.DT_F32)[0] == _lib.ERR_UNSUPPORTED
    assert train_sizes_raw(DK=64, DV=64)[0] == _lib.ERR_UNSUPPORTED
    assert train_sizes_raw(T=127)[0] == _lib.ERR_UNSUPPORTED


def test_train_pair_rejects_before_launch(L):
    """Too small a saved buffer or workspace, unaligned or missing pointers,
    and unsupported shapes return before any CUDA call (fake aligned pointers)."""
    st, sv, fw, bw = train_sizes_raw()
    assert st == _lib.OK
    P = ctypes.c_void_p(0x10000)
    U = ctypes.c_void_p(0x10008)  # not 16-byte aligned

    def fw_call(saved_bytes=sv, ws_bytes=fw, q=P, dt=_lib.DT_BF16, DK=128):
        return L.mlstm_fw_train(q, P, P, P, P, None, None, None, P, None, None, None, P,
                                saved_bytes, 1, 2, 256, DK, 128, dt, _lib.GATE_EXP, P, ws_bytes,
                                None)

    def bw_call(saved_bytes=sv, ws_bytes=bw, h=P):
        return L.mlstm_bw_saved(P, P, P, P, P, None, None, None, h, P, saved_bytes, P, P, P, P,
                                P, P, None, None, None, 1, 2, 256, 128, 128, _lib.DT_BF16,
                                _lib.GATE_EXP, P, ws_bytes, None)

    assert fw_call(saved_bytes=sv - 1) == _lib.ERR_INVALID_ARG
    assert fw_call(ws_bytes=fw - 1) == _lib.ERR_INVALID_ARG
    assert fw_call(q=U) == _lib.ERR_INVALID_ARG
    assert fw_call(q=None) == _lib.ERR_INVALID_ARG
    assert fw_call(dt=_lib.DT_F32) == _lib.ERR_UNSUPPORTED
    assert fw_call(DK=64) == _lib.ERR_UNSUPPORTED
    assert bw_call(saved_bytes=sv - 1) == _lib.ERR_INVALID_ARG
    assert bw_call(ws_bytes=bw - 1) == _lib.ERR_INVALID_ARG
    assert bw_call(h=None) == _lib.ERR_INVALID_ARG


def test_auto_picks_fused_from_half_the_sms(L):
    """AUTO takes the fused kernel from 74 (b, h) pairs up (half of a 148-SM
    B200) where it supports the shape, else the unfused tensor-core path; the
    rule depends on the shape alone, so the workspace AUTO asks for is that of
    the algorithm it runs (checked here without a GPU, through the sizes)."""
    kw = dict(T=1024, DK=128, DV=128, L=128, dt=_lib.DT_BF16)
    for NH, expect in ((73, _lib.ALGO_TC), (74, _lib.ALGO_TC_FUSED), (600, _lib.ALGO_TC_FUSED)):
        st_a, n_auto = ws(B=1, NH=NH, algo=_lib.ALGO_AUTO, **kw)
        st_e, n_exp = ws(B=1, NH=NH, algo=expect, **kw)
        st_o, n_other = ws(B=1, NH=NH, algo=_lib.ALGO_TC_FUSED + _lib.ALGO_TC - expect, **kw)
        assert st_a == st_e == st_o == _lib.OK
        assert n_other != n_exp, "the two paths need different workspaces"
        assert n_auto == n_exp, (NH, n_auto, n_exp)
    # shapes the fused kernel does not take stay unfused at any head count
    st_a, n_auto = ws(B=1, NH=600, T=1024, DK=128, DV=128, L=256, algo=_lib.ALGO_AUTO)
    st_t, n_tc = ws(B=1, NH=600, T=1024, DK=128, DV=128, L=256, algo=_lib.ALGO_TC)
    assert st_a == st_t == _lib.OK and n_auto == n_tc
