"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Sizes: every workload at a size the oracle finishes in seconds that still
spans several chunks and tiles (plus a ragged tail), and the full workload
sizes in the launch configuration bench.py times, compared on sampled heads
that the oracle recomputes in full.
"""
import numpy as np
import pytest
import torch

import parity
from mlstm_chunkwise_b200 import _lib, api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled, sweep_workload

pytestmark = pytest.mark.gpu

ALGOS = ("simt", "tc", "tc_fused")


def supported(w, algo):
    try:
        api.workspace_size(w.B, w.NH, w.T, w.DK, w.DV, w.chunk_size, w.torch_dtype, algo)
        return True
    except api.MlstmError as e:
        assert e.status == _lib.ERR_UNSUPPORTED
        return False


def run(w, x, algo="auto"):
    d = parity.to_dev(x)
    H, fin = api.mlstm_fw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], d["C0"], d["n0"],
                          d["m0"], chunk_size=w.chunk_size, gate_mode=w.gate_mode, algo=algo)
    torch.cuda.synchronize()
    st = api.last_device_error()
    assert st == _lib.OK, \
        f"device status {st}, error word 0x{_lib.lib().mlstm_last_device_error_word():08x}"
    return H, fin


SCALED = [
    # (base workload, overrides): several chunks, both q/kv tile levels, ragged tails
    ("tiny", {}),
    ("tiny", dict(T=200)),
    ("mid", dict(B=1, NH=2, T=1024)),
    ("mid", dict(B=1, NH=2, T=1000)),
    ("xlstm7b", dict(B=1, NH=2, T=1024)),
    ("xlstm7b", dict(B=1, NH=2, T=1100)),
    ("sigmoid_long", dict(B=1, NH=2, T=2048)),
    ("sigmoid_long", dict(B=1, NH=2, T=1500)),
]


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("name,over", SCALED, ids=[f"{n}-{o.get('T', 'full')}" for n, o in SCALED])
def test_workload_scaled(name, over, algo):
    w = scaled(WORKLOADS[name], **over) if over else WORKLOADS[name]
    if not supported(w, algo):
        pytest.skip(f"{algo} does not support {w}")
    x = make_inputs(w)
    H, fin = run(w, x, algo)
    ref = parity.oracle_run(x, w.gate_mode)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"{w.name}/{algo}")


@pytest.mark.parametrize("T,L", [(1024, 64), (1024, 256), (1024, 1024), (4096, 512),
                                 (4096, 1024)])
def test_sweep_points_scaled(T, L):
    w = sweep_workload(T, L).replace(B=1, NH=2)
    x = make_inputs(w)
    for algo in ALGOS:
        if not supported(w, algo):
            continue
        H, fin = run(w, x, algo)
        ref = parity.oracle_run(x, w.gate_mode)
        parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"{w.name}/{algo}")


FULL = ["tiny", "mid", "xlstm7b", "sigmoid_long"]


@pytest.mark.parametrize("name", FULL)
def test_workload_full_size_sampled_heads(name):
    """Full size, default algorithm (the one bench.py times); two heads recomputed."""
    w = WORKLOADS[name]
    x = make_inputs(w)
    H, fin = run(w, x, "auto")
    heads = [(0, 0), (w.B - 1, w.NH - 1)]
    ref = parity.oracle_run(x, w.gate_mode, heads=heads)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], heads=heads, label=f"{w.name}/full")
    assert torch.isfinite(H).all()


@pytest.mark.parametrize("T,L", [(1024, 256), (65536, 256), (1024, 64), (65536, 64), (1024, 128),
                                 (4096, 1024)])
def test_sweep_full_size_sampled_heads(T, L):
    """Full-size sweep points in the bench's launch configuration (AUTO): the
    fused kernel at T = 1024, L = 128 (1024 heads), the wide output kernel with
    pairs of 64-token chunks, the long-chunk kernel, and the segmented state
    kernel at 16 heads."""
    w = sweep_workload(T, L)
    x = make_inputs(w)
    H, fin = run(w, x, "auto")
    heads = [(0, 0), (w.B - 1, w.NH - 1)]
    ref = parity.oracle_run(x, w.gate_mode, heads=heads)
    parity.compare(H, fin, ref, parity.TOL[w.dtype], heads=heads, label=f"{w.name}/full")


EDGE = [
    dict(B=1, NH=1, T=64, DK=64, DV=64, chunk_size=64),       # one chunk, one tile
    dict(B=1, NH=1, T=1, DK=64, DV=64, chunk_size=64),        # single token
    dict(B=1, NH=1, T=37, DK=64, DV=64, chunk_size=128),      # T < chunk
    dict(B=2, NH=1, T=300, DK=128, DV=64, chunk_size=128),    # DK != DV, ragged
    dict(B=1, NH=3, T=256, DK=64, DV=256, chunk_size=256),    # DV > DK
    dict(B=1, NH=1, T=512, DK=512, DV=128, chunk_size=256),   # widest keys
    dict(B=1, NH=1, T=128, DK=100, DV=72, chunk_size=64),     # dims that are not tile multiples
    dict(B=1, NH=1, T=4096, DK=64, DV=64, chunk_size=4096),   # largest chunk
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "x".join(str(v) for v in s.values()))
def test_edge_shapes(shape, dtype):
    w = WORKLOADS["mid"].replace(name="edge", dtype=dtype, **shape)
    x = make_inputs(w)
    ref = parity.oracle_run(x, w.gate_mode)
    for algo in ALGOS:
        if not supported(w, algo):
            continue
        H, fin = run(w, x, algo)
        parity.compare(H, fin, ref, parity.TOL[dtype], label=f"edge {shape}/{algo}")


@pytest.mark.parametrize("with_state", [False, True])
def test_empty_sequence(with_state):
    w = WORKLOADS["mid"].replace(name="empty", B=1, NH=2, T=0, DK=64, DV=64, chunk_size=64,
                                 init_state=with_state)
    x = make_inputs(w)
    H, (C_T, n_T, m_T) = run(w, x, "auto")
    assert H.shape == (1, 2, 0, 64)
    if with_state:
        assert torch.equal(C_T.cpu(), x["C0"]) and torch.equal(m_T.cpu(), x["m0"])
    else:
        assert not C_T.any() and not n_T.any() and not m_T.any()


def test_initial_state_and_sigmoid_gate():
    w = WORKLOADS["sigmoid_long"].replace(name="init", B=2, NH=2, T=640, chunk_size=128)
    x = make_inputs(w)
    x["m0"] = torch.tensor([[0.5, -1.0], [2.0, 0.0]])
    ref = parity.oracle_run(x, w.gate_mode)
    for algo in ALGOS:
        if supported(w, algo):
            H, fin = run(w, x, algo)
            parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"init/{algo}")


def test_segment_resume_on_gpu():
    """Two calls of T/2 with the carried state equal one call of T."""
    w = scaled(WORKLOADS["mid"], B=1, NH=2, T=1024, DK=128, DV=128)
    x = parity.to_dev(make_inputs(w))
    H, (C, n, m) = api.mlstm_fw(x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"], chunk_size=128)
    h = 512
    H1, (C1, n1, m1) = api.mlstm_fw(x["Q"][:, :, :h].contiguous(), x["K"][:, :, :h].contiguous(),
                                    x["V"][:, :, :h].contiguous(),
                                    x["i_pre"][:, :, :h].contiguous(),
                                    x["f_pre"][:, :, :h].contiguous(), chunk_size=128)
    H2, (C2, n2, m2) = api.mlstm_fw(x["Q"][:, :, h:].contiguous(), x["K"][:, :, h:].contiguous(),
                                    x["V"][:, :, h:].contiguous(),
                                    x["i_pre"][:, :, h:].contiguous(),
                                    x["f_pre"][:, :, h:].contiguous(), C1, n1, m1, chunk_size=128)
    Hc = torch.cat([H1, H2], dim=2).double().cpu().numpy()
    assert parity.worst_rel(Hc, H.double().cpu().numpy()) < 2e-2
    assert parity.worst_rel(C2.double().cpu().numpy(), C.double().cpu().numpy()) < 2e-2
    assert parity.m_err(m2.double().cpu().numpy(), m.double().cpu().numpy()) < 1e-5


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_chunk_states_against_oracle_snapshots(algo):
    w = scaled(WORKLOADS["xlstm7b"], B=1, NH=2, T=1024)
    if not supported(w, algo):
        pytest.skip(f"{algo} unsupported")
    x = make_inputs(w)
    d = parity.to_dev(x)
    C_s, n_s, m_s, (C_T, n_T, m_T) = api.mlstm_fw_chunk_states(
        d["K"], d["V"], d["i_pre"], d["f_pre"], chunk_size=w.chunk_size, algo=algo)
    ref = parity.oracle_run(x, w.gate_mode, snap_every=w.chunk_size)
    tol = parity.TOL[w.dtype]
    NC = w.T // w.chunk_size
    for k in range(NC):
        assert parity.worst_rel(C_s[:, :, k].double().cpu().numpy(), ref["C_snap"][:, :, k]) < tol
        assert parity.worst_rel(n_s[:, :, k].double().cpu().numpy(), ref["n_snap"][:, :, k]) < tol
        assert parity.m_err(m_s[:, :, k].double().cpu().numpy(), ref["m_snap"][:, :, k]) < 1e-5
    assert parity.m_err(m_s[:, :, NC].double().cpu().numpy(), ref["m_T"]) < 1e-5
    parity.compare(torch.zeros(1, 2, 0, 1), (C_T, n_T, m_T), dict(ref, H=np.zeros((1, 2, 0, 1))),
                   tol, label="chunk states final")


PER_TOKEN_SHAPES = {
    "mid_L128": dict(base="mid", T=768),
    # the long-chunk kernel: chunk 0 without an entering state, then m_k frames
    "d128_L512": dict(base="mid", T=1536, chunk_size=512),
    # one O buffer per item (value tiles of 256 columns), sigmoid gate, C0 given
    "d256x512_L512": dict(base="sigmoid_long", T=1536),
}


@pytest.mark.parametrize("shape", list(PER_TOKEN_SHAPES))
@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_parallel_per_token_outputs(algo, shape):
    """mlstm_fw_parallel's per-token normaliser and stabiliser (the row frame
    of the chunkwise form) against the oracle's."""
    kw = dict(PER_TOKEN_SHAPES[shape])
    w = scaled(WORKLOADS[kw.pop("base")], B=1, NH=2, **kw)
    if not supported(w, algo):
        pytest.skip(f"{algo} unsupported")
    x = make_inputs(w)
    d = parity.to_dev(x)
    C_s, n_s, m_s, _ = api.mlstm_fw_chunk_states(d["K"], d["V"], d["i_pre"], d["f_pre"],
                                                 d["C0"], d["n0"], d["m0"],
                                                 chunk_size=w.chunk_size, gate_mode=w.gate_mode,
                                                 algo=algo)
    H, n_out, m_out = api.mlstm_fw_parallel(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], C_s,
                                            n_s, d["m0"], chunk_size=w.chunk_size,
                                            gate_mode=w.gate_mode, algo=algo)
    ref = parity.oracle_run(x, w.gate_mode)
    tol = parity.TOL[w.dtype]
    assert parity.worst_rel(H.double().cpu().numpy(), ref["H"]) < tol
    assert parity.worst_rel(n_out.double().cpu().numpy(), ref["den"]) < tol
    assert parity.m_err(m_out.double().cpu().numpy(), ref["m"]) < 1e-5


def test_algorithms_agree_with_each_other():
    """Kernel-variant equivalence: every supported algorithm gives the same H."""
    w = scaled(WORKLOADS["xlstm7b"], B=1, NH=2, T=768)
    x = make_inputs(w)
    outs = {a: run(w, x, a) for a in ALGOS if supported(w, a)}
    base = outs["simt"][0].double().cpu().numpy()
    for a, (H, _) in outs.items():
        assert parity.worst_rel(H.double().cpu().numpy(), base) < 2e-2, a


def test_fp32_path_is_tight():
    """fp32 inputs take the SIMT path and match the oracle to 1e-4 at several sizes."""
    for T, L in [(256, 64), (1000, 128), (512, 512)]:
        w = WORKLOADS["tiny"].replace(name="f32", T=T, chunk_size=L)
        x = make_inputs(w)
        H, fin = run(w, x, "auto")
        ref = parity.oracle_run(x, w.gate_mode)
        parity.compare(H, fin, ref, 1e-4, label=f"f32 T{T} L{L}")


@pytest.mark.parametrize("T,L,spikes", [(512, 128, (400, 470)), (512, 256, (300, 470)),
                                        (1536, 512, (1100, 1300))])
def test_input_gate_spikes(T, L, spikes):
    """Input-gate spikes (+70) inside a query tile push the row stabilisers of
    the later rows some e^70 above the first row's, past the range where the
    gate exponent splits into a column and a row factor: the kernels fall back
    to one exponential per element there and must still match the oracle.

    The spikes sit in the last chunk.  A spike in an earlier chunk leaves every
    later chunk state dominated by one token (rank one), and then
    h = C q / |n.q| is ill-conditioned on the rows where q.k is small: the bf16
    operand copy of C that the inter-chunk tensor-core product reads rounds
    each entry by up to 2^-9 of |k_j v_d|, which such rows amplify by
    |q||k| / |q.k| (measured: 7.5% on the worst row at T=512, L=128)."""
    w = WORKLOADS["mid"].replace(name="spikes", B=1, NH=2, T=T, chunk_size=L)
    x = make_inputs(w)
    for t in spikes:
        x["i_pre"][:, :, t] = 70.0
    ref = parity.oracle_run(x, w.gate_mode)
    for algo in ALGOS:
        if supported(w, algo):
            H, fin = run(w, x, algo)
            parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"spikes L{L}/{algo}")


@pytest.mark.parametrize("T,DK,DV,init", [(960, 128, 128, False), (1000, 128, 128, True),
                                         (300, 128, 256, True), (64, 128, 128, False)])
def test_chunk64_pairs(T, DK, DV, init):
    """64-token chunks on the tensor-core path: two chunks per 128-row query
    tile with a block-diagonal causal mask and a K-stacked inter-chunk operand;
    odd chunk counts (the last tile's second chunk past T), ragged tails and an
    initial state."""
    w = WORKLOADS["mid"].replace(name="chunk64", B=1, NH=2, T=T, DK=DK, DV=DV, chunk_size=64,
                                 init_state=init)
    assert supported(w, "tc")
    x = make_inputs(w)
    ref = parity.oracle_run(x, w.gate_mode)
    H, fin = run(w, x, "tc")
    parity.compare(H, fin, ref, parity.TOL[w.dtype], label=f"chunk64 T{T} d{DK}/{DV}")
