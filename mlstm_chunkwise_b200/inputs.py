"""Seeded synthetic inputs for the mLSTM forward workloads.

This module only draws random numbers; it holds none of the method's
arithmetic.  Tests, ``bench.py`` and the oracle checks all take their inputs
from here, so the CUDA path and the oracle see identical values.

The workloads follow the shapes and distributions of the xLSTM-7B-shaped
forward pass and its companions (mid size, tiny fp32, sigmoid-input-gate long
context, chunk/length sweep).  Every draw is made in fp32 on the CPU with a
seeded ``torch.Generator`` and then rounded once (RNE) to the storage dtype.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    NH: int
    T: int
    DK: int
    DV: int
    dtype: str          # "f32" or "bf16": storage/compute type of Q, K, V and H
    gate_mode: str      # "exp", "sigmoid" or "sigmoid_plain"
    chunk_size: int
    i_mean: float       # i_pre ~ N(i_mean, 1)
    f_low: float = 3.0  # f_pre ~ U(f_low, f_high)
    f_high: float = 6.0
    init_state: bool = False   # C0, n0 ~ N(0, 0.1^2), m0 = 0
    seed: int = 1000

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, NH=2, T=256, DK=64, DV=64, dtype="f32", gate_mode="exp",
                     chunk_size=64, i_mean=0.0, seed=1000),
    "mid": Workload("mid", B=2, NH=8, T=4096, DK=128, DV=128, dtype="bf16", gate_mode="exp",
                    chunk_size=128, i_mean=0.0, seed=1001),
    "xlstm7b": Workload("xlstm7b", B=8, NH=8, T=8192, DK=256, DV=512, dtype="bf16",
                        gate_mode="exp", chunk_size=256, i_mean=-2.0, seed=1002),
    "sigmoid_long": Workload("sigmoid_long", B=2, NH=8, T=32768, DK=256, DV=512, dtype="bf16",
                             gate_mode="sigmoid", chunk_size=512, i_mean=0.0, init_state=True,
                             seed=1003),
    # the sigmoid-input-gate variant without normaliser, on the same inputs
    "sigmoid_long_plain": Workload("sigmoid_long_plain", B=2, NH=8, T=32768, DK=256, DV=512,
                                   dtype="bf16", gate_mode="sigmoid_plain", chunk_size=512,
                                   i_mean=0.0, init_state=True, seed=1003),
}

SWEEP_TOKENS = 65536
SWEEP_T = (1024, 4096, 16384, 65536)
SWEEP_CHUNKS = (64, 128, 256, 512, 1024)


def sweep_workload(T: int, chunk_size: int) -> Workload:
    """One point of the chunk/length sweep: B*T = 65536 tokens, NH=16, d=128."""
    return Workload(f"sweep_T{T}_L{chunk_size}", B=SWEEP_TOKENS // T, NH=16, T=T, DK=128, DV=128,
                    dtype="bf16", gate_mode="exp", chunk_size=chunk_size, i_mean=0.0, seed=1004)


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict of contiguous CPU tensors: Q, K [B,NH,T,DK] and V [B,NH,T,DV]
    in ``w.torch_dtype``; i_pre, f_pre [B,NH,T] fp32; and C0 [B,NH,DK,DV],
    n0 [B,NH,DK], m0 [B,NH] fp32 when ``w.init_state`` (else None).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    B, NH, T, DK, DV = w.B, w.NH, w.T, w.DK, w.DV
    dt = w.torch_dtype
    Q = torch.randn((B, NH, T, DK), generator=g, dtype=torch.float32).to(dt)
    K = torch.randn((B, NH, T, DK), generator=g, dtype=torch.float32).to(dt)
    V = torch.randn((B, NH, T, DV), generator=g, dtype=torch.float32).to(dt)
    i_pre = torch.randn((B, NH, T), generator=g, dtype=torch.float32) + w.i_mean
    f_pre = torch.rand((B, NH, T), generator=g, dtype=torch.float32) * (w.f_high - w.f_low) + w.f_low
    out = dict(Q=Q, K=K, V=V, i_pre=i_pre, f_pre=f_pre, C0=None, n0=None, m0=None)
    if w.init_state:
        out["C0"] = torch.randn((B, NH, DK, DV), generator=g, dtype=torch.float32) * 0.1
        out["n0"] = torch.randn((B, NH, DK), generator=g, dtype=torch.float32) * 0.1
        out["m0"] = torch.zeros((B, NH), dtype=torch.float32)
    return out


def scaled(w: Workload, **kw) -> Workload:
    """The same distributions at other sizes (used to keep oracle runs short)."""
    return w.replace(name=w.name + "_scaled", **kw)
