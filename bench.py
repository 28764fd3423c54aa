"""Throughput of the chunkwise mLSTM forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--algo auto|simt|tc|tc_fused] [--impl ours|reference]

One step = one full forward pass (gates -> chunk states -> outputs, or the
fused kernel) over one batch of the workload, inputs resident in HBM.  At
N > 1 (torchrun, one process per GPU) every rank runs its own batch of the same
shape (weak scaling: the path shards over independent (batch, head) pairs, so
there is no collective on the data path); the timing is the max over ranks.

Rank 0 prints one JSON line: tokens/s over all ranks, the TFLOP/s and roofline
of the dominant kernel (per-kernel CUDA events on the launch stream), the e2e
throughput through the same API with pinned host buffers and the copies inside
the timed region, the SM clocks sampled during the timed region, and (N = 1)
the fp64 CPU oracle timed on a bounded sample of the same workload.

``--impl reference`` times that oracle alone on the host cores (the only
other place this script runs it), on the same workload and metric.

``--op step | bw | train`` measure, on one GPU, the single-token step, the
backward pass (forward recomputed inside it) and a whole training step
(forward + backward through the autograd Function) instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mLSTM fw tokens/s and TFLOP/s (% bf16 TC peak) at 7B shape, T=8192"
L2_BYTES = 126 * 2**20
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16 (the datasheet's sparse figure halved)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
# fp32 FFMA peak for the SIMT kernels: 148 SMs x 128 lanes x 2 flop x clock.
SIMT_LANES = 148 * 128


def rank_seed(w, rank):
    """Every rank draws its own batch of the same workload shape."""
    return w.seed + rank


def max_over_ranks(value, device, world):
    """The largest per-rank value over all ranks (the slowest rank times the
    job).  Every rank must call it, in the same order."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step, world, ms_per_step):
    """Whole-job tokens/s: all ranks' tokens over the max-over-ranks step time."""
    return tokens_per_rank_step * world / (ms_per_step / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_per_head(T, DK, DV, L):
    """Algorithmic tensor-core FLOPs of one (b, h): state updates, the inter-chunk
    Q.C term, and the causal half of the intra-chunk QK^T and P.V."""
    return {
        "states": 2.0 * T * DK * DV,
        "inter": 2.0 * T * DK * DV,
        "intra": float(T) * L * (DK + DV),
    }


def chunk_state_bytes_written(algo_families, B, NH, T, DK, DV, L):
    """HBM bytes of chunk states written per step (the states entering every
    chunk, excluding the final state): the bf16 operand copy plus fp32 n on
    the unfused tensor-core path, fp32 C and n on the SIMT path, none in the
    fused kernel."""
    BH, NC = B * NH, -(-T // L)
    if "tc_states" in algo_families:
        return BH * NC * (DK * DV * 2 + DK * 4)
    if "simt_states" in algo_families:
        return BH * NC * (DK * DV * 4 + DK * 4)
    return 0


def kernel_bytes(fam, B, NH, T, DK, DV, L, elem):
    """Algorithmic DRAM bytes of one launch of a kernel family on the unfused
    or fused path: every input read once, every output written once (the
    chunk-state operand copy is bf16 on the tensor-core path, fp32 on SIMT)."""
    BH, NC = B * NH, -(-T // L)
    gates_rd = BH * T * 3 * 4 + BH * (NC + 1) * 4           # bcum/acol/amax, m per chunk
    final = BH * (DK * DV + DK + 1) * 4
    state_elem = 2 if fam.startswith("tc") else 4
    states = BH * NC * (DK * DV * state_elem + DK * 4)       # C_k operand + n_k
    if fam == "gates":
        return BH * T * (8 + 12)
    if fam in ("tc_states", "simt_states"):
        return BH * T * (DK + DV) * elem + states + final + BH * T * 4
    if fam in ("tc_parallel", "simt_parallel"):
        return BH * T * (2 * DK + 2 * DV) * elem + states + gates_rd
    if fam == "tc_fused":
        return BH * T * (2 * DK + 2 * DV) * elem + final + gates_rd
    raise KeyError(fam)


def method_bytes(fam, B, NH, T, DK, DV, elem, init_state):
    """The method's own DRAM bytes in one launch of a kernel family: the
    per-token inputs the family needs and the method outputs it produces, each
    moved once.  The chunk states handed between the unfused kernels, the
    second read of K and V and the gate intermediates are traffic of this
    design, not of the method, and are not counted."""
    BH = B * NH
    final = BH * (DK * DV + DK + 1) * 4
    init = final if init_state else 0
    if fam == "gates":
        return BH * T * 8
    if fam in ("tc_states", "simt_states"):
        return BH * T * (DK + DV) * elem + final + init
    if fam in ("tc_parallel", "simt_parallel"):
        return BH * T * (2 * DK + 2 * DV) * elem
    if fam == "tc_fused":
        return BH * T * ((2 * DK + 2 * DV) * elem + 8) + final + init
    raise KeyError(fam)


# DRAM bytes per launch measured with ncu (dram__bytes_read.sum +
# dram__bytes_write.sum), valid only while the kernel's sources are unchanged:
# the entry records a SHA-1 over those files and is ignored when it differs.
MEASURED_TRAFFIC = {
    # 7B shape at batch 2 (16 heads, 514.1 MB per launch), scaled by the heads
    ("tc_parallel", "xlstm7b"): {
        "bytes": 4 * 514.113024e6,
        "sources": ['tc_parallel_wide.cu', 'tc_ptx.cuh', 'tc.h', 'common.cuh'],
        "sha1": "d77ddeaa1058f329306d4f3a8ee9e25d506f9280"},
    # 7B shape at batch 5 (40 heads, unsegmented as at full size, 819.9 MB)
    ("tc_states", "xlstm7b"): {
        "bytes": 64 / 40 * 819.934208e6,
        "sources": ['tc_states.cu', 'tc_ptx.cuh', 'tc.h', 'common.cuh'],
        "sha1": "2c1f6db9734982d4cf1ed79d073bf79bb235b0a6"},
    # sigmoid_long at batch 1 (8 heads, the long-chunk kernel, 916.6 MB)
    ("tc_parallel", "sigmoid_long"): {
        "bytes": 2 * 916.586496e6,
        "sources": ['tc_parallel.cu', 'tc_ptx.cuh', 'tc.h', 'common.cuh'],
        "sha1": "71537485f494a037f68ab3f7aa374448d029ac74"},
}


def sources_sha1(files):
    import hashlib
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "mlstm_chunkwise_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(fam, workload):
    e = MEASURED_TRAFFIC.get((fam, workload))
    if e is None or sources_sha1(e["sources"]) != e["sha1"]:
        return None
    return e["bytes"]


def roofline(fam, per_launch_ms, kflops, shape, peaks, peak_src, sustained, workload,
             init_state=False):
    """Roofline entry of one kernel family: SIMT kernels against the fp32 FFMA
    rate; every other kernel under the roofline that the method's intensity
    (algorithmic FLOPs / the method's bytes) puts it (below the ridge =
    measured bf16 peak / measured HBM copy bandwidth: HBM, above: tensor).
    `frac` is on the method's bytes (or FLOPs); the fraction on the bytes this
    kernel itself moves (chunk states included) and the tensor-side fraction
    are reported beside it."""
    B, NH, T, DK, DV, L, elem = shape
    if fam.startswith("simt"):
        peak = SIMT_LANES * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        achieved = kflops / (per_launch_ms / 1e3) / 1e12
        return {"kernel": fam, "bound": "alu", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_source": f"fp32 FFMA: 148 SMs x 128 lanes x 2 x sm_max_mhz (of {peak_src})"}
    mbytes = method_bytes(fam, B, NH, T, DK, DV, elem, init_state)
    kbytes = kernel_bytes(fam, B, NH, T, DK, DV, L, elem)
    tkey = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    ridge = peaks[tkey] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    intensity = kflops / mbytes if mbytes else 0.0
    sec = per_launch_ms / 1e3
    tflops = kflops / sec / 1e12
    gbs = mbytes / sec / 1e9
    if intensity >= ridge:
        roof = {"kernel": fam, "bound": "tensor", "achieved": tflops, "peak": peaks[tkey],
                "unit": "TFLOP/s", "frac": tflops / peaks[tkey],
                "peak_source": f"{tkey} (of {peak_src})"}
    else:
        roof = {"kernel": fam, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                "peak_source": f"hbm_gbs (of {peak_src})"}
    roof.update(algorithmic_bytes=mbytes, algorithmic_flops=kflops,
                intensity_flop_per_byte=intensity, ridge_flop_per_byte=ridge,
                frac_hbm_method_bytes=gbs / peaks["hbm_gbs"],
                kernel_bytes=kbytes,
                frac_hbm_kernel_bytes=kbytes / sec / 1e9 / peaks["hbm_gbs"],
                frac_tensor=tflops / peaks[tkey],
                traffic=measured_traffic(fam, workload))
    return roof


def algorithmic_bytes(w, elem):
    BH = w.B * w.NH
    io = BH * w.T * (2 * w.DK + 2 * w.DV) * elem + BH * w.T * 8
    final = BH * (w.DK * w.DV + w.DK + 1) * 4
    init = final if w.init_state else 0
    return io + final + init


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)
# ----------------------------------------------------------------------------
_REASON_BITS = {
    "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
    "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
    "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    "display_clock_setting": 0x100,
}


class ClockSampler:
    def __init__(self, torch_dev_index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_dev_index)
            h = None
            try:
                bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id,
                                             props.pci_device_id)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons",
                   "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return int(getattr(nv, fn)(self.h))
        return 0

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((time.perf_counter(), sm, self._reasons(), pw))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: " + getattr(self, "err", "")}
        inwin = [s for s in self.samples if t0 <= s[0] <= t1]
        src = "timed region"
        if not inwin:
            inwin = [s for s in self.samples if s[0] >= t0 - 1.0]
            src = "around the timed region (no sample fell inside it)"
        if not inwin:
            inwin = self.samples
            src = "whole run"
        bits = 0
        for s in inwin:
            bits |= s[2]
        reasons = [k for k, b in _REASON_BITS.items() if bits & b and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in inwin) if inwin else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inwin),
                "power_w_max": max((s[3] for s in inwin), default=None), "window": src}


# ----------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload
# ----------------------------------------------------------------------------
def oracle_forward(oracle, c, gate_mode):
    """The oracle's forward pass for one input dict (the sigmoid variant without
    normaliser has a function of its own)."""
    if gate_mode == "sigmoid_plain":
        return oracle.mlstm_sigmoid_plain(c["Q"], c["K"], c["V"], c["i_pre"], c["f_pre"],
                                          c["C0"], c["n0"], c["m0"])
    return oracle.mlstm_recurrent(c["Q"], c["K"], c["V"], c["i_pre"], c["f_pre"], c["C0"],
                                  c["n0"], c["m0"], gate_mode=gate_mode)


def oracle_sample(w, x, target_s=15.0):
    """Time the oracle on a leading block of heads x tokens of the workload,
    sized from a short calibration run to take about `target_s` seconds.
    Returns (tokens/s, info)."""
    import torch

    import oracle
    cores = oracle.num_threads()
    BH = w.B * w.NH

    def sub(heads, tokens):
        sel = [(i // w.NH, i % w.NH) for i in range(heads)]
        out = {k: torch.stack([x[k][b, h, :tokens] for b, h in sel]).unsqueeze(0)
               for k in ("Q", "K", "V", "i_pre", "f_pre")}
        for k in ("C0", "n0", "m0"):
            out[k] = None if x[k] is None else torch.stack([x[k][b, h] for b, h in sel]).unsqueeze(0)
        return out

    def timed(heads, tokens):
        c = sub(heads, tokens)
        t0 = time.perf_counter()
        oracle_forward(oracle, c, w.gate_mode)
        return time.perf_counter() - t0

    h_cal = min(BH, cores)
    t_cal = min(w.T, 256)
    per_unit = max(timed(h_cal, t_cal), 1e-6) / (h_cal * t_cal)  # s per head-token, all cores
    units = target_s / per_unit
    if units >= BH * w.T:
        heads, tokens = BH, w.T
    else:
        tokens = w.T if units >= h_cal * w.T else max(t_cal, int(units // h_cal))
        heads = min(BH, max(h_cal, int(units // tokens) // h_cal * h_cal))
    el = timed(heads, tokens)
    return heads * tokens / el, {"heads": heads, "tokens_per_head": tokens, "seconds": el,
                                 "cores": cores}


def workload_config(w, algo):
    return {"workload": w.name, "B": w.B, "NH": w.NH, "T": w.T, "DK": w.DK, "DV": w.DV,
            "chunk_size": w.chunk_size, "gate_mode": w.gate_mode, "dtype": w.dtype,
            "init_state": w.init_state, "algo": algo,
            "l2": l2_note(w)}


def l2_note(w):
    nbytes = algorithmic_bytes(w, 2 if w.dtype == "bf16" else 4)
    if nbytes < 2 * L2_BYTES:
        return ("flushed before every timed step (a %d MB write, outside the per-step events): "
                "each step moves %.3f GB" % (2 * L2_BYTES >> 20, nbytes / 1e9))
    return "not flushed: each step moves %.2f GB (> 2 x %d MB L2)" % (nbytes / 1e9, L2_BYTES >> 20)


def pick_workload(name):
    from mlstm_chunkwise_b200.inputs import WORKLOADS, sweep_workload
    if name.startswith("sweep_"):
        _, t, l = name.split("_")
        return sweep_workload(int(t[1:]), int(l[1:]))
    return WORKLOADS[name]


# ----------------------------------------------------------------------------
# reference arm: the oracle alone
# ----------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from mlstm_chunkwise_b200.inputs import make_inputs
    w = pick_workload(args.workload)
    x = make_inputs(w)
    # size one step so that the whole K + W run stays within ~2 minutes
    budget = max(0.05, min(4.0, 120.0 / max(1, args.steps + args.warmup)))
    _, info = oracle_sample(w, x, target_s=budget)
    import oracle
    heads, tokens = info["heads"], info["tokens_per_head"]
    sel = [(i // w.NH, i % w.NH) for i in range(heads)]
    import torch
    c = {k: torch.stack([x[k][b, h, :tokens] for b, h in sel]).unsqueeze(0)
         for k in ("Q", "K", "V", "i_pre", "f_pre")}
    for k in ("C0", "n0", "m0"):
        c[k] = None if x[k] is None else torch.stack([x[k][b, h] for b, h in sel]).unsqueeze(0)

    def step():
        oracle_forward(oracle, c, w.gate_mode)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = heads * tokens * args.steps / el
    sample = (f"{heads} heads x first {tokens} tokens of {w.name} per step "
              f"(of {w.B * w.NH} heads x {w.T} tokens)")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, "oracle"), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def run_ours(args):
    import ctypes

    import torch
    import torch.distributed as dist

    from mlstm_chunkwise_b200 import _lib, api
    from mlstm_chunkwise_b200 import build as libbuild
    from mlstm_chunkwise_b200.inputs import make_inputs

    if libbuild.needs_build():
        libbuild.build()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = pick_workload(args.workload)
    if args.batch:
        w = w.replace(name=f"{w.name}_B{args.batch}", B=args.batch)
    x = make_inputs(w, seed=rank_seed(w, rank))
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    B, NH, T, DK, DV, L = w.B, w.NH, w.T, w.DK, w.DV, w.chunk_size
    elem = 2 if w.dtype == "bf16" else 4
    ws = torch.empty(max(1, api.workspace_size(B, NH, T, DK, DV, L, w.torch_dtype, args.algo)),
                     dtype=torch.uint8, device=dev)
    out = {"H": torch.empty((B, NH, T, DV), dtype=w.torch_dtype, device=dev),
           "C_T": torch.empty((B, NH, DK, DV), dtype=torch.float32, device=dev),
           "n_T": torch.empty((B, NH, DK), dtype=torch.float32, device=dev),
           "m_T": torch.empty((B, NH), dtype=torch.float32, device=dev)}

    def step_outs(inp, o):
        api.mlstm_fw(inp["Q"], inp["K"], inp["V"], inp["i_pre"], inp["f_pre"], inp["C0"],
                     inp["n0"], inp["m0"], chunk_size=L, gate_mode=w.gate_mode, algo=args.algo,
                     workspace=ws, out=o)

    def step(inp):
        step_outs(inp, out)

    # Workloads that fit in L2 twice over would be timed from a warm L2: flush
    # it (write a buffer twice its size) before every timed step and time the
    # steps alone with per-step events.
    small = algorithmic_bytes(w, elem) < 2 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if small else None

    lib = _lib.lib()
    for _ in range(max(3, args.warmup)):
        step(d)
    torch.cuda.synchronize()
    st = api.last_device_error(dev)
    if st != _lib.OK:
        raise SystemExit(f"device error after warm-up: {_lib.status_string(st)}")

    sampler = ClockSampler(local)
    sampler.start()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms_arr = (ctypes.c_double * _lib.KERNEL_COUNT)()
    n_arr = (ctypes.c_uint64 * _lib.KERNEL_COUNT)()
    lib.mlstm_profile_read(ms_arr, n_arr, _lib.KERNEL_COUNT)  # clear
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = lib.mlstm_kernel_launches()
    lib.mlstm_profile_enable(1)
    t_host0 = time.perf_counter()
    step_ev = []
    ev0.record(stream)
    for _ in range(args.steps):
        if small:
            flush_buf.fill_(1)
            e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e_a.record(stream)
            step(d)
            e_b.record(stream)
            step_ev.append((e_a, e_b))
        else:
            step(d)
    ev1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    lib.mlstm_profile_enable(0)
    launches = lib.mlstm_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    if small:  # the steps alone, without the flushes between them
        elapsed_ms = sum(a.elapsed_time(b) for a, b in step_ev)
    st = api.last_device_error(dev)
    if st != _lib.OK:
        raise SystemExit(f"device error in the timed region: {_lib.status_string(st)}")
    _lib.check(lib.mlstm_profile_read(ms_arr, n_arr, _lib.KERNEL_COUNT), "mlstm_profile_read")
    kern = {lib.mlstm_kernel_name(i).decode(): (ms_arr[i], int(n_arr[i]))
            for i in range(_lib.KERNEL_COUNT) if n_arr[i]}
    sampler.stop()
    clocks = sampler.summary(t_host0, t_host1)

    elapsed_ms = max_over_ranks(elapsed_ms, dev, world)

    # --- sustained: the same step back to back for at least a second --------
    # A K-step burst of a sub-millisecond step runs at the boost clock; over a
    # second the 1 kW power cap lowers it.  This region is judged against the
    # sustained bf16 peak.  Skipped for workloads timed with L2 flushes.
    sus = None
    if not small and not args.no_sustained:
        n_sus = max(args.steps, int(math.ceil(1000.0 * args.sustained_s /
                                              max(1e-3, elapsed_ms / args.steps))))
        sampler2 = ClockSampler(local)
        sampler2.start()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s_h0 = time.perf_counter()
        es0, es1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        es0.record(stream)
        for _ in range(n_sus):
            step(d)
        es1.record(stream)
        torch.cuda.synchronize()
        s_h1 = time.perf_counter()
        sampler2.stop()
        sus_ms = max_over_ranks(es0.elapsed_time(es1), dev, world)
        st = api.last_device_error(dev)
        if st != _lib.OK:
            raise SystemExit(f"device error in the sustained region: {_lib.status_string(st)}")
        sus = {"steps": n_sus, "seconds": sus_ms / 1e3, "ms_per_step": sus_ms / n_sus,
               "value": job_throughput(B * T, world, sus_ms / n_sus), "unit": "tokens/s",
               "clocks": sampler2.summary(s_h0, s_h1)}

    # --- e2e: pinned host inputs -> device -> mlstm_fw -> host outputs -------
    # Every step copies its own inputs in and its outputs out.  The copies run
    # on two copy streams (the link is full duplex) into double-buffered device
    # buffers, so step i's inputs travel while step i - 1 computes and step
    # i - 2's outputs travel back; the timed region spans the first input copy
    # to the last output copy.  At least 30 steps (up to 60) when --steps
    # allows, so that the pipeline's fill (the first copy in) and drain (the
    # last copy out) are spread over a run closer to steady streaming.
    e2e_steps = max(1, min(max(args.steps, 30), 60)) if args.steps >= 3 else max(1, args.steps)
    e2e_ms = float("nan")
    h2d = d2h = 0
    if not args.no_e2e:
        hx = {k: v.pin_memory() for k, v in x.items() if v is not None}
        hout = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()}
        h2d = sum(v.numel() * v.element_size() for v in hx.values())
        d2h = sum(v.numel() * v.element_size() for v in hout.values())
        dins = [dict(x, **{k: torch.empty_like(v, device=dev) for k, v in hx.items()})
                for _ in range(2)]
        douts = [out] + [{k: torch.empty_like(v) for k, v in out.items()}]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "done", "read")}

        def e2e_run(n_steps):
            for i in range(n_steps):
                b = i % 2
                if i >= 2:
                    s_in.wait_event(ev["done"][b])  # step i - 2 has read dins[b]
                with torch.cuda.stream(s_in):
                    for k, v in hx.items():
                        dins[b][k].copy_(v, non_blocking=True)
                    ev["in"][b].record(s_in)
                stream.wait_event(ev["in"][b])
                if i >= 2:
                    stream.wait_event(ev["read"][b])  # step i - 2's outputs copied out
                step_outs(dins[b], douts[b])
                ev["done"][b].record(stream)
                s_out.wait_event(ev["done"][b])
                with torch.cuda.stream(s_out):
                    for k, v in douts[b].items():
                        hout[k].copy_(v, non_blocking=True)
                    ev["read"][b].record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if not args.no_e2e:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_run(e2e_steps)
        s_out.wait_stream(s_in)
        s_out.wait_stream(stream)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dev, world)

    tokens_per_step = B * T * world
    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(B * T, world, ms_per_step)
    e2e_value = None if args.no_e2e else job_throughput(B * T, world, e2e_ms / e2e_steps)

    # --- roofline of the dominant kernel ------------------------------------
    peaks, peak_src = load_peaks()
    fph = flops_per_head(T, DK, DV, L)
    BH = B * NH
    fam_flops = {
        "tc_fused": BH * (fph["states"] + fph["inter"] + fph["intra"]),
        "tc_states": BH * fph["states"], "simt_states": BH * fph["states"],
        "tc_parallel": BH * (fph["inter"] + fph["intra"]),
        "simt_parallel": BH * (fph["inter"] + fph["intra"]),
    }
    total_flops = BH * sum(fph.values())
    top = max(kern.items(), key=lambda kv: kv[1][0])
    top_name, (top_ms, top_n) = top
    calls = max(1, args.steps)
    per_launch_ms = top_ms / calls
    sustained = elapsed_ms > 1000.0
    roof = roofline(top_name, per_launch_ms, fam_flops.get(top_name, 0.0),
                    (B, NH, T, DK, DV, L, elem), peaks, peak_src, sustained, w.name,
                    w.init_state)
    roof["per_launch_ms"] = per_launch_ms
    step_flops_s = total_flops / (ms_per_step / 1e3)
    if sus is not None:
        sus["tflops"] = total_flops * world / (sus["ms_per_step"] / 1e3) / 1e12
        sus["frac_bf16_peak_sustained"] = (total_flops / (sus["ms_per_step"] / 1e3) / 1e12) / \
            peaks["bf16_tflops_sustained"]

    algo_used = "+".join(sorted(kern))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": workload_config(w, algo_used),
        "tflops": total_flops * world / (ms_per_step / 1e3) / 1e12,
        "frac_bf16_peak": step_flops_s / 1e12 / peaks["bf16_tflops"],
        "frac_bf16_datasheet": step_flops_s / 1e12 / DATASHEET_BF16_TFLOPS,
        "frac_hbm_step": algorithmic_bytes(w, elem) / (ms_per_step / 1e3) / 1e9 /
        peaks["hbm_gbs"],
        "roofline": roof,
        "sustained": sus,
        "kernels_ms_per_step": {k: v[0] / calls for k, v in kern.items()},
        "chunk_state_bytes_written": chunk_state_bytes_written(set(kern), B, NH, T, DK, DV, L),
        "e2e": None if args.no_e2e else {
            "value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": e2e_steps,
            "overlap": "copy-in, compute and copy-out on three streams, double-buffered"},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        v, info = oracle_sample(w, x, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": v, "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
            "sample": f"{info['heads']} heads x first {info['tokens_per_head']} tokens of "
                      f"{w.name} ({info['seconds']:.1f} s)"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# single-token step (decode) at a workload's B, NH, d_qk, d_v
# ----------------------------------------------------------------------------
STEP_METRIC = "mLSTM single-token step tokens/s (one token per sequence per step)"


def step_bytes(B, NH, DK, DV, elem):
    """Algorithmic bytes of one step: the fp32 state (C, n, m) read and written
    once, q, k, v, h and the two gate pre-activations moved once."""
    state = B * NH * (DK * DV + DK + 1) * 4
    return 2 * state + B * NH * ((2 * DK + 2 * DV) * elem + 2 * 4)


def run_step(args):
    import ctypes

    import torch

    import oracle
    from mlstm_chunkwise_b200 import _lib, api
    from mlstm_chunkwise_b200 import build as libbuild

    if libbuild.needs_build():
        libbuild.build()
    if int(os.environ.get("WORLD_SIZE", "1")) != 1 or args.gpus != 1:
        raise SystemExit("--op step runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = pick_workload(args.workload)
    B = args.batch or w.B
    NH, DK, DV, dt = w.NH, w.DK, w.DV, w.torch_dtype
    elem = 2 if w.dtype == "bf16" else 4
    g = torch.Generator().manual_seed(rank_seed(w, 0))
    n_tok = args.steps + max(3, args.warmup)
    tok = {"q": torch.randn((n_tok, B, NH, DK), generator=g).to(dt),
           "k": torch.randn((n_tok, B, NH, DK), generator=g).to(dt),
           "v": torch.randn((n_tok, B, NH, DV), generator=g).to(dt),
           "i": torch.randn((n_tok, B, NH), generator=g) + w.i_mean,
           "f": torch.rand((n_tok, B, NH), generator=g) * (w.f_high - w.f_low) + w.f_low}
    dtok = {k: v.to(dev) for k, v in tok.items()}
    C = torch.zeros((B, NH, DK, DV), device=dev)
    n = torch.zeros((B, NH, DK), device=dev)
    m = torch.zeros((B, NH), device=dev)
    h = torch.empty((B, NH, DV), dtype=dt, device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step(i):
        api.mlstm_step(dtok["q"][i], dtok["k"][i], dtok["v"][i], dtok["i"][i], dtok["f"][i],
                       C, n, m, gate_mode=w.gate_mode, h=h)

    warm = max(3, args.warmup)
    for i in range(warm):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    lib = _lib.lib()
    ms_arr = (ctypes.c_double * _lib.KERNEL_COUNT)()
    n_arr = (ctypes.c_uint64 * _lib.KERNEL_COUNT)()
    lib.mlstm_profile_read(ms_arr, n_arr, _lib.KERNEL_COUNT)
    sampler = ClockSampler(0)
    sampler.start()
    stream = torch.cuda.current_stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    launches0 = lib.mlstm_kernel_launches()
    t_host0 = time.perf_counter()
    for j, (e0, e1) in enumerate(evs):
        flush.zero_()  # the state does not stay in L2 between steps
        e0.record(stream)
        step(warm + j)
        e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    launches = lib.mlstm_kernel_launches() - launches0
    sampler.stop()
    st = api.last_device_error(dev)
    if st != _lib.OK:
        raise SystemExit(f"device error in the timed region: {_lib.status_string(st)}")
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    peaks, peak_src = load_peaks()
    nbytes = step_bytes(B, NH, DK, DV, elem)
    achieved = nbytes / (ms / 1e3) / 1e9
    line = {
        "metric": STEP_METRIC, "value": B / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": warm, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"step_{w.name}", "B": B, "NH": NH, "DK": DK, "DV": DV,
                   "gate_mode": w.gate_mode, "dtype": w.dtype,
                   "l2": "flushed before every step (a %d MB write outside the events)"
                         % (2 * L2_BYTES >> 20)},
        "roofline": {"kernel": "step", "bound": "hbm", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "peak_source": f"hbm_gbs (of {peak_src})", "algorithmic_bytes": nbytes,
                     "traffic": None, "per_launch_ms": ms},
        "gpu_launches": int(launches), "e2e": None,
        "clocks": sampler.summary(t_host0, t_host1),
    }
    if not args.no_cpu_baseline:
        # the oracle's recurrence over one token from the state, for every (b, h)
        Ch, nh, mh = C.cpu(), n.cpu(), m.cpu()
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.mlstm_recurrent(tok["q"][0][:, :, None], tok["k"][0][:, :, None],
                                   tok["v"][0][:, :, None], tok["i"][0][:, :, None],
                                   tok["f"][0][:, :, None], Ch, nh, mh, gate_mode=w.gate_mode)
            reps += 1
            el = time.perf_counter() - t0
            if el > min(args.cpu_seconds, 5.0):
                break
        line["cpu_baseline"] = {"value": B * reps / el, "unit": "tokens/s",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{reps} steps of all {B * NH} heads ({el:.1f} s)"}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# backward pass at a workload's shape (bf16 with d_qk 128 or 256: tensor-core
# kernels on 128-token chunks; otherwise the fp32 CUDA-core kernels)
# ----------------------------------------------------------------------------
BW_METRIC = "mLSTM backward tokens/s (gradients of a loss on H, forward recomputed)"


def bw_flops_per_head(T, DK, DV, L):
    """Algorithmic FLOPs of the gradient kernels for one (b, h), causal halves
    counted once: the reverse state recurrence and the three inter-chunk terms
    (2 T DK DV each), and six intra-chunk contractions (T L d each: dP and P.K
    for dq, dP and P.Q for dk, S and P.dU for dv).  The recomputed forward is
    counted separately (flops_per_head)."""
    return 8.0 * T * DK * DV + 3.0 * T * L * (DK + DV)


def run_bw(args):
    import ctypes

    import torch

    from mlstm_chunkwise_b200 import _lib, api
    from mlstm_chunkwise_b200 import build as libbuild
    from mlstm_chunkwise_b200.inputs import make_inputs

    if libbuild.needs_build():
        libbuild.build()
    if int(os.environ.get("WORLD_SIZE", "1")) != 1 or args.gpus != 1:
        raise SystemExit("--op bw runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = pick_workload(args.workload)
    if args.batch:
        w = w.replace(name=f"{w.name}_B{args.batch}", B=args.batch)
    x = make_inputs(w, seed=rank_seed(w, 0))
    g = torch.Generator().manual_seed(rank_seed(w, 0) + 1)
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    dH = torch.randn((w.B, w.NH, w.T, w.DV), generator=g).to(w.torch_dtype).to(dev)
    B, NH, T, DK, DV, L = w.B, w.NH, w.T, w.DK, w.DV, w.chunk_size

    saved = None
    if args.saved:
        # the training pair's backward: the training forward once, untimed
        if api.train_sizes(B, NH, T, DK, DV, w.torch_dtype) is None:
            raise SystemExit("--saved: this shape has no training pair")
        H, _, saved = api.mlstm_fw_train(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"],
                                         d["C0"], d["n0"], d["m0"], gate_mode=w.gate_mode)

    def step():
        if saved is not None:
            api.mlstm_bw_saved(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], H, saved, dH,
                               d["C0"], d["n0"], d["m0"], gate_mode=w.gate_mode)
        else:
            api.mlstm_bw(d["Q"], d["K"], d["V"], d["i_pre"], d["f_pre"], dH, d["C0"], d["n0"],
                         d["m0"], chunk_size=L, gate_mode=w.gate_mode)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    lib = _lib.lib()
    sampler = ClockSampler(0)
    sampler.start()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = lib.mlstm_kernel_launches()
    t_host0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    launches = lib.mlstm_kernel_launches() - launches0
    sampler.stop()
    st = api.last_device_error(dev)
    if st != _lib.OK:
        raise SystemExit(f"device error in the timed region: {_lib.status_string(st)}")
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = load_peaks()
    # the tensor-core backward runs on 128-token chunks whatever chunk_size is
    tc_bw = (w.dtype == "bf16" and DK in (128, 256) and (DV == 128 or DV % 256 == 0) and DV <= 1024
             and T >= 128)
    Lb = 128 if tc_bw else L
    fph = flops_per_head(T, DK, DV, Lb)
    # the saved backward recomputes nothing: its FLOPs are the gradient kernels'
    fw_flops = 0.0 if saved is not None else B * NH * (fph["states"] + fph["inter"] + fph["intra"])
    bw_flops = B * NH * bw_flops_per_head(T, DK, DV, Lb)
    achieved = (fw_flops + bw_flops) / (ms / 1e3) / 1e12
    if tc_bw:
        algo = ("bw from the training pair's saved buffer" if saved is not None
                else "bw (tensor cores, 128-token chunks)")
        bound, peak = "tensor", peaks["bf16_tflops"]
        peak_source = f"bf16_tflops (of {peak_src})"
    else:
        algo, bound = "bw (fp32 CUDA-core kernels)", "alu"
        peak = SIMT_LANES * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        peak_source = f"fp32 FFMA: 148 SMs x 128 lanes x 2 x sm_max_mhz (of {peak_src})"
    line = {
        "metric": BW_METRIC, "value": B * T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": warm, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, algo),
        "tflops": achieved,
        "roofline": {"kernel": "bw", "bound": bound, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_source,
                     "algorithmic_flops": fw_flops + bw_flops, "traffic": None,
                     "per_launch_ms": ms},
        "gpu_launches": int(launches), "e2e": None,
        "clocks": sampler.summary(t_host0, t_host1),
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# training step: forward + backward through the autograd Function
# ----------------------------------------------------------------------------
TRAIN_METRIC = "mLSTM training step tokens/s (forward + backward through torch.autograd)"


def run_train(args):
    """One training step of the layer: mlstm_chunkwise forward, a loss
    sum(H * G) with a fixed G, and loss.backward() into every input's .grad
    (the backward recomputes the forward from the inputs).  Timed with CUDA
    events around whole steps on one GPU."""
    import torch

    from mlstm_chunkwise_b200 import _lib, api
    from mlstm_chunkwise_b200 import build as libbuild
    from mlstm_chunkwise_b200.inputs import make_inputs

    if libbuild.needs_build():
        libbuild.build()
    if int(os.environ.get("WORLD_SIZE", "1")) != 1 or args.gpus != 1:
        raise SystemExit("--op train runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = pick_workload(args.workload)
    if args.batch:
        w = w.replace(name=f"{w.name}_B{args.batch}", B=args.batch)
    x = make_inputs(w, seed=rank_seed(w, 0))
    leaves = {k: v.to(dev).requires_grad_(True) for k, v in x.items() if v is not None}
    G = torch.randn((w.B, w.NH, w.T, w.DV), generator=torch.Generator().manual_seed(7)).to(
        w.torch_dtype).to(dev)

    def step():
        for v in leaves.values():
            v.grad = None
        H, _ = api.mlstm_chunkwise(leaves["Q"], leaves["K"], leaves["V"], leaves["i_pre"],
                                   leaves["f_pre"], leaves.get("C0"), leaves.get("n0"),
                                   leaves.get("m0"), chunk_size=w.chunk_size,
                                   gate_mode=w.gate_mode)
        H.backward(G)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    lib = _lib.lib()
    sampler = ClockSampler(0)
    sampler.start()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = lib.mlstm_kernel_launches()
    t_host0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    launches = lib.mlstm_kernel_launches() - launches0
    sampler.stop()
    st = api.last_device_error(dev)
    if st != _lib.OK:
        raise SystemExit(f"device error in the timed region: {_lib.status_string(st)}")
    ms = e0.elapsed_time(e1) / args.steps
    line = {
        "metric": TRAIN_METRIC, "value": w.B * w.T / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": warm, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": workload_config(w, "mlstm_chunkwise (fw + bw)"),
        "roofline": None, "gpu_launches": int(launches), "e2e": None,
        "clocks": sampler.summary(t_host0, t_host1),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="xlstm7b")
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc", "tc_fused"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end loop (profiling runs)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller profiling captures)")
    ap.add_argument("--saved", action="store_true",
                    help="with --op bw: time mlstm_bw_saved (the training pair's backward)")
    ap.add_argument("--sustained-s", type=float, default=1.2,
                    help="seconds of the sustained region that follows the timed steps")
    ap.add_argument("--no-sustained", action="store_true")
    ap.add_argument("--op", default="fw", choices=["fw", "step", "bw", "train"],
                    help="fw: the forward pass (default); step: the single-token step; "
                         "bw: the backward pass; train: forward + backward through autograd")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "step":
        return run_step(args)
    if args.op == "train":
        return run_train(args)
    if args.op == "bw":
        return run_bw(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
