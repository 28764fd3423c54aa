"""The N > 1 logic of bench.py on CPU: two gloo ranks (world size 2) on
127.0.0.1.  The path shards over independent (b, h) pairs, so the only
cross-rank steps are the barrier and the max over ranks of the timings."""
import importlib.util
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs
        w = WORKLOADS["tiny"]
        x = make_inputs(w, seed=bench.rank_seed(w, rank))
        # each rank "times" a different amount; the job is as slow as the slowest
        local_ms = 10.0 + 5.0 * rank
        worst = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        tput = bench.job_throughput(w.B * w.T, world, worst)
        dist.barrier()
        torch.save({"worst": worst, "tput": tput, "Q": x["Q"]}, os.path.join(outdir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_two_gloo_ranks_take_the_max_and_shard_the_inputs(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [torch.load(tmp_path / f"r{i}.pt") for i in range(world)]
    assert r[0]["worst"] == r[1]["worst"] == 15.0
    # whole-job tokens/s: both ranks' tokens over the slower rank's time
    from mlstm_chunkwise_b200.inputs import WORKLOADS
    w = WORKLOADS["tiny"]
    assert r[0]["tput"] == pytest.approx(2 * w.B * w.T / 15e-3)
    # same shape, independent draws per rank
    assert r[0]["Q"].shape == r[1]["Q"].shape
    assert not torch.equal(r[0]["Q"], r[1]["Q"])


def test_single_rank_helpers_need_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    assert bench.job_throughput(1000, 1, 2.0) == pytest.approx(5e5)


@pytest.mark.timeout(120)
def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun only rank 0 times the oracle; other ranks exit 0 silently."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=110)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
