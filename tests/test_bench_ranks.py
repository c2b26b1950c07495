"""The multi-rank plumbing of bench.py on CPU, and its reference arm.

With N > 1 each rank draws its own seeded batch (its shard of the global
batch of the token-sharded data-parallel step, whose collectives are tested in
test_dp_orchestration.py and test_gpu_dp_ranks.py), and the reported time is
the slowest rank's (max over ranks, gloo world size 2 here).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"), world)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_replicas_draw_different_batches():
    w = synth.CONFIGS["tiny"]
    a = synth.make_inputs(w, seed=bench.replica_seed(w, w.N, 0))
    b = synth.make_inputs(w, seed=bench.replica_seed(w, w.N, 1))
    assert not (a.hidden_bits == b.hidden_bits).all()
    assert bench.replica_seed(w, w.N, 0) == synth.seed_for(w)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5


@pytest.mark.parametrize("steps", [1])
def test_reference_arm_prints_contract_line(steps, capsys, monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--config", "tiny", "--steps", str(steps),
                                     "--warmup", "1"])
    assert bench.main() == 0
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True


def test_reference_arm_counts_the_rows_it_times():
    """Each step times one seeded sample of bench.CPU_SAMPLE_ROWS rows (the GPU line's
    cpu_baseline times the same sample size), and the rate is computed from the rows
    actually processed."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "2", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    n = min(bench.CPU_SAMPLE_ROWS, synth.CONFIGS["tiny"].N)
    assert line["config"]["sample_rows_per_step"] == n
    assert line["cpu_baseline"]["sample"].startswith(f"{n} seeded rows")
    assert abs(line["value"] - n * 2 / (line["ms_per_step"] * 2 / 1000.0)) <= 1e-6 * line["value"]
