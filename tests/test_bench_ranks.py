"""The multi-rank plumbing of bench.py on CPU with gloo (world size 2).

With N > 1 every rank runs an independent replica (different seeded batch)
and the reported time is the slowest rank's; no collective touches the data.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


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
