"""The multi-rank plumbing of bench.py on the CPU: two ranks over gloo (127.0.0.1) take the same
collective steps as the GPU bench (a barrier, a max over ranks of each rank's time), draw different
seeded inputs per rank (independent sequences, no data-path collective), and report the whole-job
rate over the slowest rank's time.  The reference arm does its work on rank 0 only."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    from cascade_token_head_b200 import synth
    r = bench.Ranks("gloo", timeout_s=60)
    r.barrier()
    own_ms = 100.0 + 50.0 * rank                  # this rank's device time
    slowest = r.max_over_ranks(own_ms)
    rate = bench.whole_job_rate(r.world, 1000, 4, slowest)
    w = synth.tiny_fp32()
    w.seed = r.rank                               # as the bench seeds each rank's sequences
    x = synth.draw_prefill(w)["X"]
    r.barrier()
    r.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"slowest": slowest, "rate": rate, "x0": float(np.asarray(x).ravel()[0]),
                   "x_sum": float(np.asarray(x).sum())}, f)


def test_two_ranks_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["slowest"] == 150.0                          # the max over ranks, on every rank
        assert r["rate"] == pytest.approx(2 * 1000 * 4 / 0.150)
    assert res[0]["x_sum"] != res[1]["x_sum"]                  # each rank draws its own sequences


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks("gloo")
    assert (r.rank, r.world) == (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
    if r.world == 1:
        assert r.max_over_ranks(3.5) == 3.5
        r.barrier()
        r.close()


def test_reference_arm_times_exactly_the_requested_steps(capsys):
    """The reference arm (the float64 oracle) times exactly --steps units of the workload, one
    sequence per step for the BERT-shaped prefill, and reports consistent per-step numbers."""
    sys.path.insert(0, ROOT)
    import bench
    os.environ.pop("RANK", None)
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2
    assert "2 sequence(s)" in line["cpu_baseline"]["sample"]
    per_step_s = line["ms_per_step"] / 1e3
    assert line["value"] == pytest.approx(512 / per_step_s, rel=0.25)   # tokens/s of one sequence per step
    assert line["e2e"]["value"] == line["value"]
