"""bench.py with more than one rank, on the host: two gloo ranks (one process
each, as torchrun starts them) agree on the slowest rank's time and on the
whole-job rate; one process is its own maximum; under torchrun only rank 0
of the reference arm does any work or prints."""
import json
import socket
import sys

import pytest
import torch.multiprocessing as mp

import bench
import _multirank


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree(tmp_path):
    rank_ms = [12.5, 20.0]   # rank 1 is the slowest
    mp.start_processes(_multirank.rank_worker, args=(2, _free_port(), str(tmp_path), rank_ms),
                       nprocs=2, start_method="spawn", join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert got[0] == got[1]
    assert got[0]["max_ms"] == 20.0
    # every rank's units over the slowest rank's time
    assert got[0]["rate"] == pytest.approx(1000.0 * 5 * 2 / 0.020)


def test_one_process_is_its_own_maximum():
    import torch
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(10.0, 4, 1, 8.0) == pytest.approx(10.0 * 4 / 0.008)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2",
                                      "--steps", "1", "--warmup", "1"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""


def test_bench_rejects_unsupported_state_counts(monkeypatch):
    for argv in (["bench.py", "--n-states", "32"], ["bench.py", "--n-states", "65", "--backward"]):
        monkeypatch.setattr(sys, "argv", argv)
        with pytest.raises(SystemExit) as ei:
            bench.main()
        assert ei.value.code == 2
