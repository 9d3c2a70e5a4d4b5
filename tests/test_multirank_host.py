"""The N > 1 host path of bench.py on CPU: two ranks over gloo (127.0.0.1).

Every rank times its own independent copy of the workload; the job's time is the slowest
rank's and its throughput counts every rank's units.  The reference arm runs on rank 0
only; other ranks leave without work."""
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, times, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # same collective sequence as the bench: step time, then the end-to-end time
        t_step = bench.max_over_ranks(times[rank][0], ws)
        t_e2e = bench.max_over_ranks(times[rank][1], ws)
        out.put((rank, t_step, t_e2e, bench.whole_job_rate(1000, ws, t_step)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_count_all_units():
    ws, port = 2, _free_port()
    times = [(0.25, 3.0), (0.5, 2.0)]          # per rank: (step s, e2e s)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, times, out)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(ws))
    for rank, t_step, t_e2e, rate in res:
        assert t_step == 0.5 and t_e2e == 3.0           # max over ranks, the same on every rank
        assert rate == pytest.approx(2 * 1000 / 0.5)    # whole job: both ranks' units


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.whole_job_rate(10, 1, 2.0) == 5.0


class _FakeSample:
    """Stands in for the oracle sample: counts steps, scores 1000 keys per step."""
    made = []

    def __init__(self, w, kind, heads, seed=0):
        self.heads = heads
        _FakeSample.made.append(self)

    def step(self):
        return 1000

    def describe(self, dt):
        return "fake sample"


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    _FakeSample.made = []
    monkeypatch.setattr(bench, "OracleSample", _FakeSample)
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(steps=2, warmup=3, config="serving")
    bench.run_reference(args)
    assert _FakeSample.made == [] and capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    import json
    import bench
    _FakeSample.made = []
    monkeypatch.setattr(bench, "OracleSample", _FakeSample)
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    args = types.SimpleNamespace(steps=2, warmup=3, config="serving")
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "keys/s" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "serving-decode-3.5bit"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
