"""Multi-rank logic of bench.py on CPU: two gloo ranks (spawned processes) take the max of
their timed regions, draw disjoint inputs (weak scaling), and the whole-job rate counts every
rank's tokens over the slowest rank's time; the reference arm does no work off rank 0."""
import datetime
import multiprocessing as mp
import os
import socket
import types

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        seeds = bench.rank_seeds(rank, 8, 16)
    finally:
        dist.destroy_process_group()
    q.put((rank, got, seeds))


def test_two_gloo_ranks_max_time_and_disjoint_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert [got for _, got, _ in res] == [15.0, 15.0]           # both see the slowest rank
    (_, _, (rep0, x0)), (_, _, (rep1, x1)) = res
    assert not set(rep0) & set(rep1) and not set(x0) & set(x1)
    assert len(set(rep0)) == 8 and len(set(x0)) == 16


def test_whole_job_rate_counts_all_ranks_over_the_slowest():
    assert bench.whole_job_rate(1, 2, 100, 15.0) == 2 * 100 / 0.015
    assert bench.whole_job_rate(4096, 1, 20, 58.0) == 4096 * 20 / 0.058


def test_reference_arm_idle_off_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(steps=1, warmup=0)
    assert bench.reference_arm(args, None, 1) == 0


def _reference_line(capsys, monkeypatch, *extra):
    import json
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--impl", "reference", "--workload", "tiny:4", "--steps", "2", "--warmup", "3",
                       *extra]) == 0
    return json.loads(capsys.readouterr().out.strip().splitlines()[-1])


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    """The oracle as the reference arm: one JSON line with the keys the benchmark contract
    asks for, its cpu_baseline and e2e describing this run."""
    d = _reference_line(capsys, monkeypatch)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tok/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"] and "top-p" not in d["config"]["workload"]


def test_reference_arm_with_adaptive_top_p(capsys, monkeypatch):
    d = _reference_line(capsys, monkeypatch, "--top-p", "0.3")
    assert d["value"] > 0 and "adaptive top-p 0.3" in d["config"]["workload"]


def test_timed_region_has_no_instrumented_step():
    """Every timed step is an event-free graph replay, whatever --steps, --period and
    --event-steps are (the driver's --steps 20 is below the default --event-steps 32), and the
    replays add up to exactly --steps."""
    for steps in (1, 3, 19, 20, 31, 32, 33, 255, 256, 257, 5000):
        for period in (1, 16, 20, 64, 256):
            for ev in (1, 16, 20, 32, 64):
                G, n_main, rem, Ge = bench.step_plan(steps, period, ev)
                assert n_main * G + rem == steps and 0 <= rem < G and 1 <= Ge <= G
                plan = bench.timed_replays(steps, period, ev)
                assert sum(n for _, n, _ in plan) == steps
                assert not any(inst for _, _, inst in plan), (steps, period, ev)
                assert {name for name, _, _ in plan} <= {"graph", "graph_rem"}


def test_both_arms_print_the_same_config(capsys, monkeypatch):
    """The reference arm's config object is the one the GPU arm prints for the same arguments."""
    d = _reference_line(capsys, monkeypatch)
    cfg, T = bench.parse_workload("tiny:4")
    ns = types.SimpleNamespace(steps=2, warmup=3, period=256, event_steps=32, replicas=8, top_p=0.0)
    assert d["config"] == bench.line_config(cfg, T, ns, 1)
    assert "no event nodes" in d["config"]["graph"]
