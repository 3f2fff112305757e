"""Host logic of bench.py's multi-rank path, on CPU with the gloo backend.

Under torchrun every rank times its own replica of the layer; the job's
time is the maximum over the ranks and the value is ms per call over all
ranks' calls.  Two gloo ranks check that reduction and the per-call value,
and the oracle arm exits at once on every rank but 0.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = 100.0 + 25.0 * rank  # rank 1 is the slower one
        t_max = bench.max_over_ranks(local_ms, "cpu", world)
        out.put((rank, t_max, bench.per_call_ms(t_max, 10, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_every_call():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(2))
    for rank, t_max, per_call in got:
        assert t_max == 125.0  # the slower rank's time, on every rank
        assert per_call == pytest.approx(125.0 / 20)  # 2 ranks x 10 calls


def test_single_rank_reduction_is_the_local_value():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(42.5, "cpu", 1) == 42.5
    assert bench.per_call_ms(42.5, 5, 1) == pytest.approx(8.5)


def test_reference_arm_exits_on_nonzero_ranks_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    """Rank 0 of the oracle arm prints one JSON line with the contract's keys;
    the paired draw design runs through it like the others (one query block
    per head, a few seconds of CPU)."""
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--cpu-seconds", "1",
                        "--sampling", "paired"], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["higher_is_better"] is False
    assert line["config"]["sampling"] == "paired"
    assert line["value"] > 0 and line["value"] == line["cpu_baseline"]["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    # the line states what ran: ms_per_step is the measured sampled step, value the
    # full-layer estimate from it, with the sampled query blocks and the factor
    sw = line["sampled_work"]
    assert line["config"]["workload"] == "hunyuan_720p_33x45x80"
    assert 1 <= sw["timed_query_blocks_per_head"] <= sw["query_blocks_per_head"]
    assert sw["extrapolation_factor"] == pytest.approx(
        sw["query_blocks_per_head"] / sw["timed_query_blocks_per_head"])
    assert line["ms_per_step"] == pytest.approx(sw["step_seconds"] * 1e3)
    assert line["ms_per_step"] <= line["value"]
