"""The N > 1 bench path on the host: two gloo ranks on CPU.  Each rank runs its
own replica of the workload (no data-path collective); the job's time is the
maximum over ranks and the throughput counts every rank's tokens."""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 7.5 * rank, world, "cpu")
        q.put((rank, ms, bench.job_tokens_per_s(world, 4096, 100, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 17.5                        # the slower rank's time, on every rank
        assert value == pytest.approx(2 * 4096 * 100 / 17.5e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.job_tokens_per_s(1, 8192, 10, 20.0) == pytest.approx(8192 * 10 / 0.02)


def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun only rank 0 times the oracle; rank 1 exits 0 at once."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    """Rank 0 of the reference arm times the oracle on the host cores and prints
    one JSON line with the bench contract's keys; the copies it does not make are
    counted as zero bytes."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32_L256", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] >= 3
    assert line["config"]["workload"] == "tiny_f32_L256"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_ranks_draw_their_own_batches():
    """Weak scaling over replicas: every rank times the same shape on its own
    inputs; rank 0 keeps the single-GPU inputs."""
    import torch
    from token_attention_b200 import synth
    wl = synth.WORKLOADS["tiny_f32_L256"]
    r0 = bench.make_sets(wl, "cpu", 2, rank=0)
    r1 = bench.make_sets(wl, "cpu", 2, rank=1)
    single = synth.make_attn_inputs(synth.shrink(wl, seed=wl.seed))
    assert torch.equal(r0[0]["q"], torch.from_numpy(single["q"]))
    assert not torch.equal(r0[0]["q"], r0[1]["q"])
    assert not torch.equal(r0[0]["q"], r1[0]["q"]) and r0[0]["q"].shape == r1[0]["q"].shape
