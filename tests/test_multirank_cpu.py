"""The N > 1 bench path on CPU: two gloo ranks, replicas with max-over-ranks timing.

The method needs no exchange between ranks (every (sequence, head) unit is
independent), so a multi-GPU run is N independent replicas; the only
collectives are the barrier and the max of the per-rank step times.  These run
here with the gloo backend, world size 2, without a GPU.  The reference arm
(the fp64 oracle on host cores) is checked as well.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    m = d.max(times[rank])
    d.barrier()
    d.close()
    out_q.put((rank, m))


def test_two_rank_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [1.25, 3.5]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 3.5, 1: 3.5}


def test_weak_scaling_value_formula():
    sys.path.insert(0, ROOT)
    import bench

    # algorithmic bytes of the gated workload: q, k bf16 once per q/k head, v bf16, o fp32,
    # gates/betas fp32, state in + out fp32
    b = bench.prefill_bytes(2, 8192, 16, 32, 128, 128, 2, 4, 2, True)
    tok = 2 * 8192
    assert b == tok * 16 * 128 * 2 * 2 + tok * 32 * 128 * 2 + tok * 32 * 128 * 4 + tok * 32 * 8 \
        + 2 * 32 * 128 * 128 * 4 * 2
    assert bench.prefill_flops(1, 128, 128) == 2 * 64 * (3 * 128 + 2 * 128) + 6 * 128 * 128


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["unit"] == "tokens/s"
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun the reference arm runs on rank 0 alone; rank 1 prints nothing, exits 0."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""
