"""Host-side logic of bench.py: algorithmic byte accounting, weak-scaling aggregation and
the max-over-ranks reduction (world_size 2 over gloo on CPU), and the reference arm's
JSON line."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_slot_recurrent_b200.workloads import WORKLOADS  # noqa: E402


def test_prefill_algorithmic_bytes():
    # per token-head: 2 x 20 bf16 logits + v, z, y (128 bf16 each) + g = 850 B;
    # per head: final S (1024 x 128 fp32) + m (1024 fp32) = 528,384 B
    w = WORKLOADS["prefill_340m_top8"]
    assert bench.prefill_algorithmic_bytes(w) == 8 * 4096 * 8 * 850 + 64 * 528384
    w4 = WORKLOADS["prefill_1p3b_top16"]
    assert bench.prefill_algorithmic_bytes(w4) == 4 * 16384 * 16 * 850 + 64 * 528384


def test_decode_algorithmic_bytes():
    w = WORKLOADS["decode_b256"]
    per_unit = 2 * 32 * 2 + 3 * 128 * 2 + 2 + 16 * 128 * 4 * 3 + 16 * 4 * 2
    assert bench.decode_algorithmic_bytes(w) == 256 * 16 * per_unit
    assert abs(bench.decode_algorithmic_bytes(w) / 1e6 - 104.9) < 0.1


def test_weak_scaling_value():
    assert bench.weak_scaling_value(32768, 1, 1.0) == 32768e3
    assert bench.weak_scaling_value(32768, 4, 2.0) == 4 * 32768 / 2e-3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.dist_barrier(world)
        mx = bench.dist_max(1.5 + rank, world)
        q.put((rank, mx, bench.weak_scaling_value(100, world, mx)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.5, 2.5]
    assert all(abs(r[2] - 2 * 100 / 2.5e-3) < 1e-6 for r in res)


def test_reference_arm_prints_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "prefill_1p3b_top16"
