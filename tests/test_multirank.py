"""Host-side logic of the N > 1 bench path, on CPU with the gloo backend
(world size 2): every rank runs its own batch of the same shape, the job's
value is the bytes all ranks moved divided by the slowest rank's time, and
the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        r = bench.reduce_over_ranks(step_bytes=1000 + rank, ms_step=1.0 + rank,
                                    e2e_ms=2.0 + 3 * rank, dec_ms=0.5 + rank, world=world)
        q.put((rank, r))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        r = res[rank]
        assert r["ms_step"] == 2.0 and r["e2e_ms"] == 5.0 and r["dec_ms"] == 1.5
        assert r["total_bytes"] == 2001.0
        assert r["value"] == pytest.approx(2001.0 / 2.0e-3 / 1e9)
        assert r["e2e_value"] == pytest.approx(2001.0 / 5.0e-3 / 1e9)


def test_reduce_single_rank_is_plain_division():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.reduce_over_ranks(500, 2.0, 4.0, 1.0, world=1)
    assert r["value"] == pytest.approx(500 / 2.0e-3 / 1e9) and r["ms_step"] == 2.0


def test_replicas_share_shape_not_values():
    from workloads import make_workload
    a = make_workload("tiny", seed=0, shape_seed=0)
    b = make_workload("tiny", seed=1, shape_seed=0)
    assert np.array_equal(a.context_lens, b.context_lens)
    assert a.algorithmic_bytes() == b.algorithmic_bytes()
    assert not np.array_equal(a.q, b.q)
    c = make_workload("llama3_8b_decode", seed=1, shape_seed=0)
    d = make_workload("llama3_8b_decode", seed=0)
    assert np.array_equal(c.context_lens, d.context_lens)


def test_reference_arm_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
