"""KV parallelism on the host: the slice planner (pgd_kvp_plan, a host-only
entry of the C library), the rank-local block table, and the exchange +
merge over a gloo process group of 2 and 3 ranks, with each rank's split
result computed by the oracle so that the whole chain is checked against the
oracle's unsplit decode."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import paged_gqa_decode_07_b200 as pgd
from paged_gqa_decode_07_b200 import kvp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_gqa_decode_07_b200 import build
    build.build()


@pytest.mark.parametrize("W", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bs", [16, 64])
def test_plan_tiles_every_sequence_in_order(W, bs):
    rng = np.random.default_rng(W * 100 + bs)
    ctx = np.concatenate([[0, 1, bs - 1, bs, bs + 1, 3 * bs], rng.integers(0, 20 * bs, 30)])
    ctx = ctx.astype(np.int32)
    plans = [kvp.plan(ctx, bs, W, r) for r in range(W)]
    for s, n in enumerate(ctx):
        nb = -(-int(n) // bs)
        pos = 0
        for r, (start, length) in enumerate(plans):
            # contiguous, block-aligned, in rank order, as even as blocks allow
            assert start[s] == nb * r // W
            if length[s]:
                assert start[s] * bs == pos
            pos += int(length[s])
            blocks = -(-int(length[s]) // bs)
            assert blocks == nb * (r + 1) // W - nb * r // W
        assert pos == n


def test_plan_rejects_bad_arguments():
    with pytest.raises(pgd.PGDError):
        kvp.plan([5, 6], 16, 2, 2)
    with pytest.raises(pgd.PGDError):
        kvp.plan([5, -1], 16, 2, 0)
    with pytest.raises(pgd.PGDError):
        kvp.plan([5], 0, 2, 0)
    s, n = kvp.plan([], 16, 2, 1)
    assert s.size == 0 and n.size == 0


def test_local_block_table_picks_the_slice():
    bt = np.arange(40, dtype=np.int32).reshape(4, 10) + 100
    start = np.array([0, 3, 9, 0], np.int32)
    length = np.array([33, 40, 5, 0], np.int32)
    t = kvp.local_block_table(bt, start, length, 16)
    assert t.shape == (4, 3)
    assert t[0].tolist() == [100, 101, 102]
    assert t[1].tolist() == [113, 114, 115]
    assert t[2, 0] == 129


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _kvp_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from paged_gqa_decode_07_b200 import kvp as K
        from workloads import make_case
        ctx = [1, 40, 333, 1000, 0, 64, 2500]
        w = make_case(ctx, 8, 2, 32 * 4, 16, "bf16", seed=77, name="kvp")
        start, length = K.plan(w.context_lens, w.block_size, world, rank)
        table = K.local_block_table(w.block_table, start, length, w.block_size)
        o, lse = oracle.paged_decode(w.q, w.k_cache, w.v_cache, table, length,
                                     w.num_kv_heads, w.scale)
        rows = w.num_seqs * w.num_q_heads
        o_all = torch.empty((world, rows, w.head_dim), dtype=torch.float64)
        lse_all = torch.empty((world, rows), dtype=torch.float64)
        K.gather_partials(torch.from_numpy(o), torch.from_numpy(lse), o_all, lse_all)
        # the same exchange with each rank's result already in its own slot
        o_in = torch.zeros_like(o_all)
        lse_in = torch.zeros_like(lse_all)
        o_in[rank].copy_(torch.from_numpy(o).reshape(rows, -1))
        lse_in[rank].copy_(torch.from_numpy(lse).reshape(-1))
        K.gather_partials(o_in[rank], lse_in[rank], o_in, lse_in)
        same = bool(torch.equal(o_in, o_all) and torch.equal(lse_in, lse_all))
        merged, mlse = oracle.merge_partials(o_all.numpy(), lse_all.numpy())
        ref, rlse = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table,
                                        w.context_lens, w.num_kv_heads, w.scale)
        err = float(np.max(np.abs(merged - ref.reshape(rows, -1))))
        live = np.isfinite(rlse.reshape(-1))
        lerr = float(np.max(np.abs(mlse[live] - rlse.reshape(-1)[live])))
        dead_ok = same and bool(np.all(np.isneginf(mlse[~live])) and np.all(merged[~live] == 0))
        q.put((rank, err, lerr, dead_ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_kvp_exchange_and_merge_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_kvp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (e, le, d)) for r, e, le, d in (q.get(timeout=180) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        err, lerr, dead_ok = res[r]
        assert err <= 1e-12 and lerr <= 1e-12 and dead_ok, res[r]
