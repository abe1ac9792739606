"""Host-side parts of the benchmark that need no GPU: how many copies of the
K/V caches the timed loop rotates through so that no step is served from L2
by the step before it, and the algorithmic byte count behind every GB/s and
roofline figure, checked against a row-by-row count of what a step reads."""
import bench

L2 = bench.L2_BYTES


def test_one_copy_when_a_step_streams_twice_l2():
    assert bench.l2_replicas(2 * L2, 3 * L2) == 1
    assert bench.l2_replicas(10 * L2, 10 * L2) == 1


def test_enough_copies_to_stream_twice_l2_between_reuses():
    for read in (1, 1000, L2 // 3, L2 - 1, L2, 2 * L2 - 1):
        r = bench.l2_replicas(read, read)
        assert r >= 2 and r * read >= 2 * L2
        assert (r - 1) * read < 2 * L2          # no more copies than needed


def test_copies_capped_by_memory():
    # a window that reads a little of a large cache: copies bounded by the cap
    assert bench.l2_replicas(1 << 20, 8 << 30, cap_bytes=16 << 30) == 2
    assert bench.l2_replicas(1 << 20, 32 << 30, cap_bytes=16 << 30) == 1


def _brute_force_bytes(w, q_len, window):
    """Count, row by row, the K/V rows and block-table entries that at least
    one query row of the step reads; token j of a sequence of n sits at
    position n - q_len + j and sees the positions up to its own, the last
    `window` of them when window > 0."""
    rows, blocks = 0, 0
    for n in w.context_lens.tolist():
        seen = set()
        for j in range(q_len):
            p = n - q_len + j
            first = 0 if window <= 0 else max(0, p - window + 1)
            seen.update(range(first, p + 1))
        rows += len(seen)
        blocks += len({t // w.block_size for t in seen})
    e = w.elem_bytes
    kv = rows * w.num_kv_heads * w.head_dim * 2 * e
    meta = blocks * 4 + w.num_seqs * 4 + (2 * w.num_kv_heads * 4 if w.kv_dtype == "e4m3" else 0)
    qo = 2 * w.num_seqs * q_len * w.num_q_heads * w.head_dim * 2
    return kv, meta, qo


def test_algorithmic_bytes_match_a_row_by_row_count():
    from workloads import make_case
    ctx = [1, 2, 15, 16, 17, 63, 64, 65, 200, 333]
    for dtype in ("bf16", "e4m3"):
        w = make_case(ctx, 8, 2, 128, 16, dtype, seed=3)
        for q_len in (1, 2, 4):
            for window in (0, 1, 5, 16, 17, 100, 1000):
                ab = w.algorithmic_bytes(q_len, window)
                kv, meta, qo = _brute_force_bytes(w, q_len, window)
                assert (ab["kv"], ab["meta"], ab["qo"]) == (kv, meta, qo), (dtype, q_len, window)
                assert ab["decode_total"] == kv + meta + qo


def test_append_payload_bytes():
    from workloads import make_case
    w = make_case([5, 40, 17], 8, 2, 128, 16, "bf16", seed=1, append_last=True)
    n = len(w.slot_mapping)
    # k_new and v_new read, the same rows written into the caches, the slots read
    assert w.algorithmic_bytes()["append"] == 4 * n * 2 * 128 * 2 + 8 * n


def _bench_args_rc(*args):
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args],
                       capture_output=True, text=True, timeout=120)
    return r.returncode, r.stderr


def test_bench_rejects_too_few_warmup_steps():
    rc, err = _bench_args_rc("--warmup", "2")
    assert rc == 2 and "warmup" in err


def test_bench_rejects_kvp_with_other_rows():
    for extra in (["--q-len", "2"], ["--window", "64"], ["--unfused"]):
        rc, err = _bench_args_rc("--kvp", *extra)
        assert rc == 2 and "kvp" in err, extra
