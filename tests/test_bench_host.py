"""Host-side choices of the benchmark that need no GPU: how many copies of
the K/V caches the timed loop rotates through so that no step is served from
L2 by the step before it."""
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
