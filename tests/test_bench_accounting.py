"""The bench's closed-form work counts (FLOPs and bytes behind every roofline
figure) agree with the oracle's counts and with values worked out by hand."""
import bench
from oracle import hca_oracle as O


def test_nc_matches_visibility_rule():
    # entry j is visible from position t once its whole block lies outside the
    # window: nc(t) = max(0, floor((t - 127) / 128))
    assert [bench.nc_of(t) for t in (0, 126, 127, 254, 255, 382, 383)] == [0, 0, 0, 0, 1, 1, 2]
    for t in range(0, 2000, 37):
        assert bench.nc_of(t) == O.num_visible_blocks(t)


def test_visited_pairs_agree_with_oracle():
    for T in (1, 127, 128, 129, 255, 256, 1000, 4096):
        assert bench.visited_pairs(T) == O.visited_pairs(T)
    # T = 256: every position sees min(t + 1, 128) raw keys, only t = 255
    # also sees one compressed entry
    assert bench.visited_pairs(256) == sum(min(t + 1, 128) for t in range(256)) + 1


def test_prefill_bytes_32k():
    # q, g, out: 3 x T x 64 x 512 bf16; k, v: 2 x T x 512; cK, cV: 2 x 256 x 512;
    # s: T -- all bf16 (2 bytes)
    T = 32768
    by_hand = 2 * (3 * T * 64 * 512 + 2 * T * 512 + 2 * (T // 128) * 512 + T)
    assert bench.prefill_bytes(1, T) == by_hand == 6510149632


def test_decode_cache_keys():
    assert bench.decode_cache_keys([1]) == 1
    assert bench.decode_cache_keys([128]) == 128
    assert bench.decode_cache_keys([255]) == 128
    assert bench.decode_cache_keys([256]) == 129
    assert bench.decode_cache_keys([131072]) == 1023 + 128
    lens = [78841, 921936, 130194, 1, 300]
    assert bench.decode_cache_keys(lens) == O.decode_keys(lens)


def test_flops_per_pair():
    # per visited (query, key) pair and head: q.k (512 multiply-adds) and
    # p.v (512 multiply-adds), 2 FLOPs each, 64 heads
    assert bench.FLOP_PER_PAIR == 64 * (2 * 512 + 2 * 512)
    # the two prefill workloads' totals quoted beside the bench numbers
    assert round(bench.visited_pairs(32768) * bench.FLOP_PER_PAIR / 1e12, 3) == 1.092
    assert round(bench.visited_pairs(131072) * bench.FLOP_PER_PAIR / 1e13, 3) == 1.097


def test_compress_bytes():
    # per complete block: K and V rows (2 x 128 x 512 bf16), the 128 scores,
    # and the two 512-wide entries written
    assert bench.compress_bytes(1, 131072) == 1024 * (2 * 128 * 512 * 2 + 128 * 2 + 2 * 512 * 2)
    assert bench.compress_bytes(1, 131072) == 1024 * 264448
    assert bench.compress_bytes(2, 300) == 2 * 2 * 264448    # the ragged tail is not read


def test_backward_accounting():
    """Five pair-GEMMs (S, dP, dq, dk, dv) against the forward's two; the
    design's least bytes at T = 131072 (10 activations + 5 passes over P/dS)."""
    import bench
    T = 131072
    pairs = bench.visited_pairs(T)
    assert 5 * pairs * bench.FLOP_PER_PAIR // 2 == 5 * pairs * 64 * 512 * 2
    act = T * 64 * 512 * 2
    assert bench.backward_bytes(1, T) == 10 * act + 5 * pairs * 64 * 2 + 2 * T * 512 * 4


def test_backward_child_failure_is_reported_not_raised_into_the_line():
    """The backward measurement's child process, run where it cannot succeed
    (no GPU here), surfaces as an exception naming its exit code, which the
    parent records under side_errors instead of losing the line."""
    import types
    import pytest
    import torch
    import bench
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError, match="backward child exited"):
        bench.run_backward_child(types.SimpleNamespace(side_steps=4))
