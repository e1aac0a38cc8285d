"""Pins of the oracle's partition planner: brute-force properties on small
inputs and shard lengths worked out by hand for the named workloads."""
import numpy as np
import pytest

import oracle
from zero_dp_partitioned_shard_b200 import synth


def _check_plan(psi, nd, a):
    p = oracle.plan(psi, nd, a)
    L = p.shard_len
    assert L % a == 0 and L >= a
    assert p.psi_pad == nd * L and p.psi_pad >= psi
    # L is the smallest multiple of A whose Nd copies cover Psi
    assert (L - a) * nd < psi
    owner = np.full(psi, -1, dtype=np.int64)
    prev_end = 0
    for r in range(nd):
        start, n = p.shard(r)
        assert start == r * L and start % a == 0
        assert 0 <= n <= L
        if n:
            assert start == prev_end, "shards must be contiguous and in rank order"
            assert (owner[start:start + n] == -1).all(), "shards overlap"
            owner[start:start + n] = r
            prev_end = start + n
        # only the last non-empty shard may be short
        if 0 < n < L:
            assert start + n == psi
    assert (owner >= 0).all(), "shards do not cover [0, psi)"
    # brute force: the owner of flat index i is i // L
    assert np.array_equal(owner, np.arange(psi) // L)


@pytest.mark.parametrize("a", [1, 8, 256])
def test_planner_properties_bruteforce(a):
    rs = np.random.default_rng(a)
    psis = sorted(set([1, 2, 3, 7, 8, 9, 255, 256, 257, 4095, 4096, 4097, 5000]
                      + list(rs.integers(1, 5001, size=40))))
    for psi in psis:
        for nd in range(1, 18):
            _check_plan(int(psi), nd, a)


def test_named_workload_shard_lengths_by_hand():
    # 1,000,003 params over 4 ranks at A = 256: ceil(1,000,003 / 1024) = 977
    # units of 256 -> L = 250,112; the last shard holds 1,000,003 - 3 * 250,112
    # = 249,667 real elements and 445 pad
    p = oracle.plan(1_000_003, 4, 256)
    assert (p.shard_len, p.psi_pad) == (250_112, 1_000_448)
    assert p.shard(3) == (750_336, 249_667)
    assert p.shard_len - p.shard(3)[1] == 445
    # GPT-2 1.5B (1,557,611,200 params), Nd = 8: 760,553 units of 256
    p = oracle.plan(1_557_611_200, 8, 256)
    assert p.shard_len == 194_701_568 and p.shard(7)[1] == 194_700_224
    # 7.5B over 64: ceil(7.5e9 / 64) = 117,187,500 unaligned, 117,187,584 at 256
    assert oracle.plan(7_500_000_000, 64, 1).shard_len == 117_187_500
    p = oracle.plan(7_500_000_000, 64, 256)
    assert p.shard_len == 117_187_584 and p.shard(63)[1] == 117_182_208
    # 24-layer d = 2048 transformer (1,315,723,264 params), Nd = 16, 25M buckets
    p = oracle.plan(1_315_723_264, 16, 256, 25_000_000)
    assert p.shard_len == 82_232_832 and p.n_buckets == 53
    assert p.bucket_range(52) == (1_300_000_000, 15_723_264)


def test_workload_parameter_counts():
    assert sum(synth.gpt2_xl_tensor_sizes()) == 1_557_611_200
    assert sum(synth.transformer_24l_d2048_tensor_sizes()) == 1_315_723_264


def test_buckets_tile_the_flat_buffer():
    for psi, b in ((1000, 1), (1000, 7), (1000, 1000), (1000, 4096), (12345, 100)):
        p = oracle.plan(psi, 3, 8, b)
        covered = 0
        for k in range(p.n_buckets):
            s, n = p.bucket_range(k)
            assert s == covered and n > 0
            covered += n
        assert covered == psi
    assert oracle.plan(1000, 3, 8, 0).bucket_range(0) == (0, 1000)


def _segments_bruteforce(sizes, L):
    """Element by element: which owner holds each element of each tensor."""
    segs = []
    off = 0
    for t, n in enumerate(sizes):
        for j in range(n):
            flat = off + j
            o = flat // L
            if segs and segs[-1][0] == t and segs[-1][1] == o and segs[-1][2] + segs[-1][3] == j:
                segs[-1][3] += 1
            else:
                segs.append([t, o, j, 1, flat - o * L])
        off += n
    return segs


def test_tensor_segments_bruteforce():
    rs = np.random.default_rng(7)
    for trial in range(60):
        sizes = list(rs.integers(0, 300, size=int(rs.integers(1, 12))))
        psi = int(sum(sizes))
        if psi == 0:
            continue
        nd = int(rs.integers(1, 9))
        a = int(rs.choice([1, 4, 16]))
        p = oracle.plan(psi, nd, a)
        got = p.tensor_segments(sizes).tolist()
        assert got == _segments_bruteforce(sizes, p.shard_len), (sizes, nd, a)


def test_tensor_segments_of_24l_d2048_straddle_owners():
    sizes = synth.transformer_24l_d2048_tensor_sizes()
    p = oracle.plan(sum(sizes), 16, 256)
    segs = p.tensor_segments(sizes)
    # every tensor is covered exactly once, in order
    for t, n in enumerate(sizes):
        mine = segs[segs[:, 0] == t]
        assert mine[:, 3].sum() == n
        assert (mine[:, 2] == np.concatenate([[0], np.cumsum(mine[:, 3])[:-1]])).all()
    # each owner's pieces tile [0, real_len) of its shard
    for o in range(16):
        mine = segs[segs[:, 1] == o]
        assert mine[:, 3].sum() == p.shard(o)[1]
    # some tensors straddle an owner boundary
    per_tensor = np.bincount(segs[:, 0])
    assert (per_tensor > 1).sum() >= 15


def test_plan_rejects_bad_arguments():
    for args in ((0, 1, 1), (5, 0, 1), (5, 1, 0), (5, 1, 1, -1)):
        with pytest.raises(ValueError):
            oracle.plan(*args)
    with pytest.raises(ValueError):
        oracle.plan(10, 2, 1).tensor_segments([3, 3])
