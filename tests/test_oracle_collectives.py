"""Pins of the oracle's reduce-scatter / all-gather / all-reduce and gather
assembly: reduce-scatter followed by all-gather is an all-reduce (the premise
of claim C2, anthology-of-the-sota note 103, "Claims"; "ZeRO: partitioning
training state across GPUs", "How it works"), Nd = 1 is the identity, and the
sum runs in rank order."""
import numpy as np
import pytest

import oracle
from zero_dp_partitioned_shard_b200 import synth


@pytest.mark.parametrize("psi,nd,a", [(1, 1, 1), (7, 3, 1), (257, 4, 8), (1000, 5, 16),
                                      (4097, 16, 256), (50, 64, 1)])
def test_reduce_scatter_then_all_gather_is_all_reduce(psi, nd, a):
    p = oracle.plan(psi, nd, a)
    G = synth.grads_f16(nd, psi, seed=psi * 31 + nd, std=1.0, stride=p.psi_pad)
    shards = oracle.reduce_scatter(G, p)
    full = oracle.all_gather_f32(shards, p)
    ar = oracle.all_reduce(G, psi)
    assert np.array_equal(full.view(np.uint32), ar.view(np.uint32))
    # pads of the reduced shards are zero, not read from the NaN pad region
    for r in range(nd):
        start, n = p.shard(r)
        assert (shards[r, n:] == 0).all()


def test_all_reduce_nd1_is_identity():
    G = synth.grads_f16(1, 999, seed=5, std=3.0)
    assert np.array_equal(oracle.all_reduce(G, 999), G[0].view(np.float16).astype(np.float32))


def test_all_reduce_small_exact_sums_match_fp64():
    # small integers: every partial sum is exact in fp32, so any order agrees
    rs = np.random.default_rng(3)
    vals = rs.integers(-50, 51, size=(8, 500)).astype(np.float16)
    got = oracle.all_reduce(vals.view(np.uint16), 500)
    assert np.array_equal(got, vals.astype(np.float64).sum(axis=0).astype(np.float32))


def test_sum_runs_in_rank_order():
    # rank 0 holds 2^-14, ranks 1 and 2 hold +65504 and -65504.  Left to right
    # from rank 0 the small value is absorbed by 65504 and the result is 0;
    # any order that adds the two large values first keeps 2^-14.
    G = np.array([[2.0 ** -14], [65504.0], [-65504.0]], dtype=np.float16).view(np.uint16)
    assert oracle.all_reduce(G, 1)[0] == 0.0
    G_rev = G[::-1].copy()
    assert oracle.all_reduce(G_rev, 1)[0] == np.float32(2.0 ** -14)
    # a single rank's -0 stays -0 (the sum starts from rank 0's value, not +0)
    z = np.array([[0x8000]], dtype=np.uint16)
    assert oracle.all_reduce(z, 1).view(np.uint32)[0] == 0x80000000


def test_gather_params_rebuilds_the_flat_buffer():
    for psi, nd, a in ((1, 1, 1), (1000, 7, 8), (4097, 4, 256), (10, 16, 1)):
        p = oracle.plan(psi, nd, a)
        ref = synth.fp16_bits(synth.normal_f32(psi, seed=psi, std=1.0))
        shards = []
        for r in range(nd):
            s, n = p.shard(r)
            sh = np.full(p.shard_len, 0x7E00, dtype=np.uint16)  # NaN pad
            sh[:n] = ref[s:s + n]
            shards.append(sh)
        full = np.zeros(psi, dtype=np.uint16)
        oracle.gather_params(shards, p, full)
        assert np.array_equal(full, ref)
        # a NULL shard leaves its range untouched
        full2 = np.full(psi, 0x1234, dtype=np.uint16)
        skip = nd // 2
        oracle.gather_params([None if r == skip else shards[r] for r in range(nd)], p, full2)
        s, n = p.shard(skip)
        assert (full2[s:s + n] == 0x1234).all()
        mask = np.ones(psi, bool)
        mask[s:s + n] = False
        assert np.array_equal(full2[mask], ref[mask])


def test_gather_tensors_equals_slices_of_the_full_gather():
    """Gathering a tensor range (compact or in place) gives exactly the slices
    of the fully gathered buffer; every tensor range together is everything."""
    rs = np.random.default_rng(19)
    for trial in range(25):
        sizes = [int(x) for x in rs.integers(0, 400, size=int(rs.integers(1, 15)))]
        psi = sum(sizes)
        if psi == 0:
            continue
        nd = int(rs.integers(1, 7))
        p = oracle.plan(psi, nd, int(rs.choice([1, 8, 32])))
        ref = synth.fp16_bits(synth.normal_f32(psi, seed=trial, std=1.0))
        shards = []
        for r in range(nd):
            st, n = p.shard(r)
            sh = np.full(p.shard_len, 0x7E00, np.uint16)
            sh[:n] = ref[st:st + n]
            shards.append(sh)
        offs = np.concatenate([[0], np.cumsum(sizes)])
        first = int(rs.integers(0, len(sizes)))
        count = int(rs.integers(0, len(sizes) - first + 1))
        lo, hi = int(offs[first]), int(offs[first + count])
        compact = np.zeros(max(hi - lo, 1), np.uint16)
        assert oracle.gather_tensors(shards, p, sizes, first, count, compact, True) == hi - lo
        assert np.array_equal(compact[:hi - lo], ref[lo:hi])
        full = np.full(psi, 0x1234, np.uint16)
        oracle.gather_tensors(shards, p, sizes, first, count, full, False)
        assert np.array_equal(full[lo:hi], ref[lo:hi])
        assert (full[:lo] == 0x1234).all() and (full[hi:] == 0x1234).all()
        # in place, a missing shard's part is left as it is
        skip = int(rs.integers(0, nd))
        part = np.full(psi, 0x1234, np.uint16)
        n_copied = oracle.gather_tensors([None if r == skip else shards[r] for r in range(nd)], p,
                                         sizes, first, count, part, False)
        s0, n0 = p.shard(skip)
        owned = np.zeros(psi, bool)
        owned[s0:s0 + n0] = True
        inside = np.zeros(psi, bool)
        inside[lo:hi] = True
        assert np.array_equal(part[inside & ~owned], ref[inside & ~owned])
        assert (part[~inside | owned] == 0x1234).all()
        assert n_copied == int((inside & ~owned).sum())
    with pytest.raises(ValueError):
        oracle.gather_tensors([None] * p.nd, p, sizes, 0, len(sizes), np.zeros(psi, np.uint16), True)
