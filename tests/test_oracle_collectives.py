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


# --- reduce-scatter with retention (stage 2): the owner keeps its reduced
# gradient in the 16-bit format ("ZeRO: partitioning training state across
# GPUs", upskillscore.com, "How it works") ---

def _bits16(x32, storage):
    import torch
    if storage == 0:
        return np.asarray(x32, np.float32).astype(np.float16).view(np.uint16)
    t = torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("storage", [0, 1])
def test_retained_shards_of_small_integers_are_the_exact_sums(storage):
    rs = np.random.default_rng(41)
    psi, nd = 1000, 6
    p = oracle.plan(psi, nd, 8)
    vals = rs.integers(-20, 21, size=(nd, p.psi_pad)).astype(np.float32)   # every sum exact in 16 bits
    G = np.stack([_bits16(v, storage) for v in vals])
    got = oracle.reduce_scatter16(G, p, storage)
    exact = vals[:, :psi].astype(np.float64).sum(axis=0)
    for o in range(nd):
        s, n = p.shard(o)
        assert np.array_equal(got[o, :n], _bits16(exact[s:s + n], storage))
        assert (got[o, n:] == 0xFFFF).all()                  # pads are never written


@pytest.mark.parametrize("storage", [0, 1])
def test_retained_shards_are_the_fp32_shards_rounded_once(storage):
    psi, nd = 4097, 5
    p = oracle.plan(psi, nd, 16)
    if storage == 0:
        G = synth.grads_f16(nd, psi, seed=43, std=3.0, stride=p.psi_pad)
    else:
        G = synth.grads_bf16(nd, psi, seed=43, std=3.0, stride=p.psi_pad)
    got = oracle.reduce_scatter16(G, p, storage)
    if storage == 0:
        f32 = oracle.reduce_scatter(G, p)                    # pinned above, fp16 contributions
    else:
        f32 = np.zeros((nd, p.shard_len), np.float32)        # bf16 contributions widen exactly
        wide = oracle.bf16_to_float(G)
        acc = wide[0].copy()
        for r in range(1, nd):
            acc = (acc + wide[r]).astype(np.float32)
        for o in range(nd):
            s, n = p.shard(o)
            f32[o, :n] = acc[s:s + n]
    for o in range(nd):
        s, n = p.shard(o)
        assert np.array_equal(got[o, :n], _bits16(f32[o, :n], storage))


def test_retention_keeps_rank_order_and_overflows_in_fp16():
    p = oracle.plan(2, 1, 1)
    # rank order decides before the rounding: 2^-14 is absorbed left to right
    G = np.array([[2.0 ** -14] * 2, [65504.0] * 2, [-65504.0] * 2], dtype=np.float16).view(np.uint16)
    p3 = oracle.plan(2, 3, 1)
    got = oracle.reduce_scatter16(G, p3, 0)
    assert got[0, 0] == 0x0000 and got[1, 0] == 0x0000
    got_rev = oracle.reduce_scatter16(np.ascontiguousarray(G[::-1]), p3, 0)
    assert got_rev[0, 0] == 0x0400                           # 2^-14 survives the other order
    # a sum beyond 65504 is +inf in fp16 but finite in bf16
    G2 = np.array([[60000.0, 1.0], [60000.0, 1.0]], dtype=np.float32)
    p2 = oracle.plan(2, 2, 1)
    assert oracle.reduce_scatter16(G2.astype(np.float16).view(np.uint16), p2, 0)[0, 0] == 0x7C00
    b = oracle.reduce_scatter16(_bits16(G2, 1), p2, 1)[0, 0]
    assert b == _bits16(np.float32(_bits16_to_f32(_bits16(G2[0, :1], 1)[0]) * 2), 1)[0]
    assert oracle.reduce_scatter16(np.array([[0x3C00, 0x3C00]], np.uint16), p, 0)[0, 0] == 0x3C00  # Nd = 1


def _bits16_to_f32(b):
    return np.array([int(b) << 16], np.uint32).view(np.float32)[0]


def test_retention_writes_only_the_requested_range():
    psi, nd = 3001, 4
    p = oracle.plan(psi, nd, 8, 700)
    G = synth.grads_f16(nd, psi, seed=44, std=1.0, stride=p.psi_pad)
    full = oracle.reduce_scatter16(G, p, 0)
    part = np.full((nd, p.shard_len), 0x1234, np.uint16)
    b0, bn = p.bucket_range(2)
    lo, hi = b0, b0 + bn
    oracle.reduce_scatter16(G, p, 0, lo, hi, out=part)
    for o in range(nd):
        s, n = p.shard(o)
        idx = np.arange(s, s + n)
        inside = (idx >= lo) & (idx < hi)
        assert np.array_equal(part[o, :n][inside], full[o, :n][inside])
        assert (part[o, :n][~inside] == 0x1234).all() and (part[o, n:] == 0x1234).all()
    # bucket by bucket covers the same as everything at once
    acc = np.full((nd, p.shard_len), 0xFFFF, np.uint16)
    for k in range(p.n_buckets):
        b0, bn = p.bucket_range(k)
        oracle.reduce_scatter16(G, p, 0, b0, b0 + bn, out=acc)
    assert np.array_equal(acc, full)


@pytest.mark.parametrize("storage", [0, 1])
def test_step_from_retained_shards_equals_the_direct_step_when_exact(storage):
    """When every reduced value is exact in 16 bits, the step on the owners'
    retained gradients (one contribution each) is the direct step bit for bit."""
    rs = np.random.default_rng(45)
    psi, nd = 20_011, 4
    p = oracle.plan(psi, nd, 8)
    vals = rs.integers(-16, 17, size=(nd, p.psi_pad)).astype(np.float32) * np.float32(2.0 ** -6)
    G = np.stack([_bits16(v, storage) for v in vals])
    retained = oracle.reduce_scatter16(G, p, storage)
    flat = np.concatenate([retained[o, :p.shard(o)[1]] for o in range(nd)])[None, :]
    hp = oracle.HP(loss_scale=64.0, weight_decay=0.01, storage=storage)
    master = synth.normal_f32(psi, seed=46, std=0.02)
    runs = []
    for g in (np.ascontiguousarray(G[:, :psi]), flat):
        st = [master.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32),
              np.zeros(psi, np.uint16), oracle.Opt()]
        for _ in range(2):
            oracle.step(g, st[0], st[1], st[2], st[3], hp, st[4])
        runs.append(st)
    for a, b in zip(runs[0][:3], runs[1][:3]):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(runs[0][3], runs[1][3])
