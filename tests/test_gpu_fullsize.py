"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: every owned element is updated by the CUDA path, and a seeded
sample of elements (random positions plus every shard / bucket / vector
boundary) is recomputed by the oracle one by one from the exact device input
bytes.  Global properties (overflow flag, skip, the fp64 norm) are checked at
any size."""
import math
import sys
import os
import concurrent.futures as cf

import numpy as np
import pytest
import torch

import oracle
from _util import assert_bf16_close, assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402  (the benchmark's own workload setup)


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.empty_cache()


def _sample_positions(lo, hi, L, bucket, n_random, seed):
    """Relative positions in [0, hi - lo): random, plus shard, bucket and
    8-element-vector boundaries."""
    rs = np.random.default_rng(seed)
    n = hi - lo
    pos = set(rs.integers(0, n, size=n_random).tolist())
    for b in range(lo, hi + 1, L):
        for d in range(-9, 10):
            pos.add(b - lo + d)
    if bucket:
        for b in range((lo // bucket) * bucket, hi + 1, bucket):
            for d in (-1, 0, 1, 7, 8):
                pos.add(b - lo + d)
    for d in range(1, 20):
        pos.add(n - d)
        pos.add(d - 1)
    return np.array(sorted(p for p in pos if 0 <= p < n), dtype=np.int64)


def _gather_inputs(bn, pos):
    """Device input bytes at sampled positions: grads [nd, k] and state."""
    idx = torch.from_numpy(pos).cuda()
    if bn.wl["layout"] == B.ZERO_GRADS_FULL:
        flat = idx + bn.o0 * bn.L
        G = torch.stack([bn.grads[r * bn.stride + flat] for r in range(bn.nd)])
    else:
        k, i = idx // bn.L, idx % bn.L
        G = torch.stack([bn.grads[(k * bn.nd + r) * bn.stride + i] for r in range(bn.nd)])
    return G.view(torch.int16).cpu().numpy().view(np.uint16), idx


def _state_at(bn, idx, slot):
    t = lambda x: x[idx].cpu().numpy()
    return t(bn.master[slot]), t(bn.exp_avg[slot]), t(bn.exp_avg_sq[slot])


def _params_at(bn, idx):
    return bn.params.view(torch.int16)[idx + bn.o0 * bn.L].cpu().numpy().view(np.uint16)


def _opt(bn):
    return B.opt_state_from_bytes(bn.opt_state.cpu().numpy().tobytes())


def _kept_of(G, storage):
    """The oracle's retained 16-bit reduction of sampled columns G [nd, k]."""
    nd, k = G.shape
    p = oracle.plan(k, nd, 1)
    kept = oracle.reduce_scatter16(G, p, storage)
    return np.concatenate([kept[o, :p.shard(o)[1]] for o in range(nd)])


def _check_sampled_steps(bn, steps, n_random, seed, clip_from_gpu=False):
    lo, hi = bn.o0 * bn.L, bn.o0 * bn.L + bn.owned
    pos = _sample_positions(lo, hi, bn.L, bn.wl["bucket"], n_random, seed)
    G, idx = _gather_inputs(bn, pos)
    if bn.kept is not None:            # retention: the step reads the kept reduction
        G = _kept_of(G, bn.storage)[None, :]
    spec = bn.wl["mode"] == B.ZERO_MODE_SPECULATIVE
    slot = _opt(bn).cur if spec else 0
    master, m, v = _state_at(bn, idx, slot)
    P = _params_at(bn, idx)
    hp = oracle.HP(lr=bn.hp.lr, beta1=bn.hp.beta1, beta2=bn.hp.beta2, eps=bn.hp.eps,
                   weight_decay=bn.hp.weight_decay, loss_scale=bn.hp.loss_scale,
                   max_grad_norm=bn.hp.max_grad_norm, storage=bn.storage)
    opt = oracle.Opt(*(lambda o: (o.t, o.beta1_pow, o.beta2_pow))(_opt(bn)))
    results = []
    for _ in range(steps):
        bn.step()
        res = B.step_result_from_bytes(bn.result.cpu().numpy().tobytes())
        results.append(res)
        assert res.overflow == 0
        _, _, bc1, bc2 = oracle.bias_corrections(hp, opt)
        c = res.clip_coef if clip_from_gpu else 1.0
        oracle.update_elements(G, master, m, v, P, hp, c, bc1, bc2, threads=oracle.host_threads())
        b1, b2, _, _ = oracle.bias_corrections(hp, opt)
        opt = oracle.Opt(opt.t + 1, b1, b2)
    torch.cuda.synchronize()
    slot = _opt(bn).cur if spec else 0
    gm, ga, gv = _state_at(bn, idx, slot)
    assert_f32_close(gm, master, 2, "master")
    assert_f32_close(ga, m, 2, "exp_avg")
    assert_f32_close(gv, v, 2, "exp_avg_sq")
    close16 = assert_bf16_close if bn.storage == B.ZERO_STORAGE_BF16 else assert_f16_close
    close16(_params_at(bn, idx), P, 1, "params")
    for d, dst in enumerate(bn.dests):   # peer tables: every rank's buffer holds the same parameters
        got = dst.view(torch.int16)[idx + bn.o0 * bn.L].cpu().numpy().view(np.uint16)
        assert np.array_equal(got, _params_at(bn, idx)), f"destination {d}"
    assert _opt(bn).t == opt.t
    return results


def _wl(name, **over):
    wl = dict(bench._workloads()[name])
    wl.update(over)
    return wl


def test_gpt2_1p5b_stage2_nd8_speculative_sampled():
    """The benchmark workload: 1,557,611,200 params, Nd = 8, 2 steps."""
    bn = bench.Bench(_wl("gpt2-1.5b-stage2-nd8"), None, seed=3)
    try:
        assert bn.owned == 1_557_611_200 and bn.L == 194_701_568
        _check_sampled_steps(bn, steps=2, n_random=1 << 20, seed=1)
        # an inf anywhere in any rank skips the whole step: sampled state,
        # sampled parameters and the step counter are unchanged
        pos = np.array([0, 12345, 194_701_567, 1_557_611_199], dtype=np.int64)
        idx = torch.from_numpy(pos).cuda()
        slot = _opt(bn).cur
        before = _state_at(bn, idx, slot), _params_at(bn, idx), _opt(bn).t
        bn.grads[5 * bn.stride + 987_654_321] = float("inf")
        bn.step()
        res = B.step_result_from_bytes(bn.result.cpu().numpy().tobytes())
        assert res.overflow == 1 and _opt(bn).t == before[2] and _opt(bn).skipped == 1
        after = _state_at(bn, idx, _opt(bn).cur), _params_at(bn, idx)
        for a, b in zip(before[0], after[0]):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        assert np.array_equal(before[1], after[1])
    finally:
        bn.close()


def test_gpt2_1p5b_bf16_storage_sampled():
    """The benchmark workload with bfloat16 gradients and parameters."""
    bn = bench.Bench(_wl("gpt2-1.5b-stage2-nd8"), None, seed=6, storage=B.ZERO_STORAGE_BF16)
    try:
        assert bn.grads.dtype == torch.bfloat16
        _check_sampled_steps(bn, steps=2, n_random=1 << 19, seed=6)
    finally:
        bn.close()


def test_gpt2_1p5b_peer_tables_sampled():
    """The benchmark workload through peer tables (bench --peer): the rank
    contributions read through the table, every new parameter stored into all
    8 ranks' buffers; each buffer checked at the sampled positions."""
    bn = bench.Bench(_wl("gpt2-1.5b-stage2-nd8"), None, seed=7, peer=True)
    try:
        assert len(bn.dests) == 7
        _check_sampled_steps(bn, steps=2, n_random=1 << 19, seed=7)
    finally:
        bn.close()


def test_gpt2_1p5b_retention_sampled():
    """The benchmark workload with stage-2 retention (bench --retain): the kept
    fp16 reduction equals the oracle's bit for bit at the sampled positions,
    and the step on it matches the oracle's step on the same kept values."""
    bn = bench.Bench(_wl("gpt2-1.5b-stage2-nd8"), None, seed=8, retain=True)
    try:
        _check_sampled_steps(bn, steps=2, n_random=1 << 19, seed=8)
        pos = _sample_positions(0, bn.owned, bn.L, bn.wl["bucket"], 1 << 18, 9)
        G, idx = _gather_inputs(bn, pos)
        got = bn.kept.view(torch.int16)[idx].cpu().numpy().view(np.uint16)
        assert np.array_equal(got, _kept_of(G, bn.storage))
    finally:
        bn.close()


@pytest.mark.parametrize("owner,align", [(0, 256), (63, 256), (0, 1)])
def test_7p5b_nd64_stage3_owner_view_sampled(owner, align):
    """One rank of 7.5B params at Nd = 64: the owner's shard (L = 117,187,584;
    owner 63 holds the short 117,182,208; A = 1 gives L = 117,187,500 and the
    scalar path) with 64 contributions."""
    bn = bench.Bench(_wl("7.5b-nd64-stage3-owner0", owner_first=owner, align=align), None, seed=4)
    try:
        want_L = 117_187_584 if align == 256 else 117_187_500
        assert bn.L == want_L
        if owner == 63:
            assert bn.owned == 7_500_000_000 - 63 * want_L
        _check_sampled_steps(bn, steps=1, n_random=1 << 18, seed=2)
    finally:
        bn.close()


def test_7p5b_gather_assembly_sampled_windows():
    """Assemble the full 7.5B fp16 buffer from 64 seeded shards (owner 0's own
    shard already in place); compare seeded 1M-element windows with the
    oracle's gather of the same shard bytes."""
    from zero_dp_partitioned_shard_b200 import synth
    psi, nd = 7_500_000_000, 64
    p = oracle.plan(psi, nd, 256)
    L = p.shard_len
    full = torch.empty(psi, dtype=torch.float16, device="cuda")
    full.fill_(float("nan"))
    shards = torch.empty(nd - 1, L, dtype=torch.float16, device="cuda")
    for r in range(1, nd):
        synth.fill_normal_(shards[r - 1], seed=7000 + r, std=0.02)
    ptrs = [0] + [shards[r - 1].data_ptr() for r in range(1, nd)]
    plan = B.zero_plan(psi, nd, stage=3, align_elems=256)
    try:
        B.zero_gather_params(plan, ptrs, full.data_ptr(), torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
    finally:
        B.zero_plan_destroy(plan)
    rs = np.random.default_rng(5)
    starts = list(rs.integers(L, psi - (1 << 20), size=6)) + [L - 10, 63 * L - 100, psi - (1 << 20)]
    for s in starts:
        s = int(max(L, s))
        e = min(psi, s + (1 << 20))
        want = np.zeros(e - s, np.uint16)
        got = full[s:e].view(torch.int16).cpu().numpy().view(np.uint16)
        # oracle gather restricted to the window: full[r*L + i] = shard_r[i]
        for r in range(s // L, (e - 1) // L + 1):
            a, b = max(s, r * L), min(e, r * L + p.shard(r)[1])
            if a >= b or r == 0:
                continue
            sh = shards[r - 1][a - r * L:b - r * L].view(torch.int16).cpu().numpy().view(np.uint16)
            want[a - s:b - s] = sh
        mask = np.ones(e - s, bool)
        if s < L:
            mask[:L - s] = False   # owner 0's range: not gathered, left untouched
        assert np.array_equal(got[mask], want[mask])
    # owner 0's range was not written
    assert torch.isnan(full[:L]).all().item()
    del shards, full


def _streamed_oracle_norm(bn, hp, chunk=1 << 24):
    """Oracle fp64 sum of squares over all owned elements, chunk by chunk from
    the device bytes: each chunk's compensated sum keeps its compensation term,
    and all the chunks' terms are added exactly (math.fsum)."""
    starts = list(range(0, bn.owned, chunk))
    workers = oracle.host_threads()
    parts = []

    def load(s):
        e = min(bn.owned, s + chunk)
        G = torch.stack([bn.grads[r * bn.stride + s:r * bn.stride + e] for r in range(bn.nd)])
        return G.view(torch.int16).cpu().numpy().view(np.uint16)

    def chunk_sumsq(G):
        acc = np.zeros(2, np.float64)
        _, bad = oracle.grad_sumsq(G, hp, acc)
        return acc, bad

    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        for w in range(0, len(starts), workers):   # bounded host memory: one wave at a time
            wave = [load(s) for s in starts[w:w + workers]]
            parts += list(ex.map(chunk_sumsq, wave))
    total = math.fsum(x for acc, _ in parts for x in acc)
    return math.sqrt(total), any(b for _, b in parts)


def test_24l_d2048_nd16_bucketed_clip_stash_sampled_with_injection():
    """1,315,723,264 params, Nd = 16, 53 buckets of 25M, clip at 1.0, stash
    mode, with a seeded injection schedule that forces a skip."""
    from zero_dp_partitioned_shard_b200 import synth
    wl = _wl("24l-d2048-stage2-nd16-clip")
    bn = bench.Bench(wl, None, seed=5)
    try:
        assert bn.L == 82_232_832 and B.zero_plan_query(bn.plan).n_buckets == 53
        hp = oracle.HP(loss_scale=wl["S"], max_grad_norm=wl["clip"])
        # step 1: the norm of the full gradient against the streamed oracle
        ref_norm, bad = _streamed_oracle_norm(bn, hp)
        assert not bad
        res = _check_sampled_steps(bn, steps=1, n_random=1 << 18, seed=3, clip_from_gpu=True)
        assert res[0].grad_norm == pytest.approx(ref_norm, rel=1e-12)
        want_c = np.float32(wl["clip"] / ref_norm) if ref_norm > wl["clip"] else np.float32(1.0)
        assert abs(res[0].clip_coef - want_c) <= np.spacing(want_c)
        # seeded schedule (1 % of steps, step 1 forced): a skipped step then
        # a normal one, again against the oracle on sampled elements
        sched = synth.inject_schedule(4, 0.01, seed=11, nd=bn.nd, psi=bn.psi, force_step=1)
        assert 1 in sched
        t_before = _opt(bn).t
        for s in range(1, 4):
            if s in sched:
                rank, i, val = sched[s]
                saved = bn.grads[rank * bn.stride + i].clone()
                bn.grads[rank * bn.stride + i] = val
                bn.step()
                r = B.step_result_from_bytes(bn.result.cpu().numpy().tobytes())
                assert r.overflow == 1 and math.isnan(r.grad_norm)
                bn.grads[rank * bn.stride + i] = saved
            else:
                _check_sampled_steps(bn, steps=1, n_random=1 << 16, seed=10 + s, clip_from_gpu=True)
        assert _opt(bn).skipped == len([s for s in sched if 1 <= s < 4])
        assert _opt(bn).t == t_before + 3 - _opt(bn).skipped
    finally:
        bn.close()


@pytest.mark.parametrize("psi", [1 << 20, 16 << 20])
@pytest.mark.parametrize("nd", [1, 2, 8, 64])
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_sweep_points_full_parity(psi, nd, stage):
    """Sweep workloads small enough for the oracle to recompute every element."""
    if psi == 16 << 20 and nd == 64 and stage != 3:
        pytest.skip("covered by the stage-3 layout at this size")
    from _gpu import make_problem, run_gpu, run_oracle, to_oracle_hp
    pb = make_problem(psi, nd, align=256, bucket=(4 << 20) if stage == 2 else 0, steps=1,
                      seed=nd + stage, S=1.0)
    hp = B.hparams(loss_scale=1.0)
    g = run_gpu(pb, hp, layout=B.ZERO_GRADS_PER_OWNER if stage == 3 else B.ZERO_GRADS_FULL,
                stage=stage)
    o = run_oracle(pb, to_oracle_hp(hp), threads=oracle.host_threads())
    assert_f32_close(g.master, o.master, 2, "master")
    assert_f32_close(g.exp_avg, o.exp_avg, 2, "exp_avg")
    assert_f32_close(g.exp_avg_sq, o.exp_avg_sq, 2, "exp_avg_sq")
    assert_f16_close(g.params, o.params, 1, "params")
    assert [r.overflow for r in g.results] == [i["overflow"] for i in o.infos] == [0]
    assert g.opt.t == o.opt.t == 1 and g.results[-1].t == 1


@pytest.mark.parametrize("psi,nd,stage,mode", [
    (256 << 20, 1, 1, 0),      # Nd <= 2: the low-byte streams
    (256 << 20, 2, 2, 0),      # ... in 8 buckets
    (1 << 30, 64, 3, 0),       # one owner of 64 at 1B (the one-owner view)
    (64 << 20, 16, 1, 0),      # the pipelined update at its largest Nd
    (64 << 20, 16, 2, 1),      # ... re-reducing in place after a clipped statistics pass
    (48 << 20, 4, 3, 0),       # ... at Nd = 4, per-owner layout
    (27 << 20, 8, 1, 0),       # below the size from which Nd = 8 takes the pipeline (64 tiles per CTA)
    ((40 << 20) + 1000, 32, 1, 0),  # rank rows by 2-D tensor-map boxes; the last box overhangs the data
    ((40 << 20) + 1000, 24, 2, 1),  # ... Nd not a power of two, 8 buckets, clipped two-pass in place
    ((40 << 20) + 1000, 64, 3, 0),  # ... per-owner layout, all 64 owners (box rows = owner x 64 + rank)
])
def test_sweep_points_large_sampled(psi, nd, stage, mode):
    """The sweep's large points in the configuration the sweep times, and the
    kernel choices around them: every owned element is updated on the GPU,
    sampled elements (random plus every shard, bucket and vector boundary) are
    recomputed by the oracle from the device bytes over two steps."""
    free, _ = torch.cuda.mem_get_info()
    wl = bench.sweep_workload(psi, nd, stage, free, mode)
    if psi >= 1 << 30:
        assert (wl["owner_count"] == 1) == (nd == 64)   # 1B at Nd = 64 only fits as one owner's view
    bn = bench.Bench(wl, None, seed=11 + nd)
    try:
        res = _check_sampled_steps(bn, steps=2, n_random=1 << 19, seed=nd + stage, clip_from_gpu=mode != 0)
        assert [r.overflow for r in res] == [0, 0] and res[-1].t == 2
    finally:
        bn.close()
