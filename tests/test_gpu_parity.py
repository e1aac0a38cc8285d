"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element
by element, at sizes the oracle finishes in seconds.  Bars: master, momentum
and variance within 2 fp32 ulp, fp16 parameters within 1 fp16 ulp, overflow
flag, step counter, padding and untouched regions exact; global norm within
1e-12 relative (both fp64, only the summation order differs)."""
import math

import numpy as np
import pytest
import torch

import oracle
from _gpu import (INF16, PARAM_SENTINEL, dev, host, kernels_launched, make_problem, run_gpu, run_oracle,
                  to_oracle_hp)
from _util import assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import synth

pytestmark = pytest.mark.gpu

MODES = [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH]
MODE_NAMES = {0: "speculative", 1: "two_pass", 2: "stash"}


def compare(g, o, what="", norm_rel=1e-12):
    assert_f32_close(g.master, o.master, 2, what + " master")
    assert_f32_close(g.exp_avg, o.exp_avg, 2, what + " exp_avg")
    assert_f32_close(g.exp_avg_sq, o.exp_avg_sq, 2, what + " exp_avg_sq")
    assert_f16_close(g.params, o.params, 1, what + " params")
    assert len(g.results) == len(o.infos)
    for r, info in zip(g.results, o.infos):
        assert r.overflow == info["overflow"], what
        if info["overflow"] == 0 and "grad_norm" in info and not math.isnan(r.grad_norm):
            assert r.grad_norm == pytest.approx(info["grad_norm"], rel=norm_rel, abs=1e-300), what
    assert g.opt.t == o.opt.t, what
    assert g.opt.skipped == sum(i["overflow"] for i in o.infos), what


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_tiny_workload(mode, stage):
    """1,000,003 params, Nd = 4, A = 256 (uneven last shard with 445 pad),
    loss scale 1024, Adam lr 1e-3 / 0.9 / 0.999 / 1e-8, 3 steps."""
    pb = make_problem(1_000_003, 4, align=256, bucket=65_536 if stage == 2 else 0, steps=3, seed=1,
                      S=1024.0)
    hp = B.hparams(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, loss_scale=1024.0, mode=mode)
    layout = B.ZERO_GRADS_PER_OWNER if stage == 3 else B.ZERO_GRADS_FULL
    g = run_gpu(pb, hp, layout=layout, stage=stage)
    o = run_oracle(pb, to_oracle_hp(hp))
    compare(g, o, f"tiny stage {stage} {MODE_NAMES[mode]}")
    assert g.opt.t == 3 and all(r.overflow == 0 for r in g.results)


RAGGED = [
    # psi, nd, align, bucket
    (1, 1, 1, 0), (1, 4, 1, 0), (7, 3, 1, 0), (8, 1, 8, 0), (255, 2, 8, 0), (257, 5, 1, 7),
    (4097, 16, 256, 0), (4097, 16, 8, 1000), (100_003, 3, 1, 0), (100_003, 7, 16, 4096),
    (65_536, 64, 1, 0), (200_001, 64, 256, 8192), (33, 64, 1, 0),
]


@pytest.mark.parametrize("psi,nd,align,bucket", RAGGED)
@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("layout", [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER], ids=["full", "per_owner"])
def test_ragged_sizes(psi, nd, align, bucket, mode, layout):
    pb = make_problem(psi, nd, align=align, bucket=bucket, steps=2, seed=psi % 97 + nd,
                      S=65536.0, random_state=True)
    hp = B.hparams(lr=1e-3, weight_decay=0.01, loss_scale=65536.0, mode=mode)
    g = run_gpu(pb, hp, layout=layout, stage=3 if layout else 2)
    compare(g, run_oracle(pb, to_oracle_hp(hp)), f"ragged {psi}/{nd}/{align}/{bucket}")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("owner", [0, 2, 3])
@pytest.mark.parametrize("layout", [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER], ids=["full", "per_owner"])
def test_one_owner_view(mode, owner, layout):
    """One rank's view: only owner `owner` is updated; the flag and norm cover
    that owner's elements; every other owner's parameters stay untouched."""
    pb = make_problem(1_000_003, 4, align=256, steps=2, seed=7, S=1024.0)
    hp = B.hparams(loss_scale=1024.0, mode=mode)
    g = run_gpu(pb, hp, layout=layout, owner_first=owner, owner_count=1, stage=3)
    o = run_oracle(pb, to_oracle_hp(hp), lo=g.lo, hi=g.hi)
    compare(g, o, f"owner {owner}")


@pytest.mark.parametrize("mode", [B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH], ids=["two_pass", "stash"])
@pytest.mark.parametrize("bucket", [0, 50_000])
def test_global_norm_clipping(mode, bucket):
    pb = make_problem(300_007, 16, align=256, bucket=bucket, steps=3, seed=11, S=65536.0)
    hp = B.hparams(loss_scale=65536.0, max_grad_norm=0.05, mode=mode)
    g = run_gpu(pb, hp, stage=2)
    o_free = run_oracle(pb, to_oracle_hp(hp))
    # the norms agree to fp64 summation-order rounding ...
    for r, info in zip(g.results, o_free.infos):
        assert r.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12)
        assert r.grad_norm > 0.05 and r.clip_coef < 1.0
        assert abs(r.clip_coef - info["clip_coef"]) <= np.spacing(np.float32(info["clip_coef"]))
    # ... and with the GPU's fp32 coefficient fed in, the update matches
    o = run_oracle(pb, to_oracle_hp(hp), clip_overrides=[r.clip_coef for r in g.results])
    compare(g, o, "clip")


def test_no_clipping_below_threshold():
    pb = make_problem(10_001, 4, align=8, steps=1, seed=12, S=1024.0)
    hp = B.hparams(loss_scale=1024.0, max_grad_norm=1e6, mode=B.ZERO_MODE_STASH)
    g = run_gpu(pb, hp)
    assert g.results[0].clip_coef == 1.0
    compare(g, run_oracle(pb, to_oracle_hp(hp)), "no clip")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("kind", ["inf", "neg_inf_pair", "nan"])
@pytest.mark.parametrize("layout", [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER], ids=["full", "per_owner"])
def test_overflow_skips_the_step(mode, kind, layout):
    pb = make_problem(123_457, 8, align=256, bucket=0, steps=3, seed=13, S=1024.0,
                      random_state=True)
    G = pb.grads[1]
    if kind == "inf":
        G[5, 99_999] = 0x7C00
    elif kind == "neg_inf_pair":
        G[0, 17] = 0x7C00
        G[7, 17] = 0xFC00
    else:
        G[3, 123_456] = 0x7E00
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01,
                   max_grad_norm=0.0 if mode == B.ZERO_MODE_SPECULATIVE else 1.0, mode=mode)
    g = run_gpu(pb, hp, layout=layout, stage=3 if layout else 1)
    o = run_oracle(pb, to_oracle_hp(hp), clip_overrides=None if mode == 0 else
                   [r.clip_coef for r in g.results])
    compare(g, o, f"overflow {kind}")
    assert [r.overflow for r in g.results] == [0, 1, 0]
    assert g.opt.t == 2 and g.opt.skipped == 1
    assert math.isnan(g.results[1].grad_norm)


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_skipped_step_changes_no_byte(mode):
    """A step that overflows leaves master, moments and parameters bit-identical."""
    pb = make_problem(50_001, 4, align=8, steps=1, seed=14, S=1024.0, random_state=True)
    pb.grads[0][2, 40_000] = 0x7C00
    hp = B.hparams(loss_scale=1024.0, mode=mode)
    g = run_gpu(pb, hp)
    assert g.results[0].overflow == 1 and g.opt.t == 0
    for a, b in ((g.master, pb.master), (g.exp_avg, pb.exp_avg), (g.exp_avg_sq, pb.exp_avg_sq)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(g.params, pb.params)


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_non_finite_pad_is_ignored(mode):
    pb = make_problem(100_003, 4, align=256, steps=2, seed=15, S=1024.0, pad_fill=np.inf)
    hp = B.hparams(loss_scale=1024.0, mode=mode)
    g = run_gpu(pb, hp, layout=B.ZERO_GRADS_FULL)
    assert all(r.overflow == 0 for r in g.results)
    compare(g, run_oracle(pb, to_oracle_hp(hp)), "pad")


def test_average_over_nd():
    pb = make_problem(77_777, 8, align=16, steps=2, seed=16, S=512.0)
    hp = B.hparams(loss_scale=512.0, average_over_nd=True, mode=B.ZERO_MODE_TWO_PASS,
                   max_grad_norm=1e-4)
    g = run_gpu(pb, hp)
    o = run_oracle(pb, to_oracle_hp(hp), clip_overrides=[r.clip_coef for r in g.results])
    compare(g, o, "average")


def test_results_invariant_to_bucket_layout_and_mode():
    """Without clipping the parameters, moments and master do not depend on the
    bucket size, the stage layout or the execution mode (bit for bit)."""
    pb = make_problem(500_009, 8, align=256, bucket=0, steps=2, seed=17, S=65536.0,
                      random_state=True)
    hp = lambda mode: B.hparams(loss_scale=65536.0, weight_decay=0.01, mode=mode)
    ref = run_gpu(pb, hp(0), stage=1)
    for bucket in (0, 8, 4096, 100_000, 1 << 30):
        for layout in (B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER):
            for mode in MODES:
                pb.bucket = bucket
                g = run_gpu(pb, hp(mode), layout=layout, stage=3 if layout else 2)
                for a, b in ((g.master, ref.master), (g.exp_avg, ref.exp_avg),
                             (g.exp_avg_sq, ref.exp_avg_sq)):
                    assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), (bucket, layout, mode)
                assert np.array_equal(g.params, ref.params)


def test_alignment_one_scalar_path_matches_vector_path():
    """A = 1 (shard length not a multiple of 8) takes the scalar path; it gives
    the same bits as the 16-byte vector path."""
    pb = make_problem(100_003, 3, align=1, steps=2, seed=18, S=1024.0)
    hp = B.hparams(loss_scale=1024.0)
    g1 = run_gpu(pb, hp, layout=B.ZERO_GRADS_PER_OWNER, stage=3)
    pb.align = 256
    g2 = run_gpu(pb, hp, layout=B.ZERO_GRADS_PER_OWNER, stage=3)
    assert np.array_equal(g1.master.view(np.uint32), g2.master.view(np.uint32))
    assert np.array_equal(g1.params, g2.params)
    compare(g1, run_oracle(pb, to_oracle_hp(hp)), "A=1")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_run_to_run_bit_identical(mode):
    pb = make_problem(654_321, 8, align=256, steps=2, seed=19, S=65536.0)
    hp = B.hparams(loss_scale=65536.0, max_grad_norm=0.0 if mode == 0 else 0.01, mode=mode)
    a = run_gpu(pb, hp)
    b = run_gpu(pb, hp)
    for x, y in ((a.master, b.master), (a.exp_avg, b.exp_avg), (a.exp_avg_sq, b.exp_avg_sq)):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    assert np.array_equal(a.params, b.params)
    assert [r.grad_norm for r in a.results] == [r.grad_norm for r in b.results] or mode == 0


def test_checkpoint_resume_equals_uninterrupted():
    """3 uninterrupted steps == 1 step, state saved to host and restored into
    fresh buffers, then 2 more steps (optimizer bookkeeping included)."""
    pb = make_problem(200_003, 4, align=256, steps=3, seed=20, S=1024.0)
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, mode=B.ZERO_MODE_TWO_PASS,
                   max_grad_norm=0.02)
    full = run_gpu(pb, hp)
    first = run_gpu(pb, hp, steps=1)
    # resume: a new problem whose initial state is the saved one
    import copy
    pb2 = copy.copy(pb)
    pb2.master, pb2.exp_avg, pb2.exp_avg_sq = first.master, first.exp_avg, first.exp_avg_sq
    pb2.params = first.params
    pb2.grads = pb.grads[1:]
    plan = B.zero_plan(pb.psi, pb.nd, stage=1, align_elems=pb.align)
    try:
        L = B.zero_plan_query(plan).shard_len
        n_state = pb.nd * L
        st = lambda a: dev(np.concatenate([a, np.zeros(n_state - a.size, np.float32)]))
        master, m, v = st(first.master), st(first.exp_avg), st(first.exp_avg_sq)
        params = dev(first.params)
        g_dev = dev(pb.grads[1])
        opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device="cuda")
        raw = bytearray(B.OPT_STATE_BYTES)
        saved = bytes(first.opt)          # the checkpointed optimizer state
        raw[:len(saved)] = saved
        opt_state.copy_(torch.frombuffer(raw, dtype=torch.uint8))
        args = B.step_args(grads=g_dev.data_ptr(), grad_rank_stride=pb.grads[1].shape[1],
                           master=(master.data_ptr(), 0), exp_avg=(m.data_ptr(), 0),
                           exp_avg_sq=(v.data_ptr(), 0), params=params.data_ptr(),
                           opt_state=opt_state.data_ptr(), owner_count=pb.nd)
        ws = torch.empty(B.zero_workspace_bytes(plan, hp, args), dtype=torch.uint8, device="cuda")
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        s = torch.cuda.current_stream().cuda_stream
        for t in (1, 2):
            g_dev.copy_(dev(pb.grads[t]))
            B.zero_shard_step(plan, hp, args, s)
        out = host(master)[:pb.psi]
        assert np.array_equal(out.view(np.uint32), full.master.view(np.uint32))
        assert np.array_equal(host(params), full.params)
        assert B.opt_state_from_bytes(host(opt_state).tobytes()).t == 3
    finally:
        B.zero_plan_destroy(plan)


@pytest.mark.parametrize("psi,nd,align", [(1_000_003, 4, 256), (100_003, 7, 1), (4097, 64, 8),
                                          (10, 16, 1)])
def test_gather_params_matches_oracle(psi, nd, align):
    p = oracle.plan(psi, nd, align)
    full_ref = synth.fp16_bits(synth.normal_f32(psi, seed=psi, std=1.0))
    shards_h, shards_d = [], []
    for r in range(nd):
        s, n = p.shard(r)
        sh = np.full(p.shard_len, 0x7E00, dtype=np.uint16)
        sh[:n] = full_ref[s:s + n]
        shards_h.append(sh)
        shards_d.append(dev(sh))
    skip = nd // 3
    ptrs = [0 if r == skip else shards_d[r].data_ptr() for r in range(nd)]
    init = np.full(psi + 64, PARAM_SENTINEL, dtype=np.uint16)
    full_d = dev(init)
    plan = B.zero_plan(psi, nd, stage=3, align_elems=align)
    try:
        B.zero_gather_params(plan, ptrs, full_d.data_ptr(), torch.cuda.current_stream().cuda_stream)
    finally:
        B.zero_plan_destroy(plan)
    want = init[:psi].copy()
    oracle.gather_params([None if r == skip else shards_h[r] for r in range(nd)], p, want)
    got = host(full_d)
    assert np.array_equal(got[:psi], want)
    assert (got[psi:] == PARAM_SENTINEL).all()


@pytest.mark.parametrize("psi,nd,align,o0,oc", [(1_000_003, 4, 256, 0, 4), (100_003, 3, 1, 1, 2),
                                                (5, 8, 1, 0, 8)])
def test_cast_params_matches_oracle(psi, nd, align, o0, oc):
    p = oracle.plan(psi, nd, align)
    lo, hi = o0 * p.shard_len, min((o0 + oc) * p.shard_len, psi)
    x = synth.normal_f32(psi, seed=3, std=1.0) * np.float32(2.0) ** synth.normal_f32(psi, seed=4, std=12.0).astype(np.int32).clip(-40, 20)
    x = x.astype(np.float32)
    x[:min(psi, 6)] = np.array([0.0, -0.0, 65504.0, 65520.0, 2.0 ** -25, -2.0 ** -24], np.float32)[:min(psi, 6)]
    master_d = dev(np.concatenate([x[lo:hi], np.zeros(oc * p.shard_len - (hi - lo) + 8, np.float32)]))
    params_d = dev(np.full(psi, PARAM_SENTINEL, dtype=np.uint16))
    plan = B.zero_plan(psi, nd, stage=1, align_elems=align)
    try:
        B.zero_cast_params(plan, master_d.data_ptr(), params_d.data_ptr(), o0, oc,
                           torch.cuda.current_stream().cuda_stream)
    finally:
        B.zero_plan_destroy(plan)
    got = host(params_d)
    assert np.array_equal(got[lo:hi], oracle.float_to_half(x[lo:hi]))
    assert (got[:lo] == PARAM_SENTINEL).all() and (got[hi:] == PARAM_SENTINEL).all()


def test_launch_counter_counts_kernels():
    pb = make_problem(10_000, 4, align=8, steps=1, seed=21, S=1024.0)
    before = B.zero_launch_count()
    run_gpu(pb, B.hparams(loss_scale=1024.0))  # init + prep + update + commit
    assert B.zero_launch_count() - before == 4
    before = B.zero_launch_count()
    pb.bucket = 2_504
    run_gpu(pb, B.hparams(loss_scale=1024.0, mode=B.ZERO_MODE_STASH, max_grad_norm=1.0))
    # init + prep + 4 statistics launches (one per bucket) + finalize + update
    assert B.zero_launch_count() - before == 8


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("layout", [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER], ids=["full", "per_owner"])
def test_dynamic_loss_scaling_sequence(mode, layout):
    """Dynamic loss scale in the device optimizer state: 8 steps with two
    injected overflows and growth after 2 clean steps; scale, counters and
    state track the oracle step by step."""
    S0 = 2.0 ** 12
    pb = make_problem(70_001, 4, align=256, steps=8, seed=81, S=S0)
    for t, (r, i) in ((2, (1, 5_000)), (5, (3, 70_000))):
        pb.grads[t][r, i] = 0x7C00
    dyn = (S0, 2.0, 0.5, 2)
    clip = 0.0 if mode == B.ZERO_MODE_SPECULATIVE else 1e-3
    hp = B.hparams(loss_scale=1.0, weight_decay=0.01, max_grad_norm=clip, mode=mode)
    g = run_gpu(pb, hp, layout=layout, stage=3 if layout else 1, dynamic=dyn)
    o = run_oracle(pb, to_oracle_hp(hp), dynamic=dyn,
                   clip_overrides=None if not clip else [r.clip_coef for r in g.results])
    compare(g, o, "dynamic scale")
    assert [r.overflow for r in g.results] == [0, 0, 1, 0, 0, 1, 0, 0]
    assert [r.loss_scale for r in g.results] == [info["loss_scale"] for info in o.infos]
    assert [r.loss_scale for r in g.results] == [S0, 2 * S0, S0, S0, 2 * S0, S0, S0, 2 * S0]


@pytest.fixture(scope="module")
def bulk_store_problem():
    psi = 32_000_017
    pb = make_problem(psi, 6, align=256, steps=3, seed=71, S=1024.0, random_state=True)
    pb.grads[1][2, 5 * (psi // 6) + 4321] = INF16[B.ZERO_STORAGE_FP16]
    return pb


@pytest.mark.parametrize("mode", [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS], ids=["speculative", "two_pass"])
@pytest.mark.parametrize("layout", [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER], ids=["full", "per_owner"])
def test_bulk_store_pipeline_launch(mode, layout, bulk_store_problem):
    """A pipelined update whose results leave through shared memory and the
    producer's bulk stores (5 <= Nd <= 11 from the contributions): Nd = 6,
    32,000,017 parameters in one call over all owners (70 tiles of 1024
    elements per CTA at 3 CTAs on each of 148 SMs), six owner segments with
    ragged ends, an overflow in the second of three steps; every element
    against the oracle."""
    pb = bulk_store_problem
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, mode=mode,
                   max_grad_norm=0.0 if mode == B.ZERO_MODE_SPECULATIVE else 0.05)
    stage = 3 if layout == B.ZERO_GRADS_PER_OWNER else 1
    g, names = kernels_launched(lambda: run_gpu(pb, hp, layout=layout, stage=stage))
    if torch.cuda.get_device_properties(0).multi_processor_count <= 148:
        assert any("zs_update_pipe_kernel" in n for n in names), sorted(names)
    assert [r.overflow for r in g.results] == [0, 1, 0]
    o = run_oracle(pb, to_oracle_hp(hp),
                   clip_overrides=None if mode == B.ZERO_MODE_SPECULATIVE else [r.clip_coef for r in g.results])
    compare(g, o, f"bulk-store pipeline {MODE_NAMES[mode]} layout {layout}")


@pytest.mark.parametrize("nd", [5, 11])
def test_bulk_store_pipeline_range_ends(nd):
    """The ends of the bulk-store range: Nd = 5, and Nd = 11, whose results
    region still leaves room for 3 CTAs per SM (2 ring stages of 1024
    elements x 36 B).  29,600,003 parameters (just over 64 tiles per CTA),
    two steps, every element against the oracle."""
    pb = make_problem(29_600_003, nd, align=256, steps=2, seed=72 + nd, S=1024.0, random_state=True)
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, mode=B.ZERO_MODE_SPECULATIVE)
    g, names = kernels_launched(lambda: run_gpu(pb, hp))
    if torch.cuda.get_device_properties(0).multi_processor_count <= 148:
        assert any("zs_update_pipe_kernel" in n for n in names), sorted(names)
    compare(g, run_oracle(pb, to_oracle_hp(hp)), f"bulk-store pipeline Nd = {nd}")


@pytest.mark.parametrize("psi,nd,mode", [
    (30_000_000, 8, B.ZERO_MODE_SPECULATIVE),   # pipeline (>= 29.1M at 3 CTAs)
    (16_000_000, 8, B.ZERO_MODE_SPECULATIVE),   # register path (under 64 tiles per CTA)
    (1_000_000, 2, B.ZERO_MODE_SPECULATIVE),    # pipeline at any size for Nd <= 3
    (2_000_000, 4, B.ZERO_MODE_STASH),          # the stash always takes the pipeline
    (15_000_000, 17, B.ZERO_MODE_SPECULATIVE),  # tensor-map pipeline (>= 14.5M at Nd = 17)
    (8_000_000, 17, B.ZERO_MODE_SPECULATIVE),   # register path
])
def test_bench_names_the_update_kernel_that_runs(psi, nd, mode):
    """The bench line's roofline names its update kernel from the library's
    shape rules; the kernel a launch of that size actually runs is the one
    it names."""
    import bench
    pb = make_problem(psi, nd, align=256, steps=1, seed=73, S=1024.0)
    hp = B.hparams(loss_scale=1024.0, mode=mode, max_grad_norm=0.0 if mode == B.ZERO_MODE_SPECULATIVE else 1.0)
    _, names = kernels_launched(lambda: run_gpu(pb, hp))
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the shape rules are stated for 148 SMs")
    want = bench.update_kernel_name(nd, mode, False, psi)
    other = "zs_update_kernel" if want == "zs_update_pipe_kernel" else "zs_update_pipe_kernel"
    assert any(want + "<" in n or want + "I" in n for n in names), sorted(names)
    assert not any(other + "<" in n or other + "I" in n for n in names), sorted(names)
