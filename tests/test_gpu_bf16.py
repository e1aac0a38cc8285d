"""GPU parity with bfloat16 storage of the gradient contributions and the
parameters (ZERO_STORAGE_BF16): the CUDA path against the oracle run with the
same storage format.  Bars as for fp16: master, momentum and variance within
2 fp32 ulp, parameters within 1 bf16 ulp, flags and counters exact, norm within
1e-12 relative."""
import math

import numpy as np
import pytest
import torch

import oracle
from _gpu import (INF16, NAN16, PARAM_SENTINEL, dev, host, kernels_launched, make_problem, run_gpu, run_oracle,
                  to_oracle_hp)
from _util import assert_bf16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import synth

pytestmark = pytest.mark.gpu

BF = B.ZERO_STORAGE_BF16
MODES = [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH]
MODE_NAMES = {0: "speculative", 1: "two_pass", 2: "stash"}
LAYOUTS = [B.ZERO_GRADS_FULL, B.ZERO_GRADS_PER_OWNER]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def compare(g, o, what=""):
    assert_f32_close(g.master, o.master, 2, what + " master")
    assert_f32_close(g.exp_avg, o.exp_avg, 2, what + " exp_avg")
    assert_f32_close(g.exp_avg_sq, o.exp_avg_sq, 2, what + " exp_avg_sq")
    assert_bf16_close(g.params, o.params, 1, what + " params")
    assert len(g.results) == len(o.infos)
    for r, info in zip(g.results, o.infos):
        assert r.overflow == info["overflow"], what
        if info["overflow"] == 0 and "grad_norm" in info and not math.isnan(r.grad_norm):
            assert r.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12, abs=1e-300), what
    assert g.opt.t == o.opt.t, what
    assert g.opt.skipped == sum(i["overflow"] for i in o.infos), what


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_tiny_workload_bf16(mode, stage):
    pb = make_problem(1_000_003, 4, align=256, bucket=65_536 if stage == 2 else 0, steps=3, seed=2,
                      S=1.0, storage=BF)
    hp = B.hparams(lr=1e-3, weight_decay=0.01, loss_scale=1.0, mode=mode)
    layout = B.ZERO_GRADS_PER_OWNER if stage == 3 else B.ZERO_GRADS_FULL
    g = run_gpu(pb, hp, layout=layout, stage=stage)
    compare(g, run_oracle(pb, to_oracle_hp(hp, BF)), f"bf16 stage {stage} {MODE_NAMES[mode]}")
    assert g.opt.t == 3


# (psi, nd, align, bucket): vectorised Nd <= 3 and the stash mode take the
# bulk-copy pipeline at these sizes, the others the register path; align 1
# the scalar path
RAGGED = [(1, 1, 1, 0), (7, 3, 1, 0), (4097, 2, 8, 1000), (100_003, 1, 256, 0), (100_003, 7, 16, 4096),
          (200_001, 64, 256, 8192), (65_539, 2, 1, 0)]


@pytest.mark.parametrize("psi,nd,align,bucket", RAGGED)
@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("layout", LAYOUTS, ids=["full", "per_owner"])
def test_ragged_sizes_bf16(psi, nd, align, bucket, mode, layout):
    pb = make_problem(psi, nd, align=align, bucket=bucket, steps=2, seed=psi % 89 + nd, S=256.0,
                      random_state=True, storage=BF)
    hp = B.hparams(lr=1e-3, weight_decay=0.01, loss_scale=256.0, mode=mode)
    g = run_gpu(pb, hp, layout=layout, stage=3 if layout else 2)
    compare(g, run_oracle(pb, to_oracle_hp(hp, BF)), f"bf16 ragged {psi}/{nd}/{align}/{bucket}")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("kind", ["inf", "neg_inf_pair", "nan"])
def test_overflow_skips_the_step_bf16(mode, kind):
    pb = make_problem(123_457, 8, align=256, steps=3, seed=13, S=1.0, random_state=True, storage=BF)
    G = pb.grads[1]
    if kind == "inf":
        G[5, 99_999] = INF16[BF]
    elif kind == "neg_inf_pair":
        G[0, 17] = INF16[BF]
        G[7, 17] = INF16[BF] | 0x8000
    else:
        G[3, 123_456] = NAN16[BF]
    hp = B.hparams(loss_scale=1.0, max_grad_norm=0.0 if mode == 0 else 1.0, mode=mode)
    g = run_gpu(pb, hp)
    o = run_oracle(pb, to_oracle_hp(hp, BF), clip_overrides=None if mode == 0 else
                   [r.clip_coef for r in g.results])
    compare(g, o, f"bf16 overflow {kind}")
    assert [r.overflow for r in g.results] == [0, 1, 0]


def test_rank_sum_overflow_to_inf_bf16():
    """bfloat16 has binary32's exponent range: two contributions of 2^127 x 1.5
    each are finite, their fp32 sum is +inf, and the step is skipped."""
    pb = make_problem(10_001, 2, align=8, steps=1, seed=31, S=1.0, storage=BF)
    big = np.uint16(0x7F40)   # 1.5 * 2^127
    pb.grads[0][0, 4_000] = big
    pb.grads[0][1, 4_000] = big
    hp = B.hparams(loss_scale=1.0, mode=B.ZERO_MODE_TWO_PASS)
    g = run_gpu(pb, hp)
    o = run_oracle(pb, to_oracle_hp(hp, BF))
    assert o.infos[0]["overflow"] == 1 and g.results[0].overflow == 1
    compare(g, o, "bf16 sum overflow")


@pytest.mark.parametrize("mode", [B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH], ids=["two_pass", "stash"])
def test_global_norm_clipping_bf16(mode):
    pb = make_problem(300_007, 16, align=256, bucket=50_000, steps=2, seed=11, S=1.0, std=1e-2,
                      storage=BF)
    hp = B.hparams(loss_scale=1.0, max_grad_norm=0.05, mode=mode)
    g = run_gpu(pb, hp, stage=2)
    o_free = run_oracle(pb, to_oracle_hp(hp, BF))
    for r, info in zip(g.results, o_free.infos):
        assert r.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12)
        assert r.clip_coef < 1.0
    o = run_oracle(pb, to_oracle_hp(hp, BF), clip_overrides=[r.clip_coef for r in g.results])
    compare(g, o, "bf16 clip")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_dynamic_loss_scaling_bf16(mode):
    S0 = 2.0 ** 8
    pb = make_problem(70_001, 4, align=256, steps=6, seed=83, S=S0, storage=BF)
    pb.grads[2][1, 5_000] = INF16[BF]
    hp = B.hparams(loss_scale=1.0, mode=mode, max_grad_norm=0.0 if mode == 0 else 10.0)
    dyn = (S0, 2.0, 0.5, 2)
    g = run_gpu(pb, hp, dynamic=dyn)
    o = run_oracle(pb, to_oracle_hp(hp, BF), dynamic=dyn,
                   clip_overrides=None if mode == 0 else [r.clip_coef for r in g.results])
    compare(g, o, "bf16 dynamic")
    assert [r.loss_scale for r in g.results] == [i["loss_scale"] for i in o.infos]
    assert [r.loss_scale for r in g.results] == [S0, 2 * S0, S0, S0, 2 * S0, 2 * S0]


@pytest.mark.parametrize("psi,nd,align,o0,oc", [(1_000_003, 4, 256, 0, 4), (100_003, 3, 1, 1, 2)])
def test_cast_params_bf16(psi, nd, align, o0, oc):
    p = oracle.plan(psi, nd, align)
    lo, hi = o0 * p.shard_len, min((o0 + oc) * p.shard_len, psi)
    x = synth.normal_f32(psi, seed=5, std=1.0) * np.float32(2.0) ** synth.normal_f32(psi, seed=6, std=40.0).astype(np.int32).clip(-140, 127)
    x = x.astype(np.float32)
    specials = np.array([0.0, -0.0, 3.3895314e38, 3.4028235e38, 1e-45, -1.1754944e-38], np.float32)
    x[:6] = specials
    master_d = dev(np.concatenate([x[lo:hi], np.zeros(oc * p.shard_len - (hi - lo) + 8, np.float32)]))
    params_d = dev(np.full(psi, PARAM_SENTINEL, dtype=np.uint16))
    plan = B.zero_plan(psi, nd, stage=1, align_elems=align)
    try:
        B.zero_cast_params(plan, master_d.data_ptr(), params_d.data_ptr(), o0, oc,
                           torch.cuda.current_stream().cuda_stream, storage=BF)
    finally:
        B.zero_plan_destroy(plan)
    got = host(params_d)
    assert np.array_equal(got[lo:hi], oracle.float_to_bf16(x[lo:hi]))
    assert (got[:lo] == PARAM_SENTINEL).all() and (got[hi:] == PARAM_SENTINEL).all()


def test_storage_formats_differ_only_in_rounding():
    """The same fp32 draws stored as fp16 and as bf16: the master weights of the
    two runs differ (different rounding of the contributions), each matching its
    own oracle."""
    a = make_problem(50_001, 4, align=8, steps=1, seed=41, S=1.0, storage=B.ZERO_STORAGE_FP16)
    b = make_problem(50_001, 4, align=8, steps=1, seed=41, S=1.0, storage=BF)
    hp = B.hparams(loss_scale=1.0)
    ga, gb = run_gpu(a, hp), run_gpu(b, hp)
    assert not np.array_equal(ga.master, gb.master)
    assert_f32_close(gb.master, run_oracle(b, to_oracle_hp(hp, BF)).master, 2, "bf16")


@pytest.mark.parametrize("psi,nd", [(30_000_007, 8), (15_000_011, 17)], ids=["bulk_stores_nd8", "tensor_map_nd17"])
def test_pipeline_launches_bf16(psi, nd):
    """Launches large enough for the bulk-copy pipeline with bfloat16
    storage: Nd = 8 (results through the producer's bulk stores; 29,097,984
    elements give 64 tiles per CTA) and Nd = 17 (rank rows as 2-D tensor-map
    boxes; 14,548,992 elements).  Two steps, every element against the
    oracle run with the same storage format."""
    pb = make_problem(psi, nd, align=256, steps=2, seed=91 + nd, S=1.0, random_state=True, storage=BF)
    hp = B.hparams(lr=1e-3, weight_decay=0.01, loss_scale=1.0, mode=B.ZERO_MODE_SPECULATIVE)
    g, names = kernels_launched(lambda: run_gpu(pb, hp))
    if torch.cuda.get_device_properties(0).multi_processor_count <= 148:
        assert any("zs_update_pipe_kernel" in n for n in names), sorted(names)
    compare(g, run_oracle(pb, to_oracle_hp(hp, BF)), f"bf16 pipeline Nd = {nd}")
