"""GPU parity of the stage-2 reduce-scatter with retention
(``zero_reduce_scatter``) and of the step on the retained gradients
(``ZERO_GRADS_REDUCED``) against the oracle's ``reduce_scatter16`` and
``step``.  The retained values are 16-bit roundings of the same fp32
rank-order sums on both sides, so they must agree bit for bit; the step on
them is held to the other parity tests' bars."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from _gpu import (CANARY, INF16, NAN16, PARAM_SENTINEL, STATE_SENTINEL, dev, host, make_problem, run_oracle,
                  to_oracle_hp)
from _util import assert_bf16_close, assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B

pytestmark = pytest.mark.gpu

MODES = [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH]
MODE_NAMES = {0: "speculative", 1: "two_pass", 2: "stash"}
SHARD_SENTINEL = np.uint16(0x7DDD)
SOURCES = ["full", "per_owner", "peers"]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


class Source:
    """The Nd contributions on the device in one of the reduce-scatter's
    source layouts, for owners o0 .. o0 + oc - 1."""

    def __init__(self, pb, plan_info, kind, o0, oc):
        self.kind, self.pb, self.o0, self.oc = kind, pb, o0, oc
        self.L, self.psi_pad = plan_info.shard_len, plan_info.psi_pad
        self.nan = NAN16[pb.storage]
        self.load(0)

    def load(self, t):
        pb, L = self.pb, self.L
        G = pb.grads[t]
        if self.kind == "per_owner":
            blk = np.full((self.oc, pb.nd, L), self.nan, np.uint16)
            for j in range(self.oc):
                s = (self.o0 + j) * L
                n = max(0, min(L, pb.psi - s))
                blk[j, :, :n] = G[:, s:s + n]
            self.buf = dev(blk)
        elif self.kind == "full":
            self.buf = dev(G)
        else:   # one separately allocated buffer per rank
            self.bufs = [dev(np.ascontiguousarray(G[r])) for r in range(pb.nd)]

    def args(self, **kw):
        if self.kind == "peers":
            a = B.step_args(grads=0, grad_rank_stride=0, **kw)
            return B.attach_peers(a, B.peer_args([b.data_ptr() for b in self.bufs]))
        layout = B.ZERO_GRADS_PER_OWNER if self.kind == "per_owner" else B.ZERO_GRADS_FULL
        stride = self.L if self.kind == "per_owner" else self.psi_pad
        return B.step_args(grads=self.buf.data_ptr(), grad_rank_stride=stride, grad_layout=layout, **kw)

    def release(self, lo, hi):
        """Overwrites flat range [lo, hi) of every rank's contribution with NaN:
        the ranks' buffers are free once the owner has reduced them."""
        if self.kind == "full":
            self.buf.view(torch.int16)[:, lo:hi] = int(np.int16(self.nan.view(np.int16)))
        elif self.kind == "peers":
            for b in self.bufs:
                b.view(torch.int16)[lo:hi] = int(np.int16(self.nan.view(np.int16)))
        else:
            for j in range(self.oc):
                s = (self.o0 + j) * self.L
                a, b = max(lo, s) - s, min(hi, s + self.L) - s
                if a < b:
                    self.buf.view(torch.int16)[j, :, a:b] = int(np.int16(self.nan.view(np.int16)))


def dummy_state():
    return dict(master=(0, 0), exp_avg=(0, 0), exp_avg_sq=(0, 0), params=0, opt_state=0)


@pytest.mark.parametrize("kind", SOURCES)
@pytest.mark.parametrize("storage", [B.ZERO_STORAGE_FP16, B.ZERO_STORAGE_BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("psi,nd,align,o0,oc", [(1_000_003, 4, 256, 0, 4), (100_003, 7, 1, 2, 3),
                                                (4097, 16, 8, 0, 16), (33, 64, 1, 30, 4), (5, 1, 1, 0, 1)])
def test_reduce_scatter_keeps_the_oracle_sums(kind, storage, psi, nd, align, o0, oc):
    pb = make_problem(psi, nd, align=align, steps=1, seed=psi % 53 + nd, S=1.0, std=1.0, storage=storage)
    plan = B.zero_plan(psi, nd, stage=2, align_elems=align)
    try:
        info = B.zero_plan_query(plan)
        L = info.shard_len
        src = Source(pb, info, kind, o0, oc)
        out = dev(np.full(oc * L + CANARY, SHARD_SENTINEL, np.uint16))
        B.zero_reduce_scatter(plan, src.args(owner_first=o0, owner_count=oc, storage=storage, **dummy_state()),
                              out.data_ptr(), -1, torch.cuda.current_stream().cuda_stream)
        got = host(out)
    finally:
        B.zero_plan_destroy(plan)
    p = oracle.plan(psi, nd, align)
    want = oracle.reduce_scatter16(pb.grads[0], p, storage)
    for j in range(oc):
        n = p.shard(o0 + j)[1]
        assert np.array_equal(got[j * L:j * L + n], want[o0 + j, :n]), f"owner {o0 + j}"
        assert (got[j * L + n:(j + 1) * L] == SHARD_SENTINEL).all(), "pad written"
    assert (got[oc * L:] == SHARD_SENTINEL).all(), "guard written"


@pytest.mark.parametrize("kind", SOURCES)
def test_bucket_by_bucket_with_release(kind):
    """Each bucket reduced as soon as it is complete, then its part of every
    rank's buffer released (overwritten): the kept shards equal the oracle's."""
    psi, nd = 300_007, 4
    pb = make_problem(psi, nd, align=256, bucket=40_000, steps=1, seed=71, S=1.0, std=1.0)
    plan = B.zero_plan(psi, nd, stage=2, align_elems=256, bucket_elems=40_000)
    try:
        info = B.zero_plan_query(plan)
        L = info.shard_len
        src = Source(pb, info, kind, 0, nd)
        out = dev(np.full(nd * L + CANARY, SHARD_SENTINEL, np.uint16))
        args = src.args(owner_first=0, owner_count=nd, **dummy_state())
        stream = torch.cuda.current_stream().cuda_stream
        for k in reversed(range(info.n_buckets)):        # a backward pass produces the last bucket first
            b0, bn = B.zero_plan_bucket(plan, k)
            B.zero_reduce_scatter(plan, args, out.data_ptr(), k, stream)
            src.release(b0, b0 + bn)
        got = host(out)
    finally:
        B.zero_plan_destroy(plan)
    p = oracle.plan(psi, nd, 256, 40_000)
    want = oracle.reduce_scatter16(pb.grads[0], p, 0)
    for o in range(nd):
        n = p.shard(o)[1]
        assert np.array_equal(got[o * L:o * L + n], want[o, :n])


@dataclasses.dataclass
class Retained:
    master: np.ndarray
    exp_avg: np.ndarray
    exp_avg_sq: np.ndarray
    params: np.ndarray
    results: list
    shards: np.ndarray
    opt: object


def run_retained(pb, hp, *, kind="full", o0=0, oc=None, dynamic=None):
    """Per step: reduce-scatter with retention on the GPU, then the step on
    the retained shards (REDUCED layout)."""
    nd, psi = pb.nd, pb.psi
    oc = nd if oc is None else oc
    plan = B.zero_plan(psi, nd, stage=2, align_elems=pb.align, bucket_elems=pb.bucket)
    try:
        info = B.zero_plan_query(plan)
        L = info.shard_len
        lo, hi = o0 * L, max(o0 * L, min((o0 + oc) * L, psi))
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE
        src = Source(pb, info, kind, o0, oc)
        shards = dev(np.full(oc * L + CANARY, SHARD_SENTINEL, np.uint16))

        def state_buf(x):
            h = np.full(oc * L + CANARY, STATE_SENTINEL, np.uint32)
            if x is not None:
                h[:hi - lo] = x[lo:hi].view(np.uint32)
            return dev(h.view(np.float32))

        master = [state_buf(pb.master), state_buf(None) if spec else None]
        m = [state_buf(pb.exp_avg), state_buf(None) if spec else None]
        v = [state_buf(pb.exp_avg_sq), state_buf(None) if spec else None]
        stash = state_buf(None) if hp.mode == B.ZERO_MODE_STASH else None
        p_h = np.full(psi + CANARY, PARAM_SENTINEL, np.uint16)
        p_h[:psi] = pb.params
        params = dev(p_h)
        opt = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device="cuda")
        res = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device="cuda")
        ptr = lambda t: t.data_ptr() if t is not None else 0
        step = B.step_args(grads=shards.data_ptr(), grad_rank_stride=0, grad_layout=B.ZERO_GRADS_REDUCED,
                           owner_first=o0, owner_count=oc, master=tuple(map(ptr, master)),
                           exp_avg=tuple(map(ptr, m)), exp_avg_sq=tuple(map(ptr, v)), params=params.data_ptr(),
                           grad_stash=ptr(stash), opt_state=opt.data_ptr(), result=res.data_ptr(),
                           storage=pb.storage)
        nb = B.zero_workspace_bytes(plan, hp, step)
        ws = torch.zeros(nb + 256, dtype=torch.uint8, device="cuda")
        step.workspace, step.workspace_bytes = ws.data_ptr(), nb
        stream = torch.cuda.current_stream().cuda_stream
        if dynamic is None:
            B.zero_opt_state_init(opt.data_ptr(), stream)
        else:
            B.zero_opt_state_init_dynamic(opt.data_ptr(), *dynamic, stream=stream)
        results = []
        for t in range(len(pb.grads)):
            if t > 0:
                src.load(t)
            red = src.args(owner_first=o0, owner_count=oc, storage=pb.storage, **dummy_state())
            B.zero_reduce_scatter(plan, red, shards.data_ptr(), -1, stream)
            B.zero_shard_step(plan, hp, step, stream)
            results.append(B.step_result_from_bytes(host(res).tobytes()))
        o = B.opt_state_from_bytes(host(opt).tobytes())
        cur = o.cur if spec else 0
        out_p = host(params)
        assert (out_p[psi:] == PARAM_SENTINEL).all()
        assert np.array_equal(out_p[:lo], pb.params[:lo]) and np.array_equal(out_p[hi:psi], pb.params[hi:psi])
        return Retained(host(master[cur])[:hi - lo].copy(), host(m[cur])[:hi - lo].copy(),
                        host(v[cur])[:hi - lo].copy(), out_p[:psi].copy(), results, host(shards), o)
    finally:
        B.zero_plan_destroy(plan)


def oracle_retained(pb, hp_o, *, o0=0, oc=None, clip_overrides=None, dynamic=None):
    """The oracle's definition: the owners keep reduce_scatter16's values and
    the step takes them as its single contribution."""
    nd, psi = pb.nd, pb.psi
    oc = nd if oc is None else oc
    p = oracle.plan(psi, nd, pb.align, pb.bucket)
    L = p.shard_len
    lo, hi = o0 * L, max(o0 * L, min((o0 + oc) * L, psi))
    flat = []
    for G in pb.grads:
        kept = oracle.reduce_scatter16(G, p, pb.storage)
        row = np.zeros((1, psi), np.uint16)
        for o in range(nd):
            s, n = p.shard(o)
            row[0, s:s + n] = kept[o, :n]
        flat.append(row)
    q = dataclasses.replace(pb, grads=flat, nd=1)
    return run_oracle(q, hp_o, lo=lo, hi=hi, clip_overrides=clip_overrides, dynamic=dynamic)


def compare(g, o, storage, what):
    assert_f32_close(g.master, o.master, 2, what + " master")
    assert_f32_close(g.exp_avg, o.exp_avg, 2, what + " exp_avg")
    assert_f32_close(g.exp_avg_sq, o.exp_avg_sq, 2, what + " exp_avg_sq")
    (assert_bf16_close if storage else assert_f16_close)(g.params, o.params, 1, what + " params")
    for r, info in zip(g.results, o.infos):
        assert r.overflow == info["overflow"], what
        if info["overflow"] == 0 and "grad_norm" in info and not math.isnan(r.grad_norm):
            assert r.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12), what
    assert g.opt.t == o.opt.t


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("storage", [B.ZERO_STORAGE_FP16, B.ZERO_STORAGE_BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("kind", SOURCES)
def test_step_on_retained_gradients_matches_oracle(mode, storage, kind):
    pb = make_problem(250_007, 4, align=256, steps=3, seed=72, S=1024.0, random_state=True, storage=storage)
    clip = 0.0 if mode == B.ZERO_MODE_SPECULATIVE else 0.05
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, max_grad_norm=clip, mode=mode)
    g = run_retained(pb, hp, kind=kind)
    o = oracle_retained(pb, to_oracle_hp(hp, storage),
                        clip_overrides=None if not clip else [r.clip_coef for r in g.results])
    compare(g, o, storage, f"retained {MODE_NAMES[mode]} {kind}")
    if clip:
        assert all(r.clip_coef < 1.0 for r in g.results)


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_retained_owner_subset_and_ragged(mode):
    pb = make_problem(100_003, 7, align=1, steps=2, seed=73, S=256.0, random_state=True)
    hp = B.hparams(loss_scale=256.0, mode=mode)
    g = run_retained(pb, hp, kind="per_owner", o0=2, oc=3)
    compare(g, oracle_retained(pb, to_oracle_hp(hp), o0=2, oc=3), 0, "retained subset")


def test_retained_sum_beyond_fp16_skips_the_step():
    """Two contributions of 40000: the fp32 sum is finite, the kept fp16 value
    is inf, and the step on it is skipped (the fused step would not skip)."""
    pb = make_problem(10_001, 2, align=8, steps=2, seed=74, S=1.0)
    big = np.float16(40000.0).view(np.uint16)
    pb.grads[0][0, 1234] = big
    pb.grads[0][1, 1234] = big
    hp = B.hparams(loss_scale=1.0, mode=B.ZERO_MODE_TWO_PASS)
    g = run_retained(pb, hp)
    o = oracle_retained(pb, to_oracle_hp(hp))
    assert [r.overflow for r in g.results] == [1, 0] == [i["overflow"] for i in o.infos]
    compare(g, o, 0, "retained overflow")


def test_retained_average_divides_by_the_plan_nd():
    pb = make_problem(50_001, 4, align=8, steps=2, seed=75, S=256.0)
    hp = B.hparams(loss_scale=256.0, average_over_nd=True)
    g = run_retained(pb, hp)
    hp_o = to_oracle_hp(B.hparams(loss_scale=256.0 * 4))       # the oracle sees one contribution
    compare(g, oracle_retained(pb, hp_o), 0, "retained average")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_retained_dynamic_loss_scaling(mode):
    S0 = 2.0 ** 10
    pb = make_problem(70_001, 4, align=256, steps=5, seed=76, S=S0)
    pb.grads[2][3, 60_000] = INF16[B.ZERO_STORAGE_FP16]
    dyn = (S0, 2.0, 0.5, 2)
    hp = B.hparams(loss_scale=1.0, mode=mode, max_grad_norm=0.0 if mode == 0 else 10.0)
    g = run_retained(pb, hp, dynamic=dyn)
    o = oracle_retained(pb, to_oracle_hp(hp), dynamic=dyn,
                        clip_overrides=None if mode == 0 else [r.clip_coef for r in g.results])
    compare(g, o, 0, "retained dynamic")
    assert [r.loss_scale for r in g.results] == [i["loss_scale"] for i in o.infos]
