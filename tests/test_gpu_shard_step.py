"""The ShardStep object (buffers + C-ABI marshalling around zero_shard_step)
against the oracle: all owners, a stage-3 owner view with clipping, bf16
with dynamic loss scaling, a checkpoint round trip through state_dict /
load_state_dict, and CUDA-graph replay of captured steps -- the last two
must equal the uninterrupted direct run bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from _util import assert_bf16_close, assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import synth
from zero_dp_partitioned_shard_b200.shard_step import ShardStep

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _grads(nd, psi, psi_pad, t, S, storage=B.ZERO_STORAGE_FP16):
    draw = synth.grads_bf16 if storage == B.ZERO_STORAGE_BF16 else synth.grads_f16
    return draw(nd, psi, seed=300 + t, std=1e-3, scale=S, stride=psi_pad, pad_fill=0.0)


def _load(step, G):
    if step.stage == 3:
        L, o0 = step.L, step.owner_first
        blk = np.zeros((step.owner_count, step.nd, L), np.uint16)
        for j in range(step.owner_count):
            s = (o0 + j) * L
            n = max(0, min(L, step.psi - s))
            blk[j, :, :n] = G[:, s:s + n]
        step.grads.view(torch.int16).copy_(torch.from_numpy(blk.view(np.int16)))
    else:
        step.grads.view(torch.int16).copy_(torch.from_numpy(G.view(np.int16)))


def _run_oracle(G_list, master0, lo, hi, hp, clips=None, dynamic=None):
    m = master0[lo:hi].copy()
    a = np.zeros(hi - lo, np.float32)
    v = np.zeros(hi - lo, np.float32)
    P = (oracle.float_to_bf16 if hp.storage else oracle.float_to_half)(master0)[lo:hi].copy()
    opt = oracle.Opt() if dynamic is None else oracle.Opt(loss_scale=dynamic[0], growth_factor=dynamic[1],
                                                          backoff_factor=dynamic[2], growth_interval=dynamic[3])
    for t, G in enumerate(G_list):
        oracle.step(np.ascontiguousarray(G[:, lo:hi]), m, a, v, P, hp, opt,
                    clip_override=None if clips is None else clips[t])
    return m, a, v, P, opt


@pytest.mark.parametrize("mode", [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS], ids=["speculative", "two_pass"])
def test_all_owners_match_the_oracle(mode):
    psi, nd, S = 400_003, 4, 1024.0
    step = ShardStep(psi, nd, lr=1e-3, weight_decay=0.01, loss_scale=S, mode=mode, bucket=100_000)
    try:
        master0 = synth.normal_f32(psi, seed=301, std=0.02)
        step.load_master(torch.from_numpy(master0))
        G_list = [_grads(nd, psi, step.psi_pad, t, S) for t in range(3)]
        for G in G_list:
            _load(step, G)
            step.step()
        m, a, v = (x.cpu().numpy()[:psi] for x in step.live_state())
        P = step.params.view(torch.int16).cpu().numpy().view(np.uint16)
        assert step.result().t == 3
    finally:
        step.close()
    om, oa, ov, oP, _ = _run_oracle(G_list, master0, 0, psi, oracle.HP(loss_scale=S, weight_decay=0.01))
    assert_f32_close(m, om, 2, "master")
    assert_f32_close(a, oa, 2, "exp_avg")
    assert_f32_close(v, ov, 2, "exp_avg_sq")
    assert_f16_close(P, oP, 1, "params")


def test_stage3_owner_view_with_clipping():
    psi, nd, S = 300_007, 8, 65536.0
    step = ShardStep(psi, nd, stage=3, owner_first=5, owner_count=2, loss_scale=S, max_grad_norm=0.05,
                     mode=B.ZERO_MODE_STASH)
    try:
        lo, hi = step.owned_range
        master0 = synth.normal_f32(psi, seed=302, std=0.02)
        step.load_master(torch.from_numpy(master0))
        G_list = [_grads(nd, psi, step.psi_pad, t, S) for t in range(2)]
        clips = []
        for G in G_list:
            _load(step, G)
            step.step()
            clips.append(step.result().clip_coef)
        m = step.live_state()[0].cpu().numpy()
        P = step.params.view(torch.int16).cpu().numpy().view(np.uint16)
    finally:
        step.close()
    assert all(c < 1.0 for c in clips)
    om, _, _, oP, _ = _run_oracle(G_list, master0, lo, hi, oracle.HP(loss_scale=S, max_grad_norm=0.05), clips)
    L = -(-psi // (nd * 256)) * 256
    got = np.concatenate([m[j * L:j * L + max(0, min(L, psi - (5 + j) * L))] for j in range(2)])
    assert_f32_close(got, om, 2, "master")
    assert_f16_close(P[lo:hi], oP, 1, "params")
    assert (P[:lo] == 0).all() and (P[hi:] == 0).all()      # other owners' parameters untouched


def test_bf16_with_dynamic_loss_scaling():
    psi, nd, S0 = 100_003, 4, 2.0 ** 10
    dyn = (S0, 2.0, 0.5, 2)
    step = ShardStep(psi, nd, loss_scale=1.0, dynamic_scale=dyn, storage=B.ZERO_STORAGE_BF16)
    try:
        master0 = synth.normal_f32(psi, seed=303, std=0.02)
        step.load_master(torch.from_numpy(master0))
        G_list = [_grads(nd, psi, step.psi_pad, t, S0, B.ZERO_STORAGE_BF16) for t in range(4)]
        G_list[1][2, 777] = 0x7F80                     # +inf in bf16: one skipped step
        scales = []
        for G in G_list:
            _load(step, G)
            step.step()
            scales.append(step.result().loss_scale)
        m = step.live_state()[0].cpu().numpy()[:psi]
        P = step.params.view(torch.int16).cpu().numpy().view(np.uint16)
    finally:
        step.close()
    om, _, _, oP, opt = _run_oracle(G_list, master0, 0, psi, oracle.HP(storage=B.ZERO_STORAGE_BF16), dynamic=dyn)
    assert_f32_close(m, om, 2, "master")
    assert_bf16_close(P, oP, 1, "params")
    assert scales[-1] == opt.loss_scale and scales[1] == S0 / 2


@pytest.mark.parametrize("mode", [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_STASH], ids=["speculative", "stash"])
def test_checkpoint_round_trip_is_bit_exact(mode):
    psi, nd, S = 200_003, 4, 1024.0
    kw = dict(loss_scale=S, weight_decay=0.01, mode=mode, max_grad_norm=0.0 if mode == 0 else 1.0)
    master0 = synth.normal_f32(psi, seed=304, std=0.02)
    G_list = [_grads(nd, psi, -(-psi // (nd * 256)) * 256 * nd, t, S) for t in range(3)]

    def fresh():
        s = ShardStep(psi, nd, **kw)
        s.load_master(torch.from_numpy(master0))
        return s

    a = fresh()
    for G in G_list:
        _load(a, G)
        a.step()
    want = a.state_dict()
    a.close()
    b = fresh()
    _load(b, G_list[0])
    b.step()
    sd = b.state_dict()
    b.close()
    c = ShardStep(psi, nd, **kw)
    c.load_state_dict(sd)
    for G in G_list[1:]:
        _load(c, G)
        c.step()
    got = c.state_dict()
    c.close()
    for k in ("master", "exp_avg", "exp_avg_sq", "params"):
        assert torch.equal(got[k], want[k]), k
    ga, wa = B.opt_state_from_bytes(got["opt_state"].numpy().tobytes()), \
        B.opt_state_from_bytes(want["opt_state"].numpy().tobytes())
    assert (ga.t, ga.beta1_pow, ga.beta2_pow, ga.skipped) == (wa.t, wa.beta1_pow, wa.beta2_pow, wa.skipped)


@pytest.mark.parametrize("mode", [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_STASH], ids=["speculative", "stash"])
def test_graph_replay_equals_direct_steps(mode):
    """A step captured as a CUDA graph: capturing applies no step, and each
    replay advances the device state like a direct call (counter, bias
    corrections, live slot), so 4 replays equal 4 direct steps bit for bit."""
    psi, nd, S = 150_001, 4, 1024.0
    kw = dict(loss_scale=S, weight_decay=0.01, mode=mode, max_grad_norm=0.0 if mode == 0 else 1.0, bucket=40_000)
    master0 = synth.normal_f32(psi, seed=305, std=0.02)
    G = _grads(nd, psi, -(-psi // (nd * 256)) * 256 * nd, 0, S)
    direct = ShardStep(psi, nd, **kw)
    direct.load_master(torch.from_numpy(master0))
    _load(direct, G)
    for _ in range(4):
        direct.step()
    want = direct.state_dict()
    direct.close()
    g = ShardStep(psi, nd, **kw)
    g.load_master(torch.from_numpy(master0))
    _load(g, G)
    before = g.state_dict()
    launches = B.zero_launch_count()
    B.zero_shard_step_prepare(g.plan, g.hp, g.args)
    assert B.zero_launch_count() == launches          # prepare launches nothing
    graph = g.capture()                  # prepares again, then records one step
    torch.cuda.synchronize()
    assert g.opt().t == 0
    after = g.state_dict()
    for k in before:
        assert torch.equal(after[k], before[k]), f"capture changed {k}"
    for _ in range(4):
        graph.replay()
    torch.cuda.synchronize()
    got = g.state_dict()
    assert g.result().t == 4
    del graph
    g.close()
    for k in ("master", "exp_avg", "exp_avg_sq", "params"):
        assert torch.equal(got[k], want[k]), k
