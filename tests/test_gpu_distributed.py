"""The split step (zero_shard_step_begin / _end around the vote) on the GPU.

* begin + end with nothing in between equal zero_shard_step bit for bit;
* Nd owners, each with its own buffers, workspace and step state, as separate
  processes would hold them (emulated one after another in this process, with
  the votes summed on the device between the halves), reproduce the oracle's
  single-process step, including a skip caused by one rank's inf;
* ZeroDPStep runs end to end over a real NCCL process group (world size 1)."""
import math
import socket

import numpy as np
import pytest
import torch

import oracle
from _gpu import PARAM_SENTINEL, dev, host, make_problem, run_gpu, to_oracle_hp
from _util import assert_bf16_close, assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B

pytestmark = pytest.mark.gpu

MODES = [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


class _Owner:
    """The buffers one process owning shard `o` would hold."""

    def __init__(self, plan, pb, o, hp):
        L = B.zero_plan_query(plan).shard_len
        self.o, self.L = o, L
        s, n = B.zero_plan_shard(plan, o)
        self.s, self.n = s, n
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE

        def shard(src):
            h = np.zeros(L, np.float32)
            if src is not None:
                h[:n] = src[s:s + n]
            return dev(h)

        self.master = [shard(pb.master), shard(None) if spec else None]
        self.m = [shard(pb.exp_avg), shard(None) if spec else None]
        self.v = [shard(pb.exp_avg_sq), shard(None) if spec else None]
        self.stash = shard(None) if hp.mode == B.ZERO_MODE_STASH else None
        self.params = dev(np.full(pb.nd * L, PARAM_SENTINEL, np.uint16))
        self.params[s:s + n] = dev(pb.params[s:s + n])
        blk = np.zeros((pb.nd, L), np.uint16)     # what the exchange delivers to owner o
        blk[:, :n] = pb.grads[0][:, s:s + n]
        self.recv = dev(blk.reshape(-1))
        self.opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device="cuda")
        self.result = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device="cuda")
        ptr = lambda t: t.data_ptr() if t is not None else 0
        self.args = B.step_args(grads=self.recv.data_ptr(), grad_rank_stride=L,
                                grad_layout=B.ZERO_GRADS_PER_OWNER, owner_first=o, owner_count=1,
                                master=tuple(map(ptr, self.master)), exp_avg=tuple(map(ptr, self.m)),
                                exp_avg_sq=tuple(map(ptr, self.v)), params=self.params.data_ptr(),
                                grad_stash=ptr(self.stash), opt_state=self.opt_state.data_ptr(),
                                result=self.result.data_ptr())
        self.ws = torch.zeros(B.zero_workspace_bytes(plan, hp, self.args), dtype=torch.uint8,
                              device="cuda")
        self.args.workspace, self.args.workspace_bytes = self.ws.data_ptr(), self.ws.numel()
        self.vote = self.ws[B.ZERO_VOTE_OFFSET:B.ZERO_VOTE_OFFSET + 16].view(torch.float64)
        B.zero_opt_state_init(self.opt_state.data_ptr(), torch.cuda.current_stream().cuda_stream)

    def live(self):
        opt = B.opt_state_from_bytes(host(self.opt_state).tobytes())
        k = opt.cur if self.master[1] is not None else 0
        return (host(self.master[k])[:self.n], host(self.m[k])[:self.n], host(self.v[k])[:self.n],
                host(self.params)[self.s:self.s + self.n], opt,
                B.step_result_from_bytes(host(self.result).tobytes()))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("bucket", [0, 40_000])
def test_begin_end_equals_single_call(mode, bucket):
    pb = make_problem(300_007, 4, align=256, bucket=bucket, steps=2, seed=51, S=1024.0,
                      random_state=True)
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01,
                   max_grad_norm=0.0 if mode == B.ZERO_MODE_SPECULATIVE else 0.02, mode=mode)
    ref = run_gpu(pb, hp, stage=2)

    def split(plan, hp_, args, stream):
        B.zero_shard_step_begin(plan, hp_, args, stream)
        B.zero_shard_step_end(plan, hp_, args, stream)

    orig = B.zero_shard_step
    try:
        B.zero_shard_step = split       # run_gpu calls B.zero_shard_step
        got = run_gpu(pb, hp, stage=2)
    finally:
        B.zero_shard_step = orig
    for a, b in ((got.master, ref.master), (got.exp_avg, ref.exp_avg), (got.exp_avg_sq, ref.exp_avg_sq)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(got.params, ref.params)
    for a, b in zip(got.results, ref.results):
        assert (a.overflow, a.t, a.skipped, a.clip_coef) == (b.overflow, b.t, b.skipped, b.clip_coef)
        assert (math.isnan(a.grad_norm) and math.isnan(b.grad_norm)) or a.grad_norm == b.grad_norm


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("nd,inject", [(4, False), (3, True), (8, False)])
def test_owners_in_separate_buffers_with_summed_votes_match_the_oracle(mode, nd, inject):
    pb = make_problem(200_003, nd, align=256, steps=1, seed=52 + nd, S=1024.0)
    if inject:
        pb.grads[0][nd - 1, 123_457] = 0x7C00
    clip = 0.0 if mode == B.ZERO_MODE_SPECULATIVE else 0.02
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, max_grad_norm=clip, mode=mode)
    plan = B.zero_plan(pb.psi, nd, stage=3, align_elems=256)
    stream = torch.cuda.current_stream().cuda_stream
    try:
        owners = [_Owner(plan, pb, o, hp) for o in range(nd)]
        for ow in owners:
            B.zero_shard_step_begin(plan, hp, ow.args, stream)
        total = torch.stack([ow.vote for ow in owners]).sum(dim=0)   # the all-reduce
        for ow in owners:
            ow.vote.copy_(total)
            B.zero_shard_step_end(plan, hp, ow.args, stream)
        torch.cuda.synchronize()
        lives = [ow.live() for ow in owners]
    finally:
        B.zero_plan_destroy(plan)
    res = [lv[5] for lv in lives]
    assert len({(r.overflow, r.t, r.skipped, r.clip_coef) for r in res}) == 1, "owners disagree"
    ref_master, ref_m, ref_v = pb.master.copy(), pb.exp_avg.copy(), pb.exp_avg_sq.copy()
    ref_P = pb.params.copy()
    info = oracle.step(np.ascontiguousarray(pb.grads[0][:, :pb.psi]), ref_master, ref_m, ref_v, ref_P,
                       to_oracle_hp(hp), oracle.Opt(), clip_override=res[0].clip_coef if clip else None)
    assert res[0].overflow == info["overflow"] == int(inject)
    if not inject and clip:
        assert res[0].grad_norm == pytest.approx(info["grad_norm"], rel=1e-12)
    got = [np.concatenate([lv[k] for lv in lives]) for k in range(4)]
    assert_f32_close(got[0], ref_master, 2, "master")
    assert_f32_close(got[1], ref_m, 2, "exp_avg")
    assert_f32_close(got[2], ref_v, 2, "exp_avg_sq")
    assert_f16_close(got[3], ref_P, 1, "params")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("storage", [B.ZERO_STORAGE_FP16, B.ZERO_STORAGE_BF16], ids=["fp16", "bf16"])
def test_zero_dp_step_over_an_nccl_group(storage):
    import torch.distributed as dist
    from zero_dp_partitioned_shard_b200 import distributed as D
    from zero_dp_partitioned_shard_b200 import synth
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    bf = storage == B.ZERO_STORAGE_BF16
    try:
        psi = 1_000_003
        hp = B.hparams(loss_scale=1024.0, weight_decay=0.01)
        zs = D.ZeroDPStep(psi, hp, align=256, storage=storage)
        master0 = synth.normal_f32(psi, seed=5, std=0.02)
        zs.load_master(torch.from_numpy(master0))
        draw = synth.grads_bf16 if bf else synth.grads_f16
        grads = [draw(1, psi, seed=60 + t, std=1e-3, scale=1024.0, stride=zs.psi_pad,
                      pad_fill=0.0)[0] for t in range(2)]
        for G in grads:
            zs.step(torch.from_numpy(G.view(np.int16)).cuda().view(zs.dtype))
        torch.cuda.synchronize()
        master, m, v = (x.cpu().numpy()[:psi] for x in zs.live_state())
        params = zs.params.view(torch.int16).cpu().numpy().view(np.uint16)[:psi]
        res = B.step_result_from_bytes(zs.result.cpu().numpy().tobytes())
        zs.close()
    finally:
        dist.destroy_process_group()
    ref_master, ref_m, ref_v = master0.copy(), np.zeros(psi, np.float32), np.zeros(psi, np.float32)
    ref_P = oracle.float_to_bf16(master0) if bf else oracle.float_to_half(master0)
    opt = oracle.Opt()
    for G in grads:
        oracle.step(G[None, :psi].copy(), ref_master, ref_m, ref_v, ref_P,
                    oracle.HP(loss_scale=1024.0, weight_decay=0.01, storage=storage), opt)
    assert res.t == 2 and res.overflow == 0 and res.status == 0
    assert_f32_close(master, ref_master, 2, "master")
    assert_f32_close(v, ref_v, 2, "exp_avg_sq")
    (assert_bf16_close if bf else assert_f16_close)(params, ref_P, 1, "params")
