"""zero_shard_step_static_scratch -- the step for callers that cannot allocate
device memory (the scratch lives in a fixed array inside the library) --
against the regular zero_shard_step with a caller workspace.  Both run the
same kernels on the same inputs, so two calls in a row must give bit-equal
state, parameters and results; any difference would mean stale contents of
the shared array leaked into a step.  The array is first filled by an
unrelated clipped call, so the claim that nothing in it has to start at zero
is exercised on purpose.  Collected last on purpose, and self-contained so
that it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _buffers(psi, nd, L, mode, master0, grads):
    n_state = nd * L
    dev = torch.device("cuda")

    def state(src=None):
        t = torch.zeros(n_state, dtype=torch.float32, device=dev)
        if src is not None:
            t[:psi].copy_(torch.from_numpy(src))
        return t

    spec = mode == B.ZERO_MODE_SPECULATIVE
    return dict(
        master=[state(master0), state() if spec else None],
        m=[state(), state() if spec else None],
        v=[state(), state() if spec else None],
        stash=state() if mode == B.ZERO_MODE_STASH else None,
        params=torch.from_numpy(synth.fp16_bits(master0)).to(dev),
        grads=torch.from_numpy(grads[0]).to(dev),
        opt_state=torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device=dev),
        result=torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device=dev),
    )


def _run(entry, psi, nd, align, bucket, mode, clip, grads, master0):
    plan = B.zero_plan(psi, nd, stage=2, align_elems=align, bucket_elems=bucket)
    try:
        info = B.zero_plan_query(plan)
        buf = _buffers(psi, nd, info.shard_len, mode, master0, grads)
        ptr = lambda t: t.data_ptr() if t is not None else 0
        hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, max_grad_norm=clip, mode=mode)
        args = B.step_args(grads=buf["grads"].data_ptr(), grad_rank_stride=info.psi_pad,
                           owner_count=nd, master=tuple(map(ptr, buf["master"])),
                           exp_avg=tuple(map(ptr, buf["m"])), exp_avg_sq=tuple(map(ptr, buf["v"])),
                           params=buf["params"].data_ptr(), grad_stash=ptr(buf["stash"]),
                           opt_state=buf["opt_state"].data_ptr(), result=buf["result"].data_ptr())
        ws = None
        if entry is B.zero_shard_step:
            ws = torch.empty(B.zero_workspace_bytes(plan, hp, args), dtype=torch.uint8, device="cuda")
            args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
        stream = torch.cuda.current_stream().cuda_stream
        B.zero_opt_state_init(buf["opt_state"].data_ptr(), stream)
        results = []
        for t in range(2):   # two calls in a row
            buf["grads"].copy_(torch.from_numpy(grads[t]))
            entry(plan, hp, args, stream)
            results.append(B.step_result_from_bytes(buf["result"].cpu().numpy().tobytes()))
        torch.cuda.synchronize()
        opt = B.opt_state_from_bytes(buf["opt_state"].cpu().numpy().tobytes())
        cur = opt.cur if mode == B.ZERO_MODE_SPECULATIVE else 0
        out = {k: buf[k][cur].cpu().numpy()[:psi] for k in ("master", "m", "v")}
        out["params"] = buf["params"].cpu().numpy()
        return out, results, opt
    finally:
        B.zero_plan_destroy(plan)


def _fill_scratch_with_another_call():
    """An unrelated clipped two-pass call with its own sizes and data, so the
    shared array holds a foreign header and foreign norm partials."""
    psi, nd = 300_017, 4
    psi_pad = nd * (-(-psi // (nd * 256)) * 256)
    grads = [synth.grads_f16(nd, psi, seed=90 + t, std=1e-2, scale=8.0, stride=psi_pad) for t in range(2)]
    _run(B.zero_shard_step_static_scratch, psi, nd, 256, 50_000, B.ZERO_MODE_TWO_PASS, 1e-3, grads,
         synth.normal_f32(psi, seed=91, std=0.5))


@pytest.mark.parametrize("mode,clip,bucket", [
    (B.ZERO_MODE_SPECULATIVE, 0.0, 0),
    (B.ZERO_MODE_TWO_PASS, 0.05, 65_536),
    (B.ZERO_MODE_STASH, 0.05, 0),
])
def test_static_scratch_step_matches_the_workspace_step(mode, clip, bucket):
    psi, nd, align = 400_003, 8, 256
    psi_pad = nd * (-(-psi // (nd * align)) * align)   # every rank holds a full gradient
    grads = [synth.grads_f16(nd, psi, seed=40 + t, std=1e-3, scale=1024.0, stride=psi_pad)
             for t in range(2)]
    master0 = synth.normal_f32(psi, seed=41, std=0.02)
    ref, ref_res, ref_opt = _run(B.zero_shard_step, psi, nd, align, bucket, mode, clip, grads, master0)
    _fill_scratch_with_another_call()
    got, got_res, got_opt = _run(B.zero_shard_step_static_scratch, psi, nd, align, bucket, mode,
                                 clip, grads, master0)
    for k in ("master", "m", "v", "params"):
        assert np.array_equal(got[k].view(np.uint32 if k != "params" else np.uint16),
                              ref[k].view(np.uint32 if k != "params" else np.uint16)), k
    for a, b in zip(got_res, ref_res):
        assert (a.overflow, a.t, a.skipped) == (b.overflow, b.t, b.skipped)
        assert a.clip_coef == b.clip_coef
        assert (np.isnan(a.grad_norm) and np.isnan(b.grad_norm)) or a.grad_norm == b.grad_norm
    assert (got_opt.t, got_opt.skipped) == (ref_opt.t, ref_opt.skipped) == (2, 0)
    if clip > 0:
        assert got_res[0].clip_coef < 1.0


def test_static_scratch_rejects_calls_beyond_its_size():
    """70 buckets of 4M elements need 70 x 2048 fp64 partials (> 1 MiB): the
    call is refused before anything is launched."""
    psi, nd = 70 * (4 << 20), 8
    plan = B.zero_plan(psi, nd, stage=2, align_elems=256, bucket_elems=4 << 20)
    fake = 1 << 40   # aligned addresses that the rejected call never touches
    try:
        hp = B.hparams(loss_scale=1.0, max_grad_norm=1.0, mode=B.ZERO_MODE_TWO_PASS)
        args = B.step_args(grads=fake, grad_rank_stride=psi, owner_count=nd, master=(fake, 0),
                           exp_avg=(fake, 0), exp_avg_sq=(fake, 0), params=fake, opt_state=fake)
        assert B.zero_workspace_bytes(plan, hp, args) > B.ZERO_STATIC_SCRATCH_BYTES
        before = B.zero_launch_count()
        with pytest.raises(B.ZeroError) as e:
            B.zero_shard_step_static_scratch(plan, hp, args, torch.cuda.current_stream().cuda_stream)
        assert e.value.status == B.ZERO_ERR_WORKSPACE
        assert "static scratch" in B.zero_last_error()
        assert B.zero_launch_count() == before
    finally:
        B.zero_plan_destroy(plan)
