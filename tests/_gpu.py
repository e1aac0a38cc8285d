"""GPU test harness: runs the library through its C ABI on host-prepared
inputs (torch only allocates and copies), and runs the oracle on the same
inputs.  Inputs come from zero_dp_partitioned_shard_b200.synth; expected values
come only from the oracle."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from zero_dp_partitioned_shard_b200 import binding as B

STATE_SENTINEL = np.uint32(0x7FBADBAD)   # a NaN bit pattern no kernel produces
PARAM_SENTINEL = np.uint16(0x7DDD)       # a NaN bit pattern
CANARY = 64                              # guard elements after every buffer


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


@dataclasses.dataclass
class Problem:
    psi: int
    nd: int
    align: int
    bucket: int
    grads: list            # per step: uint16 [nd, stride >= psi] (FULL layout)
    master: np.ndarray     # fp32 [psi]
    exp_avg: np.ndarray
    exp_avg_sq: np.ndarray
    params: np.ndarray     # uint16 [psi]
    storage: int = 0       # 16-bit format of grads and params (B.ZERO_STORAGE_*)


# a quiet NaN in each 16-bit format, for pads the kernels must not read
NAN16 = {B.ZERO_STORAGE_FP16: np.uint16(0x7E00), B.ZERO_STORAGE_BF16: np.uint16(0x7FC0)}
INF16 = {B.ZERO_STORAGE_FP16: np.uint16(0x7C00), B.ZERO_STORAGE_BF16: np.uint16(0x7F80)}


def make_problem(psi, nd, align=256, bucket=0, steps=1, seed=0, S=1024.0, std=1e-3,
                 random_state=False, pad_fill=np.nan, storage=B.ZERO_STORAGE_FP16):
    from zero_dp_partitioned_shard_b200 import synth
    pl = oracle.plan(psi, nd, align, bucket)
    draw = synth.grads_bf16 if storage == B.ZERO_STORAGE_BF16 else synth.grads_f16
    grads = [draw(nd, psi, seed=seed * 100 + t, std=std, scale=S, stride=pl.psi_pad,
                  pad_fill=pad_fill) for t in range(steps)]
    master = synth.normal_f32(psi, seed=seed * 100 + 91, std=0.02)
    if random_state:
        m = synth.normal_f32(psi, seed=seed * 100 + 92, std=1e-4)
        v = np.abs(synth.normal_f32(psi, seed=seed * 100 + 93, std=1e-7))
    else:
        m = np.zeros(psi, np.float32)
        v = np.zeros(psi, np.float32)
    params = synth.bf16_bits(master) if storage == B.ZERO_STORAGE_BF16 else synth.fp16_bits(master)
    return Problem(psi, nd, align, bucket, grads, master, m, v, params, storage)


@dataclasses.dataclass
class GpuResult:
    master: np.ndarray     # live slot, real elements of the call's owners (flat)
    exp_avg: np.ndarray
    exp_avg_sq: np.ndarray
    params: np.ndarray     # full [psi]
    results: list          # per step StepResult
    opt: B.OptState
    lo: int
    hi: int


def run_gpu(pb: Problem, hp: B.HParams, *, layout=B.ZERO_GRADS_FULL, owner_first=0,
            owner_count=None, stage=1, steps=None, check_guards=True, dynamic=None) -> GpuResult:
    """dynamic: (initial_scale, growth_factor, backoff_factor, growth_interval)
    switches dynamic loss scaling on."""
    nd, psi = pb.nd, pb.psi
    oc = nd if owner_count is None else owner_count
    o0 = owner_first
    plan = B.zero_plan(psi, nd, stage=stage, align_elems=pb.align, bucket_elems=pb.bucket)
    try:
        L = B.zero_plan_query(plan).shard_len
        lo, hi = o0 * L, max(o0 * L, min((o0 + oc) * L, psi))
        n_state = oc * L
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE

        def state_buf(src):
            h = np.full(n_state + CANARY, STATE_SENTINEL, dtype=np.uint32)
            if src is not None:
                h[:hi - lo] = src[lo:hi].view(np.uint32)
            return dev(h.view(np.float32))

        master = [state_buf(pb.master), state_buf(None) if spec else None]
        m = [state_buf(pb.exp_avg), state_buf(None) if spec else None]
        v = [state_buf(pb.exp_avg_sq), state_buf(None) if spec else None]
        params_h = np.full(psi + CANARY, PARAM_SENTINEL, dtype=np.uint16)
        params_h[:psi] = pb.params
        params = dev(params_h)
        stash = state_buf(None) if hp.mode == B.ZERO_MODE_STASH else None

        def grads_buf(G):
            if layout == B.ZERO_GRADS_FULL:
                return dev(G), G.shape[1]
            blk = np.full((oc, nd, L), NAN16[pb.storage], dtype=np.uint16)
            for j in range(oc):
                s = (o0 + j) * L
                n = max(0, min(L, psi - s))
                blk[j, :, :n] = G[:, s:s + n]
            return dev(blk), L

        g_dev, stride = grads_buf(pb.grads[0])
        opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device="cuda")
        result = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device="cuda")
        ptr = lambda t: t.data_ptr() if t is not None else 0
        args = B.step_args(grads=g_dev.data_ptr(), grad_rank_stride=stride, grad_layout=layout,
                           owner_first=o0, owner_count=oc,
                           master=(ptr(master[0]), ptr(master[1])), exp_avg=(ptr(m[0]), ptr(m[1])),
                           exp_avg_sq=(ptr(v[0]), ptr(v[1])), params=params.data_ptr(),
                           grad_stash=ptr(stash), opt_state=opt_state.data_ptr(),
                           result=result.data_ptr(), storage=pb.storage)
        ws_bytes = B.zero_workspace_bytes(plan, hp, args)
        ws = torch.empty(ws_bytes + 4096, dtype=torch.uint8, device="cuda")
        args.workspace = ws.data_ptr()
        args.workspace_bytes = ws_bytes
        stream = torch.cuda.current_stream().cuda_stream
        if dynamic is None:
            B.zero_opt_state_init(opt_state.data_ptr(), stream)
        else:
            B.zero_opt_state_init_dynamic(opt_state.data_ptr(), *dynamic, stream=stream)
        results = []
        n_steps = len(pb.grads) if steps is None else steps
        for t in range(n_steps):
            if t > 0:
                g_new, _ = grads_buf(pb.grads[t])
                g_dev.copy_(g_new)
            B.zero_shard_step(plan, hp, args, stream)
            results.append(B.step_result_from_bytes(host(result).tobytes()))
        opt = B.opt_state_from_bytes(host(opt_state).tobytes())
        cur = opt.cur if spec else 0
        out_m = host(master[cur])
        out_a = host(m[cur])
        out_v = host(v[cur])
        out_p = host(params)
        if check_guards:
            # pads and guard regions of every state slot stay untouched
            for arrs in (master, m, v):
                for k, t in enumerate(arrs):
                    if t is None:
                        continue
                    h = host(t).view(np.uint32)
                    assert (h[hi - lo:] == STATE_SENTINEL).all(), "state pad or guard written"
            assert (out_p[psi:] == PARAM_SENTINEL).all(), "params guard written"
            assert np.array_equal(out_p[:lo], pb.params[:lo]), "params of other owners written"
            assert np.array_equal(out_p[hi:psi], pb.params[hi:psi]), "params of other owners written"
        return GpuResult(out_m[:hi - lo].copy(), out_a[:hi - lo].copy(), out_v[:hi - lo].copy(),
                         out_p[:psi].copy(), results, opt, lo, hi)
    finally:
        B.zero_plan_destroy(plan)


@dataclasses.dataclass
class OracleResult:
    master: np.ndarray
    exp_avg: np.ndarray
    exp_avg_sq: np.ndarray
    params: np.ndarray     # full [psi]
    infos: list
    opt: oracle.Opt


def run_oracle(pb: Problem, hp: oracle.HP, lo=0, hi=None, steps=None, clip_overrides=None,
               threads=1, dynamic=None) -> OracleResult:
    """The oracle's step over flat range [lo, hi) (the owners of one call).
    Each info also records the loss scale after its step."""
    hi = pb.psi if hi is None else hi
    master = pb.master[lo:hi].copy()
    m = pb.exp_avg[lo:hi].copy()
    v = pb.exp_avg_sq[lo:hi].copy()
    params = pb.params.copy()
    sub_p = params[lo:hi].copy()
    opt = oracle.Opt()
    if dynamic is not None:
        opt = oracle.Opt(loss_scale=dynamic[0], growth_factor=dynamic[1], backoff_factor=dynamic[2],
                         growth_interval=dynamic[3])
    infos = []
    n_steps = len(pb.grads) if steps is None else steps
    for t in range(n_steps):
        G = np.ascontiguousarray(pb.grads[t][:, lo:hi])
        c = None if clip_overrides is None else clip_overrides[t]
        if hi > lo:
            infos.append(oracle.step(G, master, m, v, sub_p, hp, opt, clip_override=c,
                                     threads=threads))
            infos[-1]["loss_scale"] = opt.loss_scale
        else:
            infos.append({"overflow": 0})
            opt.t += 1
    params[lo:hi] = sub_p
    return OracleResult(master, m, v, params, infos, opt)


def to_oracle_hp(hp: B.HParams, storage: int = B.ZERO_STORAGE_FP16) -> oracle.HP:
    return oracle.HP(lr=hp.lr, beta1=hp.beta1, beta2=hp.beta2, eps=hp.eps,
                     weight_decay=hp.weight_decay, loss_scale=hp.loss_scale,
                     max_grad_norm=hp.max_grad_norm, average_over_nd=bool(hp.average_over_nd),
                     storage=storage)


def kernels_launched(fn):
    """Runs fn() and returns (its result, the names of the kernels of this
    library that it launched), from the library's own launch record
    (zero_recent_kernels: mangled C++ names, up to the last 64 launches)."""
    before = B.zero_launch_count()
    out = fn()
    torch.cuda.synchronize()
    n = B.zero_launch_count() - before
    assert 0 < n <= 64, f"{n} launches: the record holds the last 64"
    return out, set(B.zero_recent_kernels(n))
