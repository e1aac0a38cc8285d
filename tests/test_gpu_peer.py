"""GPU parity of the fused reduce-scatter + update + all-gather over peer
tables, with the Nd ranks emulated in one process on one GPU: every rank has
its own gradient buffer and its own full parameter buffer, and each rank's
call reads all gradient buffers through the table and stores its new
parameters into every rank's parameter buffer.  The per-rank calls are the
split step (begin, the votes summed on the host in rank order as the
all-reduce would, end), in stream order, so no kernel waits on another.
Every rank's parameter buffer and every shard's state must match the oracle
at the bars of the other parity tests, and the strided call on the same data
exactly."""
import math

import numpy as np
import pytest
import torch

from _gpu import (CANARY, INF16, NAN16, PARAM_SENTINEL, STATE_SENTINEL, dev, host, kernels_launched,
                  make_problem, run_gpu, run_oracle, to_oracle_hp)
from _util import assert_bf16_close, assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B

pytestmark = pytest.mark.gpu

MODES = [B.ZERO_MODE_SPECULATIVE, B.ZERO_MODE_TWO_PASS, B.ZERO_MODE_STASH]
MODE_NAMES = {0: "speculative", 1: "two_pass", 2: "stash"}


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def run_peer(pb, hp, *, per_rank=True, misalign=False, dynamic=None, stage=2):
    """Runs pb's steps through peer tables.  per_rank: one call per owner
    (split step, host-summed vote); else one call over all owners.  Returns
    (per-rank params [nd][psi], master/m/v of the live slots concatenated
    over the owners [psi], per-step results of call 0, per-call results)."""
    nd, psi = pb.nd, pb.psi
    plan = B.zero_plan(psi, nd, stage=stage, align_elems=pb.align, bucket_elems=pb.bucket)
    try:
        info = B.zero_plan_query(plan)
        L, psi_pad = info.shard_len, info.psi_pad
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE
        off = 1 if misalign else 0
        nan16 = NAN16[pb.storage]
        # one gradient buffer and one full parameter buffer per rank
        g_store = [dev(np.full(psi_pad + off + CANARY, nan16, np.uint16)) for _ in range(nd)]
        p_h = np.full(psi + off + CANARY, PARAM_SENTINEL, np.uint16)
        p_h[off:off + psi] = pb.params
        p_store = [dev(p_h) for _ in range(nd)]
        g_ptr = [t.data_ptr() + 2 * off for t in g_store]
        p_ptr = [t.data_ptr() + 2 * off for t in p_store]

        def load_grads(t):
            G = pb.grads[t]
            for r in range(nd):
                row = np.full(psi_pad + off + CANARY, nan16, np.uint16)
                row[off:off + G.shape[1]] = G[r]
                g_store[r].copy_(torch.from_numpy(row))

        calls = [(r, 1) for r in range(nd)] if per_rank else [(0, nd)]
        C = []
        stream = torch.cuda.current_stream().cuda_stream
        for o0, oc in calls:
            lo, hi = o0 * L, max(o0 * L, min((o0 + oc) * L, psi))

            def state_buf(src):
                h = np.full(oc * L + CANARY, STATE_SENTINEL, np.uint32)
                if src is not None:
                    h[:hi - lo] = src[lo:hi].view(np.uint32)
                return dev(h.view(np.float32))

            c = dict(o0=o0, oc=oc, lo=lo, hi=hi,
                     master=[state_buf(pb.master), state_buf(None) if spec else None],
                     m=[state_buf(pb.exp_avg), state_buf(None) if spec else None],
                     v=[state_buf(pb.exp_avg_sq), state_buf(None) if spec else None],
                     stash=state_buf(None) if hp.mode == B.ZERO_MODE_STASH else None,
                     opt=torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device="cuda"),
                     res=torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device="cuda"), results=[])
            ptr = lambda t: t.data_ptr() if t is not None else 0
            own = o0 if per_rank else 0
            dests = [p_ptr[q] for q in range(nd) if q != own]
            args = B.step_args(grads=0, grad_rank_stride=0, owner_first=o0, owner_count=oc,
                               master=tuple(map(ptr, c["master"])), exp_avg=tuple(map(ptr, c["m"])),
                               exp_avg_sq=tuple(map(ptr, c["v"])), params=p_ptr[own],
                               grad_stash=ptr(c["stash"]), opt_state=c["opt"].data_ptr(),
                               result=c["res"].data_ptr(), storage=pb.storage)
            B.attach_peers(args, B.peer_args(g_ptr, dests))
            nb = B.zero_workspace_bytes(plan, hp, args)
            c["ws"] = torch.zeros(nb + 256, dtype=torch.uint8, device="cuda")
            args.workspace, args.workspace_bytes = c["ws"].data_ptr(), nb
            c["args"] = args
            if dynamic is None:
                B.zero_opt_state_init(c["opt"].data_ptr(), stream)
            else:
                B.zero_opt_state_init_dynamic(c["opt"].data_ptr(), *dynamic, stream=stream)
            C.append(c)

        for t in range(len(pb.grads)):
            load_grads(t)
            if per_rank:
                for c in C:
                    B.zero_shard_step_begin(plan, hp, c["args"], stream)
                torch.cuda.synchronize()
                votes = [c["ws"][B.ZERO_VOTE_OFFSET:B.ZERO_VOTE_OFFSET + 16].view(torch.float64).cpu()
                         for c in C]
                total = votes[0].clone()
                for v in votes[1:]:
                    total += v
                for c in C:
                    c["ws"][B.ZERO_VOTE_OFFSET:B.ZERO_VOTE_OFFSET + 16].view(torch.float64).copy_(total)
                for c in C:
                    B.zero_shard_step_end(plan, hp, c["args"], stream)
            else:
                B.zero_shard_step(plan, hp, C[0]["args"], stream)
            for c in C:
                c["results"].append(B.step_result_from_bytes(host(c["res"]).tobytes()))

        params = [host(t)[off:off + psi].copy() for t in p_store]
        for t in p_store:
            h = host(t)
            assert (h[:off] == PARAM_SENTINEL).all() and (h[off + psi:] == PARAM_SENTINEL).all(), \
                "parameter guard written"
        master = np.zeros(psi, np.float32)
        m = np.zeros(psi, np.float32)
        v = np.zeros(psi, np.float32)
        for c in C:
            opt = B.opt_state_from_bytes(host(c["opt"]).tobytes())
            cur = opt.cur if spec else 0
            n = c["hi"] - c["lo"]
            for dst, pair in ((master, c["master"]), (m, c["m"]), (v, c["v"])):
                live = host(pair[cur])
                dst[c["lo"]:c["hi"]] = live[:n]
                for buf in pair:
                    if buf is not None:
                        assert (host(buf).view(np.uint32)[n:] == STATE_SENTINEL).all(), "state pad written"
            c["opt_final"] = opt
        return params, master, m, v, C
    finally:
        B.zero_plan_destroy(plan)


def check(pb, hp, params, master, m, v, C, o, what):
    close16 = assert_bf16_close if pb.storage == B.ZERO_STORAGE_BF16 else assert_f16_close
    for r, P in enumerate(params):
        close16(P, o.params, 1, f"{what}: rank {r} params")
    assert_f32_close(master, o.master, 2, what + " master")
    assert_f32_close(m, o.exp_avg, 2, what + " exp_avg")
    assert_f32_close(v, o.exp_avg_sq, 2, what + " exp_avg_sq")
    for c in C:
        assert c["opt_final"].t == o.opt.t, what
        for r, info in zip(c["results"], o.infos):
            assert r.overflow == info["overflow"], what
            if info["overflow"] == 0 and "grad_norm" in info and not math.isnan(r.grad_norm):
                assert r.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12), what


def clip_of(hp):
    return None if hp.max_grad_norm <= 0 else hp.max_grad_norm


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
@pytest.mark.parametrize("storage", [B.ZERO_STORAGE_FP16, B.ZERO_STORAGE_BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("per_rank", [True, False], ids=["per_rank", "one_call"])
def test_peer_step_matches_oracle(mode, storage, per_rank):
    pb = make_problem(300_007, 4, align=256, bucket=65_536, steps=3, seed=61, S=1024.0,
                      random_state=True, storage=storage)
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01,
                   max_grad_norm=0.0 if mode == B.ZERO_MODE_SPECULATIVE else 0.05, mode=mode)
    params, master, m, v, C = run_peer(pb, hp, per_rank=per_rank)
    o = run_oracle(pb, to_oracle_hp(hp, storage),
                   clip_overrides=None if not clip_of(hp) else [r.clip_coef for r in C[0]["results"]])
    check(pb, hp, params, master, m, v, C, o, f"peer {MODE_NAMES[mode]}")
    if clip_of(hp):
        assert all(r.clip_coef < 1.0 for r in C[0]["results"])
        # every rank took the same global clip coefficient
        for c in C[1:]:
            assert [r.clip_coef for r in c["results"]] == [r.clip_coef for r in C[0]["results"]]


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_overflow_anywhere_skips_every_rank(mode):
    """A +inf in one rank's contribution to another rank's shard: every rank
    skips, and every rank's parameter buffer is left as it was."""
    pb = make_problem(100_003, 4, align=8, steps=3, seed=62, S=1024.0, random_state=True)
    L = -(-100_003 // (4 * 8)) * 8
    pb.grads[1][2, 3 * L + 17] = INF16[B.ZERO_STORAGE_FP16]   # rank 2, owner 3's shard
    hp = B.hparams(loss_scale=1024.0, mode=mode, max_grad_norm=0.0 if mode == 0 else 1.0)
    params, master, m, v, C = run_peer(pb, hp)
    o = run_oracle(pb, to_oracle_hp(hp),
                   clip_overrides=None if mode == 0 else [r.clip_coef for r in C[0]["results"]])
    check(pb, hp, params, master, m, v, C, o, "peer overflow")
    for c in C:
        assert [r.overflow for r in c["results"]] == [0, 1, 0]


@pytest.mark.parametrize("psi,nd,align", [(1, 1, 1), (7, 3, 1), (4097, 2, 8), (100_003, 7, 16),
                                          (33, 64, 1), (65_536, 64, 8)])
@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_ragged_sizes(psi, nd, align, mode):
    """Empty owners, one rank (no destinations), Nd = 2 (the stash pipeline
    with destinations), a full table of 64 ranks, scalar paths."""
    pb = make_problem(psi, nd, align=align, steps=2, seed=psi % 31 + nd, S=256.0, random_state=True)
    hp = B.hparams(loss_scale=256.0, weight_decay=0.01, mode=mode)
    params, master, m, v, C = run_peer(pb, hp)
    check(pb, hp, params, master, m, v, C, run_oracle(pb, to_oracle_hp(hp)), f"peer ragged {psi}/{nd}")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_unaligned_buffers_take_the_scalar_path(mode):
    pb = make_problem(50_001, 4, align=8, steps=2, seed=63, S=1024.0)
    hp = B.hparams(loss_scale=1024.0, mode=mode)
    params, master, m, v, C = run_peer(pb, hp, misalign=True)
    check(pb, hp, params, master, m, v, C, run_oracle(pb, to_oracle_hp(hp)), "peer unaligned")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_tables_equal_the_strided_call(mode):
    """The same data through the strided all-owner call and through peer
    tables: bit-identical state and parameters."""
    pb = make_problem(200_003, 8, align=256, bucket=50_000, steps=2, seed=64, S=1024.0, random_state=True)
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, mode=mode,
                   max_grad_norm=0.0 if mode == 0 else 0.05)
    g = run_gpu(pb, hp, stage=2)
    params, master, m, v, C = run_peer(pb, hp, per_rank=False)
    for P in params:
        assert np.array_equal(P, g.params)
    for a, b in ((master, g.master), (m, g.exp_avg), (v, g.exp_avg_sq)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.fixture(scope="module")
def pipeline_sized_problem():
    psi = 33_554_437
    pb = make_problem(psi, 8, align=256, steps=3, seed=66, S=1024.0, random_state=True)
    pb.grads[1][5, 7 * (psi // 8) + 1234] = INF16[B.ZERO_STORAGE_FP16]
    return pb


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_pipeline_launch(mode, pipeline_sized_problem):
    """One call over all 8 owners, large enough for the bulk-copy pipeline
    (at least 64 tiles of 1024 elements per CTA at 3 CTAs on each of 148
    SMs: 29,097,984 elements), so the producer copies every rank row from its
    own table entry and the consumers store into all 8 parameter buffers.
    Ragged Psi, an inf in the second step: bit-identical to the strided call
    on the same data, and within the oracle's bars."""
    pb = pipeline_sized_problem
    hp = B.hparams(loss_scale=1024.0, weight_decay=0.01, mode=mode,
                   max_grad_norm=0.0 if mode == 0 else 0.05)
    (params, master, m, v, C), names = kernels_launched(lambda: run_peer(pb, hp, per_rank=False))
    if torch.cuda.get_device_properties(0).multi_processor_count <= 148:
        assert any("zs_update_pipe_kernel" in n for n in names), sorted(names)
        # the kernel the bench line names for this launch is the one that ran
        import bench
        assert any(bench.update_kernel_name(8, mode, True, pb.psi) in n for n in names), sorted(names)
    assert [r.overflow for r in C[0]["results"]] == [0, 1, 0]
    g = run_gpu(pb, hp, stage=2)
    for P in params:
        assert np.array_equal(P, g.params)
    for a, b in ((master, g.master), (m, g.exp_avg), (v, g.exp_avg_sq)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    o = run_oracle(pb, to_oracle_hp(hp), clip_overrides=None if mode == 0 else [r.clip_coef for r in C[0]["results"]])
    check(pb, hp, params, master, m, v, C, o, f"peer pipeline {MODE_NAMES[mode]}")


@pytest.mark.parametrize("mode", MODES, ids=lambda m: MODE_NAMES[m])
def test_peer_dynamic_loss_scaling(mode):
    S0 = 2.0 ** 12
    pb = make_problem(70_001, 4, align=256, steps=5, seed=65, S=S0)
    pb.grads[2][1, 5_000] = INF16[B.ZERO_STORAGE_FP16]
    dyn = (S0, 2.0, 0.5, 2)
    hp = B.hparams(loss_scale=1.0, mode=mode, max_grad_norm=0.0 if mode == 0 else 10.0)
    params, master, m, v, C = run_peer(pb, hp, dynamic=dyn)
    o = run_oracle(pb, to_oracle_hp(hp), dynamic=dyn,
                   clip_overrides=None if mode == 0 else [r.clip_coef for r in C[0]["results"]])
    check(pb, hp, params, master, m, v, C, o, "peer dynamic")
    for c in C:
        assert [r.loss_scale for r in c["results"]] == [i["loss_scale"] for i in o.infos]
