"""The benchmark's sharded harness (``bench.py --sharded``) on the CPU: two
gloo ranks, each owning one shard, with the oracle as the local compute.

The harness is what the GPU run shares with this test: the warm-up, the
barrier-bracketed timed region and the slowest rank's time (``sharded_loop``),
and the volumes and bounds of ``sharded_report``, checked against the
accounting of ``zero_state_bytes``.  The local step is the one-process-per-GPU
protocol of the library's collectives -- exchange of gradient slices, vote
all-reduce, all-gather of the 16-bit shards -- so after warm-up plus timed
steps every rank must hold the single-process oracle's parameters."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PSI, S, STEPS, WARMUP = 30_011, 1024.0, 2, 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(nd):
    sys.path.insert(0, ROOT)
    import oracle
    from zero_dp_partitioned_shard_b200 import synth
    p = oracle.plan(PSI, nd, 256)
    grads = synth.grads_f16(nd, PSI, seed=61, std=1e-3, scale=S, stride=p.psi_pad, pad_fill=0.0)
    master = synth.normal_f32(PSI, seed=62, std=0.02)
    return p, grads, master


class OracleOwnerStep:
    """One process's step of the sharded protocol, the oracle doing the
    arithmetic of its own shard (speculative-free: the vote decides first)."""

    def __init__(self, rank, world, hp):
        import oracle
        import torch
        self.O, self.T = oracle, torch
        self.p, grads, master = _problem(world)
        self.rank, self.world, self.hp = rank, world, hp
        self.L = self.p.shard_len
        s, n = self.p.shard(rank)
        self.s, self.n = s, n
        self.mine = torch.from_numpy(grads[rank].view(np.float16).copy())
        self.master = master[s:s + n].copy()
        self.m = np.zeros(n, np.float32)
        self.v = np.zeros(n, np.float32)
        self.opt = oracle.Opt()
        self.P_full = torch.from_numpy(np.zeros(world * self.L, np.uint16).view(np.float16))
        self.P_full[:PSI] = torch.from_numpy(oracle.float_to_half(master).view(np.float16))
        self.calls = 0

    def __call__(self, k):
        from zero_dp_partitioned_shard_b200 import distributed as D
        O, T = self.O, self.T
        recv = T.empty_like(self.mine)
        D.exchange_gradients(self.mine, recv)
        block = np.ascontiguousarray(recv.numpy().view(np.uint16).reshape(self.world, self.L)[:, :self.n])
        sumsq, bad = O.grad_sumsq(block, self.hp) if self.n else (0.0, False)
        vote = T.tensor([sumsq, 1.0 if bad else 0.0], dtype=T.float64)
        D.reduce_vote(vote)
        assert vote[1].item() == 0.0
        P_shard = O.float_to_half(self.master)
        b1, b2, bc1, bc2 = O.bias_corrections(self.hp, self.opt)
        if self.n:
            O.update_elements(block, self.master, self.m, self.v, P_shard, self.hp, 1.0, bc1, bc2)
        self.opt = O.Opt(self.opt.t + 1, b1, b2)
        self.P_full[self.rank * self.L:self.rank * self.L + self.n] = T.from_numpy(P_shard.view(np.float16))
        D.gather_params(self.P_full, self.L)
        self.calls += 1


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from zero_dp_partitioned_shard_b200 import binding as B
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        hp = oracle.HP(loss_scale=S, weight_decay=0.01)
        step = OracleOwnerStep(rank, world, hp)
        ms_max = bench.sharded_loop(step, STEPS, WARMUP, world, bench.HostTimer(), device="cpu")
        rep = bench.sharded_report(PSI, world, step.L, STEPS, ms_max, 2.0 + rank, "nccl", 6500.0,
                                   B.zero_state_bytes(PSI, world, 2, 256))
        out.put((rank, step.calls, ms_max, rep, step.P_full.numpy().view(np.uint16)[:PSI].copy()))
    finally:
        dist.destroy_process_group()


def test_sharded_harness_on_two_gloo_ranks():
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = sorted([out.get(timeout=180) for _ in range(world)], key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p, grads, master = _problem(world)
    L = p.shard_len
    # every rank ran warm-up + timed steps and agrees on the slowest time
    assert all(g[1] == WARMUP + STEPS for g in got)
    assert got[0][2] == got[1][2] > 0
    for _, _, ms_max, rep, _ in got:
        ex, acc = rep["exchange"], rep["accounting"]
        # 2 (Nd-1) L elements each way: gradient slices out, own parameters out
        assert ex["elements_each_way"] == 2 * (world - 1) * L
        assert ex["bytes_each_way"] == 4 * (world - 1) * L
        assert ex["link_bound_ms"] == pytest.approx(4 * (world - 1) * L / 770e9 * 1e3)
        # the pages' 2 Psi per step (stages 1-2), and its ring share (Nd-1)/Nd
        assert acc["comm_elems_pages"] == 2 * PSI
        assert acc["comm_elems_ring"] == pytest.approx(2 * PSI * (world - 1) / world)
        assert acc["exchanged_over_ring"] == pytest.approx(world * L / PSI)   # padding only
        assert rep["step_ms"] == pytest.approx(ms_max / STEPS)
        assert rep["update"]["alg_bytes"] == L * (2 * world + 26)
    # the parameters every rank holds equal the single-process oracle's
    hp = oracle.HP(loss_scale=S, weight_decay=0.01)
    ref_master = master.copy()
    ref_m = np.zeros(PSI, np.float32)
    ref_v = np.zeros(PSI, np.float32)
    ref_P = oracle.float_to_half(master)
    opt = oracle.Opt()
    for _ in range(WARMUP + STEPS):
        oracle.step(np.ascontiguousarray(grads[:, :PSI]), ref_master, ref_m, ref_v, ref_P, hp, opt)
    for g in got:
        assert np.array_equal(g[4], ref_P)
    assert math.isfinite(got[0][3]["exchange"]["link_frac"])
