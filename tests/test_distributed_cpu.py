"""The multi-process ZeRO-DP protocol on the CPU with gloo (world sizes 2 and
3): the library's collectives (exchange of gradient slices, vote
all-reduce, in-place all-gather) composed with the oracle as each process's
local compute must reproduce the single-process oracle step.

This checks the protocol's algebra -- the per-owner exchange layout, that the
global overflow decision and norm decompose into a sum of per-owner votes,
and the all-gather layout -- on host ranks; the GPU side of the same split
step is covered by tests/test_gpu_distributed.py."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


PSI, S = 50_021, 1024.0


def _problem(nd, inject):
    """Every rank's local fp16 gradient (seeded by rank) and the initial state."""
    sys.path.insert(0, ROOT)
    import oracle
    from zero_dp_partitioned_shard_b200 import synth
    p = oracle.plan(PSI, nd, 8)
    grads = synth.grads_f16(nd, PSI, seed=77, std=1e-3, scale=S, stride=p.psi_pad, pad_fill=0.0)
    if inject:
        grads[nd - 1, PSI // 3] = 0x7C00   # +inf in one rank's gradient
    master = synth.normal_f32(PSI, seed=78, std=0.02)
    return p, grads, master


def _worker(rank, world, port, inject, clip, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from zero_dp_partitioned_shard_b200 import distributed as D
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p, grads, master = _problem(world, inject)
        L = p.shard_len
        hp = oracle.HP(loss_scale=S, weight_decay=0.01, max_grad_norm=clip)
        # 1. exchange: this rank's gradient in, its shard's contributions out
        # bit patterns travel as fp16 tensors: the collectives only move bytes
        mine = torch.from_numpy(grads[rank].view(np.float16).copy())
        recv = torch.empty_like(mine)
        D.exchange_gradients(mine, recv)
        block = recv.numpy().view(np.uint16).reshape(world, L)
        s, n = p.shard(rank)
        # 2. local half: this owner's sum of squares and non-finite flag
        sumsq, bad = oracle.grad_sumsq(np.ascontiguousarray(block[:, :n]), hp) if n else (0.0, False)
        vote = torch.tensor([sumsq, 1.0 if bad else 0.0], dtype=torch.float64)
        # 3. the global vote
        D.reduce_vote(vote)
        skip = vote[1].item() != 0.0
        norm = math.sqrt(vote[0].item())
        c = np.float32(clip / norm) if (clip > 0 and norm > clip) else np.float32(1.0)
        # 4. own shard's update with the global decision
        m_shard = master[s:s + n].copy()
        mo = np.zeros(n, np.float32)
        vo = np.zeros(n, np.float32)
        P_full = torch.zeros(world * L, dtype=torch.float16)
        P_shard = oracle.float_to_half(m_shard)
        if not skip and n:
            _, _, bc1, bc2 = oracle.bias_corrections(hp, oracle.Opt())
            oracle.update_elements(np.ascontiguousarray(block[:, :n]), m_shard, mo, vo, P_shard, hp,
                                   float(c), bc1, bc2)
        P_full[rank * L:rank * L + n] = torch.from_numpy(P_shard.view(np.float16))
        # 5. all-gather of the fp16 shards
        D.gather_params(P_full, L)
        out.put((rank, skip, norm, float(c), m_shard, P_full.numpy().view(np.uint16)[:PSI].copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,inject,clip", [(2, False, 0.0), (3, False, 1e-3), (2, True, 0.0),
                                               (3, True, 1e-3)])
def test_gloo_protocol_matches_single_process_oracle(world, inject, clip):
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, inject, clip, out)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = sorted([out.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    # the single-process definition on the same inputs
    p, grads, master = _problem(world, inject)
    hp = oracle.HP(loss_scale=S, weight_decay=0.01, max_grad_norm=clip)
    ref_master = master.copy()
    ref_P = oracle.float_to_half(master)
    info = oracle.step(np.ascontiguousarray(grads[:, :PSI]), ref_master, np.zeros(PSI, np.float32),
                       np.zeros(PSI, np.float32), ref_P, hp, oracle.Opt(),
                       clip_override=results[0][3] if clip > 0 else None)
    assert all(r[1] == bool(info["overflow"]) for r in results)
    if not info["overflow"]:
        for r in results:
            assert r[2] == pytest.approx(info["grad_norm"], rel=1e-14)
    got_master = np.concatenate([r[4] for r in results])
    assert np.array_equal(got_master.view(np.uint32), ref_master.view(np.uint32))
    for r in results:   # every process holds the same, complete parameter buffer
        assert np.array_equal(r[5], ref_P)


def _tables_worker(rank, world, port, out):
    """Host side of the fused peer step: the IPC exports travel in rank order
    and become one gradient table (this process's own buffer at its rank) and
    the other ranks' parameter buffers as destinations."""
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_dp_partitioned_shard_b200 import distributed as D
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = (f"grad-export-{rank}".encode(), f"param-export-{rank}".encode())
        handles = D.exchange_handles(mine)
        opened_here = []

        def opener(h):        # stands in for zero_ipc_open: a distinct address per export
            opened_here.append(h)
            return 1_000_000 + int(h.decode().rsplit("-", 1)[1]) * 10 + (1 if h.startswith(b"param") else 0)

        own = (7, 8)
        grads, dests, opened = D.peer_tables(handles, rank, own, opener)
        vote = torch.tensor([float(rank + 1), 1.0 if rank == world - 1 else 0.0], dtype=torch.float64)
        D.reduce_vote(vote)
        out.put((rank, handles, grads, dests, opened, opened_here, vote.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_peer_tables_from_exchanged_exports(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_tables_worker, args=(r, world, port, out)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = sorted([out.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, handles, grads, dests, opened, opened_here, vote in got:
        assert [h[0] for h in handles] == [f"grad-export-{r}".encode() for r in range(world)]
        assert grads[rank] == 7                       # own gradient: not mapped, the local address
        others = [r for r in range(world) if r != rank]
        assert [grads[r] for r in others] == [1_000_000 + r * 10 for r in others]
        assert dests == [1_000_000 + r * 10 + 1 for r in others]   # other ranks' parameters, rank order
        assert sorted(opened) == sorted([1_000_000 + r * 10 for r in others] + dests)
        assert len(opened_here) == 2 * (world - 1)    # nothing of its own is mapped
        assert vote == [world * (world + 1) / 2, 1.0]
