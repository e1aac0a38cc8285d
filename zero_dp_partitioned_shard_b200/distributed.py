"""The ZeRO-DP step across real data-parallel processes, one process per GPU.

Process r owns shard r of the flat model state (fp32 master, momentum,
variance; "ZeRO memory optimization: training large models", trishampatil.com,
sections "ZeRO-1" to "ZeRO-3").  One step, as that page's figure under
"Forward/Backward Under ZeRO-3" and the upskillscore.com guide ("How it
works") describe it -- reduce-scatter the gradient, update the own shard,
all-gather the parameters -- maps onto:

1. ``exchange_gradients``: an all-to-all of the flat fp16 gradient's
   L-element slices, after which process o holds every rank's contribution to
   shard o as ``[Nd][L]`` (the reduce-scatter's input in the library's
   per-owner layout).  The sum itself is taken by the fused kernel in rank
   order and fp32, exactly as a single process does; an fp16 reduce-scatter
   would round every partial sum instead.
2. ``zero_shard_step_begin`` on the own shard (update or statistics pass).
3. ``reduce_vote``: a sum-all-reduce of the 16-byte vote, so every process
   sees the global overflow flag and the global sum of squares.
4. ``zero_shard_step_end`` (commit, or decision + in-place update).
5. ``gather_params``: an in-place all-gather of the fp16 shards into the full
   parameter buffer.

Per step a process sends (Nd-1)/Nd of the Psi gradient elements and receives
(Nd-1)/Nd of the Psi parameter elements: the 2 Psi of ZeRO stages 1 and 2.
The collectives are torch.distributed's (NCCL on GPUs); every arithmetic step
runs in the library's kernels.

``ZeroDPPeerStep`` moves the same 2 Psi without the exchange and the
all-gather: the processes map each other's gradient and parameter buffers
(CUDA IPC), and the step's kernels load the contributions to their shard
straight from every rank's gradient buffer and store each new parameter into
every rank's parameter buffer, over NVLink, in the same pass as the
arithmetic.  Stream-ordered collectives around the step keep the processes in
step; no kernel waits on another GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as B


def exchange_gradients(grad_flat: torch.Tensor, recv: torch.Tensor, group=None) -> None:
    """All-to-all of L-element slices: ``recv[r*L:(r+1)*L]`` receives rank r's
    slice of the shard this process owns.  Both tensors hold Nd*L fp16."""
    dist.all_to_all_single(recv, grad_flat, group=group)


def _nccl(group=None) -> bool:
    return dist.get_backend(group) == "nccl"


def reduce_vote(vote: torch.Tensor, group=None) -> None:
    """Sum of the fp64[2] votes of all processes, in place (through host
    memory for a process group without device collectives)."""
    if vote.is_cuda and not _nccl(group):
        host = vote.cpu()
        dist.all_reduce(host, op=dist.ReduceOp.SUM, group=group)
        vote.copy_(host)
        return
    dist.all_reduce(vote, op=dist.ReduceOp.SUM, group=group)


def stream_barrier(group=None, device=None) -> None:
    """Orders this process's later stream work after the work every process
    has enqueued so far: an all-reduce of one element on the stream (NCCL:
    it completes only once every process's stream has reached it), or a
    host barrier after draining the stream (other backends)."""
    if _nccl(group):
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        dist.all_reduce(torch.zeros(1, device=dev), group=group)
    else:
        torch.cuda.current_stream(device).synchronize()
        dist.barrier(group=group)


def exchange_handles(local, group=None) -> list:
    """Every process's ``local`` (picklable: here the IPC exports of its
    buffers), in rank order."""
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, local, group=group)
    return out


def peer_tables(handles, rank: int, own, opener):
    """Pointer tables from the exchanged exports: ``handles[r]`` = (gradient,
    parameters) exports of rank r, ``own`` = this process's (gradient,
    parameters) addresses, ``opener`` maps an export to a local address.
    Returns (rank_grads in rank order, param_dests of the other ranks in rank
    order, the addresses opened)."""
    rank_grads, dests, opened = [], [], []
    for r, (hg, hp) in enumerate(handles):
        if r == rank:
            rank_grads.append(own[0])
            continue
        g, p = opener(hg), opener(hp)
        opened += [g, p]
        rank_grads.append(g)
        dests.append(p)
    return rank_grads, dests, opened


def gather_params(params_full: torch.Tensor, shard_len: int, group=None) -> None:
    """In-place all-gather: rank r's fp16 shard at ``params_full[r*L:(r+1)*L]``
    ends up in every process's buffer at the same place."""
    r = dist.get_rank(group)
    dist.all_gather_into_tensor(params_full, params_full[r * shard_len:(r + 1) * shard_len],
                                group=group)


class ZeroDPStep:
    """The shard step of this process inside a data-parallel process group.

    ``psi`` parameters are partitioned over the group's Nd processes; this
    process owns shard ``rank``.  Buffers live on the current CUDA device:
    ``params`` (fp16, Nd*L elements, the first psi are the model's) is the
    all-gathered parameter buffer after every step.
    """

    def __init__(self, psi: int, hp: B.HParams, *, group=None, align: int = 256,
                 bucket: int = 0, stage: int = 2, device=None, storage: int = B.ZERO_STORAGE_FP16):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.hp = hp
        self.storage = storage
        self.dtype = torch.bfloat16 if storage == B.ZERO_STORAGE_BF16 else torch.float16
        self.plan = B.zero_plan(psi, self.world, stage=stage, align_elems=align, bucket_elems=bucket)
        info = B.zero_plan_query(self.plan)
        self.psi, self.L, self.psi_pad = psi, info.shard_len, info.psi_pad
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE
        f32 = lambda: torch.zeros(self.L, dtype=torch.float32, device=dev)
        self.master = [f32(), f32() if spec else None]
        self.exp_avg = [f32(), f32() if spec else None]
        self.exp_avg_sq = [f32(), f32() if spec else None]
        self.stash = f32() if hp.mode == B.ZERO_MODE_STASH else None
        self.params = torch.zeros(self.psi_pad, dtype=self.dtype, device=dev)
        self.recv = torch.zeros(self.psi_pad, dtype=self.dtype, device=dev)
        self.opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device=dev)
        self.result = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device=dev)
        ptr = lambda t: t.data_ptr() if t is not None else 0
        self.args = B.step_args(
            grads=self.recv.data_ptr(), grad_rank_stride=self.L, grad_layout=B.ZERO_GRADS_PER_OWNER,
            owner_first=self.rank, owner_count=1, master=tuple(map(ptr, self.master)),
            exp_avg=tuple(map(ptr, self.exp_avg)), exp_avg_sq=tuple(map(ptr, self.exp_avg_sq)),
            params=self.params.data_ptr(), grad_stash=ptr(self.stash),
            opt_state=self.opt_state.data_ptr(), result=self.result.data_ptr(), storage=storage)
        ws_bytes = B.zero_workspace_bytes(self.plan, hp, self.args)
        self.workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
        self.args.workspace = self.workspace.data_ptr()
        self.args.workspace_bytes = ws_bytes
        off = B.ZERO_VOTE_OFFSET
        self.vote = self.workspace[off:off + 16].view(torch.float64)
        B.zero_opt_state_init(self.opt_state.data_ptr(), self._stream())

    def _stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    def load_master(self, master_full: torch.Tensor) -> None:
        """Initialise this process's fp32 shard from the full fp32 master
        (any device) and all-gather the 16-bit cast into ``params``."""
        s, n = B.zero_plan_shard(self.plan, self.rank)
        self.master[0].zero_()
        self.master[0][:n].copy_(master_full[s:s + n])
        B.zero_cast_params(self.plan, self.master[0].data_ptr(), self.params.data_ptr(), self.rank, 1,
                           self._stream(), storage=self.storage)
        gather_params(self.params, self.L, self.group)

    def step(self, grad_flat: torch.Tensor) -> torch.Tensor:
        """One ZeRO-DP step from this process's local 16-bit gradient (Nd*L
        elements, pads zero, the storage format's dtype).  Returns the device
        result struct (raw bytes)."""
        assert grad_flat.dtype == self.dtype and grad_flat.numel() == self.psi_pad
        stream = self._stream()
        exchange_gradients(grad_flat, self.recv, self.group)
        B.zero_shard_step_begin(self.plan, self.hp, self.args, stream)
        reduce_vote(self.vote, self.group)
        B.zero_shard_step_end(self.plan, self.hp, self.args, stream)
        gather_params(self.params, self.L, self.group)
        return self.result

    def live_state(self):
        """(master, exp_avg, exp_avg_sq) of the live slot of this shard."""
        cur = B.opt_state_from_bytes(self.opt_state.cpu().numpy().tobytes()).cur
        pick = lambda pair: pair[cur] if pair[1] is not None else pair[0]
        return pick(self.master), pick(self.exp_avg), pick(self.exp_avg_sq)

    def close(self) -> None:
        B.zero_plan_destroy(self.plan)
        self.plan = 0


class ZeroDPPeerStep:
    """The shard step of this process with the reduce-scatter and the
    all-gather done by the step's own kernels over peer memory.

    ``grads`` (16-bit, Nd*L elements) is this process's gradient, written by
    its backward pass before ``step``; ``params`` (Nd*L elements, the first psi
    the model's) holds every owner's new parameters after ``step``.  Both are
    mapped into every other process of the group.  One step:

    1. ``stream_barrier``: every process's gradient is complete;
    2. ``zero_shard_step_begin`` on the own shard, reading the Nd gradients
       through the peer table (SPECULATIVE: the update, which also stores the
       new parameters into every process's ``params``);
    3. ``reduce_vote`` (the global skip / norm decision);
    4. ``zero_shard_step_end`` (TWO_PASS / STASH: the update and its stores;
       SPECULATIVE: on a skip, the old parameters are stored back);
    5. ``stream_barrier``: every process's parameters are complete and its
       gradient buffer may be overwritten.
    """

    def __init__(self, psi: int, hp: B.HParams, *, group=None, align: int = 256,
                 bucket: int = 0, stage: int = 2, device=None, storage: int = B.ZERO_STORAGE_FP16):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.hp = hp
        self.storage = storage
        self.plan = B.zero_plan(psi, self.world, stage=stage, align_elems=align, bucket_elems=bucket)
        info = B.zero_plan_query(self.plan)
        self.psi, self.L, self.psi_pad = psi, info.shard_len, info.psi_pad
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        h16 = torch.bfloat16 if storage == B.ZERO_STORAGE_BF16 else torch.float16
        spec = hp.mode == B.ZERO_MODE_SPECULATIVE
        f32 = lambda: torch.zeros(self.L, dtype=torch.float32, device=dev)
        self.master = [f32(), f32() if spec else None]
        self.exp_avg = [f32(), f32() if spec else None]
        self.exp_avg_sq = [f32(), f32() if spec else None]
        self.stash = f32() if hp.mode == B.ZERO_MODE_STASH else None
        self.grads = torch.zeros(self.psi_pad, dtype=h16, device=dev)
        self.params = torch.zeros(self.psi_pad, dtype=h16, device=dev)
        self.opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device=dev)
        self.result = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        mine = (B.zero_ipc_export(self.grads.data_ptr()), B.zero_ipc_export(self.params.data_ptr()))
        handles = exchange_handles(mine, group)
        rank_grads, self.dests, self._opened = peer_tables(
            handles, self.rank, (self.grads.data_ptr(), self.params.data_ptr()), B.zero_ipc_open)
        self.peers = B.peer_args(rank_grads, self.dests)
        ptr = lambda t: t.data_ptr() if t is not None else 0
        self.args = B.step_args(
            grads=0, grad_rank_stride=0, grad_layout=B.ZERO_GRADS_FULL,
            owner_first=self.rank, owner_count=1, master=tuple(map(ptr, self.master)),
            exp_avg=tuple(map(ptr, self.exp_avg)), exp_avg_sq=tuple(map(ptr, self.exp_avg_sq)),
            params=self.params.data_ptr(), grad_stash=ptr(self.stash),
            opt_state=self.opt_state.data_ptr(), result=self.result.data_ptr(), storage=storage)
        B.attach_peers(self.args, self.peers)
        ws_bytes = B.zero_workspace_bytes(self.plan, hp, self.args)
        self.workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
        self.args.workspace = self.workspace.data_ptr()
        self.args.workspace_bytes = ws_bytes
        off = B.ZERO_VOTE_OFFSET
        self.vote = self.workspace[off:off + 16].view(torch.float64)
        B.zero_opt_state_init(self.opt_state.data_ptr(), self._stream())

    def _stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    def load_master(self, master_full: torch.Tensor) -> None:
        """Initialises this process's fp32 shard from the full fp32 master and
        stores its 16-bit cast into every process's ``params``."""
        s, n = B.zero_plan_shard(self.plan, self.rank)
        self.master[0].zero_()
        self.master[0][:n].copy_(master_full[s:s + n])
        for dst in [self.params.data_ptr()] + list(self.dests):
            B.zero_cast_params(self.plan, self.master[0].data_ptr(), dst, self.rank, 1, self._stream(),
                               storage=self.storage)
        stream_barrier(self.group, self.device)

    def step(self) -> torch.Tensor:
        """One ZeRO-DP step from the gradients in every process's ``grads``.
        Returns the device result struct (raw bytes)."""
        stream = self._stream()
        stream_barrier(self.group, self.device)
        B.zero_shard_step_begin(self.plan, self.hp, self.args, stream)
        reduce_vote(self.vote, self.group)
        B.zero_shard_step_end(self.plan, self.hp, self.args, stream)
        stream_barrier(self.group, self.device)
        return self.result

    def live_state(self):
        """(master, exp_avg, exp_avg_sq) of the live slot of this shard."""
        cur = B.opt_state_from_bytes(self.opt_state.cpu().numpy().tobytes()).cur
        pick = lambda pair: pair[cur] if pair[1] is not None else pair[0]
        return pick(self.master), pick(self.exp_avg), pick(self.exp_avg_sq)

    def close(self) -> None:
        """Unmaps the peers' buffers (after every process has finished with
        them) and releases the plan."""
        stream_barrier(self.group, self.device)
        torch.cuda.synchronize(self.device)
        for p in self._opened:
            B.zero_ipc_close(p)
        self._opened = []
        dist.barrier(group=self.group)
        B.zero_plan_destroy(self.plan)
        self.plan = 0
