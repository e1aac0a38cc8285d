"""The one-process-per-rank fused step (``ZeroDPPeerStep``) with two processes
sharing one GPU: each exports its gradient and parameter buffers with CUDA
IPC, maps the other's, and runs the step whose kernels read both gradient
buffers and store into both parameter buffers.  The process group is gloo:
the barriers around the step and the vote all-reduce run on the host after
the streams have drained, so neither process's kernels ever wait on the
other's.  Every rank's parameters and shard state must match the oracle."""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PSI, S, STEPS, ALIGN = 50_021, 1024.0, 3, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(nd, inject):
    sys.path.insert(0, ROOT)
    import oracle
    from zero_dp_partitioned_shard_b200 import synth
    p = oracle.plan(PSI, nd, ALIGN)
    grads = [synth.grads_f16(nd, PSI, seed=90 + t, std=1e-3, scale=S, stride=p.psi_pad, pad_fill=0.0)
             for t in range(STEPS)]
    if inject:
        grads[1][nd - 1, PSI // 5] = 0x7C00     # +inf in the last rank, owner 0's shard
    master = synth.normal_f32(PSI, seed=91, std=0.02)
    return p, grads, master


def _worker(rank, world, port, mode, clip, inject, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_dp_partitioned_shard_b200 import binding as B
    from zero_dp_partitioned_shard_b200 import distributed as D
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p, grads, master = _inputs(world, inject)
        hp = B.hparams(loss_scale=S, weight_decay=0.01, max_grad_norm=clip, mode=mode)
        step = D.ZeroDPPeerStep(PSI, hp, align=ALIGN, stage=2)
        step.load_master(torch.from_numpy(master).cuda())
        results = []
        for t in range(STEPS):
            step.grads.copy_(torch.from_numpy(grads[t][rank].view(np.float16)).cuda())
            res = step.step()
            results.append(bytes(B.step_result_from_bytes(res.cpu().numpy().tobytes())))
        torch.cuda.synchronize()
        s, n = B.zero_plan_shard(step.plan, rank)
        mm, ea, es = (x[:n].cpu().numpy() for x in step.live_state())
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), params=step.params[:PSI].cpu().view(torch.int16).numpy(),
                 master=mm, exp_avg=ea, exp_avg_sq=es, start=s, n=n,
                 results=np.frombuffer(b"".join(results), np.uint8))
        step.close()
    finally:
        dist.destroy_process_group()


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("mode,clip,inject", [(0, 0.0, False), (0, 0.0, True), (1, 0.05, False),
                                              (2, 0.05, True)],
                         ids=["speculative", "speculative-overflow", "two_pass-clip", "stash-clip-overflow"])
def test_two_processes_one_gpu_match_oracle(tmp_path, mode, clip, inject):
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    import oracle
    from _util import assert_f16_close, assert_f32_close
    from zero_dp_partitioned_shard_b200 import binding as B
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), mode, clip, inject, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    p, grads, master = _inputs(world, inject)
    outs = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    k = ctypes.sizeof(B.StepResult)
    res = [[B.StepResult.from_buffer_copy(o["results"].tobytes()[i * k:(i + 1) * k]) for i in range(STEPS)]
           for o in outs]
    clips = [r.clip_coef for r in res[0]]
    hp = oracle.HP(loss_scale=S, weight_decay=0.01, max_grad_norm=clip)
    m = master.copy()
    ea = np.zeros(PSI, np.float32)
    es = np.zeros(PSI, np.float32)
    P = oracle.float_to_half(master)
    opt = oracle.Opt()
    infos = []
    for t in range(STEPS):
        infos.append(oracle.step(np.ascontiguousarray(grads[t][:, :PSI]), m, ea, es, P, hp, opt,
                                 clip_override=clips[t] if clip > 0 else None))
    for r, o in enumerate(outs):
        assert_f16_close(o["params"].view(np.uint16), P, 1, f"rank {r} params")
        s, n = int(o["start"]), int(o["n"])
        assert_f32_close(o["master"], m[s:s + n], 2, f"rank {r} master")
        assert_f32_close(o["exp_avg"], ea[s:s + n], 2, f"rank {r} exp_avg")
        assert_f32_close(o["exp_avg_sq"], es[s:s + n], 2, f"rank {r} exp_avg_sq")
        for got, info in zip(res[r], infos):
            assert got.overflow == info["overflow"]
            if info["overflow"] == 0 and clip > 0:
                assert got.grad_norm == pytest.approx(info["grad_norm"], rel=1e-12)
    assert [r.overflow for r in res[0]] == [0, 1 if inject else 0, 0]
