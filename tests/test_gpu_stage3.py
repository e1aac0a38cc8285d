"""Stage-3 on-demand gathering on the GPU: zero_gather_tensors against the
oracle's definition (compact and in place, odd tensor sizes and alignments
so pieces take both the vector and the scalar path), and the layer schedule's
forward and backward passes -- every layer's gathered parameters equal the
oracle's, and the gathered volume plus the gradient reduce-scatter is the
3 Psi the pages give for stage 3."""
import numpy as np
import pytest
import torch

import oracle
from _gpu import dev, host
from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import stage3, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _shards(p, ref):
    host_sh, dev_sh = [], []
    for r in range(p.nd):
        s, n = p.shard(r)
        sh = np.full(p.shard_len, 0x7E00, np.uint16)
        sh[:n] = ref[s:s + n]
        host_sh.append(sh)
        dev_sh.append(dev(sh))
    return host_sh, dev_sh


GATHERS = {"kernel": B.zero_gather_tensors, "dma": B.zero_gather_tensors_dma}


@pytest.mark.parametrize("engine", sorted(GATHERS))
@pytest.mark.parametrize("nd,align,seed", [(3, 1, 1), (8, 8, 2), (4, 256, 3), (16, 256, 4)])
def test_gather_tensors_matches_oracle(nd, align, seed, engine):
    gather = GATHERS[engine]
    rs = np.random.default_rng(seed)
    sizes = [int(x) for x in rs.integers(1, 40_000, size=40)] + [7, 1600, 4800, 13]
    psi = sum(sizes)
    p = oracle.plan(psi, nd, align)
    ref = synth.fp16_bits(synth.normal_f32(psi, seed=seed, std=1.0))
    host_sh, dev_sh = _shards(p, ref)
    plan = B.zero_plan(psi, nd, stage=3, align_elems=align, tensor_sizes=sizes)
    stream = torch.cuda.current_stream().cuda_stream
    try:
        for first, count in ((0, len(sizes)), (3, 5), (len(sizes) - 4, 4), (10, 1), (0, 0)):
            want = np.zeros(max(1, psi), np.uint16)
            n_ref = oracle.gather_tensors(host_sh, p, sizes, first, count, want, True)
            out = dev(np.full(max(1, n_ref) + 64, 0x7DDD, np.uint16))
            n = gather(plan, first, count, [t.data_ptr() for t in dev_sh], out.data_ptr(), True, stream)
            got = host(out)
            assert n == n_ref
            assert np.array_equal(got[:n], want[:n]) and (got[n:] == 0x7DDD).all()
        # in place, with one owner's part already there (NULL shard)
        skip = nd // 2
        full_init = np.full(psi, 0x1234, np.uint16)
        s0, n0 = p.shard(skip)
        full_init[s0:s0 + n0] = ref[s0:s0 + n0]
        full = dev(full_init)
        ptrs = [0 if r == skip else dev_sh[r].data_ptr() for r in range(nd)]
        gather(plan, 2, len(sizes) - 5, ptrs, full.data_ptr(), False, stream)
        want = full_init.copy()
        oracle.gather_tensors([None if r == skip else host_sh[r] for r in range(nd)], p, sizes,
                              2, len(sizes) - 5, want, False)
        assert np.array_equal(host(full), want)
        with pytest.raises(B.ZeroError):   # compact needs every owner's shard
            gather(plan, 0, len(sizes), ptrs, out.data_ptr(), True, stream)
    finally:
        B.zero_plan_destroy(plan)


@pytest.mark.parametrize("engine", ["kernel", "dma"])
def test_layer_schedule_forward_backward_and_volume(engine):
    n_layer, d = 6, 96
    sizes = synth.transformer_tensor_sizes(n_layer, d, 1000, 64)
    psi, nd = sum(sizes), 4
    p = oracle.plan(psi, nd, 8)
    ref = synth.fp16_bits(synth.normal_f32(psi, seed=9, std=0.02))
    host_sh, dev_sh = _shards(p, ref)
    layers = [(12 * i, 12) for i in range(n_layer)] + [(12 * n_layer, 4)]
    plan = B.zero_plan(psi, nd, stage=3, align_elems=8, tensor_sizes=sizes)
    try:
        sched = stage3.LayerGatherSchedule(plan, layers, [t.data_ptr() for t in dev_sh], sizes, engine=engine)
        seen = {"fwd": [], "bwd": []}
        sched.forward(lambda i, w: seen["fwd"].append((i, w.clone())))
        sched.backward(lambda i, w: seen["bwd"].append((i, w.clone())))
        torch.cuda.synchronize()
        assert [i for i, _ in seen["fwd"]] == list(range(len(layers)))
        assert [i for i, _ in seen["bwd"]] == list(reversed(range(len(layers))))
        for pas in ("fwd", "bwd"):
            for i, w in seen[pas]:
                first, count = layers[i]
                want = np.zeros(psi, np.uint16)
                n = oracle.gather_tensors(host_sh, p, sizes, first, count, want, True)
                assert np.array_equal(w.cpu().numpy().view(np.uint16), want[:n]), (pas, i)
        # two parameter gathers per step plus the gradient reduce-scatter
        assert sched.gathered == 2 * psi
        assert sched.gathered + psi == oracle.state_bytes(psi, nd, 3)["comm_elems"]
    finally:
        B.zero_plan_destroy(plan)


@pytest.mark.parametrize("engine", ["kernel", "dma"])
def test_layer_schedule_graph_replay_matches_eager(engine):
    """The forward + backward passes captured once as a CUDA graph: each
    replay gathers every layer again (the shards change between replays),
    and each layer equals the oracle's gather of the current shards."""
    n_layer, d = 5, 64
    sizes = synth.transformer_tensor_sizes(n_layer, d, 500, 32)
    psi, nd = sum(sizes), 4
    p = oracle.plan(psi, nd, 8)
    layers = [(12 * i, 12) for i in range(n_layer)] + [(12 * n_layer, 4)]
    plan = B.zero_plan(psi, nd, stage=3, align_elems=8, tensor_sizes=sizes)
    try:
        ref = synth.fp16_bits(synth.normal_f32(psi, seed=21, std=0.02))
        host_sh, dev_sh = _shards(p, ref)
        sched = stage3.LayerGatherSchedule(plan, layers, [t.data_ptr() for t in dev_sh], sizes, engine=engine)
        cap = max(sched.sizes)
        outs = {pas: torch.zeros(len(layers), cap, dtype=torch.float16, device="cuda") for pas in ("fwd", "bwd")}
        fwd = lambda i, w: outs["fwd"][i, :w.numel()].copy_(w)
        bwd = lambda i, w: outs["bwd"][i, :w.numel()].copy_(w)
        sched.forward(fwd)                       # eager first: caches and launch geometry
        sched.backward(bwd)
        g_fwd = sched.capture(range(len(layers)), fwd)
        g_bwd = sched.capture(reversed(range(len(layers))), bwd)
        for seed in (22, 23):
            ref = synth.fp16_bits(synth.normal_f32(psi, seed=seed, std=0.02))
            new_host, new_dev = _shards(p, ref)
            for r in range(nd):              # same device buffers, new contents
                dev_sh[r].copy_(new_dev[r])
            outs["fwd"].zero_()
            outs["bwd"].zero_()
            g_fwd.replay()
            g_bwd.replay()
            torch.cuda.synchronize()
            for pas in ("fwd", "bwd"):
                got = outs[pas].cpu().numpy().view(np.uint16)
                for i, (first, count) in enumerate(layers):
                    want = np.zeros(psi, np.uint16)
                    n = oracle.gather_tensors(new_host, p, sizes, first, count, want, True)
                    assert np.array_equal(got[i, :n], want[:n]), (seed, pas, i)
        del g_fwd, g_bwd
    finally:
        B.zero_plan_destroy(plan)
