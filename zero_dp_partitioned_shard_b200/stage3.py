"""Stage-3 parameter schedule: gather a layer's parameters just before use,
release them after.

ZeRO stage 3 keeps only the owned 1/Nd of the fp16 parameters; when the
forward or backward pass reaches a layer, the layer's parameters are gathered
from their owners, used, and released ("ZeRO memory optimization: training
large models", trishampatil.com, "ZeRO-3" and the figure under
"Forward/Backward Under ZeRO-3").  The two parameter gathers (forward and
backward) plus the gradient reduce-scatter make stage 3's 3 Psi of
communication per step ("ZeRO: partitioning training state across GPUs",
upskillscore.com, "How it works").

``LayerGatherSchedule`` runs that pattern on the GPU with the library's
``zero_gather_tensors``: two compact layer buffers, the next layer's gather
issued on a side stream while the current layer is in use (prefetch), and a
buffer reused only after the work that used it has finished (release).
Consecutive gathers fill different buffers and only read the shards, so each
buffer has its own copy stream and one gather's tail overlaps the next one's
start.  ``engine="dma"`` moves the layers with the copy engines
(``zero_gather_tensors_dma``) instead of a copy kernel, so a gather can run
beside compute that holds every SM.
"""
from __future__ import annotations

import torch

from . import binding as B


class LayerGatherSchedule:
    """``layers``: list of (first_tensor, n_tensors) of the plan's tensor list;
    ``shard_ptrs``: the owners' fp16 shard addresses (one per owner);
    ``engine``: "kernel" (a copy kernel) or "dma" (the copy engines)."""

    def __init__(self, plan: int, layers, shard_ptrs, tensor_sizes, device=None, engine: str = "kernel"):
        if engine not in ("kernel", "dma"):
            raise ValueError(f"unknown engine {engine!r}")
        self._gather = B.zero_gather_tensors if engine == "kernel" else B.zero_gather_tensors_dma
        self.plan = plan
        self.layers = list(layers)
        self.shard_ptrs = list(shard_ptrs)
        self.sizes = [sum(tensor_sizes[f:f + n]) for f, n in self.layers]
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        cap = max(self.sizes) if self.sizes else 1
        self.buffers = [torch.empty(cap, dtype=torch.float16, device=dev) for _ in range(2)]
        self.copy_streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]   # one per buffer
        self.gathered = 0   # elements gathered so far (the communication volume)

    def _issue(self, layer: int, slot: int, free: torch.cuda.Event, ready: torch.cuda.Event) -> None:
        first, count = self.layers[layer]
        cs = self.copy_streams[slot]
        cs.wait_event(free)                           # the slot's last use has finished
        n = self._gather(self.plan, first, count, self.shard_ptrs, self.buffers[slot].data_ptr(), True,
                         cs.cuda_stream)
        ready.record(cs)
        self.gathered += n

    def run(self, order, use) -> None:
        """Visits the layers in ``order`` (forward: ascending, backward:
        descending); ``use(layer, params)`` runs on the current stream with the
        layer's gathered fp16 parameters and must not keep them."""
        order = list(order)
        if not order:
            return
        main = torch.cuda.current_stream(self.device)
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        free = [torch.cuda.Event(), torch.cuda.Event()]
        for ev in free:
            ev.record(main)
        self._issue(order[0], 0, free[0], ready[0])
        for k, layer in enumerate(order):
            slot = k & 1
            if k + 1 < len(order):                    # prefetch the next layer
                self._issue(order[k + 1], slot ^ 1, free[slot ^ 1], ready[slot ^ 1])
            main.wait_event(ready[slot])
            use(layer, self.buffers[slot][:self.sizes[layer]])
            free[slot].record(main)                   # release after use
        for cs in self.copy_streams:
            main.wait_stream(cs)

    def forward(self, use) -> None:
        self.run(range(len(self.layers)), use)

    def backward(self, use) -> None:
        self.run(reversed(range(len(self.layers))), use)

    def capture(self, order, use) -> torch.cuda.CUDAGraph:
        """Records ``run(order, use)`` once as a CUDA graph: every layer's
        gather, the side-stream prefetch and the release ordering become
        graph nodes, and ``replay()`` re-issues the whole pass with one launch
        instead of a host round per layer.  ``use`` must be capturable (work
        enqueued on the current stream, no host synchronisation).  The
        schedule's buffers stay the graph's: do not run the schedule eagerly
        while a replay may be in flight.  Replays do not add to
        ``gathered``; the capture counts one pass."""
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(self.device)
        with torch.cuda.graph(graph):
            self.run(order, use)
        return graph
