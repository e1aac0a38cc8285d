"""The shard step as one object: device buffers, C-ABI arguments and the
optimizer state of a ZeRO-DP partitioned Adam step on one GPU.

``ShardStep`` owns what ``zero_shard_step`` needs -- the Nd ranks' gradient
buffers (or the per-owner contributions of stage 3), the fp32 master /
momentum / variance of the owners it updates (two slots in speculative
mode), the full 16-bit parameter buffer, the device optimizer state, the
result struct and the workspace -- and marshals them into the call.  Every
step of the arithmetic runs in the library's kernels; this module only
allocates and passes pointers.

    step = ShardStep(psi, nd, lr=1e-3, weight_decay=0.01, loss_scale=1024.0)
    step.load_master(master_fp32)          # fp32 [psi], any device
    step.grads[r, :psi] = rank_r_gradient  # 16-bit, one row per rank
    result = step.step()                   # enqueued; result() reads it back
"""
from __future__ import annotations

import torch

from . import binding as B


class ShardStep:
    """One simulated data-parallel group (or one owner's view of it) on the
    current CUDA device.

    psi / tensor_sizes: the flat parameter count, or the tensor list whose
    sizes sum to it.  nd: data-parallel degree.  owner_first / owner_count:
    the owners this object updates (default: all).  stage 1 and 2 keep full
    per-rank gradients ``grads`` [nd, psi_pad]; stage 3 keeps the owners'
    contributions ``grads`` [owner_count, nd, L].  mode: ``B.ZERO_MODE_*``;
    max_grad_norm > 0 needs TWO_PASS or STASH.  dynamic_scale: (initial
    scale, growth factor, backoff factor, growth interval) keeps the loss
    scale in the device state.  storage: ``B.ZERO_STORAGE_FP16`` or ``_BF16``.
    """

    def __init__(self, psi: int | None = None, nd: int = 1, *, tensor_sizes=None, stage: int = 2,
                 align: int = 256, bucket: int = 0, owner_first: int = 0, owner_count: int | None = None,
                 lr: float = 1e-3, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 loss_scale: float = 1.0, max_grad_norm: float = 0.0, average_over_nd: bool = False,
                 mode: int = B.ZERO_MODE_SPECULATIVE, dynamic_scale=None,
                 storage: int = B.ZERO_STORAGE_FP16, device=None):
        if psi is None:
            if tensor_sizes is None:
                raise ValueError("give psi or tensor_sizes")
            psi = int(sum(tensor_sizes))
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        dev = self.device
        self.plan = B.zero_plan(psi, nd, stage=stage, align_elems=align, bucket_elems=bucket,
                                tensor_sizes=tensor_sizes)
        try:
            info = B.zero_plan_query(self.plan)
            self.psi, self.nd, self.stage = psi, nd, stage
            self.L, self.psi_pad = info.shard_len, info.psi_pad
            self.owner_first = owner_first
            self.owner_count = nd if owner_count is None else owner_count
            self.storage = storage
            self.dtype = torch.bfloat16 if storage == B.ZERO_STORAGE_BF16 else torch.float16
            self.hp = B.hparams(lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, weight_decay=weight_decay,
                                loss_scale=loss_scale, max_grad_norm=max_grad_norm,
                                average_over_nd=average_over_nd, mode=mode)
            oc, L = self.owner_count, self.L
            spec = mode == B.ZERO_MODE_SPECULATIVE
            f32 = lambda: torch.zeros(oc * L, dtype=torch.float32, device=dev)
            self.master = [f32(), f32() if spec else None]
            self.exp_avg = [f32(), f32() if spec else None]
            self.exp_avg_sq = [f32(), f32() if spec else None]
            self.stash = f32() if mode == B.ZERO_MODE_STASH else None
            if stage == 3:
                self.grads = torch.zeros(oc, nd, L, dtype=self.dtype, device=dev)
                layout, stride = B.ZERO_GRADS_PER_OWNER, L
            else:
                self.grads = torch.zeros(nd, self.psi_pad, dtype=self.dtype, device=dev)
                layout, stride = B.ZERO_GRADS_FULL, self.psi_pad
            self.params = torch.zeros(psi, dtype=self.dtype, device=dev)
            self.opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device=dev)
            self.result_buf = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device=dev)
            ptr = lambda t: t.data_ptr() if t is not None else 0
            self.args = B.step_args(
                grads=self.grads.data_ptr(), grad_rank_stride=stride, grad_layout=layout,
                owner_first=owner_first, owner_count=oc, master=tuple(map(ptr, self.master)),
                exp_avg=tuple(map(ptr, self.exp_avg)), exp_avg_sq=tuple(map(ptr, self.exp_avg_sq)),
                params=self.params.data_ptr(), grad_stash=ptr(self.stash),
                opt_state=self.opt_state.data_ptr(), result=self.result_buf.data_ptr(), storage=storage)
            n = B.zero_workspace_bytes(self.plan, self.hp, self.args)
            self.workspace = torch.empty(n, dtype=torch.uint8, device=dev)
            self.args.workspace, self.args.workspace_bytes = self.workspace.data_ptr(), n
            if dynamic_scale is None:
                B.zero_opt_state_init(self.opt_state.data_ptr(), self._stream())
            else:
                B.zero_opt_state_init_dynamic(self.opt_state.data_ptr(), *dynamic_scale, stream=self._stream())
        except Exception:
            B.zero_plan_destroy(self.plan)
            raise

    def _stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    @property
    def owned_range(self) -> tuple[int, int]:
        """Flat [lo, hi) of the parameters this object updates."""
        lo = self.owner_first * self.L
        return lo, max(lo, min((self.owner_first + self.owner_count) * self.L, self.psi))

    def load_master(self, master_full: torch.Tensor) -> None:
        """Sets the owners' fp32 master from the full fp32 master (psi values,
        any device) and writes its 16-bit cast into their part of ``params``."""
        for j in range(self.owner_count):
            s, n = B.zero_plan_shard(self.plan, self.owner_first + j)
            self.master[0][j * self.L:(j + 1) * self.L].zero_()
            self.master[0][j * self.L:j * self.L + n].copy_(master_full[s:s + n])
        B.zero_cast_params(self.plan, self.master[0].data_ptr(), self.params.data_ptr(), self.owner_first,
                           self.owner_count, self._stream(), storage=self.storage)

    def step(self) -> torch.Tensor:
        """Enqueues one step on the current stream; returns the device result
        struct (``result()`` reads it back)."""
        B.zero_shard_step(self.plan, self.hp, self.args, self._stream())
        return self.result_buf

    def capture(self, steps: int = 1) -> torch.cuda.CUDAGraph:
        """Records ``steps`` consecutive steps as one CUDA graph; each
        ``replay()`` then runs them with a single launch.  Capturing applies
        no step: the first replay is the next step.  Everything a step
        depends on stays in device memory (the step counter, the bias
        corrections, the live slot, the dynamic loss scale), so each replay
        continues from the last one rather than repeating it.  The buffers
        must not move; refill ``grads`` in stream order between replays."""
        # load the step's kernels and size their grids before the capture
        # opens; this launches nothing and leaves the state untouched
        B.zero_shard_step_prepare(self.plan, self.hp, self.args)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(steps):
                self.step()
        return graph

    def result(self) -> B.StepResult:
        """The last step's result (synchronises with the device)."""
        return B.step_result_from_bytes(self.result_buf.cpu().numpy().tobytes())

    def opt(self) -> B.OptState:
        return B.opt_state_from_bytes(self.opt_state.cpu().numpy().tobytes())

    def live_state(self):
        """(master, exp_avg, exp_avg_sq) of the live slot, [owner_count * L]."""
        cur = self.opt().cur if self.master[1] is not None else 0
        return self.master[cur], self.exp_avg[cur], self.exp_avg_sq[cur]

    def state_dict(self) -> dict:
        """Host copies of everything a later step depends on: the live fp32
        state, the 16-bit parameters and the optimizer state bytes."""
        m, a, v = self.live_state()
        return {"master": m.cpu(), "exp_avg": a.cpu(), "exp_avg_sq": v.cpu(),
                "params": self.params.view(torch.int16).cpu(), "opt_state": self.opt_state.cpu()}

    def load_state_dict(self, sd: dict) -> None:
        """Restores a state_dict into slot 0 (the opt state's live-slot index
        is reset to match)."""
        self.master[0].copy_(sd["master"])
        self.exp_avg[0].copy_(sd["exp_avg"])
        self.exp_avg_sq[0].copy_(sd["exp_avg_sq"])
        self.params.view(torch.int16).copy_(sd["params"])
        raw = bytearray(sd["opt_state"].numpy().tobytes())
        st = B.OptState.from_buffer(raw)
        st.cur = 0
        self.opt_state.copy_(torch.frombuffer(raw, dtype=torch.uint8))

    def close(self) -> None:
        if self.plan:
            B.zero_plan_destroy(self.plan)
            self.plan = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
