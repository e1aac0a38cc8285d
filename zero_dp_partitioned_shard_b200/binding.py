"""ctypes binding of ``libzero_shard.so`` (declared in ``include/zero_shard.h``).

Argument marshalling only: every function below has the name of the C entry
point it calls, converts Python values / integer device addresses into the C
structs, and raises :class:`ZeroError` (carrying the status code and the
library's message) when the call returns a non-zero status.  All device work
runs in the library's CUDA kernels; there is no Python or CPU fallback, and a
missing library raises at first use.

Device buffers are passed as integer addresses (``tensor.data_ptr()``) and
streams / events as their raw handles (``torch.cuda.Stream.cuda_stream``,
``torch.cuda.Event.cuda_event``), so this module does not depend on torch.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzero_shard.so")

ZERO_OK = 0
ZERO_ERR_INVALID_ARG = 1
ZERO_ERR_ALIGNMENT = 2
ZERO_ERR_CUDA = 3
ZERO_ERR_WORKSPACE = 4
ZERO_ERR_TIMEOUT = 5
ZERO_ERR_UNSUPPORTED = 6

ZERO_MODE_SPECULATIVE = 0
ZERO_MODE_TWO_PASS = 1
ZERO_MODE_STASH = 2

ZERO_GRADS_FULL = 0
ZERO_GRADS_PER_OWNER = 1
ZERO_GRADS_REDUCED = 2

ZERO_STORAGE_FP16 = 0
ZERO_STORAGE_BF16 = 1

ZERO_MAX_PEERS = 64

ZERO_STATIC_SCRATCH_BYTES = 1 << 20  # static scratch of zero_shard_step_static_scratch
ZERO_VOTE_OFFSET = 128               # byte offset of the split step's fp64[2] vote in the workspace

OPT_STATE_BYTES = 64   # device allocation for zero_opt_state (64 bytes)
RESULT_BYTES = 64      # device allocation for zero_step_result (40 bytes used)


class ZeroError(RuntimeError):
    def __init__(self, status: int, func: str, message: str):
        super().__init__(f"{func}: status {status} ({message})")
        self.status = status


class PlanDesc(C.Structure):
    _fields_ = [("psi", C.c_int64), ("align_elems", C.c_int64), ("bucket_elems", C.c_int64),
                ("tensor_sizes", C.c_void_p), ("nd", C.c_int32), ("stage", C.c_int32),
                ("n_tensors", C.c_int32), ("reserved", C.c_int32)]


class PlanInfo(C.Structure):
    _fields_ = [("psi", C.c_int64), ("psi_pad", C.c_int64), ("shard_len", C.c_int64),
                ("align_elems", C.c_int64), ("bucket_elems", C.c_int64),
                ("n_buckets", C.c_int64), ("n_segments", C.c_int64),
                ("nd", C.c_int32), ("stage", C.c_int32)]


class Segment(C.Structure):
    _fields_ = [("tensor", C.c_int64), ("owner", C.c_int64), ("offset_in_tensor", C.c_int64),
                ("length", C.c_int64), ("offset_in_shard", C.c_int64)]


class StateReport(C.Structure):
    _fields_ = [("params_bytes", C.c_double), ("grads_bytes", C.c_double),
                ("optim_bytes", C.c_double), ("total_bytes", C.c_double),
                ("params_bytes_padded", C.c_int64), ("grads_bytes_padded", C.c_int64),
                ("optim_bytes_padded", C.c_int64), ("total_bytes_padded", C.c_int64),
                ("reduction", C.c_double), ("comm_elems", C.c_double),
                ("comm_bytes", C.c_double), ("comm_elems_ring", C.c_double)]


class OptState(C.Structure):
    _fields_ = [("t", C.c_int64), ("beta1_pow", C.c_double), ("beta2_pow", C.c_double),
                ("skipped", C.c_int64), ("cur", C.c_int32), ("reserved", C.c_int32),
                ("loss_scale", C.c_float), ("good_steps", C.c_int32), ("growth_factor", C.c_float),
                ("backoff_factor", C.c_float), ("growth_interval", C.c_int32), ("reserved2", C.c_int32)]


class StepResult(C.Structure):
    _fields_ = [("grad_norm", C.c_double), ("t", C.c_int64), ("skipped", C.c_int64),
                ("clip_coef", C.c_float), ("overflow", C.c_int32), ("status", C.c_int32),
                ("loss_scale", C.c_float)]


class HParams(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float),
                ("eps", C.c_float), ("weight_decay", C.c_float), ("loss_scale", C.c_float),
                ("max_grad_norm", C.c_float), ("average_over_nd", C.c_int32),
                ("mode", C.c_int32), ("reserved", C.c_int32)]


class StepArgs(C.Structure):
    _fields_ = [("grads", C.c_void_p), ("grad_rank_stride", C.c_int64),
                ("grad_layout", C.c_int32), ("owner_first", C.c_int32),
                ("owner_count", C.c_int32), ("storage", C.c_int32),
                ("master", C.c_void_p * 2), ("exp_avg", C.c_void_p * 2),
                ("exp_avg_sq", C.c_void_p * 2), ("params", C.c_void_p),
                ("grad_stash", C.c_void_p), ("opt_state", C.c_void_p), ("result", C.c_void_p),
                ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t),
                ("timing_events", C.c_void_p * 2), ("peers", C.c_void_p)]


class PeerArgs(C.Structure):
    _fields_ = [("rank_grads", C.c_void_p * ZERO_MAX_PEERS),
                ("param_dests", C.c_void_p * ZERO_MAX_PEERS),
                ("n_param_dests", C.c_int32), ("reserved", C.c_int32)]


class IpcHandle(C.Structure):
    _fields_ = [("handle", C.c_ubyte * 64), ("offset", C.c_int64), ("device", C.c_int32),
                ("reserved", C.c_int32)]


_lib = None
_P = C.c_void_p
_S = C.c_int32

# name -> (restype, argtypes) of every exported symbol of include/zero_shard.h
SIGNATURES = {
    "zero_plan": (_S, [C.POINTER(PlanDesc), C.POINTER(_P)]),
    "zero_plan_query": (_S, [_P, C.POINTER(PlanInfo)]),
    "zero_plan_shard": (_S, [_P, C.c_int32, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
    "zero_plan_bucket": (_S, [_P, C.c_int64, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]),
    "zero_plan_segments": (_S, [_P, _P, C.c_int64, C.POINTER(C.c_int64)]),
    "zero_plan_destroy": (None, [_P]),
    "zero_state_bytes": (_S, [C.c_int64, C.c_int32, C.c_int32, C.c_int64, C.POINTER(StateReport)]),
    "zero_opt_state_init": (_S, [_P, _P]),
    "zero_opt_state_init_dynamic": (_S, [_P, C.c_float, C.c_float, C.c_float, C.c_int32, _P]),
    "zero_workspace_bytes": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs), C.POINTER(C.c_size_t)]),
    "zero_shard_step": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs), _P]),
    "zero_shard_step_static_scratch": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs), _P]),
    "zero_shard_step_prepare": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs)]),
    "zero_shard_step_begin": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs), _P]),
    "zero_shard_step_end": (_S, [_P, C.POINTER(HParams), C.POINTER(StepArgs), _P]),
    "zero_gather_params": (_S, [_P, _P, _P, _P]),
    "zero_reduce_scatter": (_S, [_P, C.POINTER(StepArgs), C.c_int64, _P, _P]),
    "zero_gather_tensors": (_S, [_P, C.c_int32, C.c_int32, _P, _P, C.c_int32, C.POINTER(C.c_int64), _P]),
    "zero_gather_tensors_dma": (_S, [_P, C.c_int32, C.c_int32, _P, _P, C.c_int32, C.POINTER(C.c_int64), _P]),
    "zero_cast_params": (_S, [_P, _P, _P, C.c_int32, C.c_int32, C.c_int32, _P]),
    "zero_ipc_export": (_S, [_P, C.POINTER(IpcHandle)]),
    "zero_ipc_open": (_S, [C.POINTER(IpcHandle), C.POINTER(_P)]),
    "zero_ipc_close": (_S, [_P]),
    "zero_abi_version": (C.c_int32, []),
    "zero_strerror": (C.c_char_p, [_S]),
    "zero_last_error": (C.c_char_p, []),
    "zero_launch_count": (C.c_uint64, []),
    "zero_recent_kernels": (C.c_int32, [C.POINTER(C.c_char_p), C.c_int32]),
    "zero_set_wait_budget": (C.c_int64, [C.c_int64]),
}


def lib() -> C.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python zero_dp_partitioned_shard_b200/build.py` "
                "(there is no CPU fallback)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.zero_abi_version() != 9:
            raise ImportError("libzero_shard.so ABI version mismatch")
        _lib = L
    return _lib


def _check(status: int, func: str) -> None:
    if status != ZERO_OK:
        raise ZeroError(status, func, lib().zero_last_error().decode())


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def zero_plan(psi: int, nd: int, stage: int = 1, align_elems: int = 256, bucket_elems: int = 0,
              tensor_sizes=None) -> int:
    """Returns an opaque plan handle; release it with zero_plan_destroy."""
    sizes = None
    if tensor_sizes is not None:
        sizes = (C.c_int64 * len(tensor_sizes))(*[int(x) for x in tensor_sizes])
    d = PlanDesc(psi, align_elems, bucket_elems, C.cast(sizes, C.c_void_p) if sizes else None,
                 nd, stage, len(tensor_sizes) if tensor_sizes is not None else 0, 0)
    h = C.c_void_p()
    _check(lib().zero_plan(C.byref(d), C.byref(h)), "zero_plan")
    return h.value


def zero_plan_query(plan: int) -> PlanInfo:
    info = PlanInfo()
    _check(lib().zero_plan_query(plan, C.byref(info)), "zero_plan_query")
    return info


def zero_plan_shard(plan: int, owner: int) -> tuple[int, int]:
    s, n = C.c_int64(), C.c_int64()
    _check(lib().zero_plan_shard(plan, owner, C.byref(s), C.byref(n)), "zero_plan_shard")
    return s.value, n.value


def zero_plan_bucket(plan: int, k: int) -> tuple[int, int]:
    s, n = C.c_int64(), C.c_int64()
    _check(lib().zero_plan_bucket(plan, k, C.byref(s), C.byref(n)), "zero_plan_bucket")
    return s.value, n.value


def zero_plan_segments(plan: int) -> list[tuple[int, int, int, int, int]]:
    n = C.c_int64()
    _check(lib().zero_plan_segments(plan, None, 0, C.byref(n)), "zero_plan_segments")
    arr = (Segment * max(n.value, 1))()
    _check(lib().zero_plan_segments(plan, C.cast(arr, C.c_void_p), n.value, C.byref(n)),
           "zero_plan_segments")
    return [(s.tensor, s.owner, s.offset_in_tensor, s.length, s.offset_in_shard)
            for s in arr[:n.value]]


def zero_plan_destroy(plan: int) -> None:
    if plan:
        lib().zero_plan_destroy(plan)


def zero_state_bytes(psi: int, nd: int, stage: int, align_elems: int = 1) -> dict:
    r = StateReport()
    _check(lib().zero_state_bytes(psi, nd, stage, align_elems, C.byref(r)), "zero_state_bytes")
    return {name: getattr(r, name) for name, _ in StateReport._fields_}


def zero_opt_state_init(opt_state: int, stream: int = 0) -> None:
    _check(lib().zero_opt_state_init(opt_state, stream), "zero_opt_state_init")


def zero_opt_state_init_dynamic(opt_state: int, initial_scale: float, growth_factor: float = 2.0,
                                backoff_factor: float = 0.5, growth_interval: int = 2000,
                                stream: int = 0) -> None:
    _check(lib().zero_opt_state_init_dynamic(opt_state, initial_scale, growth_factor, backoff_factor,
                                             growth_interval, stream), "zero_opt_state_init_dynamic")


def zero_workspace_bytes(plan: int, hp: HParams, args: StepArgs) -> int:
    n = C.c_size_t()
    _check(lib().zero_workspace_bytes(plan, C.byref(hp), C.byref(args), C.byref(n)),
           "zero_workspace_bytes")
    return n.value


def zero_shard_step(plan: int, hp: HParams, args: StepArgs, stream: int = 0) -> None:
    _check(lib().zero_shard_step(plan, C.byref(hp), C.byref(args), stream), "zero_shard_step")


def zero_shard_step_prepare(plan: int, hp: HParams, args: StepArgs) -> None:
    """Validates a step and loads / sizes its kernels without launching anything."""
    _check(lib().zero_shard_step_prepare(plan, C.byref(hp), C.byref(args)), "zero_shard_step_prepare")


def zero_shard_step_static_scratch(plan: int, hp: HParams, args: StepArgs, stream: int = 0) -> None:
    """zero_shard_step with the library's static device scratch (args.workspace ignored)."""
    _check(lib().zero_shard_step_static_scratch(plan, C.byref(hp), C.byref(args), stream),
           "zero_shard_step_static_scratch")


def zero_shard_step_begin(plan: int, hp: HParams, args: StepArgs, stream: int = 0) -> None:
    """First half of a split step: ends with this call's vote at workspace + ZERO_VOTE_OFFSET."""
    _check(lib().zero_shard_step_begin(plan, C.byref(hp), C.byref(args), stream), "zero_shard_step_begin")


def zero_shard_step_end(plan: int, hp: HParams, args: StepArgs, stream: int = 0) -> None:
    """Second half of a split step, after the votes of all owners were summed in place."""
    _check(lib().zero_shard_step_end(plan, C.byref(hp), C.byref(args), stream), "zero_shard_step_end")


def zero_reduce_scatter(plan: int, args: StepArgs, grad_shards: int, bucket: int = -1, stream: int = 0) -> None:
    """Keeps the owners' reduced gradients (16-bit, [owner_count * L]) for a
    later step with grad_layout ZERO_GRADS_REDUCED; bucket < 0: everything."""
    _check(lib().zero_reduce_scatter(plan, C.byref(args), bucket, grad_shards, stream), "zero_reduce_scatter")


def zero_gather_params(plan: int, shard_ptrs, params_full: int, stream: int = 0) -> None:
    arr = (C.c_void_p * len(shard_ptrs))(*[p if p else None for p in shard_ptrs])
    _check(lib().zero_gather_params(plan, C.cast(arr, C.c_void_p), params_full, stream),
           "zero_gather_params")


def zero_gather_tensors(plan: int, first_tensor: int, n_tensors: int, shard_ptrs, out: int,
                        compact: bool, stream: int = 0) -> int:
    """Gathers a tensor range from the owners' shards; returns the elements copied."""
    arr = (C.c_void_p * len(shard_ptrs))(*[p if p else None for p in shard_ptrs])
    n = C.c_int64()
    _check(lib().zero_gather_tensors(plan, first_tensor, n_tensors, C.cast(arr, C.c_void_p), out,
                                     int(compact), C.byref(n), stream), "zero_gather_tensors")
    return n.value


def zero_gather_tensors_dma(plan: int, first_tensor: int, n_tensors: int, shard_ptrs, out: int,
                            compact: bool, stream: int = 0) -> int:
    """zero_gather_tensors moved by the copy engines; returns the elements copied."""
    arr = (C.c_void_p * len(shard_ptrs))(*[p if p else None for p in shard_ptrs])
    n = C.c_int64()
    _check(lib().zero_gather_tensors_dma(plan, first_tensor, n_tensors, C.cast(arr, C.c_void_p), out,
                                         int(compact), C.byref(n), stream), "zero_gather_tensors_dma")
    return n.value


def zero_cast_params(plan: int, master: int, params: int, owner_first: int, owner_count: int,
                     stream: int = 0, storage: int = ZERO_STORAGE_FP16) -> None:
    _check(lib().zero_cast_params(plan, master, params, owner_first, owner_count, storage, stream),
           "zero_cast_params")


def zero_ipc_export(dev_ptr: int) -> bytes:
    """The CUDA IPC export of a device buffer, as bytes to send to other processes."""
    h = IpcHandle()
    _check(lib().zero_ipc_export(dev_ptr, C.byref(h)), "zero_ipc_export")
    return bytes(h)


def zero_ipc_open(handle: bytes) -> int:
    """Maps a buffer exported by another process; returns its address here."""
    h = IpcHandle.from_buffer_copy(handle)
    p = C.c_void_p()
    _check(lib().zero_ipc_open(C.byref(h), C.byref(p)), "zero_ipc_open")
    return p.value


def zero_ipc_close(dev_ptr: int) -> None:
    _check(lib().zero_ipc_close(dev_ptr), "zero_ipc_close")


def zero_abi_version() -> int:
    return lib().zero_abi_version()


def zero_strerror(status: int) -> str:
    return lib().zero_strerror(status).decode()


def zero_last_error() -> str:
    return lib().zero_last_error().decode()


def zero_launch_count() -> int:
    return lib().zero_launch_count()


def zero_recent_kernels(max_names: int = 64) -> list:
    """Names of the kernels the library launched last (oldest first, mangled
    C++ names), up to the last 64 launches in the process."""
    buf = (C.c_char_p * max_names)()
    n = lib().zero_recent_kernels(buf, max_names)
    if n < 0:
        raise ValueError("zero_recent_kernels: bad arguments")
    return [buf[i].decode() for i in range(n)]


def zero_set_wait_budget(cycles: int) -> int:
    """Sets the per-wait cycle budget of the pipelined update (0 = default, < 0 =
    expire at once); returns the previous value."""
    return lib().zero_set_wait_budget(cycles)


# ---------------------------------------------------------------------------
# struct builders
# ---------------------------------------------------------------------------

def hparams(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, loss_scale=1.0,
            max_grad_norm=0.0, average_over_nd=False, mode=ZERO_MODE_SPECULATIVE) -> HParams:
    return HParams(lr, beta1, beta2, eps, weight_decay, loss_scale, max_grad_norm,
                   int(average_over_nd), mode, 0)


def step_args(*, grads: int, grad_rank_stride: int, master, exp_avg, exp_avg_sq, params: int,
              opt_state: int, workspace: int = 0, workspace_bytes: int = 0, result: int = 0,
              grad_layout: int = ZERO_GRADS_FULL, owner_first: int = 0, owner_count: int = 1,
              grad_stash: int = 0, timing_events=(0, 0), storage: int = ZERO_STORAGE_FP16) -> StepArgs:
    """master/exp_avg/exp_avg_sq: (slot0, slot1) device addresses (slot1 may be 0)."""
    a = StepArgs()
    a.grads = grads
    a.grad_rank_stride = grad_rank_stride
    a.grad_layout = grad_layout
    a.owner_first = owner_first
    a.owner_count = owner_count
    a.storage = storage
    for k in range(2):
        a.master[k] = master[k] or None
        a.exp_avg[k] = exp_avg[k] or None
        a.exp_avg_sq[k] = exp_avg_sq[k] or None
        a.timing_events[k] = timing_events[k] or None
    a.params = params
    a.grad_stash = grad_stash or None
    a.opt_state = opt_state
    a.result = result or None
    a.workspace = workspace or None
    a.workspace_bytes = workspace_bytes
    return a


def peer_args(rank_grads, param_dests=()) -> PeerArgs:
    """Peer tables: rank_grads[r] = rank r's gradient buffer, param_dests = the
    other full parameter buffers that receive every new parameter."""
    if len(rank_grads) > ZERO_MAX_PEERS or len(param_dests) > ZERO_MAX_PEERS:
        raise ValueError(f"at most {ZERO_MAX_PEERS} ranks and destinations")
    q = PeerArgs()
    for r, g in enumerate(rank_grads):
        q.rank_grads[r] = g or None
    for d, p in enumerate(param_dests):
        q.param_dests[d] = p or None
    q.n_param_dests = len(param_dests)
    return q


def attach_peers(args: StepArgs, peers: PeerArgs | None) -> StepArgs:
    """Points args at the peer tables (None detaches them); args keeps them alive."""
    args._peers_ref = peers
    args.peers = C.cast(C.pointer(peers), C.c_void_p) if peers is not None else None
    return args


def opt_state_from_bytes(raw: bytes) -> OptState:
    return OptState.from_buffer_copy(raw[:C.sizeof(OptState)])


def step_result_from_bytes(raw: bytes) -> StepResult:
    return StepResult.from_buffer_copy(raw[:C.sizeof(StepResult)])
