"""CPU oracle of the ZeRO-DP partitioned mixed-precision Adam shard step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product library in ``zero_dp_partitioned_shard_b200`` never imports, links or
executes anything here, and shares no code with it.

This module is argument marshalling around ``oracle.c`` (plain C, fp32 IEEE
arithmetic, no contraction): every definition and every citation lives there.
Arrays are numpy; fp16 data is carried as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os

import numpy as np

from . import build as _build

_lib = None


class PlanT(C.Structure):
    _fields_ = [
        ("psi", C.c_int64), ("psi_pad", C.c_int64), ("shard_len", C.c_int64),
        ("align", C.c_int64), ("bucket", C.c_int64), ("n_buckets", C.c_int64),
        ("nd", C.c_int32), ("pad_", C.c_int32),
    ]


class StateReport(C.Structure):
    _fields_ = [
        ("params_bytes", C.c_double), ("grads_bytes", C.c_double),
        ("optim_bytes", C.c_double), ("total_bytes", C.c_double),
        ("params_bytes_padded", C.c_int64), ("grads_bytes_padded", C.c_int64),
        ("optim_bytes_padded", C.c_int64), ("total_bytes_padded", C.c_int64),
        ("reduction", C.c_double), ("comm_elems", C.c_double),
        ("comm_bytes", C.c_double), ("comm_elems_ring", C.c_double),
    ]


class HParams(C.Structure):
    _fields_ = [
        ("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float),
        ("eps", C.c_float), ("weight_decay", C.c_float),
        ("loss_scale", C.c_float), ("max_grad_norm", C.c_float),
        ("average_over_nd", C.c_int32), ("storage", C.c_int32),
    ]


class OptState(C.Structure):
    _fields_ = [("t", C.c_int64), ("beta1_pow", C.c_double), ("beta2_pow", C.c_double),
                ("loss_scale", C.c_float), ("good_steps", C.c_int32), ("growth_factor", C.c_float),
                ("backoff_factor", C.c_float), ("growth_interval", C.c_int32), ("pad_", C.c_int32)]


class StepInfo(C.Structure):
    _fields_ = [
        ("overflow", C.c_int32), ("clip_coef", C.c_float),
        ("sumsq", C.c_double), ("grad_norm", C.c_double),
        ("bc1", C.c_float), ("bc2", C.c_float),
    ]


_P = C.c_void_p
_I64 = C.c_int64
_I32 = C.c_int32


def lib():
    """Load (building first if needed) ``liboracle.so``."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        sig = {
            "oracle_half_to_float": (C.c_float, [C.c_uint16]),
            "oracle_float_to_half": (C.c_uint16, [C.c_float]),
            "oracle_half_to_float_array": (None, [_P, _P, _I64]),
            "oracle_bf16_to_float_array": (None, [_P, _P, _I64]),
            "oracle_float_to_bf16_array": (None, [_P, _P, _I64]),
            "oracle_float_to_half_array": (None, [_P, _P, _I64]),
            "oracle_plan": (C.c_int, [_I64, _I32, _I64, _I64, C.POINTER(PlanT)]),
            "oracle_shard": (None, [C.POINTER(PlanT), _I32, C.POINTER(_I64), C.POINTER(_I64)]),
            "oracle_bucket": (None, [C.POINTER(PlanT), _I64, C.POINTER(_I64), C.POINTER(_I64)]),
            "oracle_tensor_segments": (_I64, [C.POINTER(PlanT), _P, _I32, _P, _I64]),
            "oracle_state_bytes": (C.c_int, [_I64, _I32, _I32, _I64, C.POINTER(StateReport)]),
            "oracle_all_reduce": (None, [_P, _I64, _I32, _I64, _P]),
            "oracle_reduce_scatter": (None, [_P, _I64, C.POINTER(PlanT), _P]),
            "oracle_reduce_scatter16": (None, [_P, _I64, C.POINTER(PlanT), _I32, _I64, _I64, _P]),
            "oracle_all_gather_f32": (None, [_P, C.POINTER(PlanT), _P]),
            "oracle_gather_params": (None, [_P, C.POINTER(PlanT), _P]),
            "oracle_gather_tensors": (_I64, [C.POINTER(PlanT), _P, _I32, _I32, _I32, _P, _P, _I32]),
            "oracle_bias_corrections": (None, [C.POINTER(HParams), C.POINTER(OptState),
                                               C.POINTER(C.c_double), C.POINTER(C.c_double),
                                               C.POINTER(C.c_float), C.POINTER(C.c_float)]),
            "oracle_update_elements": (None, [_P, _I64, _I32, _I64, _P, _P, _P, _P,
                                              C.POINTER(HParams), C.c_float, C.c_float,
                                              C.c_float, C.c_int]),
            "oracle_step": (C.c_int, [_P, _I64, _I32, _I64, _P, _P, _P, _P,
                                      C.POINTER(HParams), C.POINTER(OptState),
                                      _I32, C.c_float, C.c_int, C.POINTER(StepInfo)]),
            "oracle_grad_sumsq": (C.c_double, [_P, _I64, _I32, _I64, C.POINTER(HParams),
                                               _P, C.POINTER(_I32)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


# --------------------------------------------------------------------------
# binary16
# --------------------------------------------------------------------------

def half_to_float(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    lib().oracle_half_to_float_array(_ptr(h), _ptr(out), h.size)
    return out


def bf16_to_float(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    lib().oracle_bf16_to_float_array(_ptr(h), _ptr(out), h.size)
    return out


def float_to_bf16(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    lib().oracle_float_to_bf16_array(_ptr(f), _ptr(out), f.size)
    return out


def float_to_half(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    lib().oracle_float_to_half_array(_ptr(f), _ptr(out), f.size)
    return out


# --------------------------------------------------------------------------
# plan / accounting
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Plan:
    psi: int
    nd: int
    align: int
    bucket: int
    shard_len: int
    psi_pad: int
    n_buckets: int

    def _c(self) -> PlanT:
        return PlanT(self.psi, self.psi_pad, self.shard_len, self.align, self.bucket,
                     self.n_buckets, self.nd, 0)

    def shard(self, r: int) -> tuple[int, int]:
        s, n = _I64(), _I64()
        p = self._c()
        lib().oracle_shard(C.byref(p), r, C.byref(s), C.byref(n))
        return s.value, n.value

    def bucket_range(self, k: int) -> tuple[int, int]:
        s, n = _I64(), _I64()
        p = self._c()
        lib().oracle_bucket(C.byref(p), k, C.byref(s), C.byref(n))
        return s.value, n.value

    def tensor_segments(self, sizes) -> np.ndarray:
        sizes = np.ascontiguousarray(sizes, dtype=np.int64)
        p = self._c()
        n = lib().oracle_tensor_segments(C.byref(p), _ptr(sizes), len(sizes), None, 0)
        if n < 0:
            raise ValueError("tensor sizes do not add up to psi")
        out = np.zeros((max(n, 1), 5), dtype=np.int64)
        lib().oracle_tensor_segments(C.byref(p), _ptr(sizes), len(sizes), _ptr(out), n)
        return out[:n]


def plan(psi: int, nd: int, align: int = 256, bucket: int = 0) -> Plan:
    p = PlanT()
    if lib().oracle_plan(psi, nd, align, bucket, C.byref(p)) != 0:
        raise ValueError(f"invalid plan arguments psi={psi} nd={nd} align={align} bucket={bucket}")
    return Plan(p.psi, p.nd, p.align, p.bucket, p.shard_len, p.psi_pad, p.n_buckets)


def state_bytes(psi: int, nd: int, stage: int, align: int = 1) -> dict:
    r = StateReport()
    if lib().oracle_state_bytes(psi, nd, stage, align, C.byref(r)) != 0:
        raise ValueError("invalid accounting arguments")
    return {name: getattr(r, name) for name, _ in StateReport._fields_}


# --------------------------------------------------------------------------
# collectives
# --------------------------------------------------------------------------

def all_reduce(G: np.ndarray, n: int) -> np.ndarray:
    """G: uint16 [nd, stride] rank buffers; returns fp32 [n] rank-order sums."""
    G = np.ascontiguousarray(G, dtype=np.uint16)
    out = np.empty(n, dtype=np.float32)
    lib().oracle_all_reduce(_ptr(G), G.shape[1], G.shape[0], n, _ptr(out))
    return out


def reduce_scatter(G: np.ndarray, p: Plan) -> np.ndarray:
    """Returns fp32 [nd, L]: each owner's reduced slice (pads zero)."""
    G = np.ascontiguousarray(G, dtype=np.uint16)
    assert G.shape[0] == p.nd and G.shape[1] >= p.psi
    out = np.empty((p.nd, p.shard_len), dtype=np.float32)
    pc = p._c()
    lib().oracle_reduce_scatter(_ptr(G), G.shape[1], C.byref(pc), _ptr(out))
    return out


def reduce_scatter16(G: np.ndarray, p: Plan, storage: int = 0, lo: int = 0, hi: int | None = None,
                     out: np.ndarray | None = None) -> np.ndarray:
    """The owners' retained 16-bit reduced gradients [nd, L] (uint16 bits):
    the rank-order fp32 sum rounded once to the storage format, written for
    flat indices in [lo, hi) only (into ``out`` if given; fresh pads are
    0xFFFF, a NaN in both formats, and are never written)."""
    G = np.ascontiguousarray(G, dtype=np.uint16)
    assert G.shape[0] == p.nd and G.shape[1] >= p.psi
    hi = p.psi if hi is None else hi
    if out is None:
        out = np.full((p.nd, p.shard_len), 0xFFFF, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == p.nd * p.shard_len
    pc = p._c()
    lib().oracle_reduce_scatter16(_ptr(G), G.shape[1], C.byref(pc), int(storage), int(lo), int(hi), _ptr(out))
    return out


def all_gather_f32(shards: np.ndarray, p: Plan) -> np.ndarray:
    shards = np.ascontiguousarray(shards, dtype=np.float32)
    out = np.zeros(p.psi, dtype=np.float32)
    pc = p._c()
    lib().oracle_all_gather_f32(_ptr(shards), C.byref(pc), _ptr(out))
    return out


def gather_params(shards, p: Plan, full: np.ndarray) -> np.ndarray:
    """shards: list of nd uint16 arrays (or None); assembles into ``full`` in place."""
    assert full.dtype == np.uint16 and full.size >= p.psi and full.flags["C_CONTIGUOUS"]
    keep = []
    ptrs = (C.c_void_p * p.nd)()
    for r, s in enumerate(shards):
        if s is None:
            ptrs[r] = None
        else:
            s = np.ascontiguousarray(s, dtype=np.uint16)
            keep.append(s)
            ptrs[r] = s.ctypes.data
    pc = p._c()
    lib().oracle_gather_params(ptrs, C.byref(pc), _ptr(full))
    return full


def gather_tensors(shards, p: Plan, sizes, first: int, count: int, out: np.ndarray,
                   compact: bool) -> int:
    """Assembles tensors first..first+count-1 from the owners' fp16 shards
    (list of nd uint16 arrays or None) into ``out``; returns elements written."""
    sizes = np.ascontiguousarray(sizes, dtype=np.int64)
    keep = []
    ptrs = (C.c_void_p * p.nd)()
    for r, sh in enumerate(shards):
        if sh is None:
            ptrs[r] = None
        else:
            sh = np.ascontiguousarray(sh, dtype=np.uint16)
            keep.append(sh)
            ptrs[r] = sh.ctypes.data
    assert out.dtype == np.uint16 and out.flags["C_CONTIGUOUS"]
    pc = p._c()
    n = lib().oracle_gather_tensors(C.byref(pc), _ptr(sizes), len(sizes), first, count, ptrs,
                                    _ptr(out), int(compact))
    if n < 0:
        raise ValueError("gather_tensors: bad range, sizes or missing shard")
    return n


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------

@dataclasses.dataclass
class HP:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0
    loss_scale: float = 1.0
    max_grad_norm: float = 0.0
    average_over_nd: bool = False
    storage: int = 0          # 16-bit format of gradients and parameters: 0 fp16, 1 bf16

    def _c(self) -> HParams:
        return HParams(self.lr, self.beta1, self.beta2, self.eps, self.weight_decay,
                       self.loss_scale, self.max_grad_norm, int(self.average_over_nd),
                       int(self.storage))


@dataclasses.dataclass
class Opt:
    t: int = 0
    beta1_pow: float = 1.0
    beta2_pow: float = 1.0
    loss_scale: float = 0.0        # > 0: dynamic loss scaling with this current scale
    good_steps: int = 0
    growth_factor: float = 2.0
    backoff_factor: float = 0.5
    growth_interval: int = 2000

    def _c(self) -> OptState:
        return OptState(self.t, self.beta1_pow, self.beta2_pow, self.loss_scale, self.good_steps,
                        self.growth_factor, self.backoff_factor, self.growth_interval, 0)

    def _update(self, o: OptState) -> None:
        self.t, self.beta1_pow, self.beta2_pow = o.t, o.beta1_pow, o.beta2_pow
        self.loss_scale, self.good_steps = o.loss_scale, o.good_steps


def bias_corrections(hp: HP, opt: Opt):
    """(beta1^(t+1), beta2^(t+1), fp32 bc1, fp32 bc2) for the next step."""
    h, o = hp._c(), opt._c()
    b1, b2, c1, c2 = C.c_double(), C.c_double(), C.c_float(), C.c_float()
    lib().oracle_bias_corrections(C.byref(h), C.byref(o), C.byref(b1), C.byref(b2),
                                  C.byref(c1), C.byref(c2))
    return b1.value, b2.value, np.float32(c1.value), np.float32(c2.value)


def step(G: np.ndarray, master: np.ndarray, exp_avg: np.ndarray, exp_avg_sq: np.ndarray,
         params: np.ndarray, hp: HP, opt: Opt, clip_override: float | None = None,
         threads: int = 1) -> dict:
    """One step over all owners, in place.

    G: uint16 [nd, stride] (stride >= psi); master/exp_avg/exp_avg_sq: fp32 [psi];
    params: uint16 [psi].  ``opt`` is advanced unless the step is skipped.
    """
    G = np.ascontiguousarray(G, dtype=np.uint16)
    psi = params.size
    for a, dt in ((master, np.float32), (exp_avg, np.float32), (exp_avg_sq, np.float32),
                  (params, np.uint16)):
        assert a.dtype == dt and a.flags["C_CONTIGUOUS"] and a.size == psi
    h = hp._c()
    o = opt._c()
    info = StepInfo()
    rc = lib().oracle_step(_ptr(G), G.shape[1], G.shape[0], psi, _ptr(master), _ptr(exp_avg),
                           _ptr(exp_avg_sq), _ptr(params), C.byref(h), C.byref(o),
                           int(clip_override is not None),
                           float(clip_override if clip_override is not None else 0.0),
                           threads, C.byref(info))
    if rc != 0:
        raise ValueError("oracle_step rejected its arguments")
    opt._update(o)
    return {name: getattr(info, name) for name, _ in StepInfo._fields_}


def update_elements(G: np.ndarray, master: np.ndarray, exp_avg: np.ndarray,
                    exp_avg_sq: np.ndarray, params: np.ndarray, hp: HP, clip_coef: float,
                    bc1: float, bc2: float, threads: int = 1) -> None:
    """The per-element update with known global quantities, in place.

    G: uint16 [nd, n] -- the n elements' contributions, rank-major.
    """
    G = np.ascontiguousarray(G, dtype=np.uint16)
    n = G.shape[1]
    for a, dt in ((master, np.float32), (exp_avg, np.float32), (exp_avg_sq, np.float32),
                  (params, np.uint16)):
        assert a.dtype == dt and a.flags["C_CONTIGUOUS"] and a.size == n
    h = hp._c()
    lib().oracle_update_elements(_ptr(G), n, G.shape[0], n, _ptr(master), _ptr(exp_avg),
                                 _ptr(exp_avg_sq), _ptr(params), C.byref(h),
                                 float(clip_coef), float(bc1), float(bc2), threads)


def grad_sumsq(G: np.ndarray, hp: HP, acc: np.ndarray | None = None) -> tuple[float, bool]:
    """Compensated fp64 sum of squares of the unscaled reduced gradient of G
    [nd, n].  acc: optional float64[2] Neumaier accumulator {sum,
    compensation}, updated in place, to stream a problem through in pieces:
    one acc carried along gives the single-pass sum bit for bit; separate
    accs per piece add up exactly with math.fsum over all their terms."""
    G = np.ascontiguousarray(G, dtype=np.uint16)
    if acc is None:
        acc = np.zeros(2, np.float64)
    assert acc.dtype == np.float64 and acc.shape == (2,) and acc.flags["C_CONTIGUOUS"]
    h = hp._c()
    bad = _I32(0)
    s = lib().oracle_grad_sumsq(_ptr(G), G.shape[1], G.shape[0], G.shape[1], C.byref(h),
                                _ptr(acc), C.byref(bad))
    return s, bool(bad.value)


def host_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
