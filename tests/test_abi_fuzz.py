"""Property-based fuzzing of the step's host-side checks through
zero_workspace_bytes, which validates and plans exactly as zero_shard_step
does but never launches anything (so fake device addresses are safe).
Random plans and valid configurations (layouts, strides, owner ranges,
alignments, modes, clipping, peer tables, storage) must be planned with a
workspace of the documented size; the same configurations with one field
broken must return that field's documented status."""
import ctypes as C

from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from zero_dp_partitioned_shard_b200 import binding as B

FAKE = 1 << 40
STATUSES = {B.ZERO_OK, B.ZERO_ERR_INVALID_ARG, B.ZERO_ERR_ALIGNMENT, B.ZERO_ERR_UNSUPPORTED,
            B.ZERO_ERR_WORKSPACE}


MUTATIONS = ["none", "none", "none", "null_grads", "odd_state", "odd_params", "bad_mode", "bad_scale", "bad_beta",
             "clip_speculative", "owner_range", "owner_count", "bad_layout", "short_stride", "bad_storage",
             "no_stash", "null_slot1", "peer_null", "peer_odd", "peer_dests", "peer_layout", "reserved"]


_I, _A, _U = B.ZERO_ERR_INVALID_ARG, B.ZERO_ERR_ALIGNMENT, B.ZERO_ERR_UNSUPPORTED
EXPECTED = {"null_grads": _I, "odd_state": _A, "odd_params": _A, "bad_mode": _I, "bad_scale": _I,
            "bad_beta": _I, "clip_speculative": _U, "owner_range": _I, "owner_count": _I, "bad_layout": _I,
            "short_stride": _I, "bad_storage": _I, "no_stash": _I, "null_slot1": _I, "peer_null": _I,
            "peer_odd": _A, "peer_dests": _I, "peer_layout": _U, "reserved": _I}


@st.composite
def cases(draw):
    """A valid configuration, then at most one field broken."""
    nd = draw(st.integers(1, 70))
    psi = draw(st.integers(1, 200_000))
    plan = dict(psi=psi, nd=nd, stage=draw(st.integers(1, 3)), align_elems=draw(st.sampled_from([1, 2, 8, 256])),
                bucket_elems=draw(st.sampled_from([0, 1, 7, 1000, 65536])))
    L = -(-psi // (nd * plan["align_elems"])) * plan["align_elems"]
    mode = draw(st.integers(0, 2))
    clip = draw(st.sampled_from([0.0, 1.0])) if mode else 0.0
    hp = B.hparams(loss_scale=draw(st.sampled_from([1.0, 1024.0])), max_grad_norm=clip, mode=mode,
                   average_over_nd=draw(st.booleans()))
    o_first = draw(st.integers(0, nd - 1))
    o_count = draw(st.integers(1, nd - o_first))
    layout = draw(st.integers(0, 2))
    stride = {0: nd * L + draw(st.sampled_from([0, 8])), 1: L, 2: 0}[layout]
    vec = draw(st.booleans())
    addr = lambda k: FAKE + (k << 24) + (0 if vec else 2)      # 16-bit buffers
    addr32 = lambda k: FAKE + (k << 24) + (0 if vec else 4)    # fp32 buffers
    a = B.step_args(grads=addr(1), grad_rank_stride=stride, grad_layout=layout, owner_first=o_first,
                    owner_count=o_count, master=(addr32(2), addr32(3)), exp_avg=(addr32(4), addr32(5)),
                    exp_avg_sq=(addr32(6), addr32(7)), params=addr(8), opt_state=FAKE, result=FAKE + 64,
                    grad_stash=addr32(9), storage=draw(st.integers(0, 1)))
    peers = layout == 0 and nd <= 64 and draw(st.booleans())
    q = None
    if peers:
        q = B.peer_args([addr(20 + r) for r in range(nd)], [addr(100 + d) for d in range(draw(st.integers(0, 3)))])
        B.attach_peers(a, q)
    m = draw(st.sampled_from(MUTATIONS))
    if m == "null_grads" and not peers:
        a.grads = None
    elif m == "odd_state":
        a.master[0] = FAKE + 1
    elif m == "odd_params":
        a.params = FAKE + 1
    elif m == "bad_mode":
        hp.mode = 5
    elif m == "bad_scale":
        hp.loss_scale = draw(st.sampled_from([0.0, -1.0, float("inf"), float("nan")]))
    elif m == "bad_beta":
        hp.beta2 = 1.0
    elif m == "clip_speculative":
        hp.mode, hp.max_grad_norm = 0, 1.0
    elif m == "owner_range":
        a.owner_first = nd
    elif m == "owner_count":
        a.owner_count = 0
    elif m == "bad_layout":
        a.grad_layout = 9
    elif m == "short_stride" and layout == 0 and nd > 1 and not peers:
        a.grad_rank_stride = psi - 1 if psi > 1 else 0
    elif m == "bad_storage":
        a.storage = 2
    elif m == "no_stash":
        hp.mode = 2
        a.grad_stash = None
    elif m == "null_slot1":
        hp.mode, hp.max_grad_norm = 0, 0.0
        a.master[1] = None
    elif m == "peer_null" and peers:
        q.rank_grads[nd - 1] = None
    elif m == "peer_odd" and peers:
        q.rank_grads[0] = FAKE + 1
    elif m == "peer_dests" and peers:
        q.n_param_dests = 65
    elif m == "peer_layout" and peers:
        a.grad_layout = 1
    elif m == "reserved":
        hp.reserved = 1
    else:
        m = "none"
    return plan, hp, a, m


@settings(max_examples=600, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(cases())
def test_step_checks_return_a_documented_status(case):
    plan_kw, hp, args, mutation = case
    plan = B.zero_plan(**plan_kw)
    try:
        n = C.c_size_t(0)
        status = B.lib().zero_workspace_bytes(plan, C.byref(hp), C.byref(args), C.byref(n))
        assert status in STATUSES, status
        if mutation == "none":
            # a valid configuration is planned: the header plus the fp64
            # partials of the statistics passes (none in speculative mode)
            assert status == B.ZERO_OK, B.zero_last_error()
            assert n.value >= 256 and (n.value - 256) % 8 == 0
            if hp.mode == B.ZERO_MODE_SPECULATIVE:
                assert n.value == 256
        else:
            assert status == EXPECTED[mutation], (mutation, status, B.zero_last_error())
            assert B.zero_last_error()
    finally:
        B.zero_plan_destroy(plan)
