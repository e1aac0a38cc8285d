"""C-ABI checks that need no GPU: the library loads and exports every
function include/*.h declares, the ctypes structs match the C layout, the
host planner and accounting agree bit for bit with the oracle, and invalid
arguments are rejected before anything is launched."""
import ctypes as C
import glob
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from zero_dp_partitioned_shard_b200 import binding as B
from zero_dp_partitioned_shard_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(zero_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert {"zero_plan", "zero_shard_step", "zero_gather_params", "zero_state_bytes"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = declared - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    # the binding covers exactly the declared surface
    assert set(B.SIGNATURES) == declared
    lib = B.lib()
    for name in declared:
        assert getattr(lib, name) is not None
    assert B.zero_abi_version() == 9
    # nothing else leaks out of the library (hidden visibility)
    assert all(n.startswith("zero_") for n in exported if not n.startswith("_"))


_LAYOUT_PROBE = r"""
#include <stdio.h>
#include <stddef.h>
#include "zero_shard.h"
#define S(T) printf(#T " %zu\n", sizeof(T));
#define O(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  S(zero_plan_desc) S(zero_plan_info) S(zero_segment) S(zero_state_report)
  S(zero_opt_state) S(zero_step_result) S(zero_hparams) S(zero_step_args)
  O(zero_step_args, master) O(zero_step_args, params) O(zero_step_args, workspace_bytes)
  O(zero_step_args, timing_events) O(zero_hparams, mode) O(zero_opt_state, cur)
  O(zero_step_result, overflow) O(zero_step_result, status) O(zero_step_result, loss_scale)
  O(zero_opt_state, loss_scale) O(zero_opt_state, growth_interval) O(zero_plan_desc, nd) O(zero_plan_info, nd)
  S(zero_peer_args) S(zero_ipc_handle) O(zero_step_args, peers) O(zero_peer_args, param_dests)
  O(zero_peer_args, n_param_dests) O(zero_ipc_handle, offset) O(zero_ipc_handle, device)
  return 0;
}
"""


def test_ctypes_structs_match_the_c_header(tmp_path):
    src = tmp_path / "probe.c"
    src.write_text(_LAYOUT_PROBE)
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = dict(line.rsplit(" ", 1) for line in subprocess.run([str(exe)], capture_output=True,
                                                             text=True, check=True).stdout.split("\n") if line)
    got = {k: int(v) for k, v in got.items()}
    py = {"zero_plan_desc": B.PlanDesc, "zero_plan_info": B.PlanInfo, "zero_segment": B.Segment,
          "zero_state_report": B.StateReport, "zero_opt_state": B.OptState,
          "zero_step_result": B.StepResult, "zero_hparams": B.HParams, "zero_step_args": B.StepArgs,
          "zero_peer_args": B.PeerArgs, "zero_ipc_handle": B.IpcHandle}
    for cname, ctype in py.items():
        assert got[cname] == C.sizeof(ctype), cname
    for key, val in got.items():
        if "." in key:
            cname, field = key.split(".")
            assert getattr(py[cname], field).offset == val, key
    assert got["zero_opt_state"] <= B.OPT_STATE_BYTES and got["zero_step_result"] <= B.RESULT_BYTES


def _plan_cases():
    rs = np.random.default_rng(5)
    cases = [(1, 1, 1, 0), (7, 3, 1, 0), (1_000_003, 4, 256, 0), (1_000_003, 4, 256, 25_000),
             (1_557_611_200, 8, 256, 0), (7_500_000_000, 64, 256, 0), (7_500_000_000, 64, 1, 0),
             (1_315_723_264, 16, 256, 25_000_000), (5, 64, 8, 3)]
    for _ in range(200):
        cases.append((int(rs.integers(1, 100_000)), int(rs.integers(1, 70)),
                      int(rs.choice([1, 2, 8, 16, 256])), int(rs.choice([0, 1, 7, 1000, 4096]))))
    return cases


def test_planner_matches_oracle_bit_exact():
    for psi, nd, a, b in _plan_cases():
        ref = oracle.plan(psi, nd, a, b)
        h = B.zero_plan(psi, nd, stage=2, align_elems=a, bucket_elems=b)
        try:
            info = B.zero_plan_query(h)
            assert (info.psi, info.psi_pad, info.shard_len, info.n_buckets) == \
                   (ref.psi, ref.psi_pad, ref.shard_len, ref.n_buckets)
            for r in sorted({0, nd - 1, nd // 2}):
                assert B.zero_plan_shard(h, r) == ref.shard(r)
            for k in sorted({0, ref.n_buckets - 1}):
                assert B.zero_plan_bucket(h, k) == ref.bucket_range(k)
        finally:
            B.zero_plan_destroy(h)


def test_segments_match_oracle():
    rs = np.random.default_rng(8)
    lists = [synth.transformer_24l_d2048_tensor_sizes(), synth.gpt2_xl_tensor_sizes()]
    for _ in range(30):
        lists.append([int(x) for x in rs.integers(0, 500, size=int(rs.integers(1, 20)))])
    for sizes in lists:
        psi = sum(sizes)
        if psi == 0:
            continue
        for nd, a in ((16, 256), (8, 256), (3, 1), (7, 16)):
            ref = oracle.plan(psi, nd, a).tensor_segments(sizes)
            h = B.zero_plan(psi, nd, align_elems=a, tensor_sizes=sizes)
            try:
                got = np.array(B.zero_plan_segments(h), dtype=np.int64).reshape(-1, 5)
                assert np.array_equal(got, ref)
                assert B.zero_plan_query(h).n_segments == len(ref)
            finally:
                B.zero_plan_destroy(h)


def test_state_bytes_matches_oracle_bit_exact():
    for psi, nd, a, _ in _plan_cases()[:60]:
        for stage in range(4):
            got = B.zero_state_bytes(psi, nd, stage, a)
            ref = oracle.state_bytes(psi, nd, stage, a)
            for k, v in ref.items():
                assert got[k] == v, (psi, nd, stage, a, k)


@pytest.mark.parametrize("bad", [dict(psi=0, nd=1), dict(psi=10, nd=0), dict(psi=10, nd=2, stage=4),
                                 dict(psi=10, nd=2, align_elems=0), dict(psi=10, nd=2, bucket_elems=-1),
                                 dict(psi=10, nd=2, tensor_sizes=[3, 3])])
def test_plan_rejects_bad_descriptions(bad):
    with pytest.raises(B.ZeroError) as e:
        B.zero_plan(**bad)
    assert e.value.status == B.ZERO_ERR_INVALID_ARG


# --- validation of zero_shard_step: every case below is rejected by host-side
# checks before anything is launched (addresses are never dereferenced) ---

FAKE = 1 << 40  # 256-byte aligned fake device address


def _args(**kw):
    base = dict(grads=FAKE, grad_rank_stride=1024, master=(FAKE, FAKE), exp_avg=(FAKE, FAKE),
                exp_avg_sq=(FAKE, FAKE), params=FAKE, opt_state=FAKE, workspace=FAKE,
                workspace_bytes=1 << 20, owner_first=0, owner_count=4)
    base.update(kw)
    return B.step_args(**base)


@pytest.mark.parametrize("case,status", [
    ("owner_range", B.ZERO_ERR_INVALID_ARG), ("owner_count0", B.ZERO_ERR_INVALID_ARG),
    ("null_grads", B.ZERO_ERR_INVALID_ARG), ("null_slot1", B.ZERO_ERR_INVALID_ARG),
    ("stride_small", B.ZERO_ERR_INVALID_ARG), ("bad_layout", B.ZERO_ERR_INVALID_ARG),
    ("bad_mode", B.ZERO_ERR_INVALID_ARG), ("bad_scale", B.ZERO_ERR_INVALID_ARG),
    ("bad_beta", B.ZERO_ERR_INVALID_ARG), ("clip_spec", B.ZERO_ERR_UNSUPPORTED),
    ("stash_missing", B.ZERO_ERR_INVALID_ARG), ("misaligned_master", B.ZERO_ERR_ALIGNMENT),
    ("misaligned_params", B.ZERO_ERR_ALIGNMENT), ("small_ws", B.ZERO_ERR_WORKSPACE),
    ("null_ws", B.ZERO_ERR_WORKSPACE), ("misaligned_ws", B.ZERO_ERR_ALIGNMENT),
    ("reserved", B.ZERO_ERR_INVALID_ARG), ("bad_storage", B.ZERO_ERR_INVALID_ARG),
    ("peer_layout", B.ZERO_ERR_UNSUPPORTED), ("peer_null_grad", B.ZERO_ERR_INVALID_ARG),
    ("peer_misaligned_grad", B.ZERO_ERR_ALIGNMENT), ("peer_null_dest", B.ZERO_ERR_INVALID_ARG),
    ("peer_misaligned_dest", B.ZERO_ERR_ALIGNMENT), ("peer_n_dests", B.ZERO_ERR_INVALID_ARG),
    ("peer_reserved", B.ZERO_ERR_INVALID_ARG),
])
def test_step_validation_rejects_before_launch(case, status):
    plan = B.zero_plan(1000, 4, stage=1, align_elems=8)
    hp = B.hparams(loss_scale=1024.0)
    args = _args()
    if case == "owner_range":
        args = _args(owner_first=2, owner_count=3)
    elif case == "owner_count0":
        args = _args(owner_count=0)
    elif case == "null_grads":
        args = _args(grads=0)
    elif case == "null_slot1":
        args = _args(master=(FAKE, 0))
    elif case == "stride_small":
        args = _args(grad_rank_stride=999)
    elif case == "bad_layout":
        args = _args(grad_layout=7)
    elif case == "bad_mode":
        hp = B.hparams(loss_scale=1024.0, mode=9)
    elif case == "bad_scale":
        hp = B.hparams(loss_scale=0.0)
    elif case == "bad_beta":
        hp = B.hparams(loss_scale=1.0, beta2=1.0)
    elif case == "clip_spec":
        hp = B.hparams(loss_scale=1.0, max_grad_norm=1.0)
    elif case == "stash_missing":
        hp = B.hparams(loss_scale=1.0, mode=B.ZERO_MODE_STASH)
    elif case == "misaligned_master":
        args = _args(master=(FAKE + 2, FAKE))
    elif case == "misaligned_params":
        args = _args(params=FAKE + 1)
    elif case == "small_ws":
        args = _args(workspace_bytes=16)
    elif case == "null_ws":
        args = _args(workspace=0)
    elif case == "misaligned_ws":
        args = _args(workspace=FAKE + 16)
    elif case == "reserved":
        hp.reserved = 1
    elif case == "bad_storage":
        args = _args()
        args.storage = 2
    elif case.startswith("peer_"):
        grads = [FAKE + (r << 20) for r in range(4)]
        dests = [FAKE + (9 << 20), FAKE + (10 << 20)]
        layout = B.ZERO_GRADS_FULL
        if case == "peer_layout":
            layout = B.ZERO_GRADS_PER_OWNER
        elif case == "peer_null_grad":
            grads[2] = 0
        elif case == "peer_misaligned_grad":
            grads[1] += 1
        elif case == "peer_null_dest":
            dests[1] = 0
        elif case == "peer_misaligned_dest":
            dests[0] += 3
        q = B.peer_args(grads, dests)
        if case == "peer_n_dests":
            q.n_param_dests = B.ZERO_MAX_PEERS + 1
        elif case == "peer_reserved":
            q.reserved = 1
        args = B.attach_peers(_args(grads=0, grad_layout=layout), q)
    before = B.zero_launch_count()
    try:
        with pytest.raises(B.ZeroError) as e:
            B.zero_shard_step(plan, hp, args)
        assert e.value.status == status, B.zero_last_error()
        assert B.zero_last_error()
    finally:
        B.zero_plan_destroy(plan)
    assert B.zero_launch_count() == before


def test_peer_tables_replace_the_strided_gradients():
    """With peer tables the gradient pointer and stride are not used; a plan
    with more ranks than the tables hold is refused."""
    plan = B.zero_plan(1000, 4, stage=2, align_elems=8)
    try:
        q = B.peer_args([FAKE + (r << 20) for r in range(4)], [FAKE + (7 << 20)])
        args = B.attach_peers(_args(grads=0, grad_rank_stride=0), q)
        assert B.zero_workspace_bytes(plan, B.hparams(loss_scale=1.0), args) == 256
        B.attach_peers(args, None)
        with pytest.raises(B.ZeroError) as e:     # without the tables the null grads are an error
            B.zero_workspace_bytes(plan, B.hparams(loss_scale=1.0), args)
        assert e.value.status == B.ZERO_ERR_INVALID_ARG
    finally:
        B.zero_plan_destroy(plan)
    big = B.zero_plan(100_000, B.ZERO_MAX_PEERS + 1, stage=2, align_elems=8)
    try:
        q = B.peer_args([FAKE] * B.ZERO_MAX_PEERS)
        args = B.attach_peers(_args(grads=0, owner_count=1), q)
        with pytest.raises(B.ZeroError) as e:
            B.zero_workspace_bytes(big, B.hparams(loss_scale=1.0), args)
        assert e.value.status == B.ZERO_ERR_UNSUPPORTED
    finally:
        B.zero_plan_destroy(big)


def test_reduced_layout_and_reduce_scatter_validation():
    """The REDUCED layout takes one value per element (no stride); the
    reduce-scatter with retention accepts FULL / PER_OWNER sources only, a
    bucket inside the plan and a 2-byte aligned destination."""
    plan = B.zero_plan(1000, 4, stage=2, align_elems=8, bucket_elems=300)
    hp = B.hparams(loss_scale=1.0)
    lib = B.lib()
    try:
        red = _args(grad_layout=B.ZERO_GRADS_REDUCED, grad_rank_stride=0)
        assert B.zero_workspace_bytes(plan, hp, red) == 256
        q = B.peer_args([FAKE] * 4)
        with pytest.raises(B.ZeroError) as e:
            B.zero_workspace_bytes(plan, hp, B.attach_peers(_args(grad_layout=B.ZERO_GRADS_REDUCED), q))
        assert e.value.status == B.ZERO_ERR_UNSUPPORTED

        def reduce_status(args, bucket, out):
            before = B.zero_launch_count()
            st = lib.zero_reduce_scatter(plan, C.byref(args), bucket, out, None)
            assert B.zero_launch_count() == before        # rejected before any launch
            return st

        full = _args()
        assert reduce_status(full, 4, FAKE) == B.ZERO_ERR_INVALID_ARG           # 4 buckets: 0..3
        assert reduce_status(full, 0, None) == B.ZERO_ERR_INVALID_ARG
        assert reduce_status(full, 0, FAKE + 1) == B.ZERO_ERR_ALIGNMENT
        assert reduce_status(red, 0, FAKE) == B.ZERO_ERR_INVALID_ARG            # REDUCED is not a source
        assert reduce_status(_args(grads=0), 0, FAKE) == B.ZERO_ERR_INVALID_ARG
        assert reduce_status(_args(owner_first=3, owner_count=2), 0, FAKE) == B.ZERO_ERR_INVALID_ARG
        assert reduce_status(_args(grad_rank_stride=999), -1, FAKE) == B.ZERO_ERR_INVALID_ARG
    finally:
        B.zero_plan_destroy(plan)


def test_ipc_helpers_validate_arguments():
    lib = B.lib()
    assert lib.zero_ipc_export(None, None) == B.ZERO_ERR_INVALID_ARG
    assert lib.zero_ipc_open(None, None) == B.ZERO_ERR_INVALID_ARG
    with pytest.raises(B.ZeroError) as e:   # not an address zero_ipc_open returned
        B.zero_ipc_close(FAKE)
    assert e.value.status == B.ZERO_ERR_INVALID_ARG
    h = B.IpcHandle()
    h.offset = -1
    p = C.c_void_p()
    assert lib.zero_ipc_open(C.byref(h), C.byref(p)) == B.ZERO_ERR_INVALID_ARG


def test_workspace_bytes_per_mode():
    plan = B.zero_plan(1_315_723_264, 16, stage=2, align_elems=256, bucket_elems=25_000_000)
    try:
        args = _args(grad_rank_stride=1_315_723_264, owner_count=16, grad_stash=FAKE)
        spec = B.zero_workspace_bytes(plan, B.hparams(loss_scale=1.0), args)
        two = B.zero_workspace_bytes(plan, B.hparams(loss_scale=1.0, mode=B.ZERO_MODE_TWO_PASS,
                                                      max_grad_norm=1.0), args)
        assert spec == 256
        assert two == 256 + 53 * 2048 * 8
    finally:
        B.zero_plan_destroy(plan)


def test_strerror_names_every_status():
    for s in range(7):
        assert B.zero_strerror(s) and "unknown" not in B.zero_strerror(s)
    assert "unknown" in B.zero_strerror(99)


def test_wait_budget_hook_round_trips():
    default = B.zero_set_wait_budget(12345)
    assert default == 1 << 31
    assert B.zero_set_wait_budget(-1) == 12345
    assert B.zero_set_wait_budget(0) == -1
    assert B.zero_set_wait_budget(0) == 1 << 31


def test_gather_tensors_validation():
    no_list = B.zero_plan(100, 2, align_elems=8)
    with_list = B.zero_plan(100, 2, align_elems=8, tensor_sizes=[30, 30, 40])
    try:
        for plan, first, count in ((no_list, 0, 1), (with_list, 2, 2), (with_list, -1, 1)):
            before = B.zero_launch_count()
            with pytest.raises(B.ZeroError) as e:
                B.zero_gather_tensors(plan, first, count, [FAKE, FAKE], FAKE, True)
            assert e.value.status == B.ZERO_ERR_INVALID_ARG
            assert B.zero_launch_count() == before
        with pytest.raises(B.ZeroError) as e:    # compact gather with a missing owner shard
            B.zero_gather_tensors(with_list, 0, 3, [FAKE, 0], FAKE, True)
        assert e.value.status == B.ZERO_ERR_INVALID_ARG
    finally:
        B.zero_plan_destroy(no_list)
        B.zero_plan_destroy(with_list)


_C_CALLER = r"""
/* A plain C caller of libzero_shard.so: host-only entry points and the
 * checks that reject a step before anything is launched. */
#include <stdio.h>
#include <string.h>
#include "zero_shard.h"
#define CHECK(c) do { if (!(c)) { printf("FAIL line %d\n", __LINE__); return 1; } } while (0)
int main(void) {
    CHECK(zero_abi_version() == ZERO_SHARD_ABI_VERSION);
    /* the pages' 7.5B / Nd = 64 example, stage 3: 1.875 GB per device, 3 Psi moved */
    zero_state_report r;
    CHECK(zero_state_bytes(7500000000LL, 64, 3, 1, &r) == ZERO_OK);
    CHECK(r.total_bytes == 1.875e9 && r.comm_elems == 3 * 7.5e9);
    /* the GPT-2 1.5B-shaped plan at Nd = 8 */
    zero_plan_desc d;
    memset(&d, 0, sizeof d);
    d.psi = 1557611200; d.nd = 8; d.stage = 2; d.align_elems = 256;
    zero_plan_t* plan = NULL;
    CHECK(zero_plan(&d, &plan) == ZERO_OK && plan);
    zero_plan_info info;
    CHECK(zero_plan_query(plan, &info) == ZERO_OK);
    CHECK(info.shard_len == 194701568 && info.psi_pad == 8 * 194701568LL);
    int64_t start = 0, len = 0;
    CHECK(zero_plan_shard(plan, 7, &start, &len) == ZERO_OK && start == 7 * 194701568LL && len == 194700224);
    /* a step with no buffers is refused before any launch */
    zero_hparams hp;
    memset(&hp, 0, sizeof hp);
    hp.loss_scale = 1.0f; hp.beta1 = 0.9f; hp.beta2 = 0.999f;
    zero_step_args a;
    memset(&a, 0, sizeof a);
    a.owner_count = 8; a.grad_rank_stride = info.psi_pad;
    const uint64_t before = zero_launch_count();
    CHECK(zero_shard_step(plan, &hp, &a, NULL) == ZERO_ERR_INVALID_ARG);
    CHECK(strlen(zero_last_error()) > 0);
    CHECK(zero_launch_count() == before);
    CHECK(strcmp(zero_strerror(ZERO_ERR_UNSUPPORTED), zero_strerror(ZERO_OK)) != 0);
    zero_plan_destroy(plan);
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_caller_links_and_calls_the_library(tmp_path):
    """The ABI from C, not only through ctypes: a C program includes the
    header, links libzero_shard.so and calls its host-side entry points."""
    src = tmp_path / "caller.c"
    src.write_text(_C_CALLER)
    exe = tmp_path / "caller"
    pkg = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", pkg, "-lzero_shard", "-Wl,-rpath," + pkg], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


def test_recent_kernels_record_arguments():
    """zero_recent_kernels: argument checks, and nothing recorded before the
    first launch of the process (the CPU suite launches no kernel)."""
    lib = B.lib()
    assert lib.zero_recent_kernels(None, -1) == -1
    assert lib.zero_recent_kernels(None, 4) == -1
    assert lib.zero_recent_kernels(None, 0) == 0
    if B.zero_launch_count() == 0:
        assert B.zero_recent_kernels() == []
