"""Failure detection without a GPU fault: every wait inside the pipelined
update kernel is bounded.  The library's test hook makes every pipeline wait
expire at once (a wait that nothing satisfies in time); the kernel must then
record ZERO_ERR_TIMEOUT in the step result, leave the (speculative) state and
the step counter untouched and return, so that the very next step on the same
context runs normally and matches the oracle."""
import numpy as np
import pytest
import torch

from _gpu import make_problem, run_gpu, run_oracle, to_oracle_hp
from _util import assert_f16_close, assert_f32_close
from zero_dp_partitioned_shard_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    B.zero_set_wait_budget(0)


def test_expired_pipeline_wait_reports_timeout_and_keeps_state():
    # Nd = 2, speculative, 16-byte aligned: the bulk-copy pipelined kernel
    pb = make_problem(100_003, 2, align=256, steps=1, seed=61, S=1024.0, random_state=True)
    hp = B.hparams(loss_scale=1024.0)
    B.zero_set_wait_budget(-1)
    g = run_gpu(pb, hp)
    B.zero_set_wait_budget(0)
    r = g.results[0]
    assert r.status == B.ZERO_ERR_TIMEOUT
    assert r.overflow == 0
    assert g.opt.t == 0 and g.opt.skipped == 1
    for a, b in ((g.master, pb.master), (g.exp_avg, pb.exp_avg), (g.exp_avg_sq, pb.exp_avg_sq)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(g.params, pb.params)
    # the context is still usable: a normal step right after matches the oracle
    g2 = run_gpu(pb, hp)
    o = run_oracle(pb, to_oracle_hp(hp))
    assert g2.results[0].status == B.ZERO_OK and g2.opt.t == 1
    assert_f32_close(g2.master, o.master, 2, "master")
    assert_f16_close(g2.params, o.params, 1, "params")
