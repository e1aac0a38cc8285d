"""Pins of the oracle's accounting against the numbers the pages print."""
import os

import pytest

import oracle
from _util import read_golden

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kv(rows):
    return {r[0]: r[1:] for r in rows}


def test_sixteen_bytes_per_parameter():
    g = {k: int(v[0]) for k, v in _kv(read_golden(os.path.join(GOLDEN, "model_state_bytes_per_param.txt"))).items()}
    assert g["fp32_param_copy"] + g["fp32_momentum"] + g["fp32_variance"] == g["adam_K"]
    assert g["fp16_params"] + g["fp16_grads"] + g["adam_K"] == g["total"]
    psi = 1_000_003
    r = oracle.state_bytes(psi, 1, 0)
    assert r["params_bytes"] == g["fp16_params"] * psi
    assert r["grads_bytes"] == g["fp16_grads"] * psi
    assert r["optim_bytes"] == g["adam_K"] * psi
    assert r["total_bytes"] == g["total"] * psi


def test_7p5b_nd64_printed_memory_and_comm():
    rows = read_golden(os.path.join(GOLDEN, "zero_7p5b_nd64.txt"))
    psi = int(rows[0][1])
    nd = int(rows[1][1])
    baseline = oracle.state_bytes(psi, nd, 0)["total_bytes"]
    for row in rows[2:]:
        stage, gb, red, comm = int(row[1]), float(row[2]), float(row[3]), float(row[4])
        r = oracle.state_bytes(psi, nd, stage)
        # printed to one decimal of decimal GB
        assert round(r["total_bytes"] / 1e9, 1) == gb, (stage, r["total_bytes"])
        assert r["comm_elems"] == comm * psi
        if stage in (0, 3):
            assert baseline / r["total_bytes"] == red
        else:
            # the printed 4x / 8x are the limits as Nd grows
            far = oracle.state_bytes(psi, 1 << 30, stage)
            assert abs(far["reduction"] - red) < 1e-6 * red
            assert r["reduction"] < red
    # exact values behind the rounded figures
    assert oracle.state_bytes(psi, nd, 1)["total_bytes"] == 31_406_250_000
    assert oracle.state_bytes(psi, nd, 2)["total_bytes"] == 16_640_625_000
    assert oracle.state_bytes(psi, nd, 3)["total_bytes"] == 1_875_000_000


def test_gpt2_1p5b_model_state():
    g = _kv(read_golden(os.path.join(GOLDEN, "gpt2_1p5b_model_state.txt")))
    psi = int(g["psi"][0])
    r = oracle.state_bytes(psi, 1, 0)
    assert r["total_bytes"] / 1e9 >= float(g["model_state_gb_at_least"][0])
    assert r["params_bytes"] / 1e9 == float(g["fp16_weights_gb"][0])
    # the GPT-2 XL tensor list used by the workloads (1,557,611,200 params)
    # also clears the printed floor
    assert oracle.state_bytes(1_557_611_200, 1, 0)["total_bytes"] / 1e9 >= 24


def test_comm_volume_table():
    rows = read_golden(os.path.join(GOLDEN, "comm_volume.txt"))
    psi = 123_456_789
    for row in rows:
        if row[0] == "stage":
            stage, total, rs, ags = (int(x) for x in row[1:])
            r = oracle.state_bytes(psi, 8, stage)
            assert r["comm_elems"] == total * psi == (rs + ags) * psi
            assert r["comm_bytes"] == 2 * total * psi
        else:
            ratio = float(row[1])
            assert (oracle.state_bytes(psi, 8, 3)["comm_elems"]
                    / oracle.state_bytes(psi, 8, 0)["comm_elems"]) == ratio


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
def test_nd1_collapses_to_16psi(stage):
    psi = 987_654_321
    r = oracle.state_bytes(psi, 1, stage)
    assert r["total_bytes"] == 16 * psi
    assert r["total_bytes_padded"] == 16 * psi
    assert r["reduction"] == 1.0


def test_limits_and_linear_scaling():
    psi = 10 ** 9
    # stage 1 -> 4 Psi, stage 2 -> 2 Psi as Nd grows; stage 3 is 16 Psi / Nd
    assert abs(oracle.state_bytes(psi, 1 << 30, 1)["total_bytes"] - 4 * psi) < 1e3
    assert abs(oracle.state_bytes(psi, 1 << 30, 2)["total_bytes"] - 2 * psi) < 1e3
    for nd in (2, 8, 64, 1000):
        assert oracle.state_bytes(psi, nd, 3)["total_bytes"] == pytest.approx(16 * psi / nd, rel=1e-15)
        assert oracle.state_bytes(psi, nd, 3)["reduction"] == pytest.approx(nd, rel=1e-15)


def test_padded_bytes_use_the_shard_length():
    psi, nd, a = 1_000_003, 4, 256
    L = oracle.plan(psi, nd, a).shard_len
    assert oracle.state_bytes(psi, nd, 1, a)["total_bytes_padded"] == 4 * psi + 12 * L
    assert oracle.state_bytes(psi, nd, 2, a)["total_bytes_padded"] == 2 * psi + 14 * L
    assert oracle.state_bytes(psi, nd, 3, a)["total_bytes_padded"] == 16 * L
    r = oracle.state_bytes(psi, nd, 3, a)
    assert r["comm_elems_ring"] == pytest.approx(3 * psi * (nd - 1) / nd)


def test_rejects_bad_arguments():
    for args in ((0, 1, 1), (10, 0, 1), (10, 1, 4), (10, 1, -1)):
        with pytest.raises(ValueError):
            oracle.state_bytes(*args)
