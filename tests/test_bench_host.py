"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes per
parameter that make the roofline numerator, the moved bytes per mode, and the
lookup of ncu traffic in profiles/ (taken only from a summary captured on the
current kernels.cu)."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("nd", [1, 2, 4, 8, 16, 64])
def test_bytes_per_param_match_the_documented_formulas(nd):
    alg, spec = bench.bytes_per_param(nd, 0)
    assert alg == 2 * nd + 26 and spec == alg                 # speculative moves exactly the algorithmic bytes
    assert bench.bytes_per_param(nd, 1) == (alg, 4 * nd + 26)  # two-pass re-reads the contributions
    assert bench.bytes_per_param(nd, 2) == (alg, 2 * nd + 34)  # stash writes and reads 4 B more
    assert bench.update_launch_bytes(nd, 0) == alg
    assert bench.update_launch_bytes(nd, 2) == 30              # the stash source: 4 B instead of 2 Nd
    assert bench.update_launch_bytes(nd, 0, nd - 1) == alg + 2 * (nd - 1)   # peer tables: one store per destination


def test_named_values():
    # the per-parameter figures quoted for the workloads
    assert [bench.bytes_per_param(n, 0)[0] for n in (1, 2, 4, 8, 16, 64)] == [28, 30, 34, 42, 58, 154]


def _write(tmp, name, sha, nd, mode, per):
    os.makedirs(os.path.join(tmp, "profiles"), exist_ok=True)
    with open(os.path.join(tmp, "profiles", name), "w") as f:
        f.write(f"# capture\n\n| counter | value |\n|---|---|\n| x | 1 |\n\n"
                f"traffic_bytes_per_param: {per}\ntraffic_nd: {nd}\ntraffic_mode: {mode}\n"
                f"kernels_cu_sha256_prefix: {sha}\n")


def test_traffic_only_from_a_capture_of_the_current_kernels(tmp_path, monkeypatch):
    src_dir = tmp_path / "zero_dp_partitioned_shard_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (src_dir / "kernels.cu").write_text("// kernels v1\n")
    sha = hashlib.sha256(b"// kernels v1\n").hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic(8, 0, 1000) == (None, None)          # no summary at all
    _write(str(tmp_path), "a.md", "0123456789abcdef", 8, "speculative", 41.5)
    assert bench.profiled_traffic(8, 0, 1000) == (None, None)          # a stale capture is not used
    _write(str(tmp_path), "b.md", sha, 8, "speculative", 41.5)
    traffic, path = bench.profiled_traffic(8, 0, 1000)
    assert traffic == pytest.approx(41500.0) and path.endswith("b.md")  # scaled by the parameters
    assert bench.profiled_traffic(16, 0, 1000) == (None, None)         # another Nd
    assert bench.profiled_traffic(8, 2, 1000) == (None, None)          # another mode


def test_the_committed_profiles_carry_the_keys_the_lookup_reads():
    keys = {}
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        with open(os.path.join(ROOT, "profiles", name)) as f:
            text = f.read()
        if "traffic_bytes_per_param:" in text:
            kv = dict(line.split(":", 1) for line in text.splitlines()
                      if line.startswith(("traffic_", "kernels_cu_sha256_prefix")))
            keys[name] = {k.strip(): v.strip() for k, v in kv.items()}
    assert keys, "no profile carries traffic figures"
    for name, kv in keys.items():
        assert set(kv) == {"traffic_bytes_per_param", "traffic_nd", "traffic_mode", "kernels_cu_sha256_prefix"}, name
        assert 0 < float(kv["traffic_bytes_per_param"]) < 200 and len(kv["kernels_cu_sha256_prefix"]) == 16


def test_step_bytes_of_a_run_with_skipped_steps():
    # applied steps: (2 Nd + 26) per owned parameter + 4 per assembled one
    assert bench.step_alg_bytes(1000, 0, 8, 3, 0) == 3 * 1000 * 42
    assert bench.step_alg_bytes(100, 6300, 64, 1, 0) == 100 * 154 + 4 * 6300
    # a skipped step only read the contributions
    assert bench.step_alg_bytes(1000, 0, 16, 20, 1) == 19 * 1000 * 58 + 1000 * 32
    assert bench.step_alg_bytes(1000, 0, 16, 1, 1) == 1000 * 32


def test_sharded_report_volumes():
    comm = {"comm_elems": 2 * 1000, "comm_elems_ring": 2 * 1000 * 3 / 4}
    rep = bench.sharded_report(1000, 4, 256, 10, 20.0, 0.5, "nccl", 6500.0, comm)
    assert rep["exchange"]["elements_each_way"] == 2 * 3 * 256
    assert rep["exchange"]["bytes_each_way"] == 4 * 3 * 256
    assert rep["exchange"]["link_bound_ms"] == pytest.approx(4 * 3 * 256 / 770e9 * 1e3)
    assert rep["accounting"]["exchanged_over_ring"] == pytest.approx(4 * 256 / 1000)
    assert rep["step_ms"] == 2.0
    assert rep["update"]["alg_bytes"] == 256 * (2 * 4 + 26)
    assert rep["update"]["gbs"] == pytest.approx(256 * 34 / 0.5e-3 / 1e9)


def test_host_cpu_reports_count_and_model():
    h = bench.host_cpu()
    assert h["host_cpus"] == os.cpu_count()
    assert h["cpu_model"] is None or isinstance(h["cpu_model"], str)


class _FakeRecord:
    def __init__(self, names):
        self.names = names

    def zero_recent_kernels(self, n):
        return self.names[-n:]


def test_launched_update_kernel_reads_the_launch_record():
    pipe = "_ZN2zs21zs_update_pipe_kernelILi0ELi4ELb0ELb0ELb0ELb1ELi2EEEvNS_10UpdateArgsE"
    regs = "_ZN2zs16zs_update_kernelILi0ELb1ELb0ELb0EEEvNS_10UpdateArgsE"
    prep, commit = "_ZN2zs14zs_prep_kernelEPNS_8WsHeaderE", "_ZN2zs16zs_commit_kernelILb1ELb0ELb0EEEv"
    assert bench.launched_update_kernel(_FakeRecord([prep, pipe, commit]), "x") == \
        ("zs_update_pipe_kernel", pipe, "launch record")
    assert bench.launched_update_kernel(_FakeRecord([regs, commit, prep, regs, commit]), "x") == \
        ("zs_update_kernel", regs, "launch record")
    # the newest update kernel wins
    assert bench.launched_update_kernel(_FakeRecord([pipe, commit, regs, commit]), "x")[0] == "zs_update_kernel"
    assert bench.launched_update_kernel(_FakeRecord([prep, commit]), "fallback") == ("fallback", None, "shape rule")
