"""bench.py's helpers on the CPU: both arms' config objects are identical, the code hash that
guards the committed traffic figure ignores comments and layout but not code, and the L2 note
follows the workload's size."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_config_is_the_workload_alone(bench):
    from state_space_sequence_chunked_b200 import inputs

    for name in ("mamba2_2p7b", "mamba2_2p7b_softplus_dt", "long_n256", "mamba2_130m"):
        wl = inputs.WORKLOADS[name]
        cfg = bench.fwd_config(wl)
        assert cfg == bench.fwd_config(wl)
        assert cfg["workload"] == name and cfg["seqlen"] == wl.seqlen and cfg["dt"] == wl.dt_dist
        assert "path" not in cfg


def test_code_hash_ignores_comments_not_code(bench, tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) {  // doubles\n    return 2 * x;\n}\n")
    b.write_text("// a different comment\nint f(int x)\n{\n  return 2 * x;  // same code\n}\n")
    c.write_text("int f(int x) {\n    return 3 * x;\n}\n")
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b))
    assert bench.code_sha256(str(a)) != bench.code_sha256(str(c))
    assert bench.code_sha256(str(a), str(c)) != bench.code_sha256(str(c), str(a))


def test_traffic_record_matches_the_kernel_code(bench):
    """The committed DRAM traffic of the head-pair kernel is reported for the headline only,
    and only while the record's code hash matches the sources."""
    from state_space_sequence_chunked_b200 import inputs

    t = bench.measured_traffic(inputs.WORKLOADS["mamba2_2p7b"], "tcgen05")
    assert t is not None and 600e6 < t < 760e6
    assert bench.measured_traffic(inputs.WORKLOADS["mamba2_130m"], "tcgen05") is None
    assert bench.measured_traffic(inputs.WORKLOADS["mamba2_2p7b"], "simt") is None


def test_l2_note(bench):
    from state_space_sequence_chunked_b200 import inputs

    assert "no flush" in bench.l2_note(inputs.WORKLOADS["mamba2_2p7b"])
    assert "flushed" in bench.l2_note(inputs.WORKLOADS["mamba2_130m"])
