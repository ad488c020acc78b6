"""Host-side pieces of bench.py, checked without a GPU: the algorithmic-byte
model against the per-iteration figures of the two-pass model for the
1024x1024 Poisson (fp64 and fp32) and 128^3 diffusion systems, the rule that
a committed ncu traffic figure is used only while the library source matches
it (all of it, or the files the profiled kernel is built from), and clock
sampling that degrades to "no samples" without a GPU."""
import os

import pytest

import bench


def test_two_pass_model_bytes():
    # one sweep of A ((s_v + 4) nnz + 4 (n + 1)) plus 11 vector passes (11 s_v n)
    assert bench.per_iteration_bytes(1_048_576, 5_238_784, 8) == 159_334_404
    assert bench.per_iteration_bytes(1_048_576, 5_238_784, 4) == 92_241_924
    assert bench.per_iteration_bytes(2_097_152, 14_581_760, 8) == 367_919_108
    # the value gradient reads lambda and x, the pattern, and writes nnz values
    assert bench.grad_bytes(1_048_576, 5_238_784, 8) == 12 * 5_238_784 + 20 * 1_048_576


def _profile(tmp_path, key, body):
    d = tmp_path / "profiles"
    d.mkdir(exist_ok=True)
    (d / f"{key}.md").write_text(body)


def test_traffic_is_used_only_for_the_matching_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda files=None: "abc123")
    _profile(tmp_path, "k_launch", "traffic_bytes_per_launch: 1.5e9\nsource_digest: abc123\n")
    _profile(tmp_path, "k_iter", "traffic_bytes_per_iteration: 200\nsource_digest: abc123\n")
    _profile(tmp_path, "k_stale", "traffic_bytes_per_iteration: 200\nsource_digest: ffff00\n")
    _profile(tmp_path, "k_none", "source_digest: abc123\n")
    assert bench.profile_traffic("k_launch", 10) == 1.5e9
    assert bench.profile_traffic("k_iter", 924) == 200 * 924
    assert bench.profile_traffic("k_stale", 924) is None
    assert bench.profile_traffic("k_none", 924) is None
    assert bench.profile_traffic("k_missing", 924) is None


def test_traffic_digest_scoped_to_the_kernel_files(tmp_path, monkeypatch):
    """A summary that names its kernel's source files stays valid while other
    library files change, and goes stale when one of its own files does."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "differentiable_sparse_linear_csr_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "solver.cu").write_text("solver v1")
    (csrc / "common.cuh").write_text("common v1")
    (csrc / "other.cu").write_text("other v1")
    d = bench.source_digest(["solver.cu", "common.cuh"])
    _profile(tmp_path, "k", f"traffic_bytes_per_iteration: 100\nsource_digest: {d}\n"
                            "source_files: solver.cu common.cuh\n")
    assert bench.profile_traffic("k", 10) == 1000
    (csrc / "other.cu").write_text("other v2")
    assert bench.profile_traffic("k", 10) == 1000
    (csrc / "common.cuh").write_text("common v2")
    assert bench.profile_traffic("k", 10) is None
    # a summary without a file list is checked against every file
    _profile(tmp_path, "k_all", f"traffic_bytes_per_iteration: 100\nsource_digest: {bench.source_digest()}\n")
    assert bench.profile_traffic("k_all", 10) == 1000
    (csrc / "other.cu").write_text("other v3")
    assert bench.profile_traffic("k_all", 10) is None
    # a named file that does not exist makes the figure unusable, not an error
    _profile(tmp_path, "k_gone", f"traffic_bytes_per_iteration: 100\nsource_digest: {d}\nsource_files: gone.cu\n")
    assert bench.profile_traffic("k_gone", 10) is None


def test_source_digest_covers_the_library_source():
    d = bench.source_digest()
    assert len(d) == 16 and int(d, 16) >= 0
    assert d == bench.source_digest()


def test_edge_kernel_bytes():
    m = bench.edge_metrics(n=4, nnz=10, E=3, B=2, vbytes=8, asm_ms=1.0, grad_ms=2.0)
    assert m["assemble_bytes"] == 4 * 5 + 8 * 10 + 2 * 8 * (3 + 10 + 1)
    assert m["edge_grad_bytes"] == 8 * 3 + 2 * 8 * (2 * 4 + 3 + 1)
    assert m["assemble_gbs"] == pytest.approx(m["assemble_bytes"] / 1e-3 / 1e9)


def test_clock_sampler_without_a_gpu_returns_nothing():
    if os.path.exists("/dev/nvidiactl"):
        pytest.skip("a GPU driver is present")
    s = bench.ClockSampler(0)
    assert s.stop() is None


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the reference fields (no GPU involved)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.abspath(bench.__file__))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "c1", "--steps", "1", "--warmup", "0", "--ref-iters", "5"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["unit"] == bench.UNIT and d["metric"] == bench.METRIC
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["name"] == "c1"
