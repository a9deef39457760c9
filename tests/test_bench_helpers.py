"""Host-side pieces of bench.py that need no GPU: the roofline traffic taken
from the committed ncu summary (and dropped once the kernel source changes),
and the workload description in the JSON line."""
import hashlib
import importlib.util
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench(path):
    spec = importlib.util.spec_from_file_location("bench_under_test", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_recorded_traffic_follows_the_kernel_source(tmp_path):
    # a copy of the repository layout the function reads
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "clustered_block_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "bench.py"), tmp_path / "bench.py")
    src = csrc / "attention_tc.cu"
    src.write_text("// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "attention_tc_wan.txt").write_text(
        f"summary\n\ntraffic_bytes_per_head: 1000\nkernel_source_sha256: {sha}\n")
    bench = _load_bench(str(tmp_path / "bench.py"))
    assert bench.recorded_traffic(40) == 40000
    src.write_text("// kernel v2\n")  # the capture no longer describes the kernel
    assert bench.recorded_traffic(40) is None


def test_config_names_the_workload():
    bench = _load_bench(os.path.join(ROOT, "bench.py"))
    w = bench.WORKLOADS["wan"]
    cfg = bench.config_of(w, 1)
    assert cfg["workload"] == w.name and cfg["heads"] == 40 and cfg["n_q"] == 75600
    assert "no collective" in cfg["parallelism"]
    with pytest.raises(KeyError):
        bench.WORKLOADS["unknown"]


def test_stage_bytes_count_each_copy_once():
    """Q's permutation is timed in the k-means stage (it runs under K's
    k-means), so its bytes are counted there: the layer total stays Q, K read
    per k-means iteration, Q, K, V read and written once by the permutations,
    K read by the probe, Q, K, V read and O written by the attention.  The
    gathered layout writes no copy: 5 fewer passes over a token matrix (Q and
    K read and written, V written) and V's permutation row bytes."""
    bench = _load_bench(os.path.join(ROOT, "bench.py"))
    w = bench.WORKLOADS["wan"]
    tok = w.heads * w.n * w.d * 2
    rows = w.heads * w.n
    blocks = w.heads * w.c_q * w.c_k
    p = bench.stage_bytes(w, "permuted")
    g = bench.stage_bytes(w, "gathered")
    kmeans = 2 * w.iters * (tok + 4 * rows)
    permute = 6 * tok + 24 * rows
    total = kmeans + permute + (tok + 4 * blocks) + 9 * blocks + 4 * tok
    assert sum(p.values()) == total
    assert p["kmeans"] == kmeans + 2 * tok + 8 * rows  # with Q's permutation
    assert p["permute"] == 4 * tok + 16 * rows          # K's and V's
    assert sum(p.values()) - sum(g.values()) == 5 * tok + 4 * rows
    assert g["attention"] == p["attention"] == 4 * tok


def test_config_records_the_layout_and_the_kmeans_schedule():
    bench = _load_bench(os.path.join(ROOT, "bench.py"))
    w = bench.WORKLOADS["wan"]
    cfg = bench.config_of(w, 1, "gathered", 1)
    assert cfg["layout"].startswith("gathered") and cfg["kmeans_streams"] == 1
    cfg = bench.config_of(w, 1)
    assert cfg["layout"].startswith("permuted") and cfg["kmeans_streams"] == 2
