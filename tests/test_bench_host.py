"""bench.py's host-side helpers (no GPU): the traffic figure it reports, the
source key that ties a committed ncu figure to the kernels it measured, and
the defaults of the command line."""
import importlib.util
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_traffic_scales_a_captured_ratio(bench):
    assert bench.traffic_per_launch(None, 1e6) is None
    assert bench.traffic_per_launch({"dram_bytes_per_algorithmic_byte": 1.5}, 2e6) == pytest.approx(3e6)
    assert bench.traffic_per_launch({"dram_bytes_per_launch": 123.0}, 2e6) == 123.0


def test_code_only_drops_comments_and_spacing(bench):
    a = "int f(int x) {  // add one\n  return x + 1; /* done */\n}\n"
    b = "int f(int x) {\n/* a\n   block */ return x + 1;\n}"
    assert bench._code_only(a) == bench._code_only(b) == "int f(int x) { return x + 1; }"
    assert bench._code_only("int f(int x) { return x + 2; }") != bench._code_only(a)


def test_source_key_ignores_comments_but_not_code(bench, tmp_path):
    src = os.path.join(ROOT, "activation_sparse_ffn_predict_b200", "csrc")
    dst = tmp_path / "activation_sparse_ffn_predict_b200" / "csrc"
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.o", "*.so"))
    root = bench.ROOT
    try:
        bench.ROOT = str(tmp_path)
        base = bench.source_sha()
        cu = dst / "asffn.cu"
        text = cu.read_text()
        cu.write_text("// a new comment line\n" + text)
        assert bench.source_sha() == base
        cu.write_text(text.replace("kWaitNs = 200ull", "kWaitNs = 201ull", 1))
        assert bench.source_sha() != base
    finally:
        bench.ROOT = root


def test_traffic_record_is_used_only_for_the_kernels_it_measured(bench):
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    r = bench.traffic_record("llama70b_reglu:B1:predict")
    if rec["source_sha"] == bench.source_sha():
        assert r is not None and 1.0 <= r["dram_bytes_per_algorithmic_byte"] < 1.01
    else:
        assert r is None          # kernels changed since the capture: the bench reports null
    assert bench.traffic_record("no_such_workload:B1:predict") is None


def test_default_command_line(bench):
    a = bench.parse_args([])
    assert a.gpus == 1 and a.batch == 1 and a.mode == "predict" and a.impl == "ours"
    assert a.warmup >= 3 and a.steps >= 1
    assert a.config == "llama70b_reglu" and a.layout == "packed"     # the largest single-GPU stack
    assert not a.no_hot_prefetch and not a.l2_next      # hot-block hint on where rows are hot-first
