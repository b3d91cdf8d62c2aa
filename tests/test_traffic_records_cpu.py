"""The ncu traffic records under profiles/ that bench.py reports as
roofline.traffic: each is keyed by the SHA-256 of its kernel's sources, and
bench.py uses a record only while the sources still hash to that key.  These
tests hold the committed records to the committed sources (a kernel changed
without a new capture fails here instead of silently reporting no traffic)
and check the recorded bytes against the workloads' algorithmic bytes."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# (kernel family, workload key, algorithmic bytes of one launch or None)
RECORDS = [
    ("decode", "llama3_70b_gqa_bf16", 1_109_712_896),
    ("decode", "mixed_step_fp8_decode", 2_205_399_040),
    ("prefill", "mixed_step_fp8_prefill", None),
    ("mq", "spec_verify_bf16", 1_154_310_144),
]


@pytest.mark.parametrize("kernel,workload,algo", RECORDS)
def test_record_matches_sources(bench, kernel, workload, algo):
    t = bench.traffic_from_profile(workload, kernel)
    assert isinstance(t, int) and t > 0, f"{kernel}/{workload}: record missing or stale"
    if algo is not None:
        # every valid K/V byte read once: traffic within 2 % of the algorithmic bytes
        assert abs(t / algo - 1.0) < 0.02, (kernel, workload, t, algo)


def test_changed_sources_void_the_record(bench, tmp_path, monkeypatch):
    # the same record is used while its key matches the sources' hash, and
    # not once the sources hash to anything else
    path = tmp_path / "profiles"
    path.mkdir()
    (path / "mq_traffic.txt").write_text("mq_src_sha256_16: 0123456789abcdef\n"
                                         "spec_verify_bf16: 123\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda files: "0123456789abcdef")
    assert bench.traffic_from_profile("spec_verify_bf16", "mq") == 123
    monkeypatch.setattr(bench, "source_hash", lambda files: "fedcba9876543210")
    assert bench.traffic_from_profile("spec_verify_bf16", "mq") is None
