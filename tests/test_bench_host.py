"""Host-side logic of bench.py (no GPU): where the roofline's DRAM traffic comes from.

The traffic figure is read from a committed ncu summary and used only while the
summarised kernel's source still has the hash the summary records.
"""
import hashlib
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


@pytest.mark.parametrize("kernel", ["sparse_mla", "indexer"])
def test_committed_summaries_match_the_sources(bench, kernel):
    """Every kernel the roofline may name has a committed summary whose hash
    matches the source as committed, so the line's traffic is reproducible."""
    traffic, src = bench.traffic_from_profile(kernel)
    assert traffic is not None, src
    assert traffic > 0
    assert src == bench.TRAFFIC_SUMMARY[kernel][0]


def _write_case(tmp_path, source_text, summary_hash, traffic="1.5e+09"):
    (tmp_path / "k.cu").write_text(source_text)
    (tmp_path / "s.md").write_text(
        "# summary\n\ntraffic: %s bytes per launch (scaled); source sha256 %s\n" % (traffic, summary_hash))
    return str(tmp_path / "s.md"), str(tmp_path / "k.cu")


def test_traffic_is_used_while_the_hash_matches(bench, tmp_path, monkeypatch):
    text = "__global__ void k() {}\n"
    h = hashlib.sha256(text.encode()).hexdigest()[:16]
    summary, source = _write_case(tmp_path, text, h)
    monkeypatch.setattr(bench, "TRAFFIC_SUMMARY", {"x": (summary, source)})
    assert bench.traffic_from_profile("x") == (1.5e9, summary)


def test_traffic_is_null_once_the_kernel_changes(bench, tmp_path, monkeypatch):
    text = "__global__ void k() {}\n"
    h = hashlib.sha256(text.encode()).hexdigest()[:16]
    summary, source = _write_case(tmp_path, text + "// edited\n", h)
    monkeypatch.setattr(bench, "TRAFFIC_SUMMARY", {"x": (summary, source)})
    traffic, why = bench.traffic_from_profile("x")
    assert traffic is None and "changed" in why


def test_traffic_is_null_without_a_summary_line(bench, tmp_path, monkeypatch):
    (tmp_path / "k.cu").write_text("x")
    (tmp_path / "s.md").write_text("no figures here\n")
    monkeypatch.setattr(bench, "TRAFFIC_SUMMARY",
                        {"x": (str(tmp_path / "s.md"), str(tmp_path / "k.cu"))})
    traffic, why = bench.traffic_from_profile("x")
    assert traffic is None and "no traffic line" in why
