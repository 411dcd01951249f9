"""Host-side logic of bench.py, on CPU: the algorithmic FLOP counts behind the
roofline figures (against per-layer and per-pass totals worked out by hand),
the source hash that invalidates the recorded GEMM DRAM traffic when the GEMM
code changes (and only then), and the parsing of the clock samples taken
during the timed region."""

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from few_step_dit_b200 import synthetic as S  # noqa: E402


def test_flash_pass_flops_match_the_stated_totals():
    # with the attention width equal to the hidden width (42 heads of 128):
    # 10.17 TFLOP per full layer at 12,560 rows, 2.27 per compressed layer at
    # 3,668, 665 per 3-evaluation pass (1,281 without compression)
    w42 = S.scaled(S.WORKLOADS["flash_backbone_6x34x60"], heads=42)
    assert w42.attn_dim == w42.hidden
    assert bench.block_flops(w42, 12560) / 1e12 == pytest.approx(10.17, rel=5e-3)
    assert bench.block_flops(w42, 3668) / 1e12 == pytest.approx(2.27, rel=5e-3)
    assert bench.pass_flops(w42, True) / 1e12 == pytest.approx(665.0, rel=5e-3)
    assert bench.pass_flops(w42, False) / 1e12 == pytest.approx(1281.0, rel=5e-3)
    # the model's 56 heads of 128 (A = 7,168): 12.27 / 2.65 per layer, 795.3
    # per pass (1,545.7 without compression)
    w = S.WORKLOADS["flash_backbone_6x34x60"]
    assert bench.block_flops(w, 12560) / 1e12 == pytest.approx(12.27, rel=5e-3)
    assert bench.block_flops(w, 3668) / 1e12 == pytest.approx(2.65, rel=5e-3)
    assert bench.pass_flops(w, True) / 1e12 == pytest.approx(795.3, rel=1e-3)
    assert bench.pass_flops(w, False) / 1e12 == pytest.approx(1545.7, rel=1e-3)


def test_source_hash_follows_code_not_comments():
    texts = {rel: open(os.path.join(ROOT, rel), encoding="utf-8").read() for rel in bench.GEMM_SOURCES}
    h0 = bench.gemm_sources_sha256(read=texts.__getitem__)
    assert h0 == bench.gemm_sources_sha256()
    rel = bench.GEMM_SOURCES[0]
    commented = dict(texts)
    commented[rel] = "// a new comment line\n\n" + texts[rel].replace("\n", "   // trailing note\n", 1)
    assert bench.gemm_sources_sha256(read=commented.__getitem__) == h0
    changed = dict(texts)
    changed[rel] = texts[rel] + "\nstatic int an_extra_symbol = 1;\n"
    assert bench.gemm_sources_sha256(read=changed.__getitem__) != h0


def test_traffic_record_is_used_only_for_its_workload_and_sources(tmp_path, monkeypatch):
    rec = {"workload": "flash_backbone_6x34x60", "dram_bytes_per_launch": 123.0,
           "sources_sha256": bench.gemm_sources_sha256()}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(p))
    assert bench.gemm_traffic("flash_backbone_6x34x60") == 123.0
    assert bench.gemm_traffic("flash_backbone_6x17x30") is None
    rec["sources_sha256"] = "0" * 64
    p.write_text(json.dumps(rec))
    assert bench.gemm_traffic("flash_backbone_6x34x60") is None
    p.write_text("not json")
    assert bench.gemm_traffic("flash_backbone_6x34x60") is None


class _FakeProc:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


def test_clock_samples_median_and_reasons():
    lines = [
        "1500, 1965, 980.1, Not Active, Not Active, Not Active, Active",
        "1470, 1965, 1001.0, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 300.0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.proc = _FakeProc("\n".join(lines) + "\n")
    r = s.stop()
    assert r["sm_mhz"] == 1500.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]
    s.proc = _FakeProc("1400, 1965, 900, Active, Not Active, Not Active, Not Active\n")
    assert bench.ClockSampler.stop(s)["reasons"] == ["hw_slowdown"]
    s.proc = None
    assert bench.ClockSampler.stop(s) is None
