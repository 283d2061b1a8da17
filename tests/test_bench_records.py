"""bench.py's profile records on CPU: a record counts only for the kernel sources it was
taken on, the source hash ignores comments, and the issue-rate bound follows from the
recorded warp-instruction count."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


SOURCES = bench.KERNEL_SOURCES


@pytest.fixture
def root(tmp_path, monkeypatch):
    """A temporary root holding copies of the kernel sources, as bench.ROOT."""
    for rel in SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        with open(os.path.join(ROOT, rel)) as f:
            dst.write_text(f.read())
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


@pytest.fixture
def record(root):
    """A profiles/traffic.json keyed to the (copied) kernel sources."""
    rec = {"source_sha256_16": bench._kernel_source_hash(), "kernels": {"bf16": 4_000_000},
           "warp_inst": {"bf16": 6_000_000}}
    path = root / "profiles" / "traffic.json"
    path.write_text(json.dumps(rec))
    return path, rec


def test_record_read_when_hash_matches(record):
    assert bench._traffic("bf16") == 4_000_000
    assert bench._profile_record("warp_inst", "bf16") == 6_000_000
    assert bench._traffic("codes") is None


def test_record_ignored_for_other_sources(record):
    path, rec = record
    rec = dict(rec, source_sha256_16="0" * 16)
    path.write_text(json.dumps(rec))
    assert bench._traffic("bf16") is None
    assert bench._issue_ceiling("bf16", 1 << 24, 0.01, 1965.0, 148) is None


def test_issue_ceiling_arithmetic(record):
    n = 1 << 24
    r = bench._issue_ceiling("bf16", n, 0.010, 2000.0, 100)
    lane_inst = 32 * 6_000_000 / n
    ceiling = 4 * 32 * 100 * 2000e6 / lane_inst        # lane-instructions/s over lane-instructions per symbol
    assert r["lane_inst_per_sym"] == pytest.approx(lane_inst, abs=0.005)
    assert r["ceiling_gsym_s"] == pytest.approx(ceiling / 1e9, abs=0.05)
    assert r["achieved_gsym_s"] == pytest.approx(n / 10e-6 / 1e9, abs=0.05)
    assert r["frac"] == pytest.approx((n / 10e-6) / ceiling, abs=1e-4)
    # one warp instruction per scheduler clock: a launch of exactly that many cycles is at the bound
    cycles = 6_000_000 / (4 * 100)
    at_bound = bench._issue_ceiling("bf16", n, 1e3 * cycles / 2000e6, 2000.0, 100)
    assert at_bound["frac"] == pytest.approx(1.0, abs=1e-3)
    assert bench._issue_ceiling("bf16", n, 0.01, None, 100) is None


def test_source_hash_ignores_comments_but_not_code(root):
    base = bench._kernel_source_hash()
    cu = root / SOURCES[0]
    src = cu.read_text()
    cu.write_text("// a note\n/* and a block\n   comment */\n" + src.replace("\n", "  \n", 3))
    assert bench._kernel_source_hash() == base
    assert "kRing = 16;" in src
    cu.write_text(src.replace("kRing = 16;", "kRing = 32;", 1))
    assert bench._kernel_source_hash() != base


def test_committed_record_names_its_command():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert t["commands"] and all(c.startswith("ncu ") and "--clock-control none" in c for c in t["commands"])
    assert t["kernels"] and set(t["kernels"]) == set(t["warp_inst"])
