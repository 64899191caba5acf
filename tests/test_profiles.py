"""The ncu summaries under profiles/ and bench.py's record of the code each was captured on."""
import glob
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_summary_is_guarded_and_exists():
    on_disk = {os.path.relpath(p, ROOT) for p in glob.glob(os.path.join(ROOT, "profiles", "*.md"))}
    assert on_disk == set(bench.PROFILES), "each summary needs an entry (sources + hash) in bench.PROFILES"
    for p, t in bench.PROFILES.items():
        text = open(os.path.join(ROOT, p)).read()
        assert "ncu " in text and "--clock-control none" in text, f"{p}: the command that made it"
        assert "Kernel source at capture" in text, p
        for src in t["sources"]:
            assert os.path.exists(os.path.join(ROOT, src)), src
        assert len(t["sha256"]) == 64


def test_traffic_entries_point_at_guarded_summaries():
    for t in bench.TRAFFIC.values():
        assert t["profile"] in bench.PROFILES


def test_status_turns_stale_when_a_source_changes(monkeypatch):
    p = next(iter(bench.PROFILES))
    real = bench._sources_hash
    monkeypatch.setattr(bench, "_sources_hash", lambda srcs: "0" * 64 if srcs == bench.PROFILES[p]["sources"]
                        else real(srcs))
    assert bench.profile_status()[os.path.basename(p)] == "stale"
