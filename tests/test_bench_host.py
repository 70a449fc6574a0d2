"""Host-side logic of bench.py (no GPU): FLOP counts and the traffic record."""

import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _visible_pairs_brute(N, causal, wl, wr):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    ok = np.ones((N, N), dtype=bool)
    if causal:
        ok &= j <= i
    if wl >= 0:
        ok &= j >= i - wl
    if wr >= 0:
        ok &= j <= i + wr
    return int(ok.sum())


@pytest.mark.parametrize("N,causal,wl,wr", [
    (1, False, -1, -1), (7, True, -1, -1), (64, False, 5, 7), (64, True, 3, 0),
    (100, False, -1, 0), (100, False, 0, -1), (33, True, 40, -1), (50, False, 0, 0),
])
def test_allowed_pairs_matches_brute_force(N, causal, wl, wr):
    assert bench.allowed_pairs(N, causal, wl, wr) == _visible_pairs_brute(N, causal, wl, wr)


def test_allowed_pairs_long_local_closed_form():
    # window (L, 0), causal: row i sees min(i, L) + 1 keys; rows i < L give
    # i + 1 each (L (L + 1) / 2 in all), the N - L others L + 1 each
    N, L = 32768, 4096
    expect = L * (L + 1) // 2 + (N - L) * (L + 1)
    assert expect == 125_859_840
    assert bench.allowed_pairs(N, True, L, 0) == expect


def test_flops_fwd_counts_and_causal_half():
    assert bench.flops_fwd(8, 16, 2048, 128) == 4.0 * 8 * 16 * 2048 * 2048 * 128
    assert bench.flops_fwd(8, 16, 2048, 128, causal=True) == 0.5 * bench.flops_fwd(8, 16, 2048, 128)


def test_captured_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    with open(path) as fh:
        rec = json.load(fh)
    for call in ("fa2_fwd", "fa2_bwd"):
        assert call in rec and rec[call]["bytes"] > 0
    # a record whose hash matches the sources is reported, a stale one is not
    fake_root = tmp_path
    (fake_root / "profiles").mkdir()
    good = {"fa2_fwd": {"bytes": 123, "sources_sha256": bench.sources_hash("fa2_fwd")},
            "fa2_bwd": {"bytes": 456, "sources_sha256": "0" * 16}}
    (fake_root / "profiles" / "traffic.json").write_text(json.dumps(good))
    os.symlink(os.path.join(ROOT, "exact_attention_147_b200"), fake_root / "exact_attention_147_b200")
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.captured_traffic("fa2_fwd") == 123
    assert bench.captured_traffic("fa2_bwd") is None


def test_reference_arm_prints_the_gpu_arms_config(monkeypatch, capsys):
    # the two arms must describe the same workload with the same dict, and
    # the reference's ms_per_step is the time it measured, not an estimate
    import argparse
    monkeypatch.setattr(bench, "REF_STEP_S", 0.0)
    monkeypatch.delenv("RANK", raising=False)
    assert bench.run_reference(argparse.Namespace(steps=1, warmup=0)) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"] == bench.bench_config(bench.WORKLOAD)
    assert line["impl"] == "reference"
    assert 0 < line["ms_per_step"] < line["ms_per_full_step_extrapolated"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_key_ignores_comments_only(tmp_path, monkeypatch):
    # the committed capture stays valid across a comment-only edit of the
    # kernel sources, and not across a change of code
    import shutil
    src = os.path.join(ROOT, "exact_attention_147_b200", "csrc")
    dst = tmp_path / "exact_attention_147_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = bench.sources_hash("fa2_bwd")
    f = dst / "bwd_sm100.cuh"
    f.write_text(f.read_text() + "\n// a note\n\n")
    assert bench.sources_hash("fa2_bwd") == before
    f.write_text(f.read_text() + "\nstatic const int unused_probe_constant = 1;\n")
    assert bench.sources_hash("fa2_bwd") != before
