"""Host logic of bench.py, on the CPU: the algorithmic FLOP count behind the
attention roofline, the summary of the clock record, the guard on the stored
DRAM traffic, and the reference arm's JSON line."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
import synth
from oracle import tree as otree


def _anchors(cfg):
    rng = np.random.default_rng(cfg.seed)
    return synth.draw_anchors(rng, cfg.S, cfg.B, cfg.anchor_lo, cfg.anchor_hi)


@pytest.mark.parametrize("cfg", [
    synth.attn_config("tiny"),
    synth.attn_config("8b"),
    synth.custom_attn_config(3, (5, 64, 17), 2, 5, 8, 2, 128, "bf16"),
], ids=["tiny", "8b", "three-sequences"])
def test_attention_flops_counts_visible_keys(cfg):
    # 4*D*Hq FLOPs per visible (row, key) pair (QK^T and PV).  The keys a
    # branch row sees are its ancestors in the packed tree, itself included:
    # count them by walking the oracle's parent map.
    anchors = _anchors(cfg)
    cu = np.concatenate([[0], np.cumsum(cfg.T)])
    parent, _, _ = otree.tree_build(cu, anchors, cfg.B, cfg.W)
    keys = sum(len(otree.ancestors(parent, node)) for node in range(int(cu[-1]), len(parent)))
    assert bench.attention_flops(cfg, anchors) == 4.0 * cfg.D * cfg.Hq * keys


def test_clock_summary(tmp_path):
    rec = tmp_path / "clocks.csv"
    rec.write_text(
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "1, 1000, 1965, 300.0, 0x8, Active, Not Active, Not Active, Not Active\n"
        "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 1980, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "0, [N/A], 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "not a record\n")
    s = bench._clock_summary(str(rec), 0)
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    assert bench._clock_summary(str(rec), 1)["reasons"] == ["hw_slowdown"]
    missing = bench._clock_summary(str(tmp_path / "none.csv"), 0)
    assert missing["samples"] == 0 and missing["sm_mhz"] is None


def test_traffic_record_guard(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "e2e_tv_8b_traffic.json")
    rec = json.load(open(path))
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    # the bytes are reported only for the kernel sources they were taken on
    monkeypatch.setattr(bench, "tv_source_sha256", lambda: rec["source_sha256"])
    assert bench._ncu_traffic() == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "tv_source_sha256", lambda: "0" * 64)
    assert bench._ncu_traffic() is None


def _run_bench(args, env=None):
    return subprocess.run([sys.executable, "bench.py", *args], cwd=bench.ROOT,
                          capture_output=True, text=True, timeout=600,
                          env=dict(os.environ, **(env or {})))


def test_reference_arm_json_line():
    out = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                      "--warmup", "3"])
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in j, k
    assert j["impl"] == "reference" and j["unit"] == "rows/s" and j["value"] > 0
    assert j["steps"] == 2 and j["warmup"] == 3 and j["higher_is_better"] is True
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
    assert j["e2e"] == {"value": j["value"], "unit": "rows/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    out = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1"],
                     env={"RANK": "1", "WORLD_SIZE": "2"})
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [ln for ln in out.stdout.splitlines() if ln.startswith("{")]


def test_source_digest_ignores_comments_only():
    src = ('// header\n#include "x.h"\nint f(int a) {  /* sum */\n'
           '  const char* s = "a // b /* c */";\n  return a + \'/\';  // tail\n}\n')
    d = bench.source_digest([src])
    # comments and layout edited: same digest
    moved = ('#include "x.h"\n/* new block\n comment */ int f(int a)\n{\n'
             '  const char* s = "a // b /* c */"; return a + \'/\';\n}\n')
    assert bench.source_digest([moved]) == d
    # code edited (also inside a string literal): another digest
    assert bench.source_digest([src.replace("a + ", "a - ")]) != d
    assert bench.source_digest([src.replace("/* c */\";", "/* C */\";")]) != d
    # file boundaries count
    assert bench.source_digest([src, ""]) != d
