"""Host-side logic of bench.py (no GPU): the algorithmic byte and flop accounting behind
the roofline, the expert split between the decode and tensor-core kernels, the launch
count, the clock-record parsing and the source hash that ties stored traffic figures to
the kernel code."""
import os
import shutil

import numpy as np
import pytest

import bench
from weight_only_int4_gq4_b200 import synth


def test_matrix_and_expert_bytes_match_the_pages_sizes():
    # a 6144 x 2048 expert (gate, up: 2048 x 6144; down: 6144 x 2048) is 21,233,664 B
    # with its gs = 64 scales (the worked size of the pages' expert)
    F, H = 2048, 6144
    assert 2 * bench.per_matrix_bytes(F, H) + bench.per_matrix_bytes(H, F) == 21_233_664
    assert bench.per_matrix_bytes(1, 64) == 32 + 4


def test_split_experts_threshold():
    cfg = synth.MOE_PREFILL_E32
    cnt = np.zeros(cfg.E, np.int64)
    cnt[:4] = [0, 32, 33, 200]
    sp = bench.split_experts(cfg, cnt)
    assert sp["tc"] and sp["n_small"] == 1 and sp["rows_small"] == 32
    assert sp["n_large"] == 2 and sp["rows_large"] == 233
    # fewer than 33 tokens: everything on the decode kernels
    sp = bench.split_experts(synth.MOE_BATCHED, np.full(256, 1))
    assert not sp["tc"] and sp["n_large"] == 0 and sp["n_small"] == 256


def test_stage_work_flops_and_bytes():
    cfg = synth.MOE_PREFILL
    cnt = np.full(cfg.E, cfg.T * cfg.K // cfg.E)
    sp = bench.split_experts(cfg, cnt)
    w = bench.stage_work(cfg, sp)
    rows = cfg.T * cfg.K
    # 604 MFLOP per token at H = 6144, F = 2048, K = 8 over gate+up and down
    assert w["gate_up_large"][1] + w["down_large"][1] == pytest.approx(2.0 * rows * 3 * cfg.H * cfg.F)
    assert (w["gate_up_large"][1] + w["down_large"][1]) / cfg.T == pytest.approx(603_979_776)
    # every expert's weights are read once per step
    expert = 2 * bench.per_matrix_bytes(cfg.F, cfg.H) + bench.per_matrix_bytes(cfg.H, cfg.F)
    weights = w["gate_up_large"][0] + w["down_large"][0] + w["gate_up_small"][0] + w["down_small"][0]
    assert weights >= cfg.E * expert


def test_launch_count():
    small = {"tc": False}
    assert bench.launches_per_step(synth.MOE_BATCHED, small) == 3      # one router block, 2 decode kernels
    assert bench.launches_per_step(synth.MOE_PREFILL, {"tc": True}) == 9  # 4 routing, 2 decode, gather + 2 tc


def test_clock_summary_parsing():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
               "0, 1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
               "garbage line"]
    s = c.summary()
    assert s["sm_max_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]
    assert 1900.0 <= s["sm_mhz"] <= 1965.0


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "weight_only_int4_gq4_b200", "csrc")
    root = tmp_path / "r"
    shutil.copytree(src, root / "weight_only_int4_gq4_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.kernel_source_hash()
    f = root / "weight_only_int4_gq4_b200" / "csrc" / "gq4_common.cuh"
    f.write_text(f.read_text() + "\n// a comment\n/* another\n comment */\n")
    assert bench.kernel_source_hash() == h0
    f.write_text(f.read_text() + "\nnamespace gq4 { constexpr int kUnusedForHash = 1; }\n")
    assert bench.kernel_source_hash() != h0
