"""bench.py's host-side bookkeeping (no GPU): the padding-waste figure on hand-worked masks, the
kernel-launch count, the whole-job value in both multi-GPU modes, the traffic figure's validity
check, and the configuration record."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from sparse_attention_video_head_b200 import inputs as I  # noqa: E402


def test_fixed128_waste_hand_worked():
    # one head, two Q clusters of 64 and 192 rows, two K clusters of 128 and 128 keys
    q_off = np.array([[[0, 64, 256]]], np.int32)
    k_off = np.array([[[0, 128, 256]]], np.int32)
    # Q cluster 0 keeps K cluster 1; Q cluster 1 keeps K cluster 0
    mask = np.array([[[[0, 1], [1, 0]]]], np.uint8)
    # actual pairs: 64*128 + 192*128 = 32768; 128-blocks touched: Q block 0 x K block 1 (cluster 0), and
    # Q blocks 0-1 x K block 0 (cluster 1 spans rows 64..255) -> 3 blocks of 128*128 = 49152
    waste = bench.fixed128_waste(q_off, k_off, mask, heads=[0])
    assert abs(waste - (1 - 32768 / 49152)) < 1e-12
    # everything kept and aligned to 128: no waste
    q_al = np.array([[[0, 128, 256]]], np.int32)
    assert bench.fixed128_waste(q_al, k_off, np.ones((1, 1, 2, 2), np.uint8), heads=[0]) == 0.0


def test_kernel_launch_count_matches_the_step():
    cfg = I.CONFIGS["wan720p"]
    # per role: seeding, split prep, and per Lloyd iteration assign + re-rank + 3 sort + update;
    # then selection, 3 gathers, 3 plan kernels and the attention
    assert bench.kernel_launches(cfg) == 2 * (2 + cfg.iters * 6) + 1 + 3 + 4 == 72


def test_whole_job_value_per_mode():
    assert bench.whole_job_ms_per_layer(120.0, 4) == 30.0             # replicas: 4 layers per step
    assert bench.whole_job_ms_per_layer(120.0, 4, sharded=True) == 120.0  # heads split: one layer per step
    assert bench.whole_job_ms_per_layer(120.0, 1) == 120.0


def test_traffic_figure_only_for_the_captured_source_and_workload():
    cfg = I.CONFIGS["wan720p"]
    t = bench.attn_traffic(cfg)
    assert t is None or abs(t - bench.ATTN_TRAFFIC["bytes_captured"] * 40 / 4) < 1.0
    assert bench.attn_traffic(I.CONFIGS["hunyuan720p"]) is None
    saved = bench.ATTN_TRAFFIC["sha256"]
    try:
        bench.ATTN_TRAFFIC["sha256"] = "0" * 64  # as if the kernel had changed since the capture
        assert bench.attn_traffic(cfg) is None
    finally:
        bench.ATTN_TRAFFIC["sha256"] = saved


def test_config_record_for_both_modes():
    cfg = I.CONFIGS["wan720p"]
    c = bench.config_dict(cfg, 0.9, 16384)
    assert c["workload"] == "wan720p" and c["H"] == 40 and c["parallelism"] == "replicas"
    import dataclasses
    c2 = bench.config_dict(dataclasses.replace(cfg, H=20), 0.9, 16384, shard=(40, 2))
    assert c2["H"] == 40 and c2["parallelism"] == "heads/2"


def test_traffic_constant_matches_its_profile_summary():
    """The attention's DRAM traffic that bench.py reports comes from the ncu summary it names; the
    constant and the summary's read and write rows must agree (to the summary's rounding)."""
    import re
    path = os.path.join(ROOT, bench.ATTN_TRAFFIC["summary"])
    text = open(path).read()
    rd = float(re.search(r"dram__bytes_read\.sum \| ([0-9.]+) MB", text).group(1)) * 1e6
    wr = float(re.search(r"dram__bytes_write\.sum \| ([0-9.]+) MB", text).group(1)) * 1e6
    assert abs(bench.ATTN_TRAFFIC["bytes_captured"] - (rd + wr)) <= 0.1e6
    assert f"{bench.ATTN_TRAFFIC['heads_captured']} heads" in text
