"""bench.py's host-side arithmetic, without a GPU: the algorithmic bytes the
roofline divides by, the input rings that keep every timed launch out of L2,
and the ncu traffic lookup."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

L2_B200 = 126 * 1024 * 1024


def test_algorithmic_bytes_of_the_flux_launches():
    # 2 B bf16 in + 0.5 B codes + 1/32 B scale per element, 60 B of parameters per
    # 32-element block column
    assert bench.algorithmic_bytes(4608, 12288) == 4608 * 12288 * 2.53125 + 384 * 60 == 143350272
    assert bench.algorithmic_bytes(4608, 3072) == 4608 * 3072 * 2.53125 + 96 * 60
    ws = bench.step_workloads(0)
    assert sorted((w.M, w.d) for w in ws) == [(4608, 3072), (4608, 12288)]
    assert bench.step_bytes(ws) == bench.algorithmic_bytes(4608, 3072) + bench.algorithmic_bytes(4608, 12288)


def test_weight_bytes():
    # fp32 weights read once, codes and scales written, 60 B of parameters per block column
    assert bench.weight_bytes(12288, 3072) == 12288 * 3072 * (4 + 0.5 + 1 / 32) + 96 * 60


def test_rings_exceed_four_l2():
    for w in bench.step_workloads(0):
        depth = bench.ring_depth(w, L2_B200)
        per_launch = w.M * w.d * bench.BYTES_PER_ELEM
        assert depth >= 2
        assert depth * per_launch >= bench.RING_FACTOR_L2 * L2_B200
        # one set fewer would not be enough (the ring is the smallest that works)
        assert depth == 2 or (depth - 1) * per_launch < bench.RING_FACTOR_L2 * L2_B200
    depths = {w.d: bench.ring_depth(w, L2_B200) for w in bench.step_workloads(0)}
    assert depths == {3072: 15, 12288: 4}


def test_ncu_traffic_is_current_or_absent():
    traffic, source = bench.ncu_traffic()
    if traffic is None:
        assert "predates" in source or "no ncu summary" in source
    else:
        assert source == "ncu (current sources)"
        # DRAM traffic of one launch: the input once plus part of the output, and
        # never more than the algorithmic bytes
        assert 4608 * 12288 * 2 <= traffic <= bench.algorithmic_bytes(4608, 12288)


def test_both_arms_print_the_same_config():
    cfg = bench.step_config(1)
    assert cfg["M_per_rank"] == 4608 and cfg["d"] == [3072, 12288]
    assert bench.step_config(1) == cfg


def test_all_core_oracle_runner():
    """Two spawned processes, two steps: every step's bytes are both
    workers' tokens of both shapes plus the parameters."""
    n, steps = bench.oracle_all_cores(rows_per_worker=4, steps=2, workers=2)
    assert n == 2 and len(steps) == 2
    want = 2 * 4 * (3072 + 12288) * bench.BYTES_PER_ELEM + (96 + 384) * bench.PARAM_BYTES_PER_BLOCK_COL
    for secs, nbytes in steps:
        assert secs > 0 and nbytes == want
    assert bench.cpu_model() and bench.host_cores() >= 1
