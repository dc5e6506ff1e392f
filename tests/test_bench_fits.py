"""Host-side fits of the length sweep in bench.py."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_loglog_exact_power_law():
    ns = [512, 1024, 2048, 4096, 8192, 16384]
    ts = [3e-7 * n ** 1.7 for n in ns]
    f = bench.fit_loglog(ns, ts)
    assert abs(f["exponent"] - 1.7) < 1e-12
    assert abs(f["ci95"][0] - 1.7) < 1e-9 and abs(f["ci95"][1] - 1.7) < 1e-9


def test_loglog_interval_contains_slope_with_noise():
    rng = np.random.default_rng(1)
    ns = np.array([512, 1024, 2048, 4096, 8192, 16384])
    ts = 1e-6 * ns ** 2.0 * np.exp(rng.normal(0, 0.05, ns.size))
    f = bench.fit_loglog(ns, ts)
    assert f["ci95"][0] < f["exponent"] < f["ci95"][1]
    assert f["ci95"][0] < 2.0 < f["ci95"][1]


def test_linear_memory_fit():
    ns = [512, 1024, 4096]
    f = bench.fit_linear(ns, [1000 + 20 * n for n in ns])
    assert abs(f["bytes_per_residue"] - 20) < 1e-9 and abs(f["intercept_bytes"] - 1000) < 1e-6
    assert abs(f["r2"] - 1.0) < 1e-12


def test_prologue_bytes_matches_hand_count_for_protein_batch():
    import workloads
    wl = workloads.workload("1")
    w = bench.lifted_widths(wl)
    assert w == {"Kq": 576, "KHp": 64, "VHp": 64, "Zp": 256}
    BN, BHN = 8 * 256, 8 * 8 * 256
    reads = 2 * (BHN * (32 + 16 + 24 + 24) + BN * (12 + 512)) + BN
    writes = 2 * (BHN * (576 + 64 + 64) + BN * 256) + 32 * BHN
    assert bench.prologue_bytes(wl) == reads + writes


def test_row_ranges_cover_every_row_once():
    """--shard rows: the ranks' ranges are tile-aligned, disjoint and cover all
    rows; the split follows the valid rows (a masked tail gets few ranks)."""
    import workloads
    for N, world, valid in [(4096, 8, 4096), (2048, 3, 2048), (1000, 4, 1000), (4096, 4, 1500)]:
        mask = np.zeros((1, N), dtype=bool)
        mask[0, :valid] = True
        ranges = [bench.row_range(mask, r, world) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == N
        for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
            assert a1 == b0 and a0 < a1
        for r0, r1 in ranges:
            assert r0 % 128 == 0 and (r1 % 128 == 0 or r1 == N)
    # balanced by valid rows: with 1500 of 4096 valid, the first ranges are small
    mask = np.zeros((1, 4096), dtype=bool)
    mask[0, :1500] = True
    ranges = [bench.row_range(mask, r, 4) for r in range(4)]
    assert ranges[0][1] <= 512
    assert bench.shard_mode("auto", workloads.workload("3-4096"), 4) == "rows"
    assert bench.shard_mode("auto", workloads.workload(1), 4) == "replicas"
    assert bench.shard_mode("auto", workloads.workload("3-4096"), 1) == "replicas"
    assert bench.shard_mode("rows", workloads.workload(1), 1) == "rows"


def test_row_range_rejects_more_ranks_than_tiles():
    mask = np.ones((1, 256), dtype=bool)
    assert [bench.row_range(mask, r, 2) for r in range(2)] == [(0, 128), (128, 256)]
    raised = 0
    for r in range(3):                       # 2 tiles, 3 ranks: one rank has nothing
        try:
            bench.row_range(mask, r, 3)
        except ValueError:
            raised += 1
    assert raised == 1


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the fp64 oracle on the host cores) prints one
    JSON line with the GPU line's metric and unit, its own cpu_baseline and an
    e2e block with no host-device copies."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--workload", "1"], capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("protein-batch-bf16")


def test_live_rows_and_projection_work():
    """The projection's work is counted over rows with a non-empty
    neighbourhood only (a masked row, or one whose pair_mask row is empty,
    computes no update)."""
    import workloads
    wl = workloads.workload("1")
    inp = workloads.make_inputs(wl)
    live = int(inp["mask"].sum())
    assert bench.live_rows(inp) == live
    F = wl.H * (wl.Dv + 4 * wl.Q + wl.Cz)
    assert bench.out_proj_flops(wl, live) == 2 * live * F * wl.Cout
    w0 = workloads.workload(0)
    inp0 = workloads.make_inputs(w0)          # one valid query has an all-false pair_mask row
    assert bench.live_rows(inp0) == int(inp0["mask"].sum()) - 1


def test_default_bench_workload_is_the_longest_single_gpu_chain():
    import workloads
    wl = workloads.workload(bench.DEFAULT_WORKLOAD)
    assert (wl.B, wl.N) == (1, 16384) and wl.index == 3
