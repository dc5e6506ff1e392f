"""Multi-rank partition of the forward: pure partition properties, and a
two-rank gloo run (CPU) whose gathered shares must equal the unsharded oracle.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from protein_structure_models_b200.sharding import (batch_shards, tile_rows, tile_shards,  # noqa: E402
                                                    tile_weights)


@pytest.mark.parametrize("B,world", [(8, 2), (5, 2), (1, 2), (0, 3), (512, 8), (7, 7), (3, 4)])
def test_batch_shards_cover_once(B, world):
    sh = batch_shards(B, world)
    assert len(sh) == world
    assert sh[0][0] == 0 and sh[-1][1] == B
    for (a, b), (c, d) in zip(sh, sh[1:]):
        assert b == c
    sizes = [b - a for a, b in sh]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("weights,world", [([1] * 16, 2), ([1, 0, 0, 1, 1, 1, 0, 1], 2), ([0] * 5, 2),
                                           ([1] * 128, 8), ([1, 1, 1], 4), ([0, 0, 1], 2)])
def test_tile_shards_cover_once_and_balance(weights, world):
    sh = tile_shards(weights, world)
    assert len(sh) == world
    assert sh[0][0] == 0 and sh[-1][1] == len(weights)
    for (a, b), (c, d) in zip(sh, sh[1:]):
        assert b == c and a <= b
    total = sum(weights)
    if total:
        loads = [sum(weights[a:b]) for a, b in sh]
        # contiguous greedy split: no range exceeds its fair share by a whole tile
        assert max(loads) <= -(-total // world) + 1


def test_tile_weights_and_rows():
    mask = [False] * 4 + [True] + [False] * 8 + [True] * 2
    assert tile_weights(mask, tile=4) == [0, 1, 0, 1]
    assert tile_rows((1, 3), 15, tile=4) == (4, 12)
    assert tile_rows((3, 4), 15, tile=4) == (12, 15)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_gloo_partition_matches_unsharded():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "multirank_worker.py")]
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("RESULT ")]
    assert line, out.stdout[-2000:] + out.stderr[-2000:]
    res = json.loads(line[0][len("RESULT "):])
    assert res["world"] == 2
    assert res["max_over_ranks"] == [4.0, 4.0]
    assert [tuple(r) for r in res["batch_ranges"]] == [(0, 3), (3, 5)]
    assert res["batch_update_err"] <= 1e-12 and res["batch_local_err"] <= 1e-12
    rr = [tuple(r) for r in res["row_ranges"]]
    assert rr[0][0] == 0 and rr[-1][1] == 30 and rr[0][1] == rr[1][0]
    assert res["rows_update_err"] <= 1e-12 and res["rows_local_err"] <= 1e-12
