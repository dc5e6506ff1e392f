"""Two-rank (gloo, CPU) check of the multi-GPU partition of the IPA forward.

Run by tests/test_multirank.py under torch.distributed.run.  Each rank
computes its share with the oracle; rank 0 gathers the shares and prints one
JSON line comparing them with the unsharded result:
  - max_over_ranks returns the slowest rank's value on every rank;
  - batch_shards: samples split across ranks reproduce the whole batch;
  - tile_shards: query-row ranges (balanced by valid tiles) of one long sample
    reproduce every row, and the ranges cover the rows exactly once.
"""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402
from protein_structure_models_b200.sharding import (batch_shards, max_over_ranks, tile_rows,  # noqa: E402
                                                    tile_shards, tile_weights)


def main():
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    rank, world = dist.get_rank(), dist.get_world_size()
    res = {"world": world}

    # slowest rank
    m = max_over_ranks(1.0 + 3.0 * rank)
    res_m = [None] * world
    dist.all_gather_object(res_m, m)

    # batch split: a protein batch with padded lengths, scaled down
    wl = workloads.workload("1").with_(B=5, N=20, H=2, Cz=8, Cout=16, len_range=(6, 20))
    inp = workloads.make_inputs(wl)
    b0, b1 = batch_shards(wl.B, world)[rank]
    part = oracle.ipa_forward_dense(workloads.slice_batch(inp, list(range(b0, b1)))) if b1 > b0 else None
    parts = [None] * world
    dist.all_gather_object(parts, (b0, b1, part))

    # query-tile split of one long sample (tile of 4 rows, some fully masked tiles)
    wl2 = workloads.workload("2").with_(N=30, H=2, D=8, Dv=8, P=2, Q=2, Cz=8, Cout=16)
    inp2 = workloads.make_inputs(wl2)
    inp2["mask"][0, 8:16] = False                        # two empty query tiles
    wts = tile_weights(list(inp2["mask"][0]), tile=4)
    t0, t1 = tile_shards(wts, world)[rank]
    r0, r1 = tile_rows((t0, t1), wl2.N, tile=4)
    rows = list(range(r0, r1))
    part2 = oracle.ipa_forward_dense(inp2, rows=rows) if rows else None
    parts2 = [None] * world
    dist.all_gather_object(parts2, (r0, r1, part2))

    if rank == 0:
        res["max_over_ranks"] = res_m
        full = oracle.ipa_forward_dense(inp)
        upd = np.concatenate([p["update"] for _, _, p in parts if p is not None], axis=0)
        loc = np.concatenate([p["local_points"] for _, _, p in parts if p is not None], axis=0)
        res["batch_ranges"] = [(a, b) for a, b, _ in parts]
        res["batch_update_err"] = float(np.max(np.abs(upd - full["update"])))
        res["batch_local_err"] = float(np.max(np.abs(loc - full["local_points"])))
        full2 = oracle.ipa_forward_dense(inp2)
        upd2 = np.concatenate([p["update"] for _, _, p in parts2 if p is not None], axis=1)
        loc2 = np.concatenate([p["local_points"] for _, _, p in parts2 if p is not None], axis=1)
        res["row_ranges"] = [(a, b) for a, b, _ in parts2]
        res["tile_weights"] = wts
        res["rows_update_err"] = float(np.max(np.abs(upd2 - full2["update"])))
        res["rows_local_err"] = float(np.max(np.abs(loc2 - full2["local_points"])))
        print("RESULT " + json.dumps(res), flush=True)
    dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
