"""The multi-GPU host path on CPU: two gloo ranks split heads, run them with no
collective on the data path, reduce their timing as a max, and, gathered,
give exactly the single-process result (heads are independent).

Each rank computes its heads with the float64 oracle; the product path needs a
GPU per rank, which this test does not have."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from frame_wise_gated_scan_b200 import inputs, multi
from oracle import gdn_scan_ref

WL = inputs.Workload("multi_rank", 2, 3, 32, 4, 40, "f32", 77, "gauss", "tiny")   # 6 heads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        lo, hi = multi.head_range(WL.heads, world, rank)
        mine = {}
        for bh in range(lo, hi):
            b, h = divmod(bh, WL.H)
            mine[bh] = gdn_scan_ref(*inputs.head(WL, b, h))
        # the only collectives: the timing reduction and the result gather
        slowest = multi.max_over_ranks(10.0 + rank)
        assert slowest == 10.0 + world - 1
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        if rank == 0:              # a failed assertion here makes mp.spawn raise
            merged = {}
            for part in gathered:
                assert not set(part) & set(merged), "a head ran on two ranks"
                merged.update(part)
            assert sorted(merged) == list(range(WL.heads))
            for bh, (out, st) in merged.items():
                b, h = divmod(bh, WL.H)
                ref_out, ref_st = gdn_scan_ref(*inputs.head(WL, b, h))
                assert np.array_equal(out, ref_out) and np.array_equal(st, ref_st), bh
    finally:
        dist.destroy_process_group()


def test_head_range_partitions():
    for n in (0, 1, 5, 32, 33):
        for world in (1, 2, 3, 8):
            ranges = [multi.head_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            for (a, b), (c, d) in zip(ranges, ranges[1:]):
                assert b == c
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        multi.head_range(4, 2, 2)


def test_whole_job_rate():
    assert multi.whole_job_rate(30752, 400, 1, 1266.8) == pytest.approx(30752 * 400 / 1.2668)
    assert multi.whole_job_rate(100, 10, 4, 1000.0) == pytest.approx(4000.0)
    assert multi.max_over_ranks(3.5) == 3.5          # no process group: the value itself


def test_two_gloo_ranks_split_heads_like_one_process():
    mp.spawn(_rank_main, args=(2, _free_port()), nprocs=2, join=True)
