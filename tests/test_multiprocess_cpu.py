"""Multi-process (world size 2, gloo, CPU) tests of the request-sharded path.

The GPU work is independent per request, so the N>1 path is pure host
plumbing: split a batch, let every rank select its own requests, reduce the
timing, gather rows.  Here the oracle's select stands in for the per-rank
device call, and the gathered result must equal the single-process one."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from page_scoring_top_b200 import dist as pdist
from page_scoring_top_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        B, N, K = 7, 300, 16
        s = synth.score_rows(55, B, N, "normal")
        lo, hi = pdist.split_requests(B, world, rank)
        idx, _ = oracle.topk_rows(s[lo:hi], K)
        full = pdist.gather_rows(torch.from_numpy(idx), B)
        ms, pages = pdist.reduce_timing(10.0 + rank, 100 * (rank + 1))
        np.save(os.path.join(out_dir, "r%d.npy" % rank), full.numpy())
        with open(os.path.join(out_dir, "r%d.txt" % rank), "w") as f:
            f.write("%r %r" % (ms, pages))
    finally:
        dist.destroy_process_group()


def test_split_requests_covers_once():
    for B in (1, 2, 7, 32, 33):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = pdist.split_requests(B, world, r)
                seen.extend(range(lo, hi))
            assert seen == list(range(B))
    assert pdist.rank_seed(103, 0) == 103 and pdist.rank_seed(103, 2) == 2103


def test_reduce_without_group_is_identity():
    assert pdist.reduce_timing(3.5, 7) == (3.5, 7.0)


def test_two_rank_gloo_sharded_select(tmp_path):
    import oracle
    world = 2
    port = _free_port()
    mp.spawn(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    s = synth.score_rows(55, 7, 300, "normal")
    want, _ = oracle.topk_rows(s, 16)
    for r in range(world):
        got = np.load(tmp_path / ("r%d.npy" % r))
        assert np.array_equal(got, want)
        ms, pages = open(tmp_path / ("r%d.txt" % r)).read().split()
        assert float(ms) == 11.0 and float(pages) == 300.0
