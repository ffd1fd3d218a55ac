"""Host-side logic of bench.py: exact in-window pair counts (checked against
the oracle's key lists), the workload sharding, and the max-over-ranks
reduction with two gloo ranks on CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("N,L,R,d,bs,G", [
    (200, 10, 0, 1, 0, (0, 50)), (333, 7, 7, 3, 0, (5, 100, 200)), (300, 128, 0, 2, 16, (3,)),
    (257, 40, 40, 2, 16, (0, 128)), (100, -1, 3, 2, 0, ()), (90, 5, -1, 1, 0, (1,)),
    (64, 0, 0, 1, 0, ()), (129, 64, 64, 1, 64, ()),
])
def test_pair_counts_match_oracle_key_sets(N, L, R, d, bs, G):
    ref = sum(len(oracle.key_set(i, N, L, R, d, bs, G)) for i in range(N))
    assert bench.in_window_pairs(N, L, R, d, bs, G) == ref


@pytest.mark.parametrize("N,L,R,d,G", [
    # the layer kinds of the bench's hybrid schedule, shrunk: causal dilated
    # windows, a full causal layer, a causal window with attention sinks
    (300, 63, 0, 2, ()), (300, 31, 0, 4, ()), (300, -1, 0, 1, ()), (300, 100, 0, 1, (0, 1, 2, 3)),
])
def test_schedule_pair_counts_match_oracle(N, L, R, d, G):
    ref = sum(len(oracle.key_set(i, N, L, R, d, 0, G)) for i in range(N))
    assert bench.in_window_pairs(N, L, R, d, 0, G) == ref


def test_append_pair_count_matches_oracle():
    """The append FLOP count: token c at position p0 + c sees min(W, p0 + c + 1)
    keys -- the size of the oracle's causal key set of that position."""
    W = 64
    for p0 in (0, 10, 63, 64, 200):
        for c in range(5):
            p = p0 + c
            assert min(W, p + 1) == len(oracle.key_set(p, p + 1, W - 1, 0))


def test_workload_pair_counts():
    assert bench.in_window_pairs(8192, 4095, 0, 1, 0, (), 1, 32) == 805_371_904
    assert bench.in_window_pairs(4096, 256, 256, 1, 0, range(0, 4096, 512), 4, 12) == 100_475_520
    assert bench.in_window_pairs(16384, 128, 128, 4, 0, (), 2, 16) == 132_628_480
    assert bench.in_window_pairs(16384, 128, 128, 4, 64, (), 2, 16) == 164_626_432


def test_shard_units_partition():
    for n in (0, 1, 7, 64, 1000):
        for w in (1, 2, 3, 8):
            spans = [bench.shard_units(n, w, r) for r in range(w)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[r][1] == spans[r + 1][0] for r in range(w - 1))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_ms = [3.0, 5.0][rank]
        q.put((rank, bench.reduce_max(step_ms, world, "cpu"), bench.shard_units(64, world, rank)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]  # every rank sees the slowest rank's time
    assert res[0][2] == (0, 32) and res[1][2] == (32, 64)
