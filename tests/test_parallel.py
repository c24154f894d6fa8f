"""Head sharding and max-over-ranks timing, with world_size 2 gloo ranks on CPU."""
import os

import pytest
import torch
import torch.multiprocessing as mp

from persistent_sm_attn_b200.parallel import group_head_range, head_range, max_over_ranks


@pytest.mark.parametrize("n_heads", [0, 1, 5, 32, 128, 97])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_head_ranges_partition(n_heads, world):
    seen = []
    sizes = []
    for r in range(world):
        a, b = head_range(n_heads, r, world)
        seen.extend(range(a, b))
        sizes.append(b - a)
    assert seen == list(range(n_heads))
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("n_kv,group", [(0, 2), (1, 4), (5, 2), (8, 8), (7, 1)])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_group_head_ranges_keep_kv_heads_whole(n_kv, group, world):
    seen, sizes = [], []
    for r in range(world):
        a, b = group_head_range(n_kv * group, group, r, world)
        assert a % group == 0 and b % group == 0
        seen.extend(range(a, b))
        sizes.append((b - a) // group)
    assert seen == list(range(n_kv * group))
    assert max(sizes) - min(sizes) <= 1


def test_group_head_range_rejects_partial_groups():
    with pytest.raises(ValueError):
        group_head_range(6, 4, 0, 1)
    with pytest.raises(ValueError):
        group_head_range(8, 0, 0, 2)


def test_head_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = head_range(64, rank, world)
        # each rank "times" its own shard; the job time is the slowest rank's
        t = max_over_ranks(1.0 + rank * 0.5)
        gathered = [None] * world
        dist.all_gather_object(gathered, (a, b))
        out[rank] = (t, gathered)
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        t, ranges = res[r]
        assert t == 1.5
        assert ranges == [(0, 32), (32, 64)]


def test_max_over_ranks_without_group():
    assert max_over_ranks(3.25) == 3.25
