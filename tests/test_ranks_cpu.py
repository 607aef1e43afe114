"""Sublayers spread over ranks: the partition, and the score gather + bit
allocation run as two gloo ranks on the CPU (one process each, spawned)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from second_order_post_b200 import kronq as K
from second_order_post_b200 import ranks

N_SUBLAYERS = 7  # not a multiple of the world size: uneven shares
BUDGET = 3.0


def _scores(n):
    g = torch.Generator().manual_seed(5)
    s = torch.rand(n, generator=g, dtype=torch.float64) * 10.0
    s[3] = s[5]  # a tie: the allocator's order among equal scores must agree
    m = torch.randint(1, 50, (n,), generator=g) * 4096
    return s.tolist(), [int(v) for v in m]


@pytest.mark.parametrize("n,world", [(0, 1), (7, 1), (7, 2), (7, 3), (8, 4), (3, 5)])
def test_my_sublayers_partition(n, world):
    shares = [ranks.my_sublayers(n, world, r) for r in range(world)]
    flat = [i for sh in shares for i in sh]
    assert flat == list(range(n))
    sizes = [len(sh) for sh in shares]
    assert max(sizes) - min(sizes) <= 1


def test_my_sublayers_rejects_bad_rank():
    with pytest.raises(ValueError):
        ranks.my_sublayers(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        scores, numel = _scores(N_SUBLAYERS)
        mine = ranks.my_sublayers(N_SUBLAYERS, world, rank)
        bits = ranks.allocate_bits_across_ranks([scores[i] for i in mine],
                                                [numel[i] for i in mine],
                                                N_SUBLAYERS, BUDGET)
        slowest = ranks.max_over_ranks(10.0 + rank)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(" ".join(map(str, bits)) + f"\n{slowest}\n")
    finally:
        dist.destroy_process_group()


def test_allocation_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    scores, numel = _scores(N_SUBLAYERS)
    want = K.kronq_allocate_bits(scores, numel, BUDGET)
    for r in range(world):
        lines = (tmp_path / f"rank{r}.txt").read_text().split("\n")
        assert [int(b) for b in lines[0].split()] == want
        assert float(lines[1]) == 10.0 + world - 1
    # the budget binds: the parameter-weighted mean is within it
    mean = sum(b * m for b, m in zip(want, numel)) / sum(numel)
    assert mean <= BUDGET + 1e-12
