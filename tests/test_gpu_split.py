"""The split sublayer's product path (libkronq calls per rank, NCCL
collectives) on one GPU as a one-rank group: the token-sharded covariance
all-reduce, the replicated BiIP and factor, and the row-sharded OBS must give
bitwise the same codes, scales and zero points as the one-GPU engine."""
import datetime
import socket

import pytest
import torch

from second_order_post_b200 import synth

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_split_path_matches_engine_on_one_rank(cuda_device):
    import torch.distributed as dist
    from second_order_post_b200.engine import SublayerEngine
    from second_order_post_b200.split import ShardedSublayer
    d_out, d_in, n = 384, 512, 4096
    data = synth.small_case(d_out, d_in, n, dtype=torch.bfloat16, seed=3, device="cuda")
    W, X, G = data["W"], data["X"], data["G"]
    eng = SublayerEngine(d_out, d_in, bits=3, rot_in=(128, 4), rot_out=(128, 3), split=False)
    res = eng.run(W, X, G)
    torch.cuda.synchronize()
    eng.check_info()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        sub = ShardedSublayer(d_out, d_in, bits=3, rot_in=(128, 4), rot_out=(128, 3))
        got = sub.run(W, X, G, n)
        torch.cuda.synchronize()
        sub.ops.check()
        assert torch.equal(got.codes, res.codes)
        assert torch.equal(got.scales, res.scales)
        assert torch.equal(got.zeros, res.zeros)
        assert torch.equal(got.sens, res.sens)
    finally:
        dist.destroy_process_group()
