"""The N > 1 path of the bench: replicas with no exchange on the data path, and a
timing reduction (sum of units, max of seconds) across ranks. Checked on CPU with two
gloo ranks; no GPU is involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from delta_rule_attention_ckda_b200.replicas import aggregate_throughput, shard_sequences


def test_shards_partition_the_sequences():
    for B, H, world in [(8, 16, 1), (8, 16, 2), (8, 16, 3), (1, 16, 8), (2, 3, 4), (1, 1, 2)]:
        seen = []
        for rank in range(world):
            part = shard_sequences(B, H, world, rank)
            assert len(part) in ((B * H) // world, (B * H) // world + 1)
            seen += part
        assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
    with pytest.raises(ValueError):
        shard_sequences(2, 2, 2, 2)


def test_single_rank_aggregate():
    v, t = aggregate_throughput(1000.0, 2.0, 1)
    assert v == 500.0 and t == 2.0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r processed 100 * (r + 1) units in (r + 1) seconds
        v, t = aggregate_throughput(100.0 * (rank + 1), float(rank + 1), world)
        out[rank] = (v, t)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_aggregate():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # total units 100 + 200 over the slowest rank's 2 s, identical on both ranks
    for rank in range(world):
        v, t = res[rank]
        assert t == 2.0
        assert abs(v - 150.0) < 1e-9
