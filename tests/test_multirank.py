"""Multi-rank host logic on CPU with the gloo backend (world size 2): the max-over-ranks timing,
weak-scaling seeds and head sharding used when LiteLA runs one process per GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_attention_diffusion_litela_b200.dist import (aggregate_rate, max_over_ranks, rank_seeds,
                                                         shard_heads)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        t = max_over_ranks(10.0 + 5.0 * rank)           # rank 1 is the slowest
        seeds = rank_seeds([4000, 4001, 4002], rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        h0, h1 = shard_heads(70, world, rank)
        spans = [None] * world
        dist.all_gather_object(spans, (h0, h1))
        q.put((rank, t, gathered, spans))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, gathered, spans in results:
        assert t == 15.0                                  # every rank sees the slowest time
        flat = [s for per in gathered for s in per]
        assert len(set(flat)) == len(flat)                # weak scaling: no shared inputs
        assert gathered[0] == [4000, 4001, 4002]          # rank 0 keeps the 1-GPU seeds
        assert spans == [(0, 35), (35, 70)]               # heads split without overlap or gap


def test_aggregate_rate_and_single_process_identity():
    assert max_over_ranks(3.5) == 3.5                     # no process group: identity
    # 2 ranks x 2293760 tokens*heads per call x 60 calls in 10 ms
    assert aggregate_rate(2293760 * 60, 2, 10.0) == pytest.approx(2 * 2293760 * 60 / 0.01)
    with pytest.raises(ValueError):
        aggregate_rate(1.0, 1, 0.0)


@pytest.mark.parametrize("H,world", [(70, 1), (70, 3), (36, 8), (5, 8)])
def test_shard_heads_covers_every_head_once(H, world):
    spans = [shard_heads(H, world, r) for r in range(world)]
    covered = [h for a, b in spans for h in range(a, b)]
    assert covered == list(range(H))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_head_shards_cover_every_head_once_and_pack_their_columns():
    """shard_heads splits H heads into contiguous ranges that cover each head once (sizes differ
    by at most one); pack_head_shard takes exactly those heads' q, k and v columns."""
    for H in (1, 5, 36, 70):
        for world in (1, 2, 3, 4, 8):
            if world > H:
                continue
            spans = [shard_heads(H, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [h1 - h0 for h0, h1 in spans]
            assert max(sizes) - min(sizes) <= 1
    from linear_attention_diffusion_litela_b200.dist import pack_head_shard
    B, N, H, d = 2, 3, 5, 4
    x = torch.arange(B * N * 3 * H * d, dtype=torch.float32).reshape(B, N, 3 * H * d)
    sub = pack_head_shard(x, H, 1, 3, d)
    assert sub.shape == (B, N, 3 * 2 * d)
    full = x.view(B, N, 3, H, d)
    assert torch.equal(sub.view(B, N, 3, 2, d), full[:, :, :, 1:3])
    with pytest.raises(ValueError):
        pack_head_shard(x, H, 3, 3, d)
