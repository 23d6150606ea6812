"""Multi-rank host logic on CPU: two gloo ranks agree on the sequence
partition without communicating, every sequence lands on exactly one rank,
and the timing reduction returns the slowest rank."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from mla_latent_kv_23_b200 import shard, synth


def test_partition_covers_each_sequence_once_and_balances():
    seqlens = synth.draw_seqlens(synth.config("ragged"))
    for world in (1, 2, 3, 8):
        parts = shard.partition_sequences(seqlens, world)
        flat = sorted(b for p in parts for b in p)
        assert flat == list(range(len(seqlens)))
        loads = [shard.rank_load(seqlens, p) for p in parts]
        # greedy longest-first: max load <= 4/3 of the lower bound max(mean, longest)
        lower = max(sum(int(x) for x in seqlens) / world, int(max(seqlens)))
        assert max(loads) <= 4 / 3 * lower + 1


def test_partition_equal_lengths_is_round_robin_sized():
    parts = shard.partition_sequences([4096] * 16, 4)
    assert [len(p) for p in parts] == [4, 4, 4, 4]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, seqlens, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        parts = shard.partition_sequences(seqlens, world)
        mine = parts[rank]
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        slowest = shard.max_over_ranks(1.5 + rank)
        q.put((rank, gathered, slowest, parts))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree():
    world = 2
    seqlens = [int(x) for x in np.random.default_rng(0).integers(512, 32768, size=23)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seqlens, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, slowest, parts in results:
        assert gathered == parts                  # each rank's share is what the others computed
        assert sorted(b for g in gathered for b in g) == list(range(len(seqlens)))
        assert slowest == 1.5 + world - 1         # max over ranks
