"""Context parallelism (split-KV across ranks), host side on CPU.

Every rank holds a contiguous page range of each sequence, decodes it, and
the partial (u, lse) of all ranks meet in one all-gather and a log-sum-exp
merge.  On two and three gloo ranks, with the fp64 oracle standing in for
the GPU decode, the merged result must equal the oracle's decode of the
whole contexts; the pieces must cover every cached token exactly once."""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mla_latent_kv_23_b200 import shard, synth
from oracle import mla_oracle as orc


def small_workload(B=3, seqlens=(300, 520, 1000)):
    return synth.Workload(name="cp-small", B=B, s_q=1, n_h=4, d_model=64, d_c=64, d_h=32, d_v=32,
                          d_R=16, page_size=64, dtype="fp32", seqlens=tuple(seqlens),
                          block_table="permuted", scale=1 / math.sqrt(48.0), seed=7)


def test_pieces_cover_every_token_once():
    for seqlens in ([64, 65, 128, 4096, 1000], [64 * 7, 64 * 7 + 1]):
        for world in (1, 2, 3, 7):
            if any(-(-L // 64) < world for L in seqlens):
                with pytest.raises(ValueError):
                    shard.split_context(seqlens, world, 64)
                continue
            pieces = shard.split_context(seqlens, world, 64)
            for b, L in enumerate(seqlens):
                spans = [(pieces[r][b][0] * 64, pieces[r][b][0] * 64 + pieces[r][b][1])
                         for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == L
                for (a0, a1), (b0, _) in zip(spans, spans[1:]):
                    assert a1 == b0          # contiguous, in rank order
                assert all(a1 > a0 for a0, a1 in spans)   # every rank gets a token
                n_pages = [-(-(a1 - a0) // 64) for a0, a1 in spans]
                assert max(n_pages) - min(n_pages) <= 1


def test_local_tables_follow_the_global_table():
    w = small_workload()
    inp = synth.draw(w, with_weights=False)
    for world in (2, 3):
        for r, pieces in enumerate(shard.split_context(inp["seqlens"], world, w.page_size)):
            bt, sl = shard.local_tables(inp["block_table"], pieces, w.page_size)
            for b, (p0, n) in enumerate(pieces):
                n_p = -(-n // w.page_size)
                assert sl[b] == n
                assert list(bt[b, :n_p]) == list(inp["block_table"][b, p0:p0 + n_p])
                assert all(x == -1 for x in bt[b, n_p:])


def oracle_decode(w):
    """decode_fn stand-in: the oracle's absorbed decode of one rank's pieces."""
    def fn(q, cache, bt, sl, page_size, d_R, scale):
        wl = w.with_(B=q.shape[0], seqlens=tuple(int(x) for x in sl))
        res = orc.decode_absorbed(q.numpy(), cache.numpy(), bt.numpy(), sl.numpy(), wl)
        u = torch.zeros((q.shape[0], 1, w.n_h, w.d_c), dtype=torch.float64)
        lse = torch.zeros((q.shape[0], 1, w.n_h), dtype=torch.float64)
        for (b, r, i), (uu, ll) in res.items():
            u[b, r, i] = torch.from_numpy(uu)
            lse[b, r, i] = ll
        return u, lse
    return fn


def plain_merge(u_parts, lse_parts, u, lse):
    """The log-sum-exp merge written from its definition (test stand-in)."""
    m = lse_parts.max(dim=0).values
    wts = torch.exp(lse_parts - m)
    z = wts.sum(dim=0)
    lse.copy_(m + torch.log(z))
    u.copy_((wts.unsqueeze(-1) * u_parts).sum(dim=0) / z.unsqueeze(-1))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = small_workload()
        inp = synth.draw(w, with_weights=False)
        q = torch.from_numpy(np.ascontiguousarray(synth.random_q(w), dtype=np.float64))
        cache = torch.from_numpy(np.asarray(inp["cache"], np.float64))
        pieces = shard.split_context(inp["seqlens"], world, w.page_size)[rank]
        bt, sl = shard.local_tables(inp["block_table"], pieces, w.page_size)
        u, lse = shard.context_parallel_decode(q, cache, torch.from_numpy(bt), torch.from_numpy(sl),
                                               w.page_size, w.d_R, w.softmax_scale,
                                               decode_fn=oracle_decode(w), merge_fn=plain_merge)
        out_q.put((rank, u.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_merge_to_the_whole_context(world):
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [out_q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = small_workload()
    inp = synth.draw(w, with_weights=False)
    q = synth.random_q(w)
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w)
    for rank, u, lse in results:
        for (b, r, i), (u_ref, lse_ref) in ref.items():
            assert np.max(np.abs(u[b, r, i] - u_ref)) < 1e-10
            assert abs(lse[b, r, i] - lse_ref) < 1e-10


def test_context_parallel_needs_one_query_row():
    q = torch.zeros((1, 2, 4, 80))
    with pytest.raises(ValueError):
        shard.context_parallel_decode(q, None, None, None, 64, 16, 1.0,
                                      decode_fn=lambda *a: None, merge_fn=lambda *a: None)
