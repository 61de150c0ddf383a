"""Context-parallel Full's host logic on CPU ranks (gloo, world size 2 and 3): the shard
bounds tile the history in whole pages, and the all-gather returns every rank's partial in
rank order, so that the LSE merge of the gathered partials (here the oracle's, since CPU
ranks run no kernel) equals attention over the whole history."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_kv_recall_b200 import cp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_shard_bounds_tile_whole_pages():
    for cap in (0, 1, 16, 17, 4096, 131_088):
        for world in (1, 2, 3, 8):
            b = cp.shard_bounds(cap, world)
            assert len(b) == world and b[0][0] == 0 and b[-1][1] == cp.OPEN_END
            assert all(lo % 16 == 0 and hi % 16 == 0 for lo, hi in b)
            assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))      # contiguous
            sizes = [hi - lo for lo, hi in b[:-1]] + [16 * ((cap + 15) // 16) - b[-1][0]]
            assert max(sizes) - min(sizes) <= 16                             # balanced
    with pytest.raises(ValueError):
        cp.shard_bounds(10, 0)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from oracle import oda_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = np.random.default_rng(0)                       # same history on every rank
        B, Hq, d, n = 2, 4, 128, 300
        q = r.standard_normal((B, Hq, d))
        K = r.standard_normal((B, n, d))
        V = r.standard_normal((B, n, d))
        lo, hi = cp.shard_bounds(n, world)[rank]
        o_part = np.zeros((B, Hq, d))
        l_part = np.zeros((B, Hq))
        for b in range(B):
            pos = O.shard_positions(n - 1, lo, hi)
            for h in range(Hq):
                o_part[b, h], l_part[b, h] = O.softmax_attention(q[b, h], K[b, pos], V[b, pos],
                                                                 1 / math.sqrt(d))
        o_all, l_all = cp.gather_partials(torch.from_numpy(o_part), torch.from_numpy(l_part))
        assert o_all.shape == (world, B, Hq, d) and l_all.shape == (world, B, Hq)
        assert torch.equal(o_all[rank], torch.from_numpy(o_part))           # rank order
        err = 0.0
        for b in range(B):
            for h in range(Hq):
                mo, ml = O.lse_merge([(o_all[i, b, h].numpy(), float(l_all[i, b, h]))
                                      for i in range(world)])
                wo, wl = O.softmax_attention(q[b, h], K[b], V[b], 1 / math.sqrt(d))
                err = max(err, float(np.abs(mo - wo).max()), abs(ml - wl))
        out[rank] = err
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gathered_partials_merge_to_full_attention(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert len(res) == world and max(res.values()) < 1e-12
