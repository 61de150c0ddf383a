"""KV-head tensor parallelism's host logic on CPU ranks (gloo, world size 2 and 4): head slices
tile the heads with each query head beside its KV head, the all-gather returns slices in head
order, every rank computes the same gate from the gathered h^L, and two steps decoded slice by
slice (the oracle's attention on each rank's heads, since CPU ranks run no kernel; commits and
h_{t-1} carried from step to step) equal the oracle's ODA step over all heads."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_kv_recall_b200 import tp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_head_slices_tile_the_heads():
    for hkv, hq in ((8, 16), (8, 32), (4, 4), (2, 8)):
        for world in (1, 2, 4, 8):
            if hkv % world:
                with pytest.raises(ValueError):
                    tp.head_slice(hkv, hq, world, 0)
                continue
            sl = [tp.head_slice(hkv, hq, world, r) for r in range(world)]
            assert sl[0][0] == 0 and sl[-1][1] == hkv and sl[0][2] == 0 and sl[-1][3] == hq
            for r in range(world - 1):
                assert sl[r][1] == sl[r + 1][0] and sl[r][3] == sl[r + 1][2]
            g = hq // hkv
            for kv_lo, kv_hi, q_lo, q_hi in sl:          # a query head reads a KV head of its rank
                assert all(kv_lo <= h // g < kv_hi for h in range(q_lo, q_hi))
    with pytest.raises(ValueError):
        tp.head_slice(8, 16, 2, 2)


def _bits(rng, shape):
    return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).bfloat16() \
        .view(torch.int16).numpy().view(np.uint16)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from oracle import oda_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(7)                  # the same problem on every rank
        B, Hkv, Hq, d, L, cap, sink, window = 2, 4, 8, 128, 2, 80, 4, 16
        lengths = [40, 70]
        kh = [_bits(rng, (B, Hkv, cap, d)) for _ in range(L)]
        vh = [_bits(rng, (B, Hkv, cap, d)) for _ in range(L)]
        D, M = Hq * d, 64
        W1 = rng.standard_normal((3 * D, M)) * 0.02
        b1, w2, b2 = np.zeros(M), rng.standard_normal(M) * 0.02, 0.0
        h0 = rng.standard_normal((B, D))
        steps = []
        for _ in range(2):
            inp = {k: [_bits(rng, (B, Hq if k.startswith("q") else Hkv, d)) for _ in range(L)]
                   for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
            inp["emb"] = rng.standard_normal((B, D))
            steps.append(inp)
        # theta between the two sequences' first-step scores: one gated, one not
        probe = O.OdaDecoder(kh, vh, lengths, h0, (W1, b1, w2, b2), sink=sink, window=window,
                             theta=0.0)
        q0 = probe.step(steps[0])[2]
        theta = float(q0.mean())
        ref = O.OdaDecoder(kh, vh, lengths, h0, (W1, b1, w2, b2), sink=sink, window=window,
                           theta=theta)

        kv_lo, kv_hi, q_lo, q_hi = tp.head_slice(Hkv, Hq, world, rank)
        k_mine = [x[:, kv_lo:kv_hi].copy() for x in kh]    # this rank's pages only
        v_mine = [x[:, kv_lo:kv_hi].copy() for x in vh]
        h_prev, lens, scale = h0.copy(), list(lengths), 1 / math.sqrt(d)

        def attend(layer, b, t, pos, qb, kb, vb):
            hist = pos[pos < t]
            ks, vs = [], []
            for g in range(kv_hi - kv_lo):
                kr = O.widen_bf16(k_mine[layer][b, g, hist])
                vr = O.widen_bf16(v_mine[layer][b, g, hist])
                if pos.size and pos[-1] == t:
                    kr = np.vstack([kr, O.widen_bf16(kb[g])[None]])
                    vr = np.vstack([vr, O.widen_bf16(vb[g])[None]])
                ks.append(kr)
                vs.append(vr)
            return O.decode_attention(O.widen_bf16(qb), ks, vs, scale)[0]

        err, gates_equal, gate_match = 0.0, True, True
        for inp in steps:
            sl = {k: [x[:, (q_lo if k.startswith("q") else kv_lo):(q_hi if k.startswith("q") else kv_hi)]
                      for x in v] for k, v in inp.items() if k != "emb"}
            outs = np.zeros((L, B, q_hi - q_lo, d))
            for layer in range(L):                       # Local, this rank's heads
                for b in range(B):
                    outs[layer, b] = attend(layer, b, lens[b], O.local_positions(lens[b], sink, window),
                                            sl["q_local"][layer][b], sl["k_local"][layer][b],
                                            sl["v_local"][layer][b])
            h_l = tp.gather_heads(torch.from_numpy(outs[L - 1].copy()))     # [B][Hq][d]
            q = O.recall_score(h_prev, inp["emb"], h_l.numpy().reshape(B, D), W1, b1, w2, b2)
            g = O.gate(q, theta)
            g_all = [torch.zeros(B, dtype=torch.int64) for _ in range(world)]
            dist.all_gather(g_all, torch.from_numpy(g.astype(np.int64)))
            gates_equal &= all(torch.equal(x, g_all[0]) for x in g_all)
            for b in range(B):                           # Full for the gated, this rank's heads
                if g[b]:
                    for layer in range(L):
                        outs[layer, b] = attend(layer, b, lens[b], O.full_positions(lens[b]),
                                                sl["q_full"][layer][b], sl["k_full"][layer][b],
                                                sl["v_full"][layer][b])
            for layer in range(L):                       # commit the selected path's K/V
                for b in range(B):
                    src = "full" if g[b] else "local"
                    k_mine[layer][b, :, lens[b]] = sl["k_" + src][layer][b]
                    v_mine[layer][b, :, lens[b]] = sl["v_" + src][layer][b]
            full_out = np.stack([tp.gather_heads(torch.from_numpy(outs[layer].copy())).numpy()
                                 for layer in range(L)])
            h_prev = full_out[L - 1].reshape(B, D).copy()
            lens = [x + 1 for x in lens]
            r_out, _, r_q, r_g = ref.step(inp)
            err = max(err, float(np.abs(full_out - r_out).max()), float(np.abs(q - r_q).max()))
            gate_match &= bool(np.array_equal(g, r_g))
        commits = all(np.array_equal(k_mine[l], ref.k[l][:, kv_lo:kv_hi]) and
                      np.array_equal(v_mine[l], ref.v[l][:, kv_lo:kv_hi]) for l in range(L))
        out[rank] = (err, gates_equal, gate_match, commits, int(g.sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_parallel_steps_equal_the_oracle_step(world):
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        err, gates_equal, gate_match, commits, _ = out[rank]
        assert err < 1e-12, (rank, err)
        assert gates_equal and gate_match and commits, (rank, out[rank])
