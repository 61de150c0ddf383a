"""KV-head tensor parallelism on one GPU: N ranks' head slices (their own K/V caches of Hkv/N
heads, the shared block table) decoded in turn through HeadParallelStep, the all-gathers done
by concatenation in rank order, against the oracle's ODA step over all heads: per-layer
outputs, recall score, gate (ties excluded), committed K/V bits of every slice; and the gate
bitwise identical on every rank (each computes the recall head from the same gathered h^L)."""
import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import Q_TOL, assert_attn_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda, tp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _logical(bits, bt, caps, hkv, d=128):
    out = np.zeros((len(caps), hkv, max(caps), d), dtype=np.uint16)
    for b, cap in enumerate(caps):
        p = np.arange(cap)
        out[b, :, :cap] = bits[bt[b, p // 16], :, p % 16, :].transpose(1, 0, 2)
    return out


@pytest.mark.parametrize("world,hq,lengths", [(2, 16, [700, 300]), (4, 16, [1500, 40]),
                                              (8, 32, [900])])
def test_head_slices_in_turn_equal_the_oracle_step(world, hq, lengths):
    hkv, steps = 8, 3
    w = oda_synth.Workload(name="tp", layers=3, batch=len(lengths), num_q_heads=hq,
                           num_kv_heads=hkv, prefill=max(lengths), steps=steps,
                           seed=600 + world, sink=4, window=128)
    lay = oda_synth.make_layout(w, extra_tokens=steps + 2, device="cuda", lengths=lengths)
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda")
    h0 = oda_synth.make_h0(w, device="cuda")
    bt = lay.block_table.cpu().numpy()
    dec = O.OdaDecoder([_logical(oda_synth.bf16_bits(k), bt, lay.capacity, hkv) for k, _ in caches],
                       [_logical(oda_synth.bf16_bits(v), bt, lay.capacity, hkv) for _, v in caches],
                       lengths, h0.double().cpu().numpy(),
                       (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
                        rw.w2.double().cpu().numpy(), rw.b2), sink=w.sink, window=w.window,
                       theta=0.0)
    seq_lens = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ranks, slices, rcaches = [], [], []
    for r in range(world):
        kv_lo, kv_hi, q_lo, q_hi = tp.head_slice(hkv, hq, world, r)
        mine = [(k[:, kv_lo:kv_hi].contiguous(), v[:, kv_lo:kv_hi].contiguous()) for k, v in caches]
        kvs = [oda.make_kv(k, v, lay.block_table, seq_lens, status) for k, v in mine]
        step = tp.HeadParallelStep(kvs, hq, world, r, (rw.w1, rw.b1, rw.w2, rw.b2), 0.0,
                                   w.sink, w.window, w.batch, "cuda")
        step.set_h_prev(h0)
        ranks.append(step)
        slices.append((kv_lo, kv_hi, q_lo, q_hi))
        rcaches.append(mine)
    n_gated = 0
    for i in range(steps):
        si = oda_synth.make_step_inputs(w, i, device="cuda")
        seq_lens.copy_(torch.tensor([n + i + 1 for n in lengths], dtype=torch.int32))

        def part(name, r, l):
            kv_lo, kv_hi, q_lo, q_hi = slices[r]
            x = getattr(si, name)[l]
            return (x[:, q_lo:q_hi] if name.startswith("q") else x[:, kv_lo:kv_hi]).contiguous()

        args = lambda path, r: [[part("%s_%s" % (k, path), r, l) for l in range(w.layers)]
                                for k in ("q", "k", "v")]
        h_l = tp.join_heads([ranks[r].local_pass(*args("local", r)) for r in range(world)])
        gates = [ranks[r].gate(h_l, si.emb).clone() for r in range(world)]
        assert all(torch.equal(g, gates[0]) for g in gates)          # the same branch everywhere
        sel = tp.join_heads([ranks[r].full_pass(*args("full", r)) for r in range(world)])
        for r in range(world):
            ranks[r].set_h_prev(sel)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        outs = np.stack([tp.join_heads([ranks[r].out[l] for r in range(world)]).cpu().numpy()
                         for l in range(w.layers)])
        gate = gates[0].cpu().numpy().astype(bool)
        inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
               for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
        inp["emb"] = si.emb.double().cpu().numpy()
        ref, _, rq, rg = dec.step(inp, gate_hint=gate)
        q = ranks[0].q_out.cpu().numpy()
        assert np.abs(q - rq).max() <= Q_TOL
        sure = np.abs(rq) >= Q_TOL
        assert np.array_equal(gate[sure], rg[sure])
        assert_attn_close(outs, ref, "tp world %d step %d" % (world, i))
        n_gated += int(gate.sum())
    assert all(torch.equal(rk.full_count, ranks[0].full_count) for rk in ranks)
    for r, (kv_lo, kv_hi, _, _) in enumerate(slices):          # commits, bit-exact, per slice
        for l, (k, v) in enumerate(rcaches[r]):
            dk = _logical(oda_synth.bf16_bits(k), bt, lay.capacity, kv_hi - kv_lo)
            dv = _logical(oda_synth.bf16_bits(v), bt, lay.capacity, kv_hi - kv_lo)
            for b, n in enumerate(lengths):
                assert np.array_equal(dk[b, :, :n + steps], dec.k[l][b, kv_lo:kv_hi, :n + steps])
                assert np.array_equal(dv[b, :, :n + steps], dec.v[l][b, kv_lo:kv_hi, :n + steps])
