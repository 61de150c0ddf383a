"""Seeded random sweep through the C ABI: batch sizes that take the cluster kernel and the
split kernel, G = 1, 2, 4, ragged lengths from one token to a few thousand, and every
visibility rule (Local with random sink and window, Full with a random gate, keep lists, DA
declarations, context-parallel shards), each against the oracle's sets and attention, with
the attended-row counter exact."""
import numpy as np
import pytest
import torch

from oda_cases import SCALE, Case, assert_attn_close, assert_lse_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _case(r, seed):
    batch = int(r.choice([1, 2, 3, 5, 9]))
    G = int(r.choice([1, 2, 4]))
    lens = [int(x) for x in r.integers(1, 3000, size=batch)]
    if r.random() < 0.3:
        lens[0] = int(r.choice([1, 15, 16, 17, 2052, 2053]))
    return Case(lens, hq=8 * G, hkv=8, seed=seed)


def _check(c, run, positions_of, seqs, commit=False):
    out, lse = c.out_buffers()
    c.stats.zero_()
    run(out, lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0, oda.oda_status_string(int(c.status.item()))
    ref, rlse = c.oracle(positions_of, commit=commit, seqs=seqs)
    assert_attn_close(out.cpu().numpy()[seqs], ref[seqs])
    assert_lse_close(lse.cpu().numpy()[seqs], rlse[seqs])
    return out


@pytest.mark.parametrize("seed", range(60))
def test_random_rules_match_oracle(seed):
    r = np.random.default_rng(1000 + seed)
    c = _case(r, 500 + seed)
    allb = list(range(c.B))
    t = [n - 1 for n in c.lengths]
    rule = ["local", "full", "keep", "da", "shard"][seed % 5]
    if rule == "local":
        s, w = int(r.integers(0, 40)), int(r.integers(1, 2200))
        pos = lambda b, tt: O.local_positions(tt, s, w)
        _check(c, lambda o, l: oda.oda_decode_local(c.kv, c.q, s, w, SCALE, o, c.ws,
                                                    k_new=c.k_new, v_new=c.v_new, lse=l),
               pos, allb, commit=True)
    elif rule == "full":
        g = r.random(c.B) < 0.6
        g[0] = True
        gate = torch.tensor(g.astype(np.int32), device="cuda")
        pos = lambda b, tt: O.full_positions(tt)
        _check(c, lambda o, l: oda.oda_decode_full(c.kv, c.q, SCALE, o, c.ws, gate=gate, lse=l),
               pos, [b for b in allb if g[b]])
    elif rule == "keep":
        maxk = c.bt.shape[1]
        keep = np.full((c.B, maxk), -1, dtype=np.int32)
        counts = np.zeros(c.B, dtype=np.int32)
        for b in allb:
            k = np.sort(r.choice(t[b] // 16 + 1, size=r.integers(0, t[b] // 16 + 2), replace=False))
            keep[b, :k.size] = k
            counts[b] = k.size
        pos = lambda b, tt: O.keep_positions(tt, keep[b, :counts[b]])
        kb, kc = torch.from_numpy(keep).cuda(), torch.from_numpy(counts).cuda()
        _check(c, lambda o, l: oda.oda_decode_blockmask(c.kv, c.q, SCALE, kb, kc, o, c.ws, lse=l),
               pos, allb)
    elif rule == "da":
        kw = dict(focus_len=int(r.integers(1, 900)), recent=int(r.integers(1, 400)),
                  local_len=int(r.integers(1, 1200)))
        modes = [int(x) for x in r.integers(0, 3, size=c.B)]
        offs = [int(r.integers(0, tt + 50)) for tt in t]
        vis = oda.da_visibility(torch.tensor(modes, dtype=torch.int32, device="cuda"),
                                torch.tensor(offs, dtype=torch.int32, device="cuda"), **kw)
        pos = lambda b, tt: O.da_mode_positions(modes[b], tt, offs[b], **kw)
        _check(c, lambda o, l: oda.oda_decode(c.kv, vis, c.q, SCALE, o, c.ws, lse=l), pos, allb)
    else:
        lo = 16 * int(r.integers(0, 100))
        hi = lo + 16 * int(r.integers(1, 100))
        vis = oda.shard_visibility(lo, hi)
        pos = lambda b, tt: O.shard_positions(tt, lo, hi)
        _check(c, lambda o, l: oda.oda_decode(c.kv, vis, c.q, SCALE, o, c.ws, lse=l), pos, allb)
    want_rows = sum(len(pos(b, t[b])) for b in allb
                    if rule != "full" or b in [x for x in allb if g[x]])
    assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * want_rows
