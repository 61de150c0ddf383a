"""GPU parity of the decode kernels against the fp64 oracle, through the C ABI: Local, Full,
gated Full, keep-page masks, fused and standalone commits, the plan export, counters,
determinism and device-side error reporting. Sizes span many pages, several CTAs per
(sequence, KV head) and ragged tails."""
import numpy as np
import pytest
import torch

from oda_cases import (SCALE, Case, assert_attn_close, assert_lse_close)
from oracle import oda_oracle as O
import oda_synth
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import da, oda

pytestmark = pytest.mark.gpu

LENS = [1, 2, 16, 17, 33, 300, 2053, 5000]     # tokens including the current one


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _run(case, fn):
    fn()
    torch.cuda.synchronize()
    assert int(case.status.item()) == 0, oda.oda_status_string(int(case.status.item()))


@pytest.mark.parametrize("G", [1, 2, 4])
def test_full_matches_oracle(G):
    c = Case(LENS, hq=8 * G, hkv=8, seed=100 + G)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(out.cpu().numpy(), ref, "full G=%d" % G)
    assert_lse_close(lse.cpu().numpy(), rlse)
    st = c.stats.cpu().numpy()
    assert st[oda.ODA_STAT_ROWS] == 8 * sum(LENS)                     # every visible row, once
    assert st[oda.ODA_STAT_PAGES] == 8 * sum((n + 15) // 16 for n in LENS)


@pytest.mark.parametrize("sink,window", [(4, 256), (4, 2048), (0, 1), (7, 33), (1, 16), (20, 100)])
def test_local_matches_oracle(sink, window):
    c = Case(LENS + [9000], hq=16, hkv=8, seed=7 + window)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_local(c.kv, c.q, sink, window, SCALE, out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.local_positions(t, sink, window))
    assert_attn_close(out.cpu().numpy(), ref, "local s=%d w=%d" % (sink, window))
    assert_lse_close(lse.cpu().numpy(), rlse)
    rows = sum(len(O.local_positions(n - 1, sink, window)) for n in c.lengths)
    assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * rows


def test_maximum_batch_local_and_full():
    """The largest batch one launch takes (1024 sequences), ragged 1..700 tokens: every
    sequence's attended-row count exactly, sampled sequences against the oracle."""
    r = np.random.default_rng(11)
    lens = [int(x) for x in r.integers(1, 701, size=1024)]
    c = Case(lens, hq=16, hkv=8, seed=12, extra=0, spare_pages=0)
    seqs = list(range(0, 1024, 41)) + [1023]
    for name, fn, pos in [
            ("local", lambda o, l: oda.oda_decode_local(c.kv, c.q, 4, 128, SCALE, o, c.ws, lse=l),
             lambda b, t: O.local_positions(t, 4, 128)),
            ("full", lambda o, l: oda.oda_decode_full(c.kv, c.q, SCALE, o, c.ws, lse=l),
             lambda b, t: O.full_positions(t))]:
        c.stats.zero_()
        out, lse = c.out_buffers()
        _run(c, lambda: fn(out, lse))
        ref, rlse = c.oracle(pos, seqs=seqs)
        assert_attn_close(out.cpu().numpy()[seqs], ref[seqs], name)
        assert_lse_close(lse.cpu().numpy()[seqs], rlse[seqs])
        assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * sum(len(pos(b, n - 1))
                                                             for b, n in enumerate(lens))
    with pytest.raises(oda.OdaError):          # one more sequence is refused on the host
        big = oda.make_kv(c.kc, c.vc, torch.cat([c.bt, c.bt[:1]]),
                          torch.cat([c.seq_lens, c.seq_lens[:1]]))
        oda.oda_decode_full(big, torch.cat([c.q, c.q[:1]]), SCALE,
                            torch.zeros(1025, 16, 128, device="cuda"), c.ws)


@pytest.mark.parametrize("G,lens,sink,window", [
    (2, [1], 4, 2048), (2, [17], 4, 2048), (2, [2053], 4, 2048), (2, [40_000], 4, 2048),
    (1, [5000, 33], 4, 2048), (4, [9001, 2052], 0, 2100), (2, [700, 6000], 20, 100),
    (2, [3000], 7, 33), (2, [9000], 4, 2128), (4, [9000], 4, 2129)])
def test_local_short_window_cluster_path(G, lens, sink, window):
    """Small batches take the cluster kernel for Local (one cluster per (sequence, KV head),
    one page per warp on cluster ranks 1-15, partials merged in rank 0's shared memory):
    outputs, normalisers, attended rows and the fused commit against the oracle. Sink 4 with
    window 2128 bounds the page list at the kernel's 135 pages; window 2129 (136) takes the
    split kernel instead."""
    c = Case(lens, hq=8 * G, hkv=8, seed=90 + G + len(lens))
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_local(c.kv, c.q, sink, window, SCALE, out, c.ws,
                                         k_new=c.k_new, v_new=c.v_new, lse=lse))
    pos = lambda b, t: O.local_positions(t, sink, window)
    ref, rlse = c.oracle(pos, commit=True)
    assert_attn_close(out.cpu().numpy(), ref, "local cluster G=%d" % G)
    assert_lse_close(lse.cpu().numpy(), rlse)
    assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * sum(len(pos(b, n - 1))
                                                         for b, n in enumerate(lens))
    old_k = c.kbits
    c.snapshot()
    for b, n in enumerate(lens):
        assert np.array_equal(c.slot_bits(c.kbits, b, n - 1), c.knew_bits[b])
    pages, _, rows, _ = np.nonzero(c.kbits != old_k)
    slots = {(int(c.bt_h[b, (n - 1) // 16]), (n - 1) % 16) for b, n in enumerate(lens)}
    assert set(zip(pages.tolist(), rows.tolist())) <= slots


def _scale_rows_by_position(c, factor_of):
    """Multiply the K row of every cached position p of every sequence by factor_of(p, n)
    (n = that sequence's length), in place, and refresh the host copy."""
    f = torch.ones((c.num_blocks, 16), dtype=torch.float32)
    bt = c.bt.cpu().numpy()
    for b, n in enumerate(c.lengths):
        for p in range(n):
            f[bt[b, p // 16], p % 16] = factor_of(p, n)
    c.kc.copy_((c.kc.float() * f.to("cuda")[:, None, :, None]).to(torch.bfloat16))
    c.snapshot()


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("shape", ["rising", "sharp"])
def test_extreme_score_ranges(G, shape):
    """Scores that keep rising along the sequence (K rows scaled by 1 + 8 p / n: the running
    maximum is raised again and again, by more than any rescale margin) or that are 8x wider
    than N(0, 1) logits (about 60 base-2 units between a head's largest and typical score):
    Full and Local against the oracle."""
    c = Case([300, 2053, 5000], hq=8 * G, hkv=8, seed=300 + G)
    if shape == "rising":
        _scale_rows_by_position(c, lambda p, n: 1.0 + 8.0 * p / n)
    else:
        c.q.mul_(8.0)
        c.qbits = oda_synth.bf16_bits(c.q)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(out.cpu().numpy(), ref, "full %s G=%d" % (shape, G))
    assert_lse_close(lse.cpu().numpy(), rlse)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_local(c.kv, c.q, 4, 256, SCALE, out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.local_positions(t, 4, 256))
    assert_attn_close(out.cpu().numpy(), ref, "local %s G=%d" % (shape, G))
    assert_lse_close(lse.cpu().numpy(), rlse)


def test_local_equals_full_when_window_covers_history():
    """s + w = 260 covers t + 1 <= 260 tokens: the same visible set (bit-exact in the plan
    export), hence the same attention up to fp32 summation order (Local runs the cluster
    kernel, Full the ticketed one). At 261 tokens position 4 drops out of Local."""
    c = Case([1, 40, 259, 260, 261], hq=32, hkv=8, seed=3)
    a, la = c.out_buffers()
    b, lb = c.out_buffers()
    _run(c, lambda: oda.oda_decode_local(c.kv, c.q, 4, 256, SCALE, a, c.ws, lse=la))
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, b, c.ws, lse=lb))
    assert (a[:4] - b[:4]).abs().max().item() <= 2e-6
    assert (la[:4] - lb[:4]).abs().max().item() <= 2e-6
    assert (a[4] - b[4]).abs().max().item() > 1e-4
    ml = torch.zeros((c.B, 300), dtype=torch.uint8, device="cuda")
    mf = torch.zeros_like(ml)
    _run(c, lambda: oda.oda_visible_mask(c.kv, oda.ODA_MODE_LOCAL, ml, sink=4, window=256))
    _run(c, lambda: oda.oda_visible_mask(c.kv, oda.ODA_MODE_FULL, mf))
    assert torch.equal(ml[:4], mf[:4]) and not torch.equal(ml[4], mf[4])


def _keep_case(seed, G=4):
    c = Case([1, 17, 800, 3000, 7777, 12000], hq=8 * G, hkv=8, seed=seed)
    r = np.random.default_rng(seed)
    maxb = c.bt.shape[1]
    keep = np.full((c.B, maxb), -1, dtype=np.int32)
    counts = np.zeros(c.B, dtype=np.int32)
    for b, n in enumerate(c.lengths):
        npg = (n - 1) // 16 + 1
        if b == 0:
            k = np.arange(npg)                              # all kept
        elif b == 1:
            k = np.zeros(0, dtype=np.int64)                 # nothing kept
        else:
            k = np.sort(r.choice(npg, size=int(r.integers(1, npg + 1)), replace=False))
            k[-1] = npg - 1 if r.random() < 0.5 else k[-1]
            k = np.unique(k)
        keep[b, :k.size] = k
        counts[b] = k.size
    return c, keep, counts


@pytest.mark.parametrize("seed", [21, 22])
def test_blockmask_matches_oracle(seed):
    c, keep, counts = _keep_case(seed)
    out, lse = c.out_buffers()
    kb = torch.from_numpy(keep).cuda()
    kc = torch.from_numpy(counts).cuda()
    _run(c, lambda: oda.oda_decode_blockmask(c.kv, c.q, SCALE, kb, kc, out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.keep_positions(t, keep[b, :counts[b]]))
    assert_attn_close(out.cpu().numpy(), ref, "keep")
    assert_lse_close(lse.cpu().numpy(), rlse)
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))   # empty set
    rows = sum(len(O.keep_positions(n - 1, keep[b, :counts[b]])) for b, n in enumerate(c.lengths))
    assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * rows


def test_all_keep_equals_full_bitwise():
    c = Case([5, 333, 4097], hq=16, hkv=8, seed=9)
    maxb = c.bt.shape[1]
    keep = np.full((c.B, maxb), -1, dtype=np.int32)
    counts = np.array([(n - 1) // 16 + 1 for n in c.lengths], dtype=np.int32)
    for b, k in enumerate(counts):
        keep[b, :k] = np.arange(k)
    a, la = c.out_buffers()
    f, lf = c.out_buffers()
    _run(c, lambda: oda.oda_decode_blockmask(c.kv, c.q, SCALE, torch.from_numpy(keep).cuda(),
                                             torch.from_numpy(counts).cuda(), a, c.ws, lse=la))
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, f, c.ws, lse=lf))
    assert torch.equal(a, f) and torch.equal(la, lf)


def test_da_modes_through_blockmask():
    c = Case([70_000, 41_000], hq=32, hkv=8, seed=31)
    draws = [type("D", (), {"mode": 1, "focus_offset": 1234})(),
             type("D", (), {"mode": 2, "focus_offset": 0})()]
    pos = [n - 1 for n in c.lengths]
    keep, counts = da.keep_lists(draws, pos, max_keep=c.bt.shape[1])
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_blockmask(c.kv, c.q, SCALE, torch.from_numpy(keep).cuda(),
                                             torch.from_numpy(counts).cuda(), out, c.ws, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.da_mode_positions(draws[b].mode, t, draws[b].focus_offset))
    assert_attn_close(out.cpu().numpy(), ref, "da")
    assert_lse_close(lse.cpu().numpy(), rlse)


def test_gated_full_skips_and_commits():
    c = Case(LENS, hq=16, hkv=8, seed=41)
    gate = torch.tensor([1, 0, 1, 0, 0, 1, 0, 1], dtype=torch.int32, device="cuda")
    out, lse = c.out_buffers(fill=7.0)
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, gate=gate, k_new=c.k_new,
                                        v_new=c.v_new, lse=lse))
    g = gate.cpu().numpy().astype(bool)
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t), commit=True, seqs=np.nonzero(g)[0])
    o = out.cpu().numpy()
    assert_attn_close(o[g], ref[g], "gated")
    assert_lse_close(lse.cpu().numpy()[g], rlse[g])
    assert np.all(o[~g] == 7.0) and np.all(lse.cpu().numpy()[~g] == 7.0)   # untouched
    assert c.stats[oda.ODA_STAT_PAGES].item() == 8 * sum((n + 15) // 16 for n, k in zip(LENS, g) if k)
    old_k, old_v = c.kbits, c.vbits
    c.snapshot()
    for b, n in enumerate(LENS):
        want_k = c.knew_bits[b] if g[b] else c.slot_bits(old_k, b, n - 1)
        want_v = c.vnew_bits[b] if g[b] else c.slot_bits(old_v, b, n - 1)
        assert np.array_equal(c.slot_bits(c.kbits, b, n - 1), want_k)
        assert np.array_equal(c.slot_bits(c.vbits, b, n - 1), want_v)
    slots = {(int(c.bt_h[b, (n - 1) // 16]), (n - 1) % 16) for b, n in enumerate(LENS) if g[b]}
    pages, _, rows, _ = np.nonzero((c.kbits != old_k) | (c.vbits != old_v))
    assert set(zip(pages.tolist(), rows.tolist())) <= slots          # nothing else was written


def test_fused_local_commit_equals_standalone_append():
    c = Case([3, 100, 4096, 4097], hq=16, hkv=8, seed=51)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode_local(c.kv, c.q, 4, 256, SCALE, out, c.ws, k_new=c.k_new,
                                         v_new=c.v_new, lse=lse))
    ref, rlse = c.oracle(lambda b, t: O.local_positions(t, 4, 256), commit=True)
    assert_attn_close(out.cpu().numpy(), ref, "local+commit")
    assert_lse_close(lse.cpu().numpy(), rlse)
    fused_k, fused_v = c.kc.clone(), c.vc.clone()
    d = Case([3, 100, 4096, 4097], hq=16, hkv=8, seed=51)             # same seed: same cache
    _run(d, lambda: oda.oda_kv_append(d.kv, d.k_new, d.v_new))
    assert torch.equal(fused_k, d.kc) and torch.equal(fused_v, d.vc)
    gate = torch.tensor([0, 1, 0, 1], dtype=torch.int32, device="cuda")
    e = Case([3, 100, 4096, 4097], hq=16, hkv=8, seed=51)
    _run(e, lambda: oda.oda_kv_append(e.kv, e.k_new, e.v_new, gate=gate))
    before = d.kbits
    e.snapshot()
    for b, n in enumerate(e.lengths):
        want = e.knew_bits[b] if gate[b] else e.slot_bits(before, b, n - 1)
        assert np.array_equal(e.slot_bits(e.kbits, b, n - 1), want)


@pytest.mark.parametrize("mode", ["local", "full", "keep"])
def test_visible_mask_export_is_exact(mode):
    c, keep, counts = _keep_case(61, G=2)
    T = max(c.lengths) + 40
    mask = torch.full((c.B, T), 9, dtype=torch.uint8, device="cuda")
    gate = torch.tensor([1, 1, 0, 1, 1, 0], dtype=torch.int32, device="cuda")
    if mode == "local":
        sets = lambda b, t: O.local_positions(t, 4, 1000)
        _run(c, lambda: oda.oda_visible_mask(c.kv, oda.ODA_MODE_LOCAL, mask, sink=4, window=1000))
    elif mode == "full":
        sets = lambda b, t: O.full_positions(t) if gate[b] else np.zeros(0, np.int64)
        _run(c, lambda: oda.oda_visible_mask(c.kv, oda.ODA_MODE_FULL, mask, gate=gate))
    else:
        sets = lambda b, t: O.keep_positions(t, keep[b, :counts[b]])
        _run(c, lambda: oda.oda_visible_mask(c.kv, oda.ODA_MODE_KEEP, mask,
                                             keep_blocks=torch.from_numpy(keep).cuda(),
                                             keep_counts=torch.from_numpy(counts).cuda()))
    m = mask.cpu().numpy()
    for b, n in enumerate(c.lengths):
        want = np.zeros(T, dtype=np.uint8)
        want[sets(b, n - 1)] = 1
        assert np.array_equal(m[b], want), (mode, b)


def test_index_sets_through_attention_with_one_hot_values():
    """q = 0 makes every visible position weigh 1/|V|; V[p] = 64 e_(p mod 128) then gives
    out[d] = 64 |{p in V : p = d mod 128}| / |V|, so a single missing or extra position moves
    an output by >= 64 / |V| (>= 0.015 here), far beyond the tolerance."""
    c = Case([1, 130, 2100, 4000], hq=16, hkv=8, seed=71)
    c.q.zero_()
    onehot = torch.zeros(c.vc.shape, dtype=torch.bfloat16)
    nb = c.vc.shape[0]
    bt = c.bt.cpu()
    for b, n in enumerate(c.lengths):
        p = torch.arange(n)
        onehot[bt[b, p // 16], :, p % 16, p % 128] = 64.0
    c.vc.copy_(onehot.cuda())
    for sink, window in [(4, 256), (3, 1000), (0, 17)]:
        out, _ = c.out_buffers()
        _run(c, lambda: oda.oda_decode_local(c.kv, c.q, sink, window, SCALE, out, c.ws))
        for b, n in enumerate(c.lengths):
            vis = O.local_positions(n - 1, sink, window)
            want = 64.0 * np.bincount(vis % 128, minlength=128) / vis.size
            got = out[b].cpu().numpy()
            assert np.abs(got - want[None, :]).max() < 1e-4, (sink, window, b)
    assert nb > 0


def test_repeat_runs_are_bitwise_identical():
    c = Case(LENS, hq=32, hkv=8, seed=81)
    a, la = c.out_buffers()
    b, lb = c.out_buffers()
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, a, c.ws, lse=la))
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, b, c.ws, lse=lb))
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_long_segments_are_bitwise_repeatable_and_match_oracle(G):
    """Repeated launches over long and short segments (a 128K one spread over every CTA of the
    grid, one across share boundaries, short ones) agree bit for bit -- each partial is formed
    and merged in a fixed order -- and match the oracle; the launch-wide counters in the
    workspace stay zero."""
    lens = [131_073, 8_192 + 17, 8_191, 300, 1]
    c = Case(lens, hq=8 * G, hkv=8, seed=140 + G)
    outs = []
    for _ in range(3):
        out, lse = c.out_buffers()
        _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, lse=lse))
        outs.append((out, lse))
    for out, lse in outs[1:]:
        assert torch.equal(out, outs[0][0]) and torch.equal(lse, outs[0][1])
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(outs[0][0].cpu().numpy(), ref, "full over long segments G=%d" % G)
    assert_lse_close(outs[0][1].cpu().numpy(), rlse)
    st = c.stats.cpu().numpy()
    assert st[oda.ODA_STAT_ROWS] == 3 * 8 * sum(lens)                 # every row once per launch
    assert st[oda.ODA_STAT_PAGES] == 3 * 8 * sum((n + 15) // 16 for n in lens)
    ws_tail = c.ws.view(torch.int32)[-64:]
    assert int(ws_tail.abs().sum().item()) == 0                       # counters left zero


def test_bf16_output_within_one_ulp():
    c = Case([700, 3333], hq=16, hkv=8, seed=91)
    out, _ = c.out_buffers(dtype=torch.bfloat16)
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws))
    ref, _ = c.oracle(lambda b, t: O.full_positions(t))
    rb = torch.from_numpy(ref).to(torch.bfloat16).float()
    got = out.float().cpu()
    ulp = torch.where(rb == 0, torch.full_like(rb, 2.0 ** -133),
                      2.0 ** (torch.floor(torch.log2(rb.abs())) - 7))
    assert torch.all((got - rb).abs() <= ulp * 1.0001)


def test_device_errors_are_reported_not_trapped():
    c = Case([50, 40, 300], hq=16, hkv=8, seed=95)
    out, _ = c.out_buffers()
    bt = c.bt.clone()
    c.bt[2, 3] = c.num_blocks + 5                  # a page id outside the pool
    _run_status = lambda: (oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws), torch.cuda.synchronize())
    _run_status()
    assert int(c.status.item()) == oda.ODA_DEV_BAD_BLOCK
    c.bt.copy_(bt)
    c.status.zero_()
    c.seq_lens[1] = 0                               # empty sequence: a bad length
    _run_status()
    assert int(c.status.item()) == oda.ODA_DEV_BAD_LEN
    assert torch.all(out[1] == 0)
    c.seq_lens[1] = 10 ** 6                         # beyond the page table
    c.status.zero_()
    _run_status()
    assert int(c.status.item()) == oda.ODA_DEV_BAD_LEN
    c.seq_lens[1] = 40
    c.status.zero_()
    keep = torch.tensor([[0, 2, 1, -1], [0, 1, 2, -1], [0, 1, 2, 3]], dtype=torch.int32, device="cuda")
    counts = torch.tensor([3, 3, 3], dtype=torch.int32, device="cuda")
    oda.oda_decode_blockmask(c.kv, c.q, SCALE, keep, counts, out, c.ws)
    torch.cuda.synchronize()
    assert int(c.status.item()) == oda.ODA_DEV_BAD_KEEP_LIST     # sequence 0 is not ascending
    c.status.zero_()
    counts[2] = 9                                                  # count above max_keep
    oda.oda_decode_blockmask(c.kv, c.q, SCALE, keep, counts, out, c.ws)
    torch.cuda.synchronize()
    assert int(c.status.item()) == oda.ODA_DEV_BAD_KEEP_LIST
    # the workspace is still usable: a clean call afterwards matches the oracle
    c.status.zero_()
    good, _ = c.out_buffers()
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, good, c.ws))
    ref, _ = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(good.cpu().numpy(), ref)


def test_host_errors_raise():
    c = Case([10], hq=16, hkv=8, seed=97)
    out, _ = c.out_buffers()
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(oda.OdaError, match="WORKSPACE_TOO_SMALL"):
        oda.oda_decode_full(c.kv, c.q, SCALE, out, small)
    with pytest.raises(oda.OdaError, match="UNSUPPORTED_SHAPE"):
        oda.oda_decode_full(c.kv, c.q[:, :12].contiguous(), SCALE, out, c.ws)
