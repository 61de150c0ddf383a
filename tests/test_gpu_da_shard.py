"""Parity of the rules added on top of Local / Full / Keep, through the C ABI:

* Declarative-Attention modes compiled into page runs on the device (no keep list): outputs,
  normalisers, the exported visible sets (bit-exact) and the attended-row counter, against the
  oracle's region definitions; the device plan equals the host-built keep lists bitwise;
* context-parallel Full: the history cut into page-aligned shards, each decoded on its own
  (as one GPU of a context-parallel group would), the partials merged by oda_merge_partials,
  against the oracle's Full attention and against the single-call Full decode; the commit
  happens on the shard that holds t only;
* the LSE merge itself on random partials with empty parts and a gate;
* the random gate schedule: gate == (u < rho) bit-exact, counters."""
import math

import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import SCALE, Case, assert_attn_close, assert_lse_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import da, oda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _run(case, fn, want_status=0):
    fn()
    torch.cuda.synchronize()
    assert int(case.status.item()) == want_status, oda.oda_status_string(int(case.status.item()))


DA_KW = dict(focus_len=2000, recent=300, local_len=700)


def _da_case():
    # lengths (tokens incl. the current one) chosen so that regions start and end mid-page,
    # overlap, touch, or run past t
    c = Case([1, 17, 300, 2500, 5000, 5000, 9001, 9001, 40_000], hq=32, hkv=8, seed=61)
    modes = [0, 1, 2, 1, 1, 1, 0, 1, 2]
    offs = [0, 5, 0, 1999, 4800, 100_000, 0, 7, 0]
    return c, modes, offs


def test_da_device_compiled_modes_match_oracle():
    c, modes, offs = _da_case()
    m = torch.tensor(modes, dtype=torch.int32, device="cuda")
    o = torch.tensor(offs, dtype=torch.int32, device="cuda")
    vis = oda.da_visibility(m, o, **DA_KW)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode(c.kv, vis, c.q, SCALE, out, c.ws, lse=lse))
    pos = lambda b, t: O.da_mode_positions(modes[b], t, offs[b], **DA_KW)
    ref, rlse = c.oracle(pos)
    assert_attn_close(out.cpu().numpy(), ref, "da")
    assert_lse_close(lse.cpu().numpy(), rlse)
    rows = sum(pos(b, n - 1).size for b, n in enumerate(c.lengths))
    assert c.stats[oda.ODA_STAT_ROWS].item() == 8 * rows
    # the exported plan is the oracle's index set, position by position
    T = max(c.lengths)
    mask = torch.full((c.B, T), 7, dtype=torch.uint8, device="cuda")
    _run(c, lambda: oda.oda_visible_mask_ex(c.kv, vis, mask))
    mk = mask.cpu().numpy()
    for b, n in enumerate(c.lengths):
        want = np.zeros(T, dtype=np.uint8)
        want[pos(b, n - 1)] = 1
        assert np.array_equal(mk[b], want), b


def test_da_device_plan_equals_host_keep_lists_bitwise():
    c, modes, offs = _da_case()
    draws = [oda_synth.DaDraw(mode=mm, focus_offset=oo) for mm, oo in zip(modes, offs)]
    keep, counts = da.keep_lists(draws, [n - 1 for n in c.lengths], max_keep=c.bt.shape[1],
                                 **DA_KW)
    a, la = c.out_buffers()
    k, lk = c.out_buffers()
    vis = oda.da_visibility(torch.tensor(modes, dtype=torch.int32, device="cuda"),
                            torch.tensor(offs, dtype=torch.int32, device="cuda"), **DA_KW)
    _run(c, lambda: oda.oda_decode(c.kv, vis, c.q, SCALE, a, c.ws, lse=la))
    _run(c, lambda: oda.oda_decode_blockmask(c.kv, c.q, SCALE, torch.from_numpy(keep).cuda(),
                                             torch.from_numpy(counts).cuda(), k, c.ws, lse=lk))
    assert torch.equal(a, k) and torch.equal(la, lk)   # same pages, same split, same order


def test_da_bad_declaration_reports_and_empties():
    c = Case([100, 200], hq=16, hkv=8, seed=62)
    vis = oda.da_visibility(torch.tensor([1, 5], dtype=torch.int32, device="cuda"),
                            torch.tensor([10, 0], dtype=torch.int32, device="cuda"), **DA_KW)
    out, lse = c.out_buffers()
    _run(c, lambda: oda.oda_decode(c.kv, vis, c.q, SCALE, out, c.ws, lse=lse),
         want_status=oda.ODA_DEV_BAD_DA)
    ref, rlse = c.oracle(lambda b, t: O.da_mode_positions(1, t, 10, **DA_KW), seqs=[0])
    assert_attn_close(out[0].cpu().numpy(), ref[0], "good sequence")
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))


def _cuts(cap_tokens, parts):
    cuts = [((cap_tokens * i // parts) // 16) * 16 for i in range(parts)] + [1 << 30]
    return [(a, b) for a, b in zip(cuts, cuts[1:]) if b > a]


@pytest.mark.parametrize("parts", [1, 2, 3, 8])
def test_context_parallel_full_equals_full(parts):
    lens = [1, 16, 17, 300, 2053, 5000, 40_001]
    c = Case(lens, hq=16, hkv=8, seed=70 + parts)
    shards = _cuts(max(lens), parts)
    R = len(shards)
    o_parts = torch.full((R, c.B, c.hq, 128), float("nan"), device="cuda")
    l_parts = torch.full((R, c.B, c.hq), float("nan"), device="cuda")
    for r, (lo, hi) in enumerate(shards):
        _run(c, lambda: oda.oda_decode(c.kv, oda.shard_visibility(lo, hi), c.q, SCALE,
                                       o_parts[r], c.ws, lse=l_parts[r]))
    out, lse = c.out_buffers()
    oda.oda_merge_partials(o_parts, l_parts, out, lse=lse)
    torch.cuda.synchronize()
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(out.cpu().numpy(), ref, "cp full")
    assert_lse_close(lse.cpu().numpy(), rlse)
    # each shard on its own is the oracle's attention over that range (empty: 0, -inf)
    for r, (lo, hi) in enumerate(shards):
        sref, slse = c.oracle(lambda b, t: O.shard_positions(t, lo, hi))
        assert_attn_close(o_parts[r].cpu().numpy(), sref, "shard %d" % r)
        assert_lse_close(l_parts[r].cpu().numpy(), slse)
    f, lf = c.out_buffers()
    _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, f, c.ws, lse=lf))
    assert (out - f).abs().max().item() <= 2e-6 and (lse - lf).abs().max().item() <= 2e-5
    # the exported plan of each shard is exactly its positions, and the shards tile 0..t
    T = max(lens)
    cover = np.zeros((c.B, T), dtype=np.int64)
    for lo, hi in shards:
        mask = torch.full((c.B, T), 7, dtype=torch.uint8, device="cuda")
        _run(c, lambda: oda.oda_visible_mask_ex(c.kv, oda.shard_visibility(lo, hi), mask))
        mk = mask.cpu().numpy()
        for b, n in enumerate(lens):
            want = np.zeros(T, dtype=np.uint8)
            want[O.shard_positions(n - 1, lo, hi)] = 1
            assert np.array_equal(mk[b], want)
        cover += mk
    assert all(np.array_equal(cover[b, :n], np.ones(n)) and not cover[b, n:].any()
               for b, n in enumerate(lens))


def test_context_parallel_commit_and_gate():
    lens = [33, 700, 5000]
    c = Case(lens, hq=32, hkv=8, seed=75)
    gate = torch.tensor([1, 0, 1], dtype=torch.int32, device="cuda")
    shards = _cuts(max(lens), 4)
    R = len(shards)
    o_parts = torch.zeros((R, c.B, c.hq, 128), device="cuda")
    l_parts = torch.zeros((R, c.B, c.hq), device="cuda")
    for r, (lo, hi) in enumerate(shards):
        _run(c, lambda: oda.oda_decode(c.kv, oda.shard_visibility(lo, hi, gate=gate), c.q, SCALE,
                                       o_parts[r], c.ws, k_new=c.k_new, v_new=c.v_new,
                                       lse=l_parts[r]))
    out, lse = c.out_buffers(fill=7.0)
    oda.oda_merge_partials(o_parts, l_parts, out, gate=gate, lse=lse)
    torch.cuda.synchronize()
    g = gate.cpu().numpy().astype(bool)
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t), commit=True, seqs=np.nonzero(g)[0])
    assert_attn_close(out.cpu().numpy()[g], ref[g], "cp gated")
    assert_lse_close(lse.cpu().numpy()[g], rlse[g])
    assert torch.all(out[1] == 7.0) and torch.all(lse[1] == 7.0)
    old_k, old_v = c.kbits, c.vbits
    c.snapshot()
    for b, n in enumerate(lens):          # slot t holds k_new exactly where gated, once
        want = c.knew_bits[b] if g[b] else c.slot_bits(old_k, b, n - 1)
        assert np.array_equal(c.slot_bits(c.kbits, b, n - 1), want)
    pages, _, rows, _ = np.nonzero((c.kbits != old_k) | (c.vbits != old_v))
    slots = {(int(c.bt_h[b, (n - 1) // 16]), (n - 1) % 16) for b, n in enumerate(lens) if g[b]}
    assert set(zip(pages.tolist(), rows.tolist())) <= slots


def test_merge_partials_against_oracle():
    r = np.random.default_rng(3)
    R, Bn, Hq = 5, 3, 8
    o = r.standard_normal((R, Bn, Hq, 128)).astype(np.float32)
    l = (r.standard_normal((R, Bn, Hq)) * 4).astype(np.float32)
    l[1, 0, :] = -np.inf                       # an empty part
    l[:, 2, 3] = -np.inf                       # every part empty for one head
    gate = torch.tensor([1, 1, 1], dtype=torch.int32, device="cuda")
    out = torch.full((Bn, Hq, 128), float("nan"), device="cuda")
    lse = torch.full((Bn, Hq), float("nan"), device="cuda")
    oda.oda_merge_partials(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda(), out, gate=gate,
                           lse=lse)
    torch.cuda.synchronize()
    got, gl = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(Bn):
        for h in range(Hq):
            ro, rl = O.lse_merge([(o[i, b, h].astype(np.float64), float(l[i, b, h]))
                                  for i in range(R)])
            assert np.abs(got[b, h] - ro).max() <= 1e-5
            if rl == -math.inf:
                assert gl[b, h] == -np.inf and np.all(got[b, h] == 0)
            else:
                assert abs(gl[b, h] - rl) <= 1e-5
    ob = torch.empty((Bn, Hq, 128), dtype=torch.bfloat16, device="cuda")
    oda.oda_merge_partials(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda(), ob)
    assert torch.equal(ob, out.to(torch.bfloat16))


@pytest.mark.parametrize("rho", [0.0, 0.125, 0.5, 1.0])
def test_random_gate_schedule(rho):
    B = 1000
    u = torch.rand(B, generator=torch.Generator(device="cuda").manual_seed(9), device="cuda")
    gate = torch.full((B,), 7, dtype=torch.int32, device="cuda")
    fc = torch.zeros(2, dtype=torch.int64, device="cuda")
    oda.oda_gate_schedule(u, rho, gate, full_count=fc)
    torch.cuda.synchronize()
    want = O.random_schedule_gate(u.cpu().numpy(), rho)
    assert np.array_equal(gate.cpu().numpy().astype(bool), want)
    assert fc.cpu().tolist() == [int(want.sum()), int(want.any())]


def test_context_parallel_module_over_nccl_single_rank():
    """ContextParallelFull end to end (SHARD decode -> NCCL all-gather -> merge) in a
    one-rank NCCL group: one shard covers everything, so the result is the Full decode's,
    bit for bit (same plan and split; merging one part multiplies by 1 and adds log 1)."""
    import socket

    import torch.distributed as dist

    from sparse_kv_recall_b200 import cp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        lens = [1, 300, 5000]
        c = Case(lens, hq=16, hkv=8, seed=77)
        run = cp.ContextParallelFull(c.B, c.hq, cp.shard_bounds(max(lens), 1)[0], c.ws)
        out, lse = c.out_buffers()
        run(c.kv, c.q, SCALE, out, lse=lse)
        f, lf = c.out_buffers()
        _run(c, lambda: oda.oda_decode_full(c.kv, c.q, SCALE, f, c.ws, lse=lf))
        assert torch.equal(out, f) and torch.equal(lse, lf)
    finally:
        dist.destroy_process_group()
