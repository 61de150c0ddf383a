"""Parity at the workloads' full sizes, in the launch configuration bench.py times (the step
graph: Local with commit at every layer, recall head, IF node, gated Full with commit), on
sampled outputs the oracle computes one by one:

* 128K history, 28 layers, batch 1 (16 q / 8 KV heads);
* 16K history, 28 layers, batch 8;
* ragged 8K..64K histories, 36 layers, batch 16, 32 q / 8 KV heads (87 GB of pages);
* 1M history, 1 layer, batch 2: Declarative-Attention keep lists, one per mode.

Step 0 runs with theta = -inf (every sequence recomputes with Full) and step 1 with
theta = +inf (Local only), so both paths and both commits are exercised deterministically;
the oracle reads the seeded prefill pages (host copies of only the sampled layers and
sequences) plus the K/V it decided to commit itself."""
import math

import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import Q_TOL, assert_attn_close, assert_lse_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import da, oda
from sparse_kv_recall_b200.engine import OdaEngine, fill_staging

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()
    yield
    torch.cuda.empty_cache()


def _logical(cache, bt_row, n_tokens):
    """Host copy of one sequence's pages of one layer, in position order: uint16
    [Hkv][n_tokens][128]. The gather is a torch index on the device (plumbing only)."""
    npages = (n_tokens + 15) // 16
    pages = cache.index_select(0, bt_row[:npages].long())          # [np][Hkv][16][128]
    flat = pages.permute(1, 0, 2, 3).reshape(cache.shape[1], npages * 16, 128)
    return oda_synth.bf16_bits(flat[:, :n_tokens])


def _bits(t):
    return oda_synth.bf16_bits(t)


def _attend(q_bits, kh, vh, positions, overlay=None, heads=None):
    """fp64 attention for query heads `heads` of one sequence: kh / vh logical bits
    [Hkv][>=t+1][128]; overlay = (t, k_bits [Hkv][128], v_bits) replaces position t.
    Returns {head: (out [128], lse)}."""
    Hq = q_bits.shape[0]
    Hkv = kh.shape[0]
    G = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    out = {}
    for g in sorted({h // G for h in heads}):
        K = O.widen_bf16(kh[g][positions])
        V = O.widen_bf16(vh[g][positions])
        if overlay is not None:
            t, kn, vn = overlay
            at = np.nonzero(positions == t)[0]
            if at.size:
                K[at[0]] = O.widen_bf16(kn[g])
                V[at[0]] = O.widen_bf16(vn[g])
        for h in heads:
            if h // G == g:
                out[h] = O.softmax_attention(O.widen_bf16(q_bits[h]), K, V, SCALE)
    return out


def _run_oda(name, sample_layers, sample_seqs, sample_heads):
    w = oda_synth.WORKLOADS[name]
    lengths = oda_synth.prefill_lengths(w)
    lay = oda_synth.make_layout(w, extra_tokens=8, device="cuda")
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda")
    h0 = oda_synth.make_h0(w, device="cuda")
    L = w.layers
    want_layers = sorted(set(sample_layers) | {L - 1})
    hist = {}                                   # prefill the oracle reads, before any commit
    for l in want_layers:
        for b in sample_seqs:
            n = lengths[b]
            hist[(l, b)] = (_logical(caches[l][0], lay.block_table[b], n),
                            _logical(caches[l][1], lay.block_table[b], n))
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), -math.inf, sink=w.sink,
                    window=w.window)
    eng.set_h_prev(h0, 0)
    rec = (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
           rw.w2.double().cpu().numpy(), rw.b2)
    h_prev = h0.double().cpu().numpy()
    inputs = [oda_synth.make_step_inputs(w, step, device="cuda") for step in range(2)]
    paths = ["full", "local"]                   # step 0: theta = -inf, step 1: theta = +inf
    commit = {}                                 # (layer, b) -> [(k bits, v bits) per step]
    for step in range(2):
        if step == 1:
            eng.set_theta(math.inf)
        si, path = inputs[step], paths[step]
        fill_staging(eng.v, si, [n + step + 1 for n in lengths])
        eng.launch(step)
        torch.cuda.synchronize()
        assert int(eng.status.item()) == 0
        gate = eng.gate.cpu().numpy().astype(bool)
        assert gate.all() if step == 0 else not gate.any()
        last = {}
        for l in want_layers:
            out_dev = eng.layer_out(step, l).cpu().numpy()
            for b in sample_seqs:
                t = lengths[b] + step
                kh, vh = hist[(l, b)]
                prev = commit.get((l, b), [])
                pad = np.zeros_like(kh[:, :1])
                kfull = np.concatenate([kh] + [c[0][:, None] for c in prev] + [pad], 1)
                vfull = np.concatenate([vh] + [c[1][:, None] for c in prev] + [pad], 1)
                kn = _bits(getattr(si, "k_" + path)[l][b])
                vn = _bits(getattr(si, "v_" + path)[l][b])
                pos = (O.full_positions(t) if path == "full"
                       else O.local_positions(t, w.sink, w.window))
                heads = None if l == L - 1 else sample_heads
                ref = _attend(_bits(getattr(si, "q_" + path)[l][b]), kfull, vfull, pos,
                              overlay=(t, kn, vn), heads=heads)
                hs = sorted(ref)
                assert_attn_close(np.stack([out_dev[b, h] for h in hs]),
                                  np.stack([ref[h][0] for h in hs]),
                                  "%s step %d layer %d seq %d" % (name, step, l, b))
                if l == L - 1:
                    last[b] = np.concatenate([ref[h][0] for h in range(w.num_q_heads)])
                commit.setdefault((l, b), []).append((kn, vn))
        if step == 1:
            # recall on this Local step: h_{t-1} is the oracle's own step-0 (Full) selection
            rows = list(sample_seqs)
            qs = O.recall_score(h_prev[rows], si.emb.double().cpu().numpy()[rows],
                                np.stack([last[b] for b in rows]), *rec)
            got_q = eng.q_out.cpu().numpy()[rows]
            assert np.abs(got_q - qs).max() <= Q_TOL, (got_q, qs)
        else:
            for b in sample_seqs:
                h_prev[b] = last[b]
    # committed K/V at slots n (Full, step 0) and n + 1 (Local, step 1), bit-exact, every layer
    for l in range(L):
        for b in sample_seqs:
            for step in range(2):
                t = lengths[b] + step
                pb = int(lay.block_table[b, t // 16])
                si, path = inputs[step], paths[step]
                assert torch.equal(caches[l][0][pb, :, t % 16], getattr(si, "k_" + path)[l][b])
                assert torch.equal(caches[l][1][pb, :, t % 16], getattr(si, "v_" + path)[l][b])
    assert eng.full_count.cpu().tolist() == [w.batch, 1]
    eng.close()
    del caches, eng
    torch.cuda.empty_cache()


def test_128k_28_layers_batch1():
    _run_oda("qwen3-1.7b-128k-b1", sample_layers=[0, 13], sample_seqs=[0], sample_heads=[0, 7, 15])


def test_16k_28_layers_batch8():
    _run_oda("qwen3-1.7b-16k-b8", sample_layers=[0, 20], sample_seqs=[0, 5], sample_heads=[1, 10])


def test_ragged_36_layers_batch16():
    w = oda_synth.WORKLOADS["qwen3-8b-ragged-b16"]
    lens = oda_synth.prefill_lengths(w)
    seqs = [int(np.argmin(lens)), int(np.argmax(lens))]
    _run_oda("qwen3-8b-ragged-b16", sample_layers=[0, 17], sample_seqs=seqs, sample_heads=[0, 31])


def test_da_1m_keep_lists_all_modes():
    w = oda_synth.WORKLOADS["da-1m-b2"]
    lengths = oda_synth.prefill_lengths(w)
    lay = oda_synth.make_layout(w, extra_tokens=8, device="cuda")
    kc, vc = oda_synth.make_kv_cache(w, lay, 0, device="cuda")
    seq = torch.tensor([n + 1 for n in lengths], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stats = torch.zeros(2, dtype=torch.int64, device="cuda")
    kv = oda.make_kv(kc, vc, lay.block_table, seq, status, stats)
    ws = torch.zeros(oda.oda_decode_workspace_size(w.batch, w.num_kv_heads, w.num_q_heads),
                     dtype=torch.uint8, device="cuda")
    hist = [(_logical(kc, lay.block_table[b], lengths[b] + 1),
             _logical(vc, lay.block_table[b], lengths[b] + 1)) for b in range(w.batch)]
    q = oda_synth.make_step_inputs(w, 0, device="cuda").q_local[0]
    qb = _bits(q)
    t = [n for n in lengths]
    for modes, offs in [((0, 1), (0, 300_000)), ((2, 1), (0, t[1] + 1 - 34816))]:
        draws = [oda_synth.DaDraw(mode=m, focus_offset=o) for m, o in zip(modes, offs)]
        keep, counts = da.keep_lists(draws, t, max_keep=lay.block_table.shape[1])
        out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), device="cuda")
        lse = torch.full((w.batch, w.num_q_heads), float("nan"), device="cuda")
        stats.zero_()
        oda.oda_decode_blockmask(kv, q, SCALE, torch.from_numpy(keep).cuda(),
                                 torch.from_numpy(counts).cuda(), out, ws, lse=lse)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        rows = 0
        for b in range(w.batch):
            pos = O.da_mode_positions(draws[b].mode, t[b], draws[b].focus_offset)
            rows += pos.size
            ref = _attend(qb[b], hist[b][0], hist[b][1], pos, heads=[0, 9, 22, 31])
            got = out[b].cpu().numpy()
            assert_attn_close(np.stack([got[h] for h in sorted(ref)]),
                              np.stack([ref[h][0] for h in sorted(ref)]), "da mode %d" % draws[b].mode)
            assert_lse_close(np.array([lse[b, h].item() for h in sorted(ref)]),
                             np.array([ref[h][1] for h in sorted(ref)]))
        assert stats[0].item() == rows * w.num_kv_heads        # attended rows, exact
    del kc, vc
    torch.cuda.empty_cache()
