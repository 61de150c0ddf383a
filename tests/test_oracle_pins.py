"""Pins for the fp64 oracle, each against something other than the oracle itself: library
routines (torch SDPA, torch.nn layers, torch's bf16 conversion), closed forms, invariants,
alternative constructions from the pages' wording, and the constants the pages print."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oda_synth
from oracle import oda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oda_page_constants.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- inputs
def test_widen_bf16_matches_torch_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.widen_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ---------------------------------------------------------------- visible sets
def _local_by_slicing(t, s, w):
    hist = list(range(t + 1))
    picked = set(hist[:s]) | (set(hist[-w:]) if w > 0 else set())
    return sorted(picked)


@pytest.mark.parametrize("s", [0, 1, 4, 7])
@pytest.mark.parametrize("w", [1, 2, 16, 33, 2048])
def test_local_set_is_first_s_plus_last_w(s, w):
    for t in range(0, 90):
        got = O.local_positions(t, s, w).tolist()
        assert got == _local_by_slicing(t, s, w)
        assert len(got) == min(t + 1, s + w)      # |first s U last w| closed form
        assert got[-1] == t                        # the window counts the current token


def test_local_window_edge_at_page_constants():
    t = 131072 + 17
    pos = O.local_positions(t, 4, 2048)
    assert pos.size == 2052
    assert pos[:4].tolist() == [0, 1, 2, 3]
    assert pos[4] == t - 2047 and pos[-1] == t
    assert (t - 2048) not in set(pos.tolist())


def test_local_equals_full_when_history_short():
    for t in range(0, 300):
        if 4 + 256 >= t + 1:
            assert np.array_equal(O.local_positions(t, 4, 256), O.full_positions(t))


def test_keep_positions_against_page_mask():
    r = _rng(1)
    for _ in range(200):
        t = int(r.integers(0, 200))
        nb = t // 16 + 1
        keep = np.sort(r.choice(nb, size=int(r.integers(0, nb + 1)), replace=False))
        page_of = np.arange(t + 1) // 16
        expect = np.nonzero(np.isin(page_of, keep))[0]
        assert np.array_equal(O.keep_positions(t, keep), expect)
    assert np.array_equal(O.keep_positions(100, np.arange(100 // 16 + 1)), O.full_positions(100))
    assert O.keep_positions(100, []).size == 0


@pytest.mark.parametrize("bad", [[3, 3], [4, 2], [-1, 0], [0, 7]])
def test_keep_list_validation(bad):
    with pytest.raises(ValueError):
        O.keep_positions(100, bad)   # page 7 starts at 112 > t = 100


def test_da_focus_offset_must_be_a_position():
    with pytest.raises(ValueError):
        O.da_mode_positions(1, 100, -1)


def test_da_modes_closed_forms():
    t = 100_000
    assert np.array_equal(O.da_mode_positions(0, t), O.full_positions(t))
    loc = O.da_mode_positions(2, t)
    first_page = (t - 4095) // 16
    assert loc[0] == first_page * 16 and loc[-1] == t
    assert loc.size == t + 1 - first_page * 16
    off = 12_345
    foc = set(O.da_mode_positions(1, t, off).tolist())
    assert set(range(16)) <= foc                                   # sink page
    assert set(range((off // 16) * 16, off + 32768)) <= foc        # focused region, page-rounded
    assert set(range(t - 2047, t + 1)) <= foc                      # recent window
    assert (off // 16) * 16 - 1 not in foc and 16 not in foc
    # every visible position lies on a page that the mode touches, so counts are page multiples
    pages = {p // 16 for p in foc}
    assert len(foc) == 16 * (len(pages) - 1) + (t % 16 + 1)


# ---------------------------------------------------------------- paged reads
def test_paged_rows_roundtrip_through_random_page_table():
    r = _rng(2)
    n, Hkv, d = 83, 3, 8
    logical = r.integers(0, 65535, size=(Hkv, n, d)).astype(np.uint16)
    npages = (n + 15) // 16
    perm = r.permutation(npages + 5)[:npages]
    pool = np.zeros((npages + 5, Hkv, 16, d), dtype=np.uint16)
    for lp in range(npages):
        for row in range(16):
            p = lp * 16 + row
            if p < n:
                pool[perm[lp], :, row, :] = logical[:, p, :]
    pos = r.permutation(n)[:40]
    for g in range(Hkv):
        got = O.paged_rows(pool, perm, pos, g)
        assert np.array_equal(got, O.widen_bf16(logical[g, pos]), equal_nan=True)


# ---------------------------------------------------------------- attention
def _sdpa(q, K, V, mask, scale):
    """torch SDPA in fp64 over Hq query heads, Hkv key/value heads, one query row."""
    qt = torch.from_numpy(q)[None, :, None, :]          # [1][Hq][1][d]
    kt = torch.from_numpy(K)[None]                        # [1][Hkv][n][d]
    vt = torch.from_numpy(V)[None]
    m = torch.from_numpy(mask)[None, None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale,
                                                         enable_gqa=True)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (16, 8)])
def test_decode_attention_matches_sdpa(Hq, Hkv):
    r = _rng(Hq * 10 + Hkv)
    n, d = 57, 16
    q = r.standard_normal((Hq, d))
    K = r.standard_normal((Hkv, n, d))
    V = r.standard_normal((Hkv, n, d))
    vis = np.sort(r.choice(n, size=31, replace=False))
    mask = np.zeros(n, dtype=bool)
    mask[vis] = True
    scale = 1 / math.sqrt(d)
    out, lse = O.decode_attention(q, [K[g][vis] for g in range(Hkv)],
                                  [V[g][vis] for g in range(Hkv)], scale)
    np.testing.assert_allclose(out, _sdpa(q, K, V, mask, scale), rtol=0, atol=1e-13)
    # the normaliser is the natural log-sum-exp of the visible scores
    for h in range(Hq):
        s = K[h // (Hq // Hkv)][vis] @ q[h] * scale
        assert abs(lse[h] - float(torch.logsumexp(torch.from_numpy(s), 0))) < 1e-12


def test_attention_special_cases():
    r = _rng(3)
    d = 128
    v = r.standard_normal((1, d))
    o, lse = O.softmax_attention(r.standard_normal(d), r.standard_normal((1, d)), v, 0.1)
    assert np.array_equal(o, v[0])                                 # one token: o = v
    K, V = r.standard_normal((40, d)), r.standard_normal((40, d))
    o, lse = O.softmax_attention(np.zeros(d), K, V, 0.3)
    np.testing.assert_allclose(o, V.mean(0), atol=1e-14)           # q = 0: mean of V
    assert abs(lse - math.log(40)) < 1e-14                         # ... and lse = ln n
    q = r.standard_normal(d)
    o, _ = O.softmax_attention(q, K, np.ones((40, d)), 0.3)
    np.testing.assert_allclose(o, 1.0, atol=1e-14)                 # weights sum to 1
    o0, l0 = O.softmax_attention(q, K, V, 0.3)
    shift = 37.5                                                   # shift every score by c
    Ks = K + (shift / 0.3) * q / (q @ q)
    o1, l1 = O.softmax_attention(q, Ks, V, 0.3)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    assert abs(l1 - (l0 + shift)) < 1e-9
    o2, l2 = O.softmax_attention(q * 400, K, V, 1.0)               # huge scores stay finite
    assert np.all(np.isfinite(o2)) and math.isfinite(l2)
    o3, l3 = O.softmax_attention(q, np.zeros((0, d)), np.zeros((0, d)), 1.0)
    assert np.array_equal(o3, np.zeros(d)) and l3 == -math.inf    # empty set


def test_split_then_lse_merge_equals_whole():
    r = _rng(4)
    d = 64
    q, K, V = r.standard_normal(d), r.standard_normal((300, d)), r.standard_normal((300, d))
    o, l = O.softmax_attention(q, K, V, 0.125)
    cuts = [0, 7, 120, 121, 121, 300]                   # one empty part in the middle
    parts = [O.softmax_attention(q, K[a:b], V[a:b], 0.125) for a, b in zip(cuts, cuts[1:])]
    m = max(p[1] for p in parts)
    wts = np.array([math.exp(p[1] - m) for p in parts])
    merged = sum(w * p[0] for w, p in zip(wts, parts)) / wts.sum()
    np.testing.assert_allclose(merged, o, atol=1e-12)
    assert abs(m + math.log(wts.sum()) - l) < 1e-12
    # the oracle's merge is the same identity: unsplit attention, whatever the cut order
    for perm in ([0, 1, 2, 3, 4], [4, 2, 0, 3, 1]):
        om, lm = O.lse_merge([parts[i] for i in perm])
        np.testing.assert_allclose(om, o, atol=1e-12)
        assert abs(lm - l) < 1e-12
    oe, le = O.lse_merge([(np.zeros(d), -math.inf), (np.zeros(d), -math.inf)])
    assert np.array_equal(oe, np.zeros(d)) and le == -math.inf


def test_shards_tile_the_history():
    for t in (0, 15, 16, 1000):
        cuts = [0, 16, 48, 512, 1 << 30]
        got = np.concatenate([O.shard_positions(t, a, b) for a, b in zip(cuts, cuts[1:])])
        assert np.array_equal(got, np.arange(t + 1))        # disjoint, complete, in order
    assert O.shard_positions(10, 16, 32).size == 0          # a shard past t is empty


def test_random_schedule_gate_counts():
    u = _rng(8).random(10_000)
    assert not O.random_schedule_gate(u, 0.0).any()
    assert O.random_schedule_gate(u, 1.0).all()             # u in [0, 1)
    us = np.sort(u)
    for rho in (0.125, 0.416, 0.5):
        g = O.random_schedule_gate(u, rho)
        assert g.sum() == np.searchsorted(us, rho)          # brute count of draws below rho
        assert np.all(O.random_schedule_gate(u, rho + 0.1) >= g)   # monotone in rho


# ---------------------------------------------------------------- recall head and gate
def test_gelu_textbook_values():
    assert O.gelu(0.0) == 0.0
    assert abs(O.gelu(1.0) - 0.8413447460685429) < 1e-15          # Phi(1)
    assert abs(O.gelu(-1.0) + 0.15865525393145707) < 1e-15        # -Phi(-1)
    assert abs(O.gelu(10.0) - 10.0) < 1e-18
    assert abs(O.gelu(-10.0)) < 1e-20
    z = np.linspace(-6, 6, 101)
    ref = torch.nn.functional.gelu(torch.from_numpy(z), approximate="none").numpy()
    np.testing.assert_allclose(O.gelu(z), ref, atol=1e-15)


def test_recall_matches_torch_mlp():
    r = _rng(5)
    D, M, B = 32, 16, 3
    W1, b1 = r.normal(0, 0.2, (3 * D, M)), r.normal(0, 0.1, M)
    w2, b2 = r.normal(0, 0.2, M), 0.3
    hp, e, hl = (r.standard_normal((B, D)) for _ in range(3))
    mlp = torch.nn.Sequential(torch.nn.Linear(3 * D, M), torch.nn.GELU(),
                              torch.nn.Linear(M, 1)).double()
    with torch.no_grad():
        mlp[0].weight.copy_(torch.from_numpy(W1.T))
        mlp[0].bias.copy_(torch.from_numpy(b1))
        mlp[2].weight.copy_(torch.from_numpy(w2[None]))
        mlp[2].bias.fill_(b2)
        ref = mlp(torch.from_numpy(np.concatenate([hp, e, hl], 1)))[:, 0].numpy()
    np.testing.assert_allclose(O.recall_score(hp, e, hl, W1, b1, w2, b2), ref, atol=1e-14)


def test_recall_special_cases_and_input_order():
    r = _rng(6)
    D, M = 8, 5
    w2, b1 = r.standard_normal(M), r.standard_normal(M)
    x = [r.standard_normal((1, D)) for _ in range(3)]
    q = O.recall_score(*x, np.zeros((3 * D, M)), b1, w2, 0.25)
    ref_a = torch.nn.functional.gelu(torch.from_numpy(b1)).numpy()
    assert abs(q[0] - (ref_a @ w2 + 0.25)) < 1e-14                 # W1 = 0
    zero = np.zeros((1, D))
    assert O.recall_score(zero, zero, zero, r.standard_normal((3 * D, M)), np.zeros(M),
                          w2, -0.5)[0] == -0.5                      # zero input, b1 = 0
    # rows [2D, 3D) of W1 read the Local hidden state h^L_t, and only those
    W1 = np.zeros((3 * D, M))
    W1[2 * D:] = r.standard_normal((D, M))
    base = O.recall_score(x[0], x[1], x[2], W1, b1, w2, 0.0)
    moved = O.recall_score(x[0] + 1, x[1] - 2, x[2], W1, b1, w2, 0.0)
    assert np.array_equal(base, moved)
    assert O.recall_score(x[0], x[1], x[2] + 1, W1, b1, w2, 0.0)[0] != base[0]
    W1 = np.zeros((3 * D, M))
    W1[:D] = r.standard_normal((D, M))                              # rows [0, D): h_{t-1}
    assert np.array_equal(O.recall_score(x[0], x[1] + 3, x[2] - 1, W1, b1, w2, 0.0),
                          O.recall_score(x[0], x[1], x[2], W1, b1, w2, 0.0))


def test_gate_is_strict_and_monotone():
    assert not O.gate(0.0, 0.0)
    assert O.gate(1e-300, 0.0)
    q = _rng(7).standard_normal(1000)
    prev = None
    for th in np.linspace(-3, 3, 25):
        n = int(O.gate(q, th).sum())
        assert prev is None or n <= prev
        prev = n


# ---------------------------------------------------------------- cost model
def test_cost_model_against_counted_tokens():
    n, out_len, s, w = 100, 60, 4, 16
    full = sum(t + 1 for t in range(n, n + out_len))
    local_only = sum(len(O.local_positions(t, s, w)) for t in range(n, n + out_len))
    always = sum(O.attended_tokens(t, True, s, w) for t in range(n, n + out_len))
    assert O.attention_cost_ratio(n, out_len, 0.0, s, w) == pytest.approx(local_only / full, abs=1e-15)
    assert O.attention_cost_ratio(n, out_len, 1.0, s, w) == pytest.approx(always / full, abs=1e-15)
    r0, r1 = O.attention_cost_ratio(n, out_len, 0.0, s, w), O.attention_cost_ratio(n, out_len, 1.0, s, w)
    assert O.attention_cost_ratio(n, out_len, 0.3, s, w) == pytest.approx(r0 + 0.3 * (r1 - r0), abs=1e-15)
    # short histories: Local already covers everything
    assert O.attention_cost_ratio(10, 5, 0.0, 4, 16) == pytest.approx(1.0)


def test_page_constants_and_attention_cost_at_efficiency_point():
    g = json.load(open(GOLDEN))
    assert O.DEFAULT_SINK == g["sink"]["value"]
    assert O.DEFAULT_WINDOW == g["window"]["value"]
    assert O.DEFAULT_THETA == g["theta_default"]["value"]
    ep = g["efficiency_point"]
    ratio = O.attention_cost_ratio(ep["input_tokens"], ep["output_tokens"], ep["full_call_rate"])
    ell = g["sink"]["value"] + g["window"]["value"]
    mean_hist = ep["input_tokens"] + (ep["output_tokens"] + 1) / 2
    assert ratio == pytest.approx(ell / mean_hist + ep["full_call_rate"], rel=1e-12)
    assert round(100 * ratio, 2) == 14.06
    # the printed 24.26 % counts trunk FLOPs too, so attention alone must save more
    assert ratio < ep["main_decoding_flops_fraction"]


# ---------------------------------------------------------------- the ODA step
def _tiny(layers=2, batch=2, Hq=4, Hkv=2, d=16, n=40, s=2, w=8):
    wl = oda_synth.Workload(name="tiny", layers=layers, batch=batch, num_q_heads=Hq,
                            num_kv_heads=Hkv, prefill=n, steps=3, seed=99, sink=s, window=w,
                            head_dim=d, mlp=8)
    return wl


def _decoder(wl, theta, **kw):
    lay = oda_synth.make_layout(wl, extra_tokens=8)
    ks, vs = [], []
    for layer in range(wl.layers):
        kc, vc = oda_synth.make_kv_cache(wl, lay, layer)
        kb, vb = oda_synth.bf16_bits(kc), oda_synth.bf16_bits(vc)
        # logical history in position order, read through the page table
        cap = min(lay.capacity)
        kl = np.zeros((wl.batch, wl.num_kv_heads, cap, wl.head_dim), np.uint16)
        vl = np.zeros_like(kl)
        bt = lay.block_table.numpy()
        for b in range(wl.batch):
            for p in range(cap):
                kl[b, :, p] = kb[bt[b, p // 16], :, p % 16]
                vl[b, :, p] = vb[bt[b, p // 16], :, p % 16]
        ks.append(kl)
        vs.append(vl)
    rw = oda_synth.make_recall_weights(wl, std=0.3)
    rec = (rw.w1.double().numpy(), rw.b1.double().numpy(), rw.w2.double().numpy(), rw.b2)
    dec = O.OdaDecoder(ks, vs, oda_synth.prefill_lengths(wl), oda_synth.make_h0(wl).double().numpy(),
                       rec, sink=wl.sink, window=wl.window, theta=theta, **kw)
    return dec, ks, vs, rw


def _inp(wl, step):
    si = oda_synth.make_step_inputs(wl, step)
    d = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
         for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
    d["emb"] = si.emb.double().numpy()
    return d


def _sdpa_step(kh, vh, t, q_bits, k_bits, v_bits, positions, d):
    """Reference for one (layer, sequence): history rows 0..t-1 plus the slot-t inputs,
    attended through torch SDPA with a boolean mask."""
    K = np.concatenate([O.widen_bf16(kh[:, :t]), O.widen_bf16(k_bits)[:, None]], 1)
    V = np.concatenate([O.widen_bf16(vh[:, :t]), O.widen_bf16(v_bits)[:, None]], 1)
    mask = np.zeros(t + 1, dtype=bool)
    mask[positions] = True
    return _sdpa(O.widen_bf16(q_bits), K, V, mask, 1 / math.sqrt(d))


@pytest.mark.parametrize("theta,path", [(-math.inf, "full"), (math.inf, "local")])
def test_step_selects_and_commits(theta, path):
    wl = _tiny()
    dec, ks, vs, _ = _decoder(wl, theta)
    for step in range(2):
        inp = _inp(wl, step)
        lens = list(dec.lengths)
        out, lse, q, g = dec.step(inp)
        assert np.all(g == (path == "full"))
        for layer in range(wl.layers):
            for b in range(wl.batch):
                t = lens[b]
                pos = O.full_positions(t) if path == "full" else O.local_positions(t, wl.sink, wl.window)
                ref = _sdpa_step(ks[layer][b], vs[layer][b], t, inp["q_" + path][layer][b],
                                 inp["k_" + path][layer][b], inp["v_" + path][layer][b], pos, wl.head_dim)
                np.testing.assert_allclose(out[layer, b], ref, atol=1e-12)
                # commit: slot t now holds the selected path's K/V bits
                assert np.array_equal(dec.k[layer][b, :, t], inp["k_" + path][layer][b])
                assert np.array_equal(dec.v[layer][b, :, t], inp["v_" + path][layer][b])
                ks[layer][b, :, t] = inp["k_" + path][layer][b]
                vs[layer][b, :, t] = inp["v_" + path][layer][b]


def test_step_recall_reads_last_layer_local_and_previous_selection():
    wl = _tiny()
    dec, ks, vs, rw = _decoder(wl, 0.0)
    h0 = dec.h_prev.copy()
    inp = _inp(wl, 0)
    lens = list(dec.lengths)
    out, _, q, g = dec.step(inp)
    L = wl.layers - 1
    loc = np.stack([_sdpa_step(ks[L][b], vs[L][b], lens[b], inp["q_local"][L][b], inp["k_local"][L][b],
                               inp["v_local"][L][b], O.local_positions(lens[b], wl.sink, wl.window),
                               wl.head_dim).reshape(-1) for b in range(wl.batch)])
    mlp_in = torch.from_numpy(np.concatenate([h0, inp["emb"], loc], 1))
    z = mlp_in @ rw.w1.double() + rw.b1.double()
    ref = torch.nn.functional.gelu(z) @ rw.w2.double() + rw.b2
    np.testing.assert_allclose(q, ref.numpy(), atol=1e-12)
    # the next step's h_{t-1} is the selected last-layer output
    np.testing.assert_allclose(dec.h_prev, out[L].reshape(wl.batch, -1), atol=0)


def test_step_local_equals_full_when_window_covers_history():
    wl = _tiny(layers=1, n=10, s=4, w=64)
    a, _, _, _ = _decoder(wl, -math.inf)
    b, _, _, _ = _decoder(wl, math.inf)
    inp = _inp(wl, 0)
    oa, la, _, _ = a.step(inp)
    ob, lb, _, _ = b.step(inp)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)     # layer 0: same inputs both paths


def test_gate_hint_only_breaks_near_ties():
    wl = _tiny(layers=1)
    dec, _, _, _ = _decoder(wl, 0.0)
    inp = _inp(wl, 0)
    probe, _, _, _ = _decoder(wl, 0.0)
    _, _, q, g = probe.step(inp)
    theta = float(q[0])                       # put sequence 0 exactly on the threshold
    dec.theta = theta
    _, _, q2, g2 = dec.step(inp, gate_hint=[True, not (q[1] > theta)])
    assert g2[0]                              # tie: the hint decides
    assert g2[1] == (q[1] > theta) or abs(q[1] - theta) < 1e-3


@pytest.mark.parametrize("theta,path", [(math.inf, "local"), (-math.inf, "full")])
def test_step_per_layer_access_range(theta, path):
    """Hybrid backbones restrict only some layers to Local ([ODA] 개발자 관점): layer 1 is
    unrestricted (attends 0..t in the Local attempt too); layers 0 and 2 have their own s and
    w. Each layer is checked against SDPA with the mask built by slicing, and the recompute
    attends everything at every layer."""
    wl = _tiny(layers=3, n=40, s=2, w=8)
    sinks, windows = [2, 5, 0], [8, 8, 3]
    dec, ks, vs, _ = _decoder(wl, theta, local_layers=[1, 0, 1], sinks=sinks, windows=windows)
    for step in range(2):
        inp = _inp(wl, step)
        lens = list(dec.lengths)
        out, _, _, g = dec.step(inp)
        assert np.all(g == (path == "full"))
        for layer in range(wl.layers):
            for b in range(wl.batch):
                t = lens[b]
                if path == "full" or layer == 1:
                    pos = np.arange(t + 1)
                else:
                    pos = _local_by_slicing(t, sinks[layer], windows[layer])
                ref = _sdpa_step(ks[layer][b], vs[layer][b], t, inp["q_" + path][layer][b],
                                 inp["k_" + path][layer][b], inp["v_" + path][layer][b], pos,
                                 wl.head_dim)
                np.testing.assert_allclose(out[layer, b], ref, atol=1e-12)
                assert np.array_equal(dec.k[layer][b, :, t], inp["k_" + path][layer][b])
                ks[layer][b, :, t] = inp["k_" + path][layer][b]
                vs[layer][b, :, t] = inp["v_" + path][layer][b]


def test_window_of_one_sees_only_the_new_token():
    """s = 0, w = 1: the only visible row is the one just written, so o = v_new exactly."""
    wl = _tiny(layers=2, n=37)
    dec, _, _, _ = _decoder(wl, math.inf, sinks=[0, 0], windows=[1, 1])
    inp = _inp(wl, 0)
    out, lse, _, _ = dec.step(inp)
    G = wl.num_q_heads // wl.num_kv_heads
    for layer in range(2):
        for b in range(wl.batch):
            for h in range(wl.num_q_heads):
                v = O.widen_bf16(inp["v_local"][layer][b][h // G])
                assert np.array_equal(out[layer, b, h], v)
                s = float(O.widen_bf16(inp["q_local"][layer][b][h]) @
                          O.widen_bf16(inp["k_local"][layer][b][h // G])) / math.sqrt(wl.head_dim)
                assert lse[layer, b, h] == pytest.approx(s, abs=1e-12)


# ---------------------------------------------------------------- recall-head training objective
def test_signed_log_target_values():
    assert O.signed_log_target(0.0, 0.0) == 0.0
    assert O.signed_log_target(math.e - 1, 0.0) == pytest.approx(1.0, abs=1e-15)
    assert O.signed_log_target(0.5, 0.5 + math.e ** 2 - 1) == pytest.approx(-2.0, abs=1e-14)
    d = np.linspace(-5, 5, 41)
    np.testing.assert_allclose(O.signed_log_target(d, 0.0), -O.signed_log_target(-d, 0.0), atol=0)
    assert np.all(np.diff(O.signed_log_target(d, 0.0)) > 0)            # strictly increasing


def test_huber_closed_forms():
    assert O.huber(0.5) == 0.125 and O.huber(-0.5) == 0.125
    assert O.huber(3.0) == 2.5 and O.huber(-3.0) == 2.5                 # 1 * (3 - 1/2)
    assert O.huber(1.0) == 0.5                                          # both branches meet
    assert O.huber(4.0, delta=2.0) == 6.0                               # 2 * (4 - 1)


def test_gelu_grad_against_central_differences():
    z = np.linspace(-6, 6, 49)
    h = 1e-6
    num = (O.gelu(z + h) - O.gelu(z - h)) / (2 * h)
    np.testing.assert_allclose(O.gelu_grad(z), num, atol=1e-9)
    assert O.gelu_grad(0.0) == 0.5


def _train_case(B=3, D=3, M=4, seed=11, scale=0.7):
    r = _rng(seed)
    hp, em, hl = (r.standard_normal((B, D)) for _ in range(3))
    W1 = r.standard_normal((3 * D, M)) * scale
    b1, w2 = r.standard_normal(M) * scale, r.standard_normal(M) * scale
    gain = np.array([0.05, 8.0, -5.0])[:B]
    return hp, em, hl, W1, b1, w2, 0.3, gain


def test_recall_gradient_against_central_differences():
    hp, em, hl, W1, b1, w2, b2, gain = _train_case()
    lam = 0.2
    loss, q, dW1, db1, dw2, db2 = O.recall_loss_grad(hp, em, hl, W1, b1, w2, b2, gain, lam)
    # the residuals straddle delta = 1, so both Huber branches are exercised
    r = q - O.signed_log_target(gain, lam)
    assert (np.abs(r) < 1).any() and (np.abs(r) > 1).any()
    f = lambda W1_, b1_, w2_, b2_: O.recall_loss_grad(hp, em, hl, W1_, b1_, w2_, b2_, gain, lam)[0]
    h = 1e-6
    for arr, grad in ((W1, dW1), (b1, db1), (w2, dw2)):
        for idx in np.ndindex(arr.shape):
            up, dn = arr.copy(), arr.copy()
            up[idx] += h
            dn[idx] -= h
            args_up = [up if x is arr else x for x in (W1, b1, w2)]
            args_dn = [dn if x is arr else x for x in (W1, b1, w2)]
            num = (f(*args_up, b2) - f(*args_dn, b2)) / (2 * h)
            assert abs(num - grad[idx]) < 1e-7, (idx, num, grad[idx])
    num = (f(W1, b1, w2, b2 + h) - f(W1, b1, w2, b2 - h)) / (2 * h)
    assert abs(num - db2) < 1e-7
    # the forward half is the recall head itself
    np.testing.assert_allclose(q, O.recall_score(hp, em, hl, W1, b1, w2, b2), atol=0)


def test_recall_loss_with_silent_head_is_closed_form():
    """W1 = 0, b1 = 0, w2 = 0: q = b2 for every row, so loss = mean Huber(b2 - y), the only
    nonzero gradient is db2 = mean clip(b2 - y), and dW1, db1, dw2 vanish."""
    hp, em, hl, W1, b1, w2, _, gain = _train_case(B=3)
    W1, b1, w2 = np.zeros_like(W1), np.zeros_like(b1), np.zeros_like(w2)
    b2, lam = 0.4, 0.0
    loss, q, dW1, db1, dw2, db2 = O.recall_loss_grad(hp, em, hl, W1, b1, w2, b2, gain, lam)
    y = [math.copysign(math.log1p(abs(g)), g) for g in gain]
    assert np.all(q == b2)
    want = sum(0.5 * (b2 - t) ** 2 if abs(b2 - t) <= 1 else abs(b2 - t) - 0.5 for t in y) / 3
    assert loss == pytest.approx(want, abs=1e-15)
    assert db2 == pytest.approx(sum(min(max(b2 - t, -1), 1) for t in y) / 3, abs=1e-15)
    assert not dW1.any() and not db1.any() and not dw2.any()
