"""A whole ODA decode step (Local at every layer -> recall head -> conditional Full -> commit)
as one graph launch, over several steps, against the oracle's step: per-layer outputs,
recall scores, gates (ties within 1e-3 of theta excluded), committed K/V bits and the
Full-call counter. Includes the 1-layer 4K workload in full (64 steps)."""
import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import Q_TOL, assert_attn_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda
from sparse_kv_recall_b200.engine import OdaEngine, fill_staging

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _logical(bits, bt, caps, hkv, d):
    out = np.zeros((len(caps), hkv, max(caps), d), dtype=np.uint16)
    for b, cap in enumerate(caps):
        p = np.arange(cap)
        out[b, :, :cap] = bits[bt[b, p // 16], :, p % 16, :].transpose(1, 0, 2)
    return out


def _run_steps(w, lengths, steps, theta, use_conditional=True, recall_std=0.02, timing=False,
               step_kernels=oda.ODA_STEP_FULL_PERSISTENT, expect_kernels=None, staging_slots=1,
               **layer_ranges):
    lay = oda_synth.make_layout(w, extra_tokens=steps + 2, device="cuda", lengths=lengths)
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda", std=recall_std)
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), theta, sink=w.sink,
                    window=w.window, use_conditional=use_conditional, timing=timing,
                    step_kernels=step_kernels, staging_slots=staging_slots, **layer_ranges)
    if expect_kernels is not None:                  # launches per step: Local, gate, Full
        assert eng.graphs[0].kernels() == expect_kernels, eng.graphs[0].kernels()
    h0 = oda_synth.make_h0(w, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in evs:
        e.record()
    eng.set_h_prev(h0, 0)
    bt = lay.block_table.cpu().numpy()
    caps = lay.capacity
    kh = [_logical(oda_synth.bf16_bits(c[0]), bt, caps, w.num_kv_heads, 128) for c in caches]
    vh = [_logical(oda_synth.bf16_bits(c[1]), bt, caps, w.num_kv_heads, 128) for c in caches]
    rec = (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
           rw.w2.double().cpu().numpy(), rw.b2)
    dec = O.OdaDecoder(kh, vh, lengths, h0.double().cpu().numpy(), rec, sink=w.sink,
                       window=w.window, theta=theta, **layer_ranges)
    n_gated = 0
    n_phases = 0
    for i in range(steps):
        si = oda_synth.make_step_inputs(w, i, device="cuda")
        fill_staging(eng.views_for(i), si, [n + i + 1 for n in lengths])
        if timing:
            eng.set_events(i, evs)
        eng.launch(i)
        torch.cuda.synchronize()
        assert int(eng.status.item()) == 0
        if timing:
            phases = [evs[k].elapsed_time(evs[k + 1]) for k in range(3)]
            assert all(x >= 0 for x in phases) and phases[0] > 0
        outs = np.stack([eng.layer_out(i, l).cpu().numpy() for l in range(w.layers)])
        q = eng.q_out.cpu().numpy()
        gate = eng.gate.cpu().numpy().astype(bool)
        inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
               for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
        inp["emb"] = si.emb.double().cpu().numpy()
        inp["gate_u"] = si.gate_u.cpu().numpy()
        if layer_ranges.get("random_rho") is not None:
            ref, _, _, rg = dec.step(inp)
            assert np.array_equal(gate, rg), (i, gate, rg)   # the schedule decides, exactly
        else:
            ref, _, rq, rg = dec.step(inp, gate_hint=gate)
            assert np.abs(q - rq).max() <= Q_TOL, (i, q, rq)
            sure = np.abs(rq - theta) >= Q_TOL
            assert np.array_equal(gate[sure], rg[sure]), (i, gate, rg)
        assert_attn_close(outs, ref, "step %d" % i)
        n_gated += int(gate.sum())
        n_phases += int(gate.any())
    assert eng.full_count.cpu().tolist() == [n_gated, n_phases]
    for l, (kc, vc) in enumerate(caches):                       # committed K/V, bit-exact
        dk = _logical(oda_synth.bf16_bits(kc), bt, caps, w.num_kv_heads, 128)
        dv = _logical(oda_synth.bf16_bits(vc), bt, caps, w.num_kv_heads, 128)
        for b, n in enumerate(lengths):
            assert np.array_equal(dk[b, :, :n + steps], dec.k[l][b, :, :n + steps])
            assert np.array_equal(dv[b, :, :n + steps], dec.v[l][b, :, :n + steps])
    eng.close()
    return n_gated


@pytest.mark.parametrize("use_conditional", [True, False])
def test_step_graph_matches_oracle_ragged(use_conditional):
    w = oda_synth.Workload(name="tiny", layers=3, batch=3, num_q_heads=16, num_kv_heads=8,
                           prefill=300, steps=6, seed=77, sink=4, window=64)
    n = _run_steps(w, [300, 37, 170], 6, theta=0.0, use_conditional=use_conditional)
    assert 0 < n < 18                      # both paths exercised


def test_step_graph_per_layer_access_range():
    """Hybrid backbone: layer 1 is outside the Local restriction (attends its whole history
    in the Local attempt), layers 0 and 2 have their own sink and window."""
    w = oda_synth.Workload(name="hybrid", layers=3, batch=3, num_q_heads=16, num_kv_heads=8,
                           prefill=300, steps=5, seed=81, sink=4, window=64)
    n = _run_steps(w, [300, 37, 520], 5, theta=0.0, local_layers=[1, 0, 1], sinks=[4, 0, 0],
                   windows=[64, 64, 17])
    assert 0 < n < 15


@pytest.mark.parametrize("use_conditional", [True, False])
def test_step_graph_random_gate_schedule(use_conditional):
    """The random-timing ablation: the recall head is replaced by gate = u < rho on the
    step's uniform draws; everything downstream (IF node, gated Full, commit) is unchanged."""
    w = oda_synth.Workload(name="random", layers=2, batch=4, num_q_heads=16, num_kv_heads=8,
                           prefill=400, steps=6, seed=82, sink=4, window=64)
    n = _run_steps(w, [400, 90, 1000, 17], 6, theta=0.0, use_conditional=use_conditional,
                   random_rho=0.4)
    assert 0 < n < 24


@pytest.mark.parametrize("mode", [1, 2])
def test_step_graph_with_timing_events(mode):
    """Event nodes at the four phase boundaries (mode 1), or at the step's start and around
    the Full phase only (mode 2: the recall head stays programmatically dependent on the last
    Local layer); either way the step decodes as the oracle does."""
    w = oda_synth.Workload(name="tiny3", layers=2, batch=2, num_q_heads=16, num_kv_heads=8,
                           prefill=700, steps=4, seed=79, sink=4, window=128)
    _run_steps(w, [700, 300], 4, theta=0.0, timing=mode)


def test_step_graph_all_local_and_all_full():
    w = oda_synth.Workload(name="tiny2", layers=2, batch=2, num_q_heads=32, num_kv_heads=8,
                           prefill=500, steps=3, seed=78, sink=4, window=100)
    assert _run_steps(w, [500, 129], 3, theta=float("inf")) == 0
    assert _run_steps(w, [500, 129], 3, theta=-float("inf")) == 6


def test_pr1_reference_workload_all_steps():
    """1 layer, batch 1, 16 q / 8 KV heads, n = 4096, s = 4, w = 256, 64 steps, theta = 0."""
    w = oda_synth.WORKLOADS["pr1-ref-4k"]
    n = _run_steps(w, [w.prefill], w.steps, theta=w.theta)
    assert 0 < n < w.steps


def test_local_only_phase_graph():
    """phases = Local only (a measurement graph): every layer's Local output and commit, no
    recall head (its outputs stay untouched) and no Full pass."""
    w = oda_synth.Workload(name="tiny4", layers=2, batch=2, num_q_heads=16, num_kv_heads=8,
                           prefill=400, steps=2, seed=80, sink=4, window=64)
    lengths = [400, 150]
    lay = oda_synth.make_layout(w, extra_tokens=4, device="cuda", lengths=lengths)
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda")
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), -float("inf"), sink=w.sink,
                    window=w.window, phases=oda.ODA_PHASE_LOCAL)
    eng.q_out.fill_(7.0)
    bt = lay.block_table.cpu().numpy()
    kh = [_logical(oda_synth.bf16_bits(c[0]), bt, lay.capacity, 8, 128) for c in caches]
    vh = [_logical(oda_synth.bf16_bits(c[1]), bt, lay.capacity, 8, 128) for c in caches]
    rec = (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
           rw.w2.double().cpu().numpy(), rw.b2)
    dec = O.OdaDecoder(kh, vh, lengths, np.zeros((2, w.hidden)), rec, sink=w.sink,
                       window=w.window, theta=float("inf"))
    for i in range(2):
        si = oda_synth.make_step_inputs(w, i, device="cuda")
        fill_staging(eng.v, si, [n + i + 1 for n in lengths])
        eng.launch(i)
        torch.cuda.synchronize()
        inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
               for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
        inp["emb"] = si.emb.double().cpu().numpy()
        ref, _, _, _ = dec.step(inp)
        outs = np.stack([eng.layer_out(i, l).cpu().numpy() for l in range(w.layers)])
        assert_attn_close(outs, ref, "local-only step %d" % i)
    assert torch.all(eng.q_out == 7.0) and eng.full_count.sum().item() == 0
    for l, (kc, vc) in enumerate(caches):
        dk = _logical(oda_synth.bf16_bits(kc), bt, lay.capacity, 8, 128)
        for b, n in enumerate(lengths):
            assert np.array_equal(dk[b, :, :n + 2], dec.k[l][b, :, :n + 2])
    eng.close()


# ---- the persistent step kernels: Local at every layer + fused gate as one launch (one
# cluster per (sequence, KV head), batch x KV heads <= 9 clusters), Full as one launch ----
P = oda.ODA_STEP_PERSISTENT

def _expected_kernels(w):
    """(Local, gate, Full) launches per step the step graph should take on this device: the
    persistent Local kernel with the fused gate when its clusters fit, without it when only
    the smaller shared-memory form fits, else one launch per layer and a gate kernel."""
    G, ncl = w.num_q_heads // w.num_kv_heads, w.batch * w.num_kv_heads
    fused, _ = oda.oda_step_kernel_limits(G, w.batch, w.mlp)
    plain, _ = oda.oda_step_kernel_limits(G, w.batch, 0)
    slabs = -(-3 * w.num_q_heads * 128 // 256)              # the recall head's row slabs
    if fused >= ncl and ncl <= slabs:
        return (1, 0, 1)
    if plain >= ncl:
        return (1, 1, 1)
    return (w.layers, 1, 1)


def test_persistent_local_kernel_serves_the_default_shape():
    """Batch 1 x 8 KV heads with two query heads each (the long-context workload's shape) must
    fit the persistent Local kernel with its fused gate."""
    clusters, coop = oda.oda_step_kernel_limits(2, 1, 256)
    assert clusters >= 8, clusters


@pytest.mark.parametrize("use_conditional", [False, True])
@pytest.mark.parametrize("hq,hkv,batch,lengths", [
    (16, 8, 1, [700]),                 # G = 2, the default workload's grouping
    (32, 8, 1, [333]),                 # G = 4 (8 clusters of one CTA per SM: may not fit)
    (8, 8, 1, [512]),                  # G = 1
    (8, 4, 2, [700, 45]),              # two sequences, one shorter than the window
    (4, 2, 4, [300, 129, 1000, 16]),   # four sequences
    (8, 4, 1, [2000]),                 # four KV heads: fewer clusters than the maximum
])
def test_persistent_step_kernels_match_oracle(use_conditional, hq, hkv, batch, lengths):
    w = oda_synth.Workload(name="chain", layers=3, batch=batch, num_q_heads=hq,
                           num_kv_heads=hkv, prefill=max(lengths), steps=5, seed=90 + hq + batch,
                           sink=4, window=128)
    n = _run_steps(w, lengths, 5, theta=0.0, use_conditional=use_conditional,
                   step_kernels=P, expect_kernels=_expected_kernels(w))
    assert 0 < n < 5 * batch


def test_persistent_step_kernels_per_layer_sink_and_window():
    w = oda_synth.Workload(name="chain-ranges", layers=3, batch=1, num_q_heads=16,
                           num_kv_heads=8, prefill=900, steps=4, seed=93, sink=4, window=64)
    _run_steps(w, [900], 4, theta=0.0, sinks=[4, 0, 16], windows=[64, 17, 2000],
               step_kernels=P, expect_kernels=(1, 0, 1))


def test_persistent_step_kernels_random_schedule_and_ends():
    w = oda_synth.Workload(name="chain-random", layers=2, batch=1, num_q_heads=16,
                           num_kv_heads=8, prefill=400, steps=6, seed=94, sink=4, window=64)
    _run_steps(w, [400], 6, theta=0.0, random_rho=0.5, step_kernels=P, expect_kernels=(1, 0, 1))
    assert _run_steps(w, [400], 3, theta=float("inf"), step_kernels=P,
                      expect_kernels=(1, 0, 1)) == 0
    assert _run_steps(w, [400], 3, theta=-float("inf"), step_kernels=P,
                      expect_kernels=(1, 0, 1)) == 3


def test_persistent_step_kernels_with_timing_events():
    w = oda_synth.Workload(name="chain-timing", layers=2, batch=1, num_q_heads=16,
                           num_kv_heads=8, prefill=600, steps=3, seed=95, sink=4, window=256)
    _run_steps(w, [600], 3, theta=0.0, timing=True, step_kernels=P, expect_kernels=(1, 0, 1))


def test_shapes_outside_the_persistent_local_kernel_fall_back():
    """Batch 3 x 8 KV heads needs more clusters than the GPU holds at once: Local runs per
    layer with the recall kernel after it, Full still as one persistent launch."""
    w = oda_synth.Workload(name="chain-fallback", layers=2, batch=3, num_q_heads=16,
                           num_kv_heads=8, prefill=300, steps=3, seed=96, sink=4, window=64)
    _run_steps(w, [300, 37, 170], 3, theta=0.0, step_kernels=P, expect_kernels=(2, 1, 1))


@pytest.mark.parametrize("theta,prefill", [(float("inf"), 3000), (-float("inf"), 3000),
                                           (-float("inf"), 9000)])
def test_persistent_step_equals_per_layer(theta, prefill):
    """The persistent Full kernel runs the per-layer split pass itself, so with every step
    recomputed by Full (theta = -inf) every layer output is bitwise the per-layer launches'.
    Both Local kernels form page scores on the tensor cores, but the persistent one spreads a
    window's pages over all 16 CTAs of its cluster and the per-layer one over 15 (its rank 0
    only merges), so the partials group differently and Local outputs (theta = +inf) agree to
    fp32 rounding. The default mode (Local per layer, Full
    persistent) equals the per-layer launches bitwise at both ends. Committed K/V bits and the
    attended-row and page counters are identical either way; theta at +-inf keeps the gate out
    of it (the fused recall head sums in another order than the recall kernel). The 9000-token
    case spreads each segment over many CTAs of the grid."""
    w = oda_synth.Workload(name="chain-bitwise", layers=3, batch=1, num_q_heads=16,
                           num_kv_heads=8, prefill=prefill, steps=3, seed=97, sink=4, window=512)
    res = {}
    for sk in (oda.ODA_STEP_PERSISTENT, oda.ODA_STEP_PER_LAYER, oda.ODA_STEP_FULL_PERSISTENT):
        lay = oda_synth.make_layout(w, extra_tokens=5, device="cuda")
        caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
        rw = oda_synth.make_recall_weights(w, device="cuda")
        eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                        w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), theta, sink=w.sink,
                        window=w.window, use_conditional=False, step_kernels=sk)
        eng.set_h_prev(oda_synth.make_h0(w, device="cuda"), 0)
        outs = []
        for i in range(w.steps):
            fill_staging(eng.v, oda_synth.make_step_inputs(w, i, device="cuda"),
                         [w.prefill + i + 1])
            eng.launch(i)
            outs.append(torch.stack([eng.layer_out(i, l).clone() for l in range(w.layers)]))
        torch.cuda.synchronize()
        assert int(eng.status.item()) == 0
        res[sk] = (torch.stack(outs).cpu(), [(c[0].cpu(), c[1].cpu()) for c in caches],
                   eng.stats.cpu())
        eng.close()
    a, b = res[oda.ODA_STEP_PERSISTENT], res[oda.ODA_STEP_PER_LAYER]
    if theta < 0:
        assert torch.equal(a[0], b[0])
    else:
        assert (a[0] - b[0]).abs().max().item() <= 2e-6 * max(1.0, b[0].abs().max().item())
    for (ka, va), (kb, vb) in zip(a[1], b[1]):
        assert torch.equal(ka, kb) and torch.equal(va, vb)
    assert torch.equal(a[2], b[2])                       # rows / pages counters
    c = res[oda.ODA_STEP_FULL_PERSISTENT]
    assert torch.equal(c[0], b[0]) and torch.equal(c[2], b[2])
    for (kc, vc), (kb, vb) in zip(c[1], b[1]):
        assert torch.equal(kc, kb) and torch.equal(vc, vb)


@pytest.mark.parametrize("shape", [0, 1, 2, 3])
@pytest.mark.parametrize("hq,hkv,batch,lengths", [
    (8, 4, 1, [900]),            # two query heads per KV head
    (4, 2, 2, [700, 60]),        # inbox slots sized by the fused recall head (batch x mlp)
    (4, 4, 1, [500]),            # one query head per KV head
    (16, 4, 1, [400]),           # four query heads per KV head (no 8 x 18 instance)
])
def test_persistent_local_every_shape_matches_oracle(shape, hq, hkv, batch, lengths):
    """Each cluster shape of the persistent Local kernel (16 x 9, 14 x 10, 12 x 11, 8 x 18 CTAs
    x warps), forced through the tuning hook, with the fused recall head, against the oracle.
    Four clusters or fewer fit every shape; a group size a shape has no instance of falls back
    to one launch per layer."""
    w = oda_synth.Workload(name="chain-shape", layers=2, batch=batch, num_q_heads=hq,
                           num_kv_heads=hkv, prefill=max(lengths), steps=3,
                           seed=300 + 10 * shape + hq + batch, sink=4, window=128)
    G = hq // hkv
    expect = (w.layers, 1, 1) if (G == 4 and shape == 3) else (1, 0, 1)
    oda.oda_debug_set_local_shape(shape)
    try:
        _run_steps(w, lengths, 3, theta=0.0, use_conditional=False, step_kernels=P,
                   expect_kernels=expect)
    finally:
        oda.oda_debug_set_local_shape(-1)


@pytest.mark.parametrize("step_kernels", [oda.ODA_STEP_FULL_PERSISTENT, oda.ODA_STEP_PERSISTENT])
def test_two_staging_slots_match_oracle(step_kernels):
    """Even and odd steps read their own staging slot (so that a step's inputs can be copied
    in while the previous step runs); the decode is the oracle's either way."""
    w = oda_synth.Workload(name="slots", layers=3, batch=2, num_q_heads=16, num_kv_heads=8,
                           prefill=900, steps=5, seed=310, sink=4, window=128)
    n = _run_steps(w, [900, 333], 5, theta=0.0, use_conditional=False, staging_slots=2,
                   step_kernels=step_kernels)
    assert 0 < n < 10


def test_run_from_host_overlapped_matches_oracle():
    """The host path users call (OdaEngine.run_from_host): each step's staging image comes
    from pinned host memory on an input stream and its selected output goes back on an output
    stream while the neighbouring steps run; every step's result, read back on the host, is
    the oracle's. Recall weights large enough that no score sits within 1e-2 of theta (the
    gates are not read back)."""
    from sparse_kv_recall_b200.engine import StagingLayout
    w = oda_synth.Workload(name="host-path", layers=3, batch=2, num_q_heads=16, num_kv_heads=8,
                           prefill=700, steps=6, seed=320, sink=4, window=128)
    lengths = [700, 250]
    lay = oda_synth.make_layout(w, extra_tokens=w.steps + 2, device="cuda", lengths=lengths)
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda", std=0.5)
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), 0.0, sink=w.sink,
                    window=w.window, use_conditional=False, staging_slots=2)
    h0 = oda_synth.make_h0(w, device="cuda")
    eng.set_h_prev(h0, 0)
    bt = lay.block_table.cpu().numpy()
    dec = O.OdaDecoder([_logical(oda_synth.bf16_bits(k), bt, lay.capacity, w.num_kv_heads, 128)
                        for k, _ in caches],
                       [_logical(oda_synth.bf16_bits(v), bt, lay.capacity, w.num_kv_heads, 128)
                        for _, v in caches],
                       lengths, h0.double().cpu().numpy(),
                       (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
                        rw.w2.double().cpu().numpy(), rw.b2), sink=w.sink, window=w.window,
                       theta=0.0)
    layout = StagingLayout(w.layers, w.batch, w.num_q_heads, w.num_kv_heads, w.hidden)
    host = torch.empty((w.steps, layout.nbytes), dtype=torch.uint8, pin_memory=True)
    scratch = torch.zeros(layout.nbytes, dtype=torch.uint8, device="cuda")
    inputs = []
    for i in range(w.steps):
        si = oda_synth.make_step_inputs(w, i, device="cuda")
        fill_staging(layout.views(scratch), si, [n + i + 1 for n in lengths])
        host[i].copy_(scratch)
        inputs.append(si)
    out_host = torch.empty((w.steps, w.batch, w.hidden), dtype=torch.float32, pin_memory=True)
    assert eng.run_from_host(host, out_host, 0) == w.steps
    torch.cuda.synchronize()
    assert int(eng.status.item()) == 0
    n_gated = 0
    for i, si in enumerate(inputs):
        inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
               for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
        inp["emb"] = si.emb.double().cpu().numpy()
        ref, _, rq, rg = dec.step(inp)
        assert np.abs(rq).min() >= 1e-2, rq                   # no near-tie: the gate is sure
        assert_attn_close(out_host[i].numpy().reshape(w.batch, w.num_q_heads, 128)[None],
                          ref[-1][None], "host path step %d" % i)
        n_gated += int(rg.sum())
    assert eng.full_count.cpu().tolist()[0] == n_gated
    eng.close()
