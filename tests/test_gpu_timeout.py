"""Bounded device waits. Every wait in liboda's kernels -- a stage of bulk copies, the count a
persistent kernel's CTAs publish layer by layer -- gives up after a limit, reports
ODA_DEV_TIMEOUT in the status word and lets the kernel return, so the CUDA context stays
usable. The test hooks shorten the limit to 1 ms and make one wait run out without faulting
anything: a stage armed for bytes that no copy delivers (no copy is in flight into it), or a
count that one CTA withholds. Each test checks that the launch returns with the status set,
then that a clean call on re-zeroed workspaces matches the oracle."""
import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import SCALE, Case, assert_attn_close, assert_lse_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda
from sparse_kv_recall_b200.engine import OdaEngine, fill_staging

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


class _Stall:
    def __init__(self, kind):
        self.kind = kind

    def __enter__(self):
        oda.oda_debug_set_wait_limit(LIMIT_NS)
        oda.oda_debug_set_stall(self.kind)

    def __exit__(self, *exc):
        oda.oda_debug_set_stall(oda.ODA_STALL_NONE)
        oda.oda_debug_set_wait_limit(0)


def test_hooks_reject_unknown_kinds():
    with pytest.raises(oda.OdaError, match="INVALID_ARG"):
        oda.oda_debug_set_stall(17)
    with pytest.raises(oda.OdaError, match="INVALID_ARG"):
        oda.oda_debug_set_local_shape(4)
    oda.oda_debug_set_stall(oda.ODA_STALL_NONE)
    oda.oda_debug_set_local_shape(-1)


def test_decode_ring_wait_runs_out_then_recovers():
    c = Case([5000, 300, 17], hq=16, hkv=8, seed=501)
    out, lse = c.out_buffers()
    with _Stall(oda.ODA_STALL_DECODE_RING):
        oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, lse=lse)
        torch.cuda.synchronize()
    assert int(c.status.item()) == oda.ODA_DEV_TIMEOUT
    c.status.zero_()
    c.ws.zero_()
    out, lse = c.out_buffers()
    oda.oda_decode_full(c.kv, c.q, SCALE, out, c.ws, lse=lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t))
    assert_attn_close(out.cpu().numpy(), ref, "full after a timeout")
    assert_lse_close(lse.cpu().numpy(), rlse)


def test_local_cluster_inbox_wait_runs_out_then_recovers():
    """The per-layer Local cluster kernel (batch 1, eight KV heads: eight clusters): rank 1 of
    the first cluster withholds its partial, so rank 0's wait for its inbox runs out (every
    other partial has landed long before the 1 ms limit; the withholding CTA sends nothing),
    the kernel returns with the status set; then a clean call matches the oracle."""
    c = Case([3000], hq=16, hkv=8, seed=503)
    out, lse = c.out_buffers()
    with _Stall(oda.ODA_STALL_LOCAL_PUSH):
        oda.oda_decode_local(c.kv, c.q, 4, 256, SCALE, out, c.ws, lse=lse)
        torch.cuda.synchronize()
    assert int(c.status.item()) == oda.ODA_DEV_TIMEOUT
    c.status.zero_()
    c.ws.zero_()
    out, lse = c.out_buffers()
    oda.oda_decode_local(c.kv, c.q, 4, 256, SCALE, out, c.ws, lse=lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    ref, rlse = c.oracle(lambda b, t: O.local_positions(t, 4, 256))
    assert_attn_close(out.cpu().numpy(), ref, "local after a timeout")
    assert_lse_close(lse.cpu().numpy(), rlse)


def _engine(w, lengths, theta, step_kernels=oda.ODA_STEP_PERSISTENT, **kw):
    lay = oda_synth.make_layout(w, extra_tokens=8, device="cuda", lengths=lengths)
    caches = [oda_synth.make_kv_cache(w, lay, l, device="cuda") for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device="cuda")
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), theta, sink=w.sink,
                    window=w.window, use_conditional=False, step_kernels=step_kernels, **kw)
    h0 = oda_synth.make_h0(w, device="cuda")
    eng.set_h_prev(h0, 0)
    return eng, lay, caches, rw, h0


@pytest.mark.parametrize("kind", ["local_chain", "full_chain"])
def test_persistent_kernel_wait_runs_out_then_recovers(kind):
    """One CTA of the persistent Local (Full) kernel withholds its layer-0 count: every other
    CTA's wait for layer 1 runs out, the abort word stops the rest, both kernels return. The
    same engine's graphs, captured again without the hook, then decode the step as the oracle
    does (theta = -inf: every step recomputes with Full, so both kernels do work)."""
    w = oda_synth.Workload(name="stall", layers=3, batch=1, num_q_heads=16, num_kv_heads=8,
                           prefill=900, steps=1, seed=502, sink=4, window=128)
    theta = -float("inf")
    stall = oda.ODA_STALL_LOCAL_CHAIN if kind == "local_chain" else oda.ODA_STALL_FULL_CHAIN
    with _Stall(stall):
        eng, lay, caches, rw, h0 = _engine(w, [w.prefill], theta)
    assert eng.graphs[0].kernels() == (1, 0, 1)
    snap = [(c[0].clone(), c[1].clone()) for c in caches]
    si = oda_synth.make_step_inputs(w, 0, device="cuda")
    fill_staging(eng.v, si, [w.prefill + 1])
    eng.launch(0)
    torch.cuda.synchronize()                         # returns: no wait is unbounded
    assert int(eng.status.item()) == oda.ODA_DEV_TIMEOUT
    # Clean run of the same step: caches back to their state before it, workspaces re-zeroed,
    # graphs captured again without the hook.
    for (k0, v0), (k, v) in zip(snap, caches):
        k.copy_(k0)
        v.copy_(v0)
    eng.status.zero_()
    eng.decode_ws.zero_()
    eng.recall_ws.zero_()
    eng.full_count.zero_()
    eng.set_h_prev(h0, 0)
    eng.set_theta(theta)
    eng.launch(0)
    torch.cuda.synchronize()
    assert int(eng.status.item()) == 0
    bt = lay.block_table.cpu().numpy()

    def logical(t):
        bits = oda_synth.bf16_bits(t)
        p = np.arange(lay.capacity[0])
        out = np.zeros((1, w.num_kv_heads, lay.capacity[0], 128), np.uint16)
        out[0] = bits[bt[0, p // 16], :, p % 16, :].transpose(1, 0, 2)
        return out

    dec = O.OdaDecoder([logical(k) for k, _ in snap], [logical(v) for _, v in snap],
                       [w.prefill], h0.double().cpu().numpy(),
                       (rw.w1.double().cpu().numpy(), rw.b1.double().cpu().numpy(),
                        rw.w2.double().cpu().numpy(), rw.b2),
                       sink=w.sink, window=w.window, theta=theta)
    inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
           for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
    inp["emb"] = si.emb.double().cpu().numpy()
    ref, _, rq, rg = dec.step(inp)
    outs = np.stack([eng.layer_out(0, l).cpu().numpy() for l in range(w.layers)])
    assert_attn_close(outs, ref, "step after a timeout")
    assert eng.gate.cpu().numpy().astype(bool).tolist() == rg.tolist()
    assert eng.full_count.cpu().tolist() == [1, 1]
    eng.close()
