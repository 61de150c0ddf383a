"""oda_decode_full_noalloc: the Full decode for callers that cannot allocate device memory
(code captured into a CUDA graph under a mode that forbids allocation, plugins whose host
framework owns every allocation). Its split partials and merge tickets live in a device
array inside liboda instead of a caller workspace.

Checked through the C ABI: against the fp64 oracle (gated Full, with and without the commit of
slot t, a 128K sequence among ragged ones, one to four query heads per KV head); against the
workspace entry point on two calls in a row; a batch just under the array's limit and one over
it; a call after one that left the array's tickets non-zero; and that a rejected call queues
no work. This file is collected last so that a stop-at-first-failure run has already run
every other test; it also passes alone in a fresh process."""
import math

import numpy as np
import pytest
import torch

from oda_cases import SCALE, Case, assert_attn_close, assert_lse_close
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda

pytestmark = pytest.mark.gpu

LIMIT = 2 << 20  # bytes of the library's scratch array


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _check_against_oracle(c, out, lse, gate, commit, fill):
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t), commit=commit,
                         seqs=[b for b in range(c.B) if gate[b]])
    got = out.cpu().numpy()
    on = np.array(gate, dtype=bool)
    assert_attn_close(got[on], ref[on], "noalloc")
    assert_lse_close(lse.cpu().numpy()[on], rlse[on])
    assert np.all(got[~on] == fill)                        # gated off: rows untouched


@pytest.mark.parametrize("G", [1, 2, 4])
def test_noalloc_matches_oracle(G):
    c = Case([1, 17, 300, 5000, 131_073], hq=8 * G, hkv=8, seed=120 + G)
    gate = [1, 1, 0, 1, 1]
    g = torch.tensor(gate, dtype=torch.int32, device="cuda")
    out, lse = c.out_buffers(fill=3.0)
    oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, gate=g, lse=lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    _check_against_oracle(c, out, lse, gate, False, 3.0)


def test_noalloc_commits_slot_t_and_matches_oracle():
    c = Case([40, 1000, 70_001], hq=16, hkv=8, seed=125)
    gate = [1, 0, 1]
    g = torch.tensor(gate, dtype=torch.int32, device="cuda")
    out, lse = c.out_buffers(fill=-2.0)
    oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, gate=g, k_new=c.k_new, v_new=c.v_new,
                                lse=lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    _check_against_oracle(c, out, lse, gate, True, -2.0)
    kbits = c.kc.view(torch.int16).cpu().numpy().view(np.uint16)
    vbits = c.vc.view(torch.int16).cpu().numpy().view(np.uint16)
    for b, n in enumerate(c.lengths):                      # committed bits, exactly
        t = n - 1
        want_k = c.knew_bits[b] if gate[b] else c.slot_bits(c.kbits, b, t)
        want_v = c.vnew_bits[b] if gate[b] else c.slot_bits(c.vbits, b, t)
        assert np.array_equal(c.slot_bits(kbits, b, t), want_k)
        assert np.array_equal(c.slot_bits(vbits, b, t), want_v)


def test_noalloc_matches_workspace_entry_point_twice():
    c = Case([1, 17, 300, 5000, 40_000], hq=32, hkv=8, seed=123)
    gate = torch.tensor([1, 1, 0, 1, 1], dtype=torch.int32, device="cuda")
    ref, ref_lse = c.out_buffers(fill=3.0)
    oda.oda_decode_full(c.kv, c.q, SCALE, ref, c.ws, gate=gate, lse=ref_lse)
    torch.cuda.synchronize()
    for _ in range(2):
        out, lse = c.out_buffers(fill=3.0)
        oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, gate=gate, lse=lse)
        torch.cuda.synchronize()
        assert int(c.status.item()) == 0
        assert_attn_close(out.cpu().numpy(), ref.cpu().numpy(), "noalloc")
        assert_lse_close(lse.cpu().numpy(), ref_lse.cpu().numpy())
        assert torch.all(out[2] == 3.0)                       # gated off: untouched


def _largest_batch(hkv, hq):
    lo, hi = 1, 1024
    while lo < hi:                                            # largest batch within the array
        mid = (lo + hi + 1) // 2
        if oda.oda_decode_workspace_size(mid, hkv, hq) <= LIMIT:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_noalloc_batch_at_and_beyond_its_scratch():
    hq, hkv = 32, 8
    bmax = _largest_batch(hkv, hq)
    assert oda.oda_decode_workspace_size(bmax + 1, hkv, hq) > LIMIT
    rng = np.random.default_rng(126)
    lens = [int(x) for x in rng.integers(1, 600, size=bmax)]
    c = Case(lens, hq=hq, hkv=hkv, seed=126)
    out, lse = c.out_buffers()
    oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, lse=lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    sample = sorted(set([0, bmax - 1] + [int(x) for x in rng.integers(0, bmax, size=6)]))
    ref, rlse = c.oracle(lambda b, t: O.full_positions(t), seqs=sample)
    assert_attn_close(out.cpu().numpy()[sample], ref[sample], "noalloc at the limit")
    assert_lse_close(lse.cpu().numpy()[sample], rlse[sample])
    # one sequence more does not fit: refused before anything is queued
    c2 = Case(lens + [10], hq=hq, hkv=hkv, seed=127)
    out2 = torch.zeros(c2.B, hq, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(oda.OdaError, match="WORKSPACE_TOO_SMALL"):
        oda.oda_decode_full_noalloc(c2.kv, c2.q, SCALE, out2)
    torch.cuda.synchronize()
    assert np.all(out2.cpu().numpy() == 0)


def test_noalloc_after_a_call_that_left_tickets_set():
    """A call whose bounded wait ran out (test hook) may leave merge tickets set in the shared
    array; the next call clears them before it launches and must be right again."""
    c = Case([9000, 300, 17], hq=16, hkv=8, seed=128)
    out, lse = c.out_buffers()
    oda.oda_debug_set_wait_limit(1_000_000)
    oda.oda_debug_set_stall(oda.ODA_STALL_DECODE_RING)
    try:
        oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, lse=lse)
        torch.cuda.synchronize()
    finally:
        oda.oda_debug_set_stall(oda.ODA_STALL_NONE)
        oda.oda_debug_set_wait_limit(0)
    assert int(c.status.item()) == oda.ODA_DEV_TIMEOUT
    c.status.zero_()
    for _ in range(2):
        out, lse = c.out_buffers()
        oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, lse=lse)
        torch.cuda.synchronize()
        assert int(c.status.item()) == 0
        _check_against_oracle(c, out, lse, [1, 1, 1], False, None)


def _cudart():
    import ctypes
    for name in ("libcudart.so.12", "/usr/local/cuda/lib64/libcudart.so"):
        try:
            return ctypes.CDLL(name)
        except OSError:
            continue
    pytest.fail("no CUDA runtime library to count graph nodes with")


def test_rejected_noalloc_call_queues_no_work():
    """A call refused by a host check (here a misaligned q, then a batch beyond the array)
    records nothing into a stream being captured: the captured graph has no node. An accepted
    call records its ticket clear and its launch."""
    import ctypes
    rt = _cudart()
    c = Case([100], hq=16, hkv=8, seed=129)
    out = torch.zeros(1, 16, 128, dtype=torch.float32, device="cuda")
    raw = torch.zeros(16 * 128 * 2 + 8, dtype=torch.uint8, device="cuda")
    bad_q = raw[2:2 + 16 * 128 * 2].view(torch.bfloat16).view(1, 16, 128)   # 2-byte aligned
    s = torch.cuda.Stream()
    oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out, stream=s)   # first call: module load
    s.synchronize()
    h = ctypes.c_void_p(s.cuda_stream)

    def captured_nodes(call):
        assert rt.cudaStreamBeginCapture(h, 1) == 0               # thread-local mode
        try:
            call()
        finally:
            graph = ctypes.c_void_p()
            assert rt.cudaStreamEndCapture(h, ctypes.byref(graph)) == 0
        n = ctypes.c_size_t(0)
        assert rt.cudaGraphGetNodes(graph, None, ctypes.byref(n)) == 0
        rt.cudaGraphDestroy(graph)
        return n.value

    def rejected_misaligned():
        with pytest.raises(oda.OdaError, match="INVALID_ARG"):
            oda.oda_decode_full_noalloc(c.kv, bad_q, SCALE, out, stream=s)

    big = Case([10] * (_largest_batch(8, 16) + 1), hq=16, hkv=8, seed=130)
    out_big = torch.zeros(big.B, 16, 128, dtype=torch.float32, device="cuda")

    def rejected_too_big():
        with pytest.raises(oda.OdaError, match="WORKSPACE_TOO_SMALL"):
            oda.oda_decode_full_noalloc(big.kv, big.q, SCALE, out_big, stream=s)

    assert captured_nodes(rejected_misaligned) == 0
    assert captured_nodes(rejected_too_big) == 0
    assert captured_nodes(lambda: oda.oda_decode_full_noalloc(c.kv, c.q, SCALE, out,
                                                              stream=s)) == 2
    assert int(c.status.item()) == 0
