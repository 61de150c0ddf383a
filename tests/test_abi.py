"""liboda builds, loads and exports every entry point include/oda.h declares; host-side
argument checks return their codes without touching a GPU (no compute call is made)."""
import ctypes
import os
import re

import pytest

from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "oda.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return oda.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(oda_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "oda_decode_full" in names and len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(oda.exported_symbols()) == names


def test_status_strings_and_version(lib):
    for code, name in [(0, "ODA_OK"), (-1, "ODA_ERR_INVALID_ARG"), (-2, "ODA_ERR_UNSUPPORTED_SHAPE"),
                       (-3, "ODA_ERR_WORKSPACE_TOO_SMALL"), (-4, "ODA_ERR_CUDA"),
                       (-5, "ODA_ERR_NOT_IMPLEMENTED"), (1, "ODA_DEV_BAD_BLOCK"),
                       (2, "ODA_DEV_BAD_LEN"), (3, "ODA_DEV_BAD_KEEP_LIST"), (4, "ODA_DEV_TIMEOUT"),
                       (5, "ODA_DEV_BAD_DA")]:
        assert oda.oda_status_string(code) == name
    assert oda.oda_status_string(99) == "ODA_UNKNOWN_STATUS"
    assert oda.oda_version() == 101


def _kv(**kw):
    base = dict(k_cache=0x10000, v_cache=0x20000, block_table=0x30000, seq_lens=0x40000, batch=2,
                num_kv_heads=8, head_dim=128, block_size=16, max_blocks_per_seq=64, num_blocks=128,
                dev_status=None, stats=None)
    base.update(kw)
    return oda.oda_kv(**base)


def _local(lib, kv, hq=16, sink=4, window=256, scale=0.088, k_new=None, v_new=None, out=0x50000,
           out_dtype=0, ws=0x60000, ws_bytes=1 << 40):
    return lib.oda_decode_local(ctypes.byref(kv), 0x70000, hq, sink, window, scale, k_new, v_new, out,
                                out_dtype, None, ws, ws_bytes, None)


def test_decode_argument_checks(lib):
    I, U = oda.ODA_ERR_INVALID_ARG, oda.ODA_ERR_UNSUPPORTED_SHAPE
    assert lib.oda_decode_local(None, 0x70000, 16, 4, 256, 0.1, None, None, 0x50000, 0, None,
                                0x60000, 1, None) == I
    assert _local(lib, _kv(head_dim=64)) == U
    assert _local(lib, _kv(block_size=32)) == U
    assert _local(lib, _kv(), hq=12) == U                 # 12 query heads over 8 KV heads
    assert _local(lib, _kv(), hq=64) == U                 # group of 8 is not built
    assert _local(lib, _kv(), out_dtype=7) == I
    assert _local(lib, _kv(), scale=0.0) == I
    assert _local(lib, _kv(), scale=float("nan")) == I
    assert _local(lib, _kv(), window=0) == I
    assert _local(lib, _kv(), sink=-1) == I
    assert _local(lib, _kv(), k_new=0x80000) == I         # k_new without v_new
    assert _local(lib, _kv(k_cache=0x10008)) == I         # bulk copies need 16-byte alignment
    assert _local(lib, _kv(), ws=0x60008) == I             # workspace: 16-byte aligned
    assert _local(lib, _kv(), out=0x50002) == I            # fp32 output: 4-byte aligned
    assert _local(lib, _kv(), out=0x50001, out_dtype=1) == I   # bf16 output: 2-byte aligned
    assert _local(lib, _kv(block_table=0x30002)) == I
    assert _local(lib, _kv(dev_status=0x90001)) == I
    assert _local(lib, _kv(stats=0x90004)) == I            # u64 counters: 8-byte aligned
    kv = _kv()
    assert lib.oda_decode_full(ctypes.byref(kv), 0x70000, 16, 0.1, 0x80002, None, None, 0x50000,
                               0, None, 0x60000, 1 << 40, None) == I   # int32 gate: 4-byte
    assert _local(lib, _kv(batch=-1)) == I
    assert _local(lib, _kv(batch=2000)) == U
    assert _local(lib, _kv(batch=0)) == oda.ODA_OK         # nothing to do, nothing launched
    kv = _kv()
    assert lib.oda_decode_blockmask(ctypes.byref(kv), 0x70000, 16, 0.1, None, None, 4, 0x50000, 0,
                                    None, 0x60000, 1, None) == I
    assert lib.oda_decode_blockmask(ctypes.byref(kv), 0x70000, 16, 0.1, 0x1000, 0x2000, 65, 0x50000,
                                    0, None, 0x60000, 1, None) == I   # max_keep > pages per seq
    assert lib.oda_kv_append(ctypes.byref(_kv(num_kv_heads=40)), 0x1000, 0x2000, None, None) == U
    assert lib.oda_kv_append(ctypes.byref(_kv()), None, 0x2000, None, None) == I
    assert lib.oda_kv_append(ctypes.byref(_kv()), 0x1000, 0x2008, None, None) == I   # 16 bytes
    assert lib.oda_kv_append(ctypes.byref(_kv()), 0x1000, 0x2000, 0x3002, None) == I  # gate
    assert lib.oda_visible_mask(ctypes.byref(_kv()), 9, 4, 256, None, None, None, 0, 0x1000, 10,
                                None) == I


def test_workspace_queries(lib):
    n = ctypes.c_size_t(0)
    I = oda.ODA_ERR_INVALID_ARG
    assert lib.oda_decode_workspace_size(1, 0, 16, ctypes.byref(n)) == I
    assert lib.oda_decode_workspace_size(1, 8, 12, ctypes.byref(n)) == oda.ODA_ERR_UNSUPPORTED_SHAPE
    assert lib.oda_recall_workspace_size(1, 2048, 100, ctypes.byref(n)) == I
    sizes = []
    for b in (1, 8, 16):
        assert lib.oda_recall_workspace_size(b, 2048, 256, ctypes.byref(n)) == oda.ODA_OK
        sizes.append(n.value)
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    assert lib.oda_recall_score(0x100, 0x200, 0x300, 0, 1, 2048, 96, 0x400, 0x500, 0x600, 0.0,
                                0.0, 0x700, 0x800, None, 0, 0x900, 1 << 30, None) == I
    assert lib.oda_recall_score(0x100, 0x200, 0x300, 0, 1, 2048, 256, 0x400, 0x500, 0x600, 0.0,
                                0.0, 0x700, 0x800, None, 0, 0x900, 16,
                                None) == oda.ODA_ERR_WORKSPACE_TOO_SMALL
    # misaligned pointers are refused before any launch: fp32 input, workspace, counters
    assert lib.oda_recall_score(0x102, 0x200, 0x300, 0, 1, 2048, 256, 0x400, 0x500, 0x600, 0.0,
                                0.0, 0x700, 0x800, None, 0, 0x900, 1 << 30, None) == I
    assert lib.oda_recall_score(0x100, 0x200, 0x300, 0, 1, 2048, 256, 0x400, 0x500, 0x600, 0.0,
                                0.0, 0x700, 0x800, None, 0, 0x908, 1 << 30, None) == I
    assert lib.oda_recall_score(0x100, 0x200, 0x300, 0, 1, 2048, 256, 0x400, 0x500, 0x600, 0.0,
                                0.0, 0x700, 0x800, 0xa04, 0, 0x900, 1 << 30, None) == I


def test_step_graph_argument_checks(lib):
    h = ctypes.c_void_p(0)
    assert lib.oda_step_graph_create(None, None, ctypes.byref(h)) == oda.ODA_ERR_INVALID_ARG
    d = oda.oda_step_desc(num_layers=0)
    assert lib.oda_step_graph_create(ctypes.byref(d), None, ctypes.byref(h)) == oda.ODA_ERR_INVALID_ARG
    assert lib.oda_step_graph_launch(None, None) == oda.ODA_ERR_INVALID_ARG
    assert lib.oda_step_graph_set_events(None, None, None, None, None) == oda.ODA_ERR_INVALID_ARG
    lib.oda_step_graph_destroy(None)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(oda, "_lib", None)
    monkeypatch.setattr(oda, "_LIB_PATH", str(tmp_path / "liboda.so"))
    with pytest.raises(RuntimeError, match="liboda.so not found"):
        oda.load()


def _decode(lib, vis, kv=None, k_new=None, v_new=None):
    kv = kv or _kv()
    return lib.oda_decode(ctypes.byref(kv), ctypes.byref(vis) if vis is not None else None,
                          0x70000, 16, 0.088, k_new, v_new, 0x50000, 0, None, 0x60000, 1 << 40,
                          None)


def test_visibility_argument_checks(lib):
    I, OK = oda.ODA_ERR_INVALID_ARG, oda.ODA_OK
    V = oda.oda_visibility
    assert _decode(lib, None) == I
    assert _decode(lib, V(mode=9, window=1)) == I
    assert _decode(lib, V(mode=oda.ODA_MODE_LOCAL, sink=4, window=0)) == I
    assert _decode(lib, V(mode=oda.ODA_MODE_DA, window=1, da_focus_len=16, da_recent=16,
                          da_local_len=16)) == I                       # no mode array
    assert _decode(lib, V(mode=oda.ODA_MODE_DA, window=1, da_modes=0x1000, da_focus_offsets=0x2000,
                          da_focus_len=0, da_recent=16, da_local_len=16)) == I
    assert _decode(lib, V(mode=oda.ODA_MODE_DA, window=1, da_modes=0x1000, da_focus_offsets=0x2000,
                          da_focus_len=16, da_recent=16, da_local_len=16),
                   k_new=0x80000, v_new=0x90000) == I              # DA need not hold slot t
    for lo, hi in [(-16, 32), (8, 32), (0, 24), (32, 32), (48, 32)]:
        assert _decode(lib, V(mode=oda.ODA_MODE_SHARD, window=1, pos_lo=lo, pos_hi=hi)) == I
    assert _decode(lib, V(mode=oda.ODA_MODE_SHARD, window=1, pos_lo=0, pos_hi=32),
                   kv=_kv(batch=0)) == OK                          # nothing to do
    assert lib.oda_visible_mask_ex(ctypes.byref(_kv()), None, 0x1000, 10, None) == I


def test_merge_and_schedule_argument_checks(lib):
    I, OK = oda.ODA_ERR_INVALID_ARG, oda.ODA_OK
    assert lib.oda_merge_partials(0x1000, 0x2000, 0, 1, 16, None, 0x3000, 0, None, None) == I
    assert lib.oda_merge_partials(0x1000, 0x2000, 65, 1, 16, None, 0x3000, 0, None, None) == I
    assert lib.oda_merge_partials(0x1000, 0x2000, 2, 1, 16, None, 0x3000, 5, None, None) == I
    assert lib.oda_merge_partials(None, 0x2000, 2, 1, 16, None, 0x3000, 0, None, None) == I
    assert lib.oda_merge_partials(0x1000, 0x2000, 2, 0, 16, None, 0x3000, 0, None, None) == OK
    assert lib.oda_gate_schedule(0x1000, 4, 1.5, 0x2000, None, 0, None) == I
    assert lib.oda_gate_schedule(0x1000, 4, float("nan"), 0x2000, None, 0, None) == I
    assert lib.oda_gate_schedule(None, 4, 0.5, 0x2000, None, 0, None) == I
    assert lib.oda_gate_schedule(0x1000, 0, 0.5, 0x2000, None, 0, None) == OK
    assert lib.oda_gate_schedule(0x1002, 4, 0.5, 0x2000, None, 0, None) == I
    assert lib.oda_gate_schedule(0x1000, 4, 0.5, 0x2000, 0x3004, 0, None) == I
    assert lib.oda_merge_partials(0x1002, 0x2000, 2, 1, 16, None, 0x3000, 0, None, None) == I
    assert lib.oda_merge_partials(0x1000, 0x2000, 2, 1, 16, None, 0x3001, 1, None, None) == I


def test_recall_training_argument_checks(lib):
    I = oda.ODA_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert lib.oda_recall_train_workspace_size(1025, 2048, 256, ctypes.byref(n)) == I
    assert lib.oda_recall_train_workspace_size(8, 2048, 100, ctypes.byref(n)) == I
    assert lib.oda_recall_train_workspace_size(8, 2048, 256, ctypes.byref(n)) == oda.ODA_OK
    need = n.value
    assert need > 0

    def call(batch=8, mlp=256, delta=1.0, gain=0xa00, ws_bytes=None, ws=0x1000, dw1=0xc00):
        return lib.oda_recall_loss_grad(0x100, 0x200, 0x300, 0, batch, 2048, mlp, 0x400, 0x500,
                                        0x600, 0.0, gain, 0.0, delta, None, 0xb00, dw1, 0xd00,
                                        0xe00, 0xf00, ws, need if ws_bytes is None else ws_bytes,
                                        None)
    assert call(delta=0.0) == I
    assert call(delta=float("inf")) == I
    assert call(gain=None) == I
    assert call(mlp=96) == I
    assert call(batch=2000) == I
    assert call(ws_bytes=16) == oda.ODA_ERR_WORKSPACE_TOO_SMALL
    assert call(ws=0x1008) == I                               # workspace: 16-byte aligned
    assert call(dw1=0xc02) == I                               # fp32 output: 4-byte aligned
    assert call(batch=0) == oda.ODA_OK


def test_step_desc_checks_before_any_cuda_call(lib):
    """Per-layer access range, gate source, rho, the step-kernel mode and the timing-event
    mode are validated on the host."""
    I = oda.ODA_ERR_INVALID_ARG
    L = 2
    kvs = (oda.oda_kv * L)(_kv(), _kv())
    P = ctypes.c_void_p
    arr = lambda: (P * L)(0x1000, 0x2000)
    keep = []

    def desc(**kw):
        a = [arr() for _ in range(7)]
        keep.extend(a)
        base = dict(num_layers=L, layers=ctypes.cast(kvs, ctypes.POINTER(oda.oda_kv)),
                    num_q_heads=16, sink=4, window=256, scale=0.088,
                    q_local=ctypes.cast(a[0], ctypes.POINTER(P)),
                    k_local=ctypes.cast(a[1], ctypes.POINTER(P)),
                    v_local=ctypes.cast(a[2], ctypes.POINTER(P)),
                    q_full=ctypes.cast(a[3], ctypes.POINTER(P)),
                    k_full=ctypes.cast(a[4], ctypes.POINTER(P)),
                    v_full=ctypes.cast(a[5], ctypes.POINTER(P)),
                    out=ctypes.cast(a[6], ctypes.POINTER(P)), mlp=256)
        base.update(kw)
        return oda.oda_step_desc(**base)

    h = ctypes.c_void_p(0)
    ints = lambda *v: ctypes.cast((ctypes.c_int32 * L)(*v), ctypes.POINTER(ctypes.c_int32))
    for d in [desc(sinks=ints(4, -1)), desc(windows=ints(0, 256)), desc(window=0),
              desc(gate_source=7), desc(gate_source=oda.ODA_GATE_RANDOM, gate_u=None, rho=0.5),
              desc(gate_source=oda.ODA_GATE_RANDOM, gate_u=0x3000, rho=1.5),
              desc(step_kernels=3), desc(timing_events=3), desc(timing_events=-1)]:
        assert lib.oda_step_graph_create(ctypes.byref(d), None, ctypes.byref(h)) == I
        assert not h.value
