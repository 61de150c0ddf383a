"""ctypes binding of liboda (include/oda.h). Argument marshalling only: every step of the
decode path runs in the library's CUDA kernels. Tensors are torch CUDA tensors; their
device pointers, sizes and the current CUDA stream are passed through unchanged.

There is no fallback: if liboda.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "liboda.so")

ODA_OK = 0
ODA_ERR_INVALID_ARG = -1
ODA_ERR_UNSUPPORTED_SHAPE = -2
ODA_ERR_WORKSPACE_TOO_SMALL = -3
ODA_ERR_CUDA = -4
ODA_ERR_NOT_IMPLEMENTED = -5
ODA_DEV_BAD_BLOCK = 1
ODA_DEV_BAD_LEN = 2
ODA_DEV_BAD_KEEP_LIST = 3
ODA_DEV_TIMEOUT = 4
ODA_DEV_BAD_DA = 5
ODA_F32 = 0
ODA_BF16 = 1
ODA_MODE_LOCAL = 0
ODA_MODE_FULL = 1
ODA_MODE_KEEP = 2
ODA_MODE_DA = 3
ODA_MODE_SHARD = 4
ODA_DA_GLOBAL = 0
ODA_DA_FOCUS = 1
ODA_DA_LOCAL = 2
ODA_STAT_ROWS = 0
ODA_STAT_PAGES = 1
ODA_STATS_LEN = 2
ODA_PHASE_LOCAL = 1
ODA_PHASE_RECALL = 2
ODA_PHASE_FULL = 4
ODA_GATE_RECALL = 0
ODA_GATE_RANDOM = 1
ODA_STEP_FULL_PERSISTENT = 0
ODA_STEP_PER_LAYER = 1
ODA_STEP_PERSISTENT = 2
ODA_STALL_NONE = 0
ODA_STALL_DECODE_RING = 1
ODA_STALL_LOCAL_CHAIN = 2
ODA_STALL_FULL_CHAIN = 3
ODA_STALL_LOCAL_PUSH = 4


class OdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = "%s failed: %s (%d)" % (where, oda_status_string(code), code)
        if code == ODA_ERR_CUDA:
            msg += ": " + load().oda_last_cuda_error().decode()
        super().__init__(msg)


class oda_kv(ctypes.Structure):
    _fields_ = [
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
        ("dev_status", ctypes.c_void_p), ("stats", ctypes.c_void_p),
    ]


class oda_visibility(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32),
        ("gate", ctypes.c_void_p), ("keep_blocks", ctypes.c_void_p),
        ("keep_counts", ctypes.c_void_p), ("max_keep", ctypes.c_int32),
        ("da_modes", ctypes.c_void_p), ("da_focus_offsets", ctypes.c_void_p),
        ("da_focus_len", ctypes.c_int32), ("da_recent", ctypes.c_int32),
        ("da_local_len", ctypes.c_int32), ("pos_lo", ctypes.c_int32), ("pos_hi", ctypes.c_int32),
    ]


class oda_step_desc(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32), ("layers", ctypes.POINTER(oda_kv)),
        ("num_q_heads", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("q_local", ctypes.POINTER(ctypes.c_void_p)), ("k_local", ctypes.POINTER(ctypes.c_void_p)),
        ("v_local", ctypes.POINTER(ctypes.c_void_p)), ("q_full", ctypes.POINTER(ctypes.c_void_p)),
        ("k_full", ctypes.POINTER(ctypes.c_void_p)), ("v_full", ctypes.POINTER(ctypes.c_void_p)),
        ("out", ctypes.POINTER(ctypes.c_void_p)), ("lse", ctypes.POINTER(ctypes.c_void_p)),
        ("local_layers", ctypes.POINTER(ctypes.c_int32)), ("sinks", ctypes.POINTER(ctypes.c_int32)),
        ("windows", ctypes.POINTER(ctypes.c_int32)),
        ("h_prev", ctypes.c_void_p), ("emb", ctypes.c_void_p),
        ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p),
        ("b2", ctypes.c_float), ("theta", ctypes.c_float), ("mlp", ctypes.c_int32),
        ("q_out", ctypes.c_void_p), ("gate_out", ctypes.c_void_p), ("full_count", ctypes.c_void_p),
        ("decode_ws", ctypes.c_void_p), ("decode_ws_bytes", ctypes.c_size_t),
        ("recall_ws", ctypes.c_void_p), ("recall_ws_bytes", ctypes.c_size_t),
        ("use_conditional", ctypes.c_int32), ("timing_events", ctypes.c_int32),
        ("phases", ctypes.c_int32), ("gate_source", ctypes.c_int32),
        ("gate_u", ctypes.c_void_p), ("rho", ctypes.c_float),
        ("step_kernels", ctypes.c_int32),
    ]


_lib = None
_KV = ctypes.POINTER(oda_kv)
_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_VIS = ctypes.POINTER(oda_visibility)

_SIGNATURES = {
    "oda_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "oda_version": (ctypes.c_int, []),
    "oda_last_cuda_error": (ctypes.c_char_p, []),
    "oda_decode_workspace_size": (ctypes.c_int, [_I, _I, _I, ctypes.POINTER(_SZ)]),
    "oda_recall_workspace_size": (ctypes.c_int, [_I, _I, _I, ctypes.POINTER(_SZ)]),
    "oda_kv_append": (ctypes.c_int, [_KV, _P, _P, _P, _P]),
    "oda_decode_local": (ctypes.c_int, [_KV, _P, _I, _I, _I, _F, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "oda_decode_full": (ctypes.c_int, [_KV, _P, _I, _F, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "oda_decode_blockmask": (ctypes.c_int, [_KV, _P, _I, _F, _P, _P, _I, _P, _I, _P, _P, _SZ, _P]),
    "oda_decode_full_noalloc": (ctypes.c_int, [_KV, _P, _I, _F, _P, _P, _P, _P, _I, _P, _P]),
    "oda_visible_mask": (ctypes.c_int, [_KV, _I, _I, _I, _P, _P, _P, _I, _P, _I, _P]),
    "oda_decode": (ctypes.c_int, [_KV, _VIS, _P, _I, _F, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "oda_visible_mask_ex": (ctypes.c_int, [_KV, _VIS, _P, _I, _P]),
    "oda_merge_partials": (ctypes.c_int, [_P, _P, _I, _I, _I, _P, _P, _I, _P, _P]),
    "oda_gate_schedule": (ctypes.c_int, [_P, _I, _F, _P, _P, ctypes.c_ulonglong, _P]),
    "oda_recall_train_workspace_size": (ctypes.c_int, [_I, _I, _I, ctypes.POINTER(_SZ)]),
    "oda_recall_loss_grad": (ctypes.c_int, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _F, _P, _F,
                                            _F, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "oda_recall_score": (ctypes.c_int, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _F, _F, _P, _P, _P,
                                        ctypes.c_ulonglong, _P, _SZ, _P]),
    "oda_step_graph_create": (ctypes.c_int, [ctypes.POINTER(oda_step_desc), _P,
                                             ctypes.POINTER(ctypes.c_void_p)]),
    "oda_step_graph_launch": (ctypes.c_int, [_P, _P]),
    "oda_step_graph_set_events": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "oda_step_graph_destroy": (None, [_P]),
    "oda_step_graph_kernels": (ctypes.c_int, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I),
                                              ctypes.POINTER(_I)]),
    "oda_step_kernel_limits": (ctypes.c_int, [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "oda_debug_set_wait_limit": (ctypes.c_int, [ctypes.c_ulonglong]),
    "oda_debug_set_stall": (ctypes.c_int, [ctypes.c_int]),
    "oda_debug_set_local_shape": (ctypes.c_int, [ctypes.c_int]),
}


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load liboda.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("liboda.so not found at %s; build it with "
                               "`python -m sparse_kv_recall_b200.build`" % _LIB_PATH)
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_symbols() -> list:
    return list(_SIGNATURES)


def _check(rc: int, where: str):
    if rc != ODA_OK:
        raise OdaError(rc, where)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _out_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return ODA_F32
    if t.dtype == torch.bfloat16:
        return ODA_BF16
    raise ValueError("out must be float32 or bfloat16")


def oda_status_string(code: int) -> str:
    return load().oda_status_string(int(code)).decode()


def oda_version() -> int:
    return load().oda_version()


def make_kv(k_cache, v_cache, block_table, seq_lens, dev_status=None, stats=None) -> oda_kv:
    """oda_kv for bf16 caches [num_blocks][Hkv][16][128], int32 block_table [B][maxb] and
    int32 seq_lens [B] (tokens including the current one)."""
    nb, hkv, bs, d = k_cache.shape
    kv = oda_kv(
        k_cache=_ptr(k_cache, torch.bfloat16, "k_cache"),
        v_cache=_ptr(v_cache, torch.bfloat16, "v_cache"),
        block_table=_ptr(block_table, torch.int32, "block_table"),
        seq_lens=_ptr(seq_lens, torch.int32, "seq_lens"),
        batch=block_table.shape[0], num_kv_heads=hkv, head_dim=d, block_size=bs,
        max_blocks_per_seq=block_table.shape[1], num_blocks=nb,
        dev_status=_ptr(dev_status, torch.int32, "dev_status"),
        stats=_ptr(stats, torch.int64, "stats"))
    kv._refs = (k_cache, v_cache, block_table, seq_lens, dev_status, stats)
    return kv


def oda_decode_workspace_size(batch: int, num_kv_heads: int, num_q_heads: int) -> int:
    n = _SZ(0)
    _check(load().oda_decode_workspace_size(batch, num_kv_heads, num_q_heads, ctypes.byref(n)),
           "oda_decode_workspace_size")
    return n.value


def oda_recall_workspace_size(batch: int, hidden: int, mlp: int) -> int:
    n = _SZ(0)
    _check(load().oda_recall_workspace_size(batch, hidden, mlp, ctypes.byref(n)),
           "oda_recall_workspace_size")
    return n.value


def oda_kv_append(kv: oda_kv, k_new, v_new, gate=None, stream=None):
    _check(load().oda_kv_append(ctypes.byref(kv), _ptr(k_new, torch.bfloat16, "k_new"),
                                _ptr(v_new, torch.bfloat16, "v_new"),
                                _ptr(gate, torch.int32, "gate"), _stream(stream)), "oda_kv_append")


def oda_decode_local(kv: oda_kv, q, sink: int, window: int, scale: float, out, ws,
                     k_new=None, v_new=None, lse=None, stream=None):
    _check(load().oda_decode_local(
        ctypes.byref(kv), _ptr(q, torch.bfloat16, "q"), q.shape[1], sink, window, scale,
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(out, None, "out"), _out_dtype(out), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)), "oda_decode_local")


def oda_decode_full(kv: oda_kv, q, scale: float, out, ws, gate=None, k_new=None, v_new=None,
                    lse=None, stream=None):
    _check(load().oda_decode_full(
        ctypes.byref(kv), _ptr(q, torch.bfloat16, "q"), q.shape[1], scale,
        _ptr(gate, torch.int32, "gate"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _ptr(out, None, "out"), _out_dtype(out),
        _ptr(lse, torch.float32, "lse"), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "oda_decode_full")


def oda_decode_full_noalloc(kv: oda_kv, q, scale: float, out, gate=None, k_new=None, v_new=None,
                            lse=None, stream=None):
    """oda_decode_full for callers that cannot allocate: no workspace argument; the library's
    own per-device scratch array is used (calls that overlap on the GPU race on it)."""
    _check(load().oda_decode_full_noalloc(
        ctypes.byref(kv), _ptr(q, torch.bfloat16, "q"), q.shape[1], scale,
        _ptr(gate, torch.int32, "gate"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _ptr(out, None, "out"), _out_dtype(out),
        _ptr(lse, torch.float32, "lse"), _stream(stream)), "oda_decode_full_noalloc")


def oda_decode_blockmask(kv: oda_kv, q, scale: float, keep_blocks, keep_counts, out, ws,
                         lse=None, stream=None):
    _check(load().oda_decode_blockmask(
        ctypes.byref(kv), _ptr(q, torch.bfloat16, "q"), q.shape[1], scale,
        _ptr(keep_blocks, torch.int32, "keep_blocks"), _ptr(keep_counts, torch.int32, "keep_counts"),
        keep_blocks.shape[1], _ptr(out, None, "out"), _out_dtype(out),
        _ptr(lse, torch.float32, "lse"), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "oda_decode_blockmask")


def oda_visible_mask(kv: oda_kv, mode: int, mask, sink: int = 0, window: int = 1, gate=None,
                     keep_blocks=None, keep_counts=None, stream=None):
    max_keep = keep_blocks.shape[1] if keep_blocks is not None else 0
    _check(load().oda_visible_mask(
        ctypes.byref(kv), mode, sink, window, _ptr(gate, torch.int32, "gate"),
        _ptr(keep_blocks, torch.int32, "keep_blocks"), _ptr(keep_counts, torch.int32, "keep_counts"),
        max_keep, _ptr(mask, torch.uint8, "mask"), mask.shape[1], _stream(stream)),
        "oda_visible_mask")


def da_visibility(modes, focus_offsets, focus_len: int = 32768, recent: int = 2048,
                  local_len: int = 4096) -> oda_visibility:
    """Declarative-Attention rule: one declared mode per sequence (int32 [B], ODA_DA_*) and
    the focused region's first position (int32 [B]), compiled into page runs on the device."""
    v = oda_visibility(mode=ODA_MODE_DA, window=1,
                       da_modes=_ptr(modes, torch.int32, "modes"),
                       da_focus_offsets=_ptr(focus_offsets, torch.int32, "focus_offsets"),
                       da_focus_len=focus_len, da_recent=recent, da_local_len=local_len)
    v._refs = (modes, focus_offsets)      # the rule holds device pointers: keep them alive
    return v


def shard_visibility(pos_lo: int, pos_hi: int, gate=None) -> oda_visibility:
    """Positions [pos_lo, pos_hi) of 0..t (page-aligned): one GPU's part of a Full pass."""
    v = oda_visibility(mode=ODA_MODE_SHARD, window=1, gate=_ptr(gate, torch.int32, "gate"),
                       pos_lo=int(pos_lo), pos_hi=int(pos_hi))
    v._refs = (gate,)
    return v


def oda_decode(kv: oda_kv, vis: oda_visibility, q, scale: float, out, ws, k_new=None,
               v_new=None, lse=None, stream=None):
    """Decode attention under any visibility rule (oda_visibility)."""
    _check(load().oda_decode(
        ctypes.byref(kv), ctypes.byref(vis), _ptr(q, torch.bfloat16, "q"), q.shape[1], scale,
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(out, None, "out"), _out_dtype(out), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)), "oda_decode")


def oda_visible_mask_ex(kv: oda_kv, vis: oda_visibility, mask, stream=None):
    _check(load().oda_visible_mask_ex(ctypes.byref(kv), ctypes.byref(vis),
                                      _ptr(mask, torch.uint8, "mask"), mask.shape[1],
                                      _stream(stream)), "oda_visible_mask_ex")


def oda_merge_partials(o_parts, lse_parts, out, gate=None, lse=None, stream=None):
    """o_parts fp32 [R][B][Hq][128], lse_parts fp32 [R][B][Hq] -> out [B][Hq][128]."""
    R, B, Hq, _ = o_parts.shape
    _check(load().oda_merge_partials(
        _ptr(o_parts, torch.float32, "o_parts"), _ptr(lse_parts, torch.float32, "lse_parts"),
        R, B, Hq, _ptr(gate, torch.int32, "gate"), _ptr(out, None, "out"), _out_dtype(out),
        _ptr(lse, torch.float32, "lse"), _stream(stream)), "oda_merge_partials")


def oda_gate_schedule(u, rho: float, gate_out, full_count=None, graph_cond_handle: int = 0,
                      stream=None):
    _check(load().oda_gate_schedule(
        _ptr(u, torch.float32, "u"), u.shape[0], float(rho), _ptr(gate_out, torch.int32, "gate_out"),
        _ptr(full_count, torch.int64, "full_count"), int(graph_cond_handle), _stream(stream)),
        "oda_gate_schedule")


def oda_recall_score(h_prev, emb, h_local, w1, b1, w2, b2: float, theta: float, q_out, gate_out,
                     ws, full_count=None, graph_cond_handle: int = 0, stream=None):
    batch, hidden = h_prev.shape
    _check(load().oda_recall_score(
        _ptr(h_prev, torch.float32, "h_prev"), _ptr(emb, torch.float32, "emb"),
        _ptr(h_local, None, "h_local"), _out_dtype(h_local), batch, hidden, w1.shape[1],
        _ptr(w1, torch.float32, "w1"), _ptr(b1, torch.float32, "b1"), _ptr(w2, torch.float32, "w2"),
        float(b2), float(theta), _ptr(q_out, torch.float32, "q_out"),
        _ptr(gate_out, torch.int32, "gate_out"), _ptr(full_count, torch.int64, "full_count"),
        int(graph_cond_handle), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "oda_recall_score")


def _ptr_array(tensors: Sequence, dtype, name):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = _ptr(t, dtype, name)
    return arr


class StepGraph:
    """One ODA decode step captured as a CUDA graph by oda_step_graph_create. Holds the
    ctypes arrays the description points at for as long as the graph lives."""

    def __init__(self, kvs: Sequence[oda_kv], num_q_heads: int, sink: int, window: int,
                 scale: float, q_local, k_local, v_local, q_full, k_full, v_full, out,
                 h_prev, emb, w1, b1, w2, b2: float, theta: float, q_out, gate_out,
                 decode_ws, recall_ws, full_count=None, lse=None, local_layers=None,
                 sinks=None, windows=None, use_conditional: bool = True,
                 timing_events: int = 0, phases: int = 0, gate_u=None, rho: float = 0.0,
                 step_kernels: int = ODA_STEP_FULL_PERSISTENT):
        L = len(kvs)
        self._keep = []
        layers = (oda_kv * L)(*kvs)
        bf = torch.bfloat16
        arrs = [_ptr_array(x, bf, n) for x, n in ((q_local, "q_local"), (k_local, "k_local"),
                                                   (v_local, "v_local"), (q_full, "q_full"),
                                                   (k_full, "k_full"), (v_full, "v_full"))]
        outs = _ptr_array(out, torch.float32, "out")
        lses = _ptr_array(lse, torch.float32, "lse") if lse is not None else None
        def ints(xs, name):
            if xs is None:
                return None
            if len(xs) != L:
                raise ValueError("%s: %d entries for %d layers" % (name, len(xs), L))
            return (ctypes.c_int32 * L)(*[int(x) for x in xs])

        ll, sk, wn = ints(local_layers, "local_layers"), ints(sinks, "sinks"), ints(windows, "windows")
        self._keep += [layers, outs, lses, ll, sk, wn] + arrs
        ip = ctypes.POINTER(ctypes.c_int32)
        icast = lambda a: ctypes.cast(a, ip) if a is not None else None
        vp = ctypes.POINTER(ctypes.c_void_p)
        d = oda_step_desc(
            num_layers=L, layers=ctypes.cast(layers, ctypes.POINTER(oda_kv)),
            num_q_heads=num_q_heads, sink=sink, window=window, scale=scale,
            q_local=ctypes.cast(arrs[0], vp), k_local=ctypes.cast(arrs[1], vp),
            v_local=ctypes.cast(arrs[2], vp), q_full=ctypes.cast(arrs[3], vp),
            k_full=ctypes.cast(arrs[4], vp), v_full=ctypes.cast(arrs[5], vp),
            out=ctypes.cast(outs, vp), lse=ctypes.cast(lses, vp) if lses is not None else None,
            local_layers=icast(ll), sinks=icast(sk), windows=icast(wn),
            h_prev=_ptr(h_prev, torch.float32, "h_prev"), emb=_ptr(emb, torch.float32, "emb"),
            w1=_ptr(w1, torch.float32, "w1"), b1=_ptr(b1, torch.float32, "b1"),
            w2=_ptr(w2, torch.float32, "w2"), b2=float(b2), theta=float(theta), mlp=w1.shape[1],
            q_out=_ptr(q_out, torch.float32, "q_out"), gate_out=_ptr(gate_out, torch.int32, "gate_out"),
            full_count=_ptr(full_count, torch.int64, "full_count"),
            decode_ws=_ptr(decode_ws, None, "decode_ws"),
            decode_ws_bytes=decode_ws.numel() * decode_ws.element_size(),
            recall_ws=_ptr(recall_ws, None, "recall_ws"),
            recall_ws_bytes=recall_ws.numel() * recall_ws.element_size(),
            use_conditional=int(bool(use_conditional)), timing_events=int(timing_events),
            phases=int(phases),
            gate_source=ODA_GATE_RANDOM if gate_u is not None else ODA_GATE_RECALL,
            gate_u=_ptr(gate_u, torch.float32, "gate_u"), rho=float(rho),
            step_kernels=int(step_kernels))
        self._desc = d
        h = ctypes.c_void_p(0)
        _check(load().oda_step_graph_create(ctypes.byref(d), None, ctypes.byref(h)),
               "oda_step_graph_create")
        self._h = h

    def launch(self, stream=None):
        _check(load().oda_step_graph_launch(self._h, _stream(stream)), "oda_step_graph_launch")

    def kernels(self):
        """(Local, gate, Full) kernel launches per step of this graph; the Full count is that
        of a step whose Full phase runs (with an IF node it is skipped otherwise)."""
        a, b, c = _I(0), _I(0), _I(0)
        _check(load().oda_step_graph_kernels(self._h, ctypes.byref(a), ctypes.byref(b),
                                             ctypes.byref(c)), "oda_step_graph_kernels")
        return a.value, b.value, c.value

    def set_events(self, ev_start, ev_local, ev_recall, ev_end):
        _check(load().oda_step_graph_set_events(self._h, ev_start.cuda_event, ev_local.cuda_event,
                                                ev_recall.cuda_event, ev_end.cuda_event),
               "oda_step_graph_set_events")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load().oda_step_graph_destroy(self._h)
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def oda_step_kernel_limits(group: int, batch: int, mlp: int):
    """(max clusters of the persistent Local kernel resident at once, cooperative launches)."""
    n, c = _I(0), _I(0)
    _check(load().oda_step_kernel_limits(int(group), int(batch), int(mlp), ctypes.byref(n),
                                         ctypes.byref(c)), "oda_step_kernel_limits")
    return n.value, c.value


def oda_debug_set_wait_limit(ns: int):
    """Test hook: the limit (ns) of every bounded device wait of later launches; 0 = 1 s."""
    _check(load().oda_debug_set_wait_limit(int(ns)), "oda_debug_set_wait_limit")


def oda_debug_set_local_shape(index: int):
    """Tuning hook: shape of the persistent Local kernel in later step graphs (-1 = automatic)."""
    _check(load().oda_debug_set_local_shape(int(index)), "oda_debug_set_local_shape")


def oda_debug_set_stall(kind: int):
    """Test hook: make one bounded wait of later launches run out (ODA_STALL_*)."""
    _check(load().oda_debug_set_stall(int(kind)), "oda_debug_set_stall")


def oda_recall_train_workspace_size(batch: int, hidden: int, mlp: int) -> int:
    n = _SZ(0)
    _check(load().oda_recall_train_workspace_size(batch, hidden, mlp, ctypes.byref(n)),
           "oda_recall_train_workspace_size")
    return n.value


def oda_recall_loss_grad(h_prev, emb, h_local, w1, b1, w2, b2: float, gain, lam: float, ws,
                         loss, dw1, db1, dw2, db2, delta: float = 1.0, q_out=None, stream=None):
    """Mean Huber loss of the recall head on the signed-log targets of `gain` (fp32 [B]) and
    its gradient; loss / db2 are fp32 [1] device tensors, dw1 / db1 / dw2 shaped like the
    weights."""
    batch, hidden = h_prev.shape
    _check(load().oda_recall_loss_grad(
        _ptr(h_prev, torch.float32, "h_prev"), _ptr(emb, torch.float32, "emb"),
        _ptr(h_local, None, "h_local"), _out_dtype(h_local), batch, hidden, w1.shape[1],
        _ptr(w1, torch.float32, "w1"), _ptr(b1, torch.float32, "b1"), _ptr(w2, torch.float32, "w2"),
        float(b2), _ptr(gain, torch.float32, "gain"), float(lam), float(delta),
        _ptr(q_out, torch.float32, "q_out"), _ptr(loss, torch.float32, "loss"),
        _ptr(dw1, torch.float32, "dw1"), _ptr(db1, torch.float32, "db1"),
        _ptr(dw2, torch.float32, "dw2"), _ptr(db2, torch.float32, "db2"),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
        "oda_recall_loss_grad")
