"""Seeded synthetic inputs for the On-Demand Attention (ODA) and Declarative Attention (DA)
decode workloads.

This module only draws random numbers and lays them out. It holds none of the method's
arithmetic (no attention, no recall head, no gate, no visibility rule), so both the CUDA
path and the CPU oracle can take their inputs from it without sharing any computation.

Shapes and distributions follow the five workloads the decode path is measured on:
bf16 K/V/Q ~ N(0, 1), recall-head weights ~ N(0, 0.02) with zero biases, hidden and
embedding vectors ~ N(0, 1), paged KV cache with 16-token pages handed out through a
seeded random permutation of physical pages (so no sequence is stored contiguously).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

BLOCK_SIZE = 16
HEAD_DIM = 128

# Draw purposes: each stream of random numbers has its own seed offset so that adding a
# draw never shifts another one.
_P_BLOCKTABLE = 1
_P_KCACHE = 2
_P_VCACHE = 3
_P_STEP = 4
_P_RECALL = 5
_P_H0 = 6
_P_EMB = 7
_P_LENGTHS = 8
_P_DAMODE = 9
_P_GATE_U = 10
_P_GAIN = 11


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode workload: the attention stack's shapes, history lengths and step count."""

    name: str
    layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    prefill: int                      # history length n (uniform batches)
    steps: int                        # decode steps
    seed: int
    sink: int = 4
    window: int = 2048
    head_dim: int = HEAD_DIM
    block_size: int = BLOCK_SIZE
    mlp: int = 256                    # recall-head width
    theta: Optional[float] = None     # fixed threshold, or None = calibrate to target_rho
    target_rho: Optional[float] = None
    ragged: Optional[tuple] = None    # (lo, hi): per-sequence n ~ U[lo, hi]
    mode: str = "oda"                 # "oda" (Local + gated Full) or "da" (keep-block lists)
    da_probs: tuple = (0.2, 0.5, 0.3)  # DA modes global / focus / local
    da_focus_len: int = 32768
    da_recent: int = 2048
    da_local_len: int = 4096

    @property
    def hidden(self) -> int:
        """Recall-head hidden size: the last layer's attention output flattened (Hq * d)."""
        return self.num_q_heads * self.head_dim

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


# The five measured workloads (seed = 1234 + index).
WORKLOADS = {
    "pr1-ref-4k": Workload(
        name="pr1-ref-4k", layers=1, batch=1, num_q_heads=16, num_kv_heads=8,
        prefill=4096, steps=64, seed=1234, sink=4, window=256, theta=0.0),
    "qwen3-1.7b-16k-b8": Workload(
        name="qwen3-1.7b-16k-b8", layers=28, batch=8, num_q_heads=16, num_kv_heads=8,
        prefill=16384, steps=256, seed=1235, target_rho=0.416),
    "qwen3-1.7b-128k-b1": Workload(
        name="qwen3-1.7b-128k-b1", layers=28, batch=1, num_q_heads=16, num_kv_heads=8,
        prefill=131072, steps=1024, seed=1236, target_rho=0.125),
    "qwen3-8b-ragged-b16": Workload(
        name="qwen3-8b-ragged-b16", layers=36, batch=16, num_q_heads=32, num_kv_heads=8,
        prefill=65536, steps=128, seed=1237, target_rho=0.47, ragged=(8192, 65536)),
    "da-1m-b2": Workload(
        name="da-1m-b2", layers=1, batch=2, num_q_heads=32, num_kv_heads=8,
        prefill=1048576, steps=256, seed=1238, mode="da"),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller sizes for parity tests)."""
    return dataclasses.replace(w, **changes)


def _gen(seed: int, purpose: int, *extra: int, device="cpu") -> torch.Generator:
    s = seed * 1_000_003 + purpose * 7_919
    for e in extra:
        s = s * 31 + int(e) + 1
    g = torch.Generator(device=device)
    g.manual_seed(s % (2 ** 63))
    return g


def prefill_lengths(w: Workload) -> list:
    """History length n_b per sequence: uniform n, or seeded U[lo, hi] for ragged batches."""
    if w.ragged is None:
        return [w.prefill] * w.batch
    lo, hi = w.ragged
    g = _gen(w.seed, _P_LENGTHS)
    return [int(x) for x in torch.randint(lo, hi + 1, (w.batch,), generator=g)]


@dataclasses.dataclass
class PagedLayout:
    """Page assignment shared by all layers: block_table[b][j] = physical page of logical
    page j of sequence b (-1 where unused)."""

    block_table: torch.Tensor   # int32 [batch][max_blocks_per_seq]
    num_blocks: int
    capacity: list               # tokens each sequence can hold


def make_layout(w: Workload, extra_tokens: int, device="cpu", lengths=None,
                spare_pages: int = 0) -> PagedLayout:
    """Hand out physical pages for n_b + extra_tokens tokens per sequence (n_b from the
    workload, or the explicit `lengths`), in a seeded random order over the whole pool;
    `spare_pages` extra pages stay unassigned."""
    lens = list(lengths) if lengths is not None else prefill_lengths(w)
    caps = [n + extra_tokens for n in lens]
    per_seq = [math.ceil(c / w.block_size) for c in caps]
    total = sum(per_seq) + spare_pages
    maxb = max(per_seq)
    perm = torch.randperm(total, generator=_gen(w.seed, _P_BLOCKTABLE)).to(torch.int32)
    bt = torch.full((w.batch, maxb), -1, dtype=torch.int32)
    off = 0
    for b, nb in enumerate(per_seq):
        bt[b, :nb] = perm[off:off + nb]
        off += nb
    return PagedLayout(block_table=bt.to(device), num_blocks=total, capacity=caps)


def make_kv_cache(w: Workload, layout: PagedLayout, layer: int, device="cpu"):
    """K and V page pools of one layer, bf16 [num_blocks][Hkv][16][d], every element N(0, 1).
    Slots past a sequence's history hold noise until the decode steps overwrite them."""
    shape = (layout.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    out = []
    for purpose in (_P_KCACHE, _P_VCACHE):
        g = _gen(w.seed, purpose, layer, device=device)
        if torch.device(device).type == "cuda":
            t = torch.randn(shape, generator=g, device=device, dtype=torch.bfloat16)
        else:
            t = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
        out.append(t)
    return out[0], out[1]


@dataclasses.dataclass
class StepInputs:
    """Per-layer inputs of one decode step. q_* bf16 [B][Hq][d]; k_*, v_* bf16 [B][Hkv][d].
    The Full path's layer-0 inputs equal the Local ones: layer 0 sees the same input in both
    paths, while deeper layers see different residual streams, modelled by fresh draws."""

    q_local: list
    k_local: list
    v_local: list
    q_full: list
    k_full: list
    v_full: list
    emb: torch.Tensor           # fp32 [B][hidden], the current token's embedding
    gate_u: torch.Tensor = None  # fp32 [B] ~ U[0, 1): draws of the random gate schedule


def _bf16_normal(shape, g, device):
    if torch.device(device).type == "cuda":
        return torch.randn(shape, generator=g, device=device, dtype=torch.bfloat16)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_step_inputs(w: Workload, step: int, device="cpu") -> StepInputs:
    """All per-layer q/k/v of one step, drawn in one N(0, 1) call and split into views."""
    B, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    nq, nk = B * Hq * d, B * Hkv * d
    per_path = nq + 2 * nk
    paths = [w.layers, max(w.layers - 1, 0)]          # Local: every layer; Full: layers >= 1
    flat = _bf16_normal(((paths[0] + paths[1]) * per_path,), _gen(w.seed, _P_STEP, step,
                                                                  device=device), device)
    cols = {k: [] for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
    off = 0

    def take(n, shape):
        nonlocal off
        t = flat[off:off + n].view(shape)
        off += n
        return t

    for layer in range(w.layers):
        cols["q_local"].append(take(nq, (B, Hq, d)))
        cols["k_local"].append(take(nk, (B, Hkv, d)))
        cols["v_local"].append(take(nk, (B, Hkv, d)))
    for layer in range(w.layers):
        if layer == 0:
            for k in ("q", "k", "v"):
                cols[k + "_full"].append(cols[k + "_local"][0])
        else:
            cols["q_full"].append(take(nq, (B, Hq, d)))
            cols["k_full"].append(take(nk, (B, Hkv, d)))
            cols["v_full"].append(take(nk, (B, Hkv, d)))
    ge = _gen(w.seed, _P_EMB, step, device=device)
    emb = torch.randn((B, w.hidden), generator=ge, device=device, dtype=torch.float32)
    gu = _gen(w.seed, _P_GATE_U, step, device=device)
    gate_u = torch.rand((B,), generator=gu, device=device, dtype=torch.float32)
    return StepInputs(emb=emb, gate_u=gate_u, **cols)


def make_h0(w: Workload, device="cpu") -> torch.Tensor:
    """h_{t-1} before the first decode step, fp32 [B][hidden] ~ N(0, 1)."""
    g = _gen(w.seed, _P_H0, device=device)
    return torch.randn((w.batch, w.hidden), generator=g, device=device, dtype=torch.float32)


@dataclasses.dataclass
class RecallWeights:
    w1: torch.Tensor   # fp32 [3*hidden][mlp]
    b1: torch.Tensor   # fp32 [mlp]
    w2: torch.Tensor   # fp32 [mlp]
    b2: float


def make_recall_weights(w: Workload, device="cpu", std: float = 0.02) -> RecallWeights:
    """Untrained recall head: weights ~ N(0, std), biases zero."""
    g = _gen(w.seed, _P_RECALL)
    w1 = torch.randn((3 * w.hidden, w.mlp), generator=g, dtype=torch.float32) * std
    w2 = torch.randn((w.mlp,), generator=g, dtype=torch.float32) * std
    b1 = torch.zeros((w.mlp,), dtype=torch.float32)
    return RecallWeights(w1=w1.to(device), b1=b1.to(device), w2=w2.to(device), b2=0.0)


def make_gains(w: Workload, step: int, device="cpu") -> torch.Tensor:
    """Synthetic per-sequence gains g_t = log p^F - log p^L of Full over Local (fp32 [B]) for
    recall-head training: most steps gain almost nothing from Full (N(0, 0.1^2)), about one
    in five gains a lot (|N(0, 3^2)|), the shape the pages' recall rates imply."""
    g = _gen(w.seed, _P_GAIN, step)
    small = torch.randn((w.batch,), generator=g, dtype=torch.float32) * 0.1
    big = torch.randn((w.batch,), generator=g, dtype=torch.float32).abs() * 3.0
    pick = torch.rand((w.batch,), generator=g, dtype=torch.float32) < 0.2
    return torch.where(pick, big, small).to(device)


@dataclasses.dataclass
class DaDraw:
    """One sequence's DA declaration at one step: mode 0 = global, 1 = focus, 2 = local;
    focus_offset is the start token of the focused region (focus mode only)."""

    mode: int
    focus_offset: int


def draw_da_modes(w: Workload, step: int, positions: Sequence[int]) -> list:
    """Seeded DA declarations for one step: per sequence, a mode drawn with probabilities
    w.da_probs and, for focus, an offset ~ U[0, t + 1 - (focus_len + recent)]."""
    g = _gen(w.seed, _P_DAMODE, step)
    probs = torch.tensor(w.da_probs, dtype=torch.float64)
    out = []
    for t in positions:
        mode = int(torch.multinomial(probs, 1, generator=g))
        hi = max(0, t + 1 - (w.da_focus_len + w.da_recent))
        off = int(torch.randint(0, hi + 1, (1,), generator=g))
        out.append(DaDraw(mode=mode, focus_offset=off))
    return out


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
