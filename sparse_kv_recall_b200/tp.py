"""KV-head tensor parallelism for the ODA decode step: rank r of N owns a contiguous block of
Hkv / N KV heads -- their K/V pages at every layer -- and the Hq / N query heads that read
them, and runs its heads' Local pass, Full pass, commits and merges with no exchange (heads
are independent in attention). The recall head reads the whole last-layer Local output h^L,
so it is computed on every rank from the same inputs and every rank takes the same branch:
one all-gather of the ranks' h^L slices (B x Hq/N x 128 fp32 each) before it, and one of the
selected last-layer slices after the Full pass, which are the next step's h_{t-1}. Both go
through the process group (NCCL over NVLink on GPUs).

The step is split into phases (local_pass, gate, full_pass, selected) so that one GPU can run
N ranks in turn with the gathers done by concatenation; step() runs them with the process
group's all-gathers."""
from __future__ import annotations

import math
from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import oda


def head_slice(num_kv_heads: int, num_q_heads: int, world: int, rank: int) -> Tuple[int, int, int, int]:
    """(kv_lo, kv_hi, q_lo, q_hi) of rank `rank`: contiguous blocks of KV heads and of the
    query heads that share them (query head h reads KV head h // (Hq / Hkv))."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("0 <= rank < world required")
    if num_kv_heads % world != 0 or num_q_heads % num_kv_heads != 0:
        raise ValueError("Hkv must split evenly over the ranks and Hq over Hkv")
    per = num_kv_heads // world
    g = num_q_heads // num_kv_heads
    return rank * per, (rank + 1) * per, rank * per * g, (rank + 1) * per * g


def gather_heads(part: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's [B][Hq/N][128] slice into [B][Hq][128], heads in rank order
    (the order head_slice assigns them). One collective, contiguous output."""
    world = dist.get_world_size(group)
    buf = torch.empty((world,) + tuple(part.shape), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(buf.view(-1), part.contiguous().view(-1), group=group)
    return join_heads(list(buf.unbind(0)))


def join_heads(parts: Sequence[torch.Tensor]) -> torch.Tensor:
    """[B][Hq/N][128] slices in rank order -> [B][Hq][128]."""
    return torch.cat(list(parts), dim=1).contiguous()


class HeadParallelStep:
    """One ODA decode step over this rank's KV heads at every layer.

    kvs: per layer, this rank's oda_kv (caches [num_blocks][Hkv/N][16][128]; the block table
    and sequence lengths are those of every rank). recall: (W1 [3 hidden][mlp], b1, w2, b2) of
    the full hidden size hidden = Hq x 128, replicated on every rank."""

    def __init__(self, kvs: List[oda.oda_kv], num_q_heads: int, world: int, rank: int,
                 recall, theta: float, sink: int, window: int, batch: int, device,
                 group=None):
        self.kvs = kvs
        self.L = len(kvs)
        self.B = batch
        self.Hq = num_q_heads
        self.hkv_l = kvs[0].num_kv_heads
        self.world, self.rank, self.group = world, rank, group
        if num_q_heads % (self.hkv_l * world) != 0:
            raise ValueError("Hq must be a multiple of this rank's KV heads x the ranks")
        self.hq_l = num_q_heads // world
        self.hidden = num_q_heads * 128
        self.w1, self.b1, self.w2, self.b2 = recall
        self.theta, self.sink, self.window = float(theta), int(sink), int(window)
        self.scale = 1.0 / math.sqrt(128)
        dev = device
        self.ws = torch.zeros(oda.oda_decode_workspace_size(batch, self.hkv_l, self.hq_l),
                              dtype=torch.uint8, device=dev)
        self.recall_ws = torch.zeros(oda.oda_recall_workspace_size(batch, self.hidden,
                                                                   self.w1.shape[1]),
                                     dtype=torch.uint8, device=dev)
        self.out = [torch.zeros(batch, self.hq_l, 128, dtype=torch.float32, device=dev)
                    for _ in range(self.L)]
        self.h_prev = torch.zeros(batch, self.hidden, dtype=torch.float32, device=dev)
        self.q_out = torch.zeros(batch, dtype=torch.float32, device=dev)
        self.gate_out = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.full_count = torch.zeros(2, dtype=torch.int64, device=dev)

    # ---- phases ----
    def local_pass(self, q: Sequence, k_new: Sequence, v_new: Sequence) -> torch.Tensor:
        """Local at every layer for this rank's heads (commits slot t); returns this rank's
        slice of h^L, [B][Hq/N][128]."""
        for l in range(self.L):
            oda.oda_decode_local(self.kvs[l], q[l], self.sink, self.window, self.scale,
                                 self.out[l], self.ws, k_new=k_new[l], v_new=v_new[l])
        return self.out[self.L - 1]

    def gate(self, h_local_full: torch.Tensor, emb: torch.Tensor) -> torch.Tensor:
        """The recall head on the gathered h^L ([B][Hq][128]) with the replicated h_{t-1} and
        E(x_t): the same inputs and kernel on every rank, hence the same gate."""
        oda.oda_recall_score(self.h_prev, emb, h_local_full.view(self.B, self.hidden), self.w1,
                             self.b1, self.w2, self.b2, self.theta, self.q_out, self.gate_out,
                             self.recall_ws, full_count=self.full_count)
        return self.gate_out

    def full_pass(self, q: Sequence, k_new: Sequence, v_new: Sequence) -> torch.Tensor:
        """Full at every layer for the gated sequences of this rank's heads (their output rows
        and slot t replaced); returns this rank's selected last-layer slice."""
        for l in range(self.L):
            oda.oda_decode_full(self.kvs[l], q[l], self.scale, self.out[l], self.ws,
                                gate=self.gate_out, k_new=k_new[l], v_new=v_new[l])
        return self.out[self.L - 1]

    def set_h_prev(self, h_full: torch.Tensor):
        """h_{t-1} for the next step: the gathered selected last-layer output, [B][hidden]."""
        self.h_prev.copy_(h_full.reshape(self.B, self.hidden))

    # ---- a whole step through the process group ----
    def step(self, q_local, k_local, v_local, q_full, k_full, v_full, emb,
             gather: Optional[Callable[[torch.Tensor], torch.Tensor]] = None):
        """One decode step; returns this rank's per-layer outputs (selected) and the gate."""
        gather = gather or (lambda t: gather_heads(t, self.group))
        h_l = gather(self.local_pass(q_local, k_local, v_local))
        self.gate(h_l, emb)
        sel = gather(self.full_pass(q_full, k_full, v_full))
        self.set_h_prev(sel)
        return self.out, self.gate_out
