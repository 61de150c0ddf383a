"""ODA decode engine: host-side plumbing around liboda's step graph.

One decode step over an attention stack of L layers is one graph launch
(oda_step_graph_launch): Local with commit at every layer, the recall head on the last
layer's Local output, and the gated Full recompute inside a conditional node. Everything a
step consumes that changes from step to step (seq_lens advanced by one, per-layer q/k/v of
both paths, the token embedding) lives in one contiguous staging buffer, so a step's inputs
arrive with a single copy: device-to-device from a resident pool, or host-to-device from
pinned host memory.

The previous selected hidden state h_{t-1} and the last layer's output alternate between
two buffers, with one graph for even and one for odd steps, so that the recall head of step
i reads step i-1's selected output while step i's Local pass writes the other buffer.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import torch

from . import oda

_ALIGN = 256


class StagingLayout:
    """Byte offsets of each per-step input inside the staging buffer."""

    def __init__(self, layers: int, batch: int, hq: int, hkv: int, hidden: int, d: int = 128):
        self.layers, self.batch, self.hq, self.hkv, self.hidden, self.d = layers, batch, hq, hkv, hidden, d
        off = 0
        self.fields = {}

        def add(name, nbytes):
            nonlocal off
            self.fields[name] = (off, nbytes)
            off += (nbytes + _ALIGN - 1) // _ALIGN * _ALIGN

        add("seq_lens", 4 * batch)
        add("gate_u", 4 * batch)
        add("emb", 4 * batch * hidden)
        for path in ("local", "full"):
            for l in range(layers):
                add("q_%s_%d" % (path, l), 2 * batch * hq * d)
                add("k_%s_%d" % (path, l), 2 * batch * hkv * d)
                add("v_%s_%d" % (path, l), 2 * batch * hkv * d)
        self.nbytes = off

    def views(self, buf: torch.Tensor) -> dict:
        """Typed views of one staging buffer (uint8, nbytes long)."""
        B, Hq, Hkv, D, d = self.batch, self.hq, self.hkv, self.hidden, self.d
        v = {}
        for name, (off, nb) in self.fields.items():
            raw = buf[off:off + nb]
            if name == "seq_lens":
                v[name] = raw.view(torch.int32)
            elif name == "gate_u":
                v[name] = raw.view(torch.float32)
            elif name == "emb":
                v[name] = raw.view(torch.float32).view(B, D)
            elif name.startswith("q_"):
                v[name] = raw.view(torch.bfloat16).view(B, Hq, d)
            else:
                v[name] = raw.view(torch.bfloat16).view(B, Hkv, d)
        return v


class OdaEngine:
    """Owns the per-step device buffers and the two step graphs of an ODA decode stack.

    k_caches / v_caches: per-layer bf16 [num_blocks][Hkv][16][128]; block_table int32
    [B][max_blocks]; recall: (w1 [3 Hq*128][mlp], b1 [mlp], w2 [mlp], b2 float)."""

    def __init__(self, k_caches: Sequence[torch.Tensor], v_caches: Sequence[torch.Tensor],
                 block_table: torch.Tensor, num_q_heads: int, recall, theta: float, *,
                 sink: int = 4, window: int = 2048, use_conditional: bool = True,
                 timing: bool = False, local_layers: Optional[Sequence[int]] = None,
                 sinks: Optional[Sequence[int]] = None, windows: Optional[Sequence[int]] = None,
                 random_rho: Optional[float] = None,
                 with_lse: bool = False, with_stats: bool = True, phases: int = 0,
                 step_kernels: int = oda.ODA_STEP_FULL_PERSISTENT, staging_slots: int = 1):
        self.L = len(k_caches)
        self.B = block_table.shape[0]
        self.hq = num_q_heads
        self.hkv = k_caches[0].shape[1]
        self.hidden = num_q_heads * 128
        self.sink, self.window = sink, window
        self.scale = 1.0 / math.sqrt(128)
        self.k_caches, self.v_caches, self.block_table = list(k_caches), list(v_caches), block_table
        self.w1, self.b1, self.w2, self.b2 = recall
        self.use_conditional, self.timing = use_conditional, timing
        self.phases = phases
        self.local_layers, self.sinks, self.windows = local_layers, sinks, windows
        self.random_rho = random_rho   # not None: random gate schedule at this rate
        self.step_kernels = step_kernels
        dev = block_table.device
        self.layout = StagingLayout(self.L, self.B, self.hq, self.hkv, self.hidden)
        # One staging buffer, or two: the even steps' graph reads slot 0, the odd steps' slot
        # 1, so that step i + 1's inputs can be copied in while step i runs.
        if staging_slots not in (1, 2):
            raise ValueError("staging_slots must be 1 or 2")
        self.slots = staging_slots
        self.staging_bufs = [torch.zeros(self.layout.nbytes, dtype=torch.uint8, device=dev)
                             for _ in range(staging_slots)]
        self.staging = self.staging_bufs[0]
        self.vs = [self.layout.views(b) for b in self.staging_bufs]
        self.v = self.vs[0]
        self.seq_lens = self.v["seq_lens"]
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.stats = torch.zeros(oda.ODA_STATS_LEN, dtype=torch.int64, device=dev) if with_stats else None
        self.kvs_by_slot = [[oda.make_kv(k, v, block_table, vs["seq_lens"], self.status, self.stats)
                             for k, v in zip(self.k_caches, self.v_caches)] for vs in self.vs]
        self.kvs = self.kvs_by_slot[0]
        self.out = [torch.zeros(self.B, self.hq, 128, dtype=torch.float32, device=dev)
                    for _ in range(self.L - 1)]
        self.h = [torch.zeros(self.B, self.hidden, dtype=torch.float32, device=dev) for _ in range(2)]
        self.lse = ([torch.zeros(self.B, self.hq, dtype=torch.float32, device=dev)
                     for _ in range(self.L)] if with_lse else None)
        self.q_out = torch.zeros(self.B, dtype=torch.float32, device=dev)
        self.gate = torch.zeros(self.B, dtype=torch.int32, device=dev)
        self.full_count = torch.zeros(2, dtype=torch.int64, device=dev)  # gated seqs, Full phases
        self.decode_ws = torch.zeros(oda.oda_decode_workspace_size(self.B, self.hkv, self.hq),
                                     dtype=torch.uint8, device=dev)
        self.recall_ws = torch.zeros(oda.oda_recall_workspace_size(self.B, self.hidden,
                                                                   self.w1.shape[1]),
                                     dtype=torch.uint8, device=dev)
        self.graphs = []
        self.set_theta(theta)

    def _layer_out(self, parity: int):
        last = self.h[1 - parity].view(self.B, self.hq, 128)
        return self.out + [last]

    def set_theta(self, theta: float):
        """(Re)capture the even/odd step graphs with gate threshold theta."""
        for g in self.graphs:
            g.close()
        self.theta = float(theta)
        self.graphs = self.capture(self.theta, self.phases)

    def capture(self, theta: float, phases: int = 0):
        """An even/odd pair of step graphs over this engine's buffers with the given threshold
        and phase mask, owned by the caller (launch graphs[step % 2]; close both when done).
        The engine's own graphs are untouched."""
        graphs = []
        for parity in (0, 1):
            v = self.vs[parity % self.slots]
            names = lambda p: [v["%s_%d" % (p, l)] for l in range(self.L)]
            graphs.append(oda.StepGraph(
                self.kvs_by_slot[parity % self.slots], self.hq, self.sink, self.window, self.scale,
                names("q_local"), names("k_local"), names("v_local"),
                names("q_full"), names("k_full"), names("v_full"),
                self._layer_out(parity), self.h[parity], v["emb"], self.w1, self.b1, self.w2,
                self.b2, float(theta), self.q_out, self.gate, self.decode_ws, self.recall_ws,
                full_count=self.full_count, lse=self.lse, local_layers=self.local_layers,
                sinks=self.sinks, windows=self.windows,
                gate_u=v["gate_u"] if self.random_rho is not None else None,
                rho=self.random_rho or 0.0,
                use_conditional=self.use_conditional, timing_events=self.timing,
                phases=phases, step_kernels=self.step_kernels))
        return graphs

    def views_for(self, step: int) -> dict:
        """Staging views that step `step`'s graph reads (fill them, or copy a whole staging
        image into staging_for(step), before launching it)."""
        return self.vs[step % self.slots]

    def staging_for(self, step: int) -> torch.Tensor:
        return self.staging_bufs[step % self.slots]

    def run_from_host(self, host_inputs: torch.Tensor, out_host: torch.Tensor, first_step: int,
                      stream=None) -> int:
        """Decode len(host_inputs) steps from pinned host memory: step i's staging image
        (host_inputs[i], uint8 [staging bytes]) goes in on an input stream while step i - 1
        runs (needs two staging slots), and its selected last-layer output (its result, fp32
        [B][hidden]) comes back into out_host[i % len(out_host)] on an output stream while step
        i + 1 runs. Every copy and launch is queued without a host wait; returns the step
        index after the last one. The caller synchronises before reading out_host."""
        if self.slots != 2:
            raise ValueError("run_from_host needs an engine with staging_slots=2")
        stream = stream or torch.cuda.current_stream()
        cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()
        ran = [torch.cuda.Event() for _ in range(2)]      # the graph of this slot finished
        staged = [torch.cuda.Event() for _ in range(2)]   # this slot's inputs copied in
        read = [torch.cuda.Event() for _ in range(2)]     # this slot's output copied out
        cs_in.wait_stream(stream)
        cs_out.wait_stream(stream)
        step = first_step
        for i in range(host_inputs.shape[0]):
            k = step % 2
            if i >= 2:
                cs_in.wait_event(ran[k])          # step - 2 has read this slot
            with torch.cuda.stream(cs_in):
                self.staging_for(step).copy_(host_inputs[i], non_blocking=True)
            staged[k].record(cs_in)
            stream.wait_event(staged[k])
            if i >= 2:
                stream.wait_event(read[k])        # step - 2's output has been read out
            self.launch(step, stream)
            ran[k].record(stream)
            cs_out.wait_event(ran[k])
            with torch.cuda.stream(cs_out):
                out_host[i % out_host.shape[0]].copy_(self.selected_last(step), non_blocking=True)
            read[k].record(cs_out)
            step += 1
        stream.wait_stream(cs_in)
        stream.wait_stream(cs_out)
        return step

    def set_h_prev(self, h0: torch.Tensor, step: int = 0):
        """h_{t-1} that step `step` will read."""
        self.h[step % 2].copy_(h0)

    def launch(self, step: int, stream=None):
        self.graphs[step % 2].launch(stream)

    def set_events(self, step: int, evs):
        self.graphs[step % 2].set_events(*evs)

    def selected_last(self, step: int) -> torch.Tensor:
        """Selected last-layer output of step `step` (= h_{t-1} of the next step), [B][hidden]."""
        return self.h[(step + 1) % 2]

    def layer_out(self, step: int, layer: int) -> torch.Tensor:
        return self._layer_out(step % 2)[layer]

    def close(self):
        for g in self.graphs:
            g.close()
        self.graphs = []


def fill_staging(views: dict, step_inputs, seq_lens: Sequence[int]):
    """Copy one step's inputs (oda_synth.StepInputs or any object with the same fields) into
    staging views (of a device staging buffer or of one slot of a pool)."""
    views["seq_lens"].copy_(torch.as_tensor(seq_lens, dtype=torch.int32))
    if getattr(step_inputs, "gate_u", None) is not None:
        views["gate_u"].copy_(step_inputs.gate_u)
    views["emb"].copy_(step_inputs.emb)
    for path in ("local", "full"):
        for kind in ("q", "k", "v"):
            src = getattr(step_inputs, "%s_%s" % (kind, path))
            for l, t in enumerate(src):
                views["%s_%s_%d" % (kind, path, l)].copy_(t)
