"""Helpers for the GPU parity tests: seeded paged-KV cases built from the input module, the
oracle evaluated on the same inputs, and the acceptance tolerances.

Tolerances (bf16 inputs, fp32 accumulation): outputs max |d| <= 4e-3 and mean |d| <= 5e-4;
recall scores |d| <= 1e-3; gates, visible index sets and committed K/V bits exact. The
natural-log normaliser is compared within 1e-4: its fp32 error is a few ulp of the score
sums (|lse| < 20 here, ulp ~ 2e-6), well under that."""
import math

import numpy as np
import torch

import oda_synth
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import oda

OUT_MAX = 4e-3
OUT_MEAN = 5e-4
LSE_TOL = 1e-4
Q_TOL = 1e-3
SCALE = 1.0 / math.sqrt(128)


def assert_attn_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    d = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    assert d.max() <= OUT_MAX, "%s max|d| = %g" % (what, d.max())
    assert d.mean() <= OUT_MEAN, "%s mean|d| = %g" % (what, d.mean())


def assert_lse_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf), what
    if (~inf).any():
        d = np.abs(got[~inf] - ref[~inf])
        assert d.max() <= LSE_TOL, "%s lse max|d| = %g" % (what, d.max())


class Case:
    """A batch of sequences with explicit lengths (tokens including the current one) over a
    paged bf16 cache, plus one step's q / k_new / v_new, all from the seeded generator."""

    def __init__(self, lengths, hq, hkv, seed, extra=32, spare_pages=3):
        self.B = len(lengths)
        self.hq, self.hkv = hq, hkv
        self.lengths = list(lengths)
        self.w = oda_synth.Workload(name="case", layers=1, batch=self.B, num_q_heads=hq,
                                    num_kv_heads=hkv, prefill=max(lengths), steps=1, seed=seed)
        lay = oda_synth.make_layout(self.w, extra_tokens=extra, device="cuda",
                                    lengths=self.lengths, spare_pages=spare_pages)
        self.num_blocks = lay.num_blocks
        self.bt = lay.block_table
        self.kc, self.vc = oda_synth.make_kv_cache(self.w, lay, 0, device="cuda")
        si = oda_synth.make_step_inputs(self.w, 0, device="cuda")
        self.q, self.k_new, self.v_new = si.q_local[0], si.k_local[0], si.v_local[0]
        self.seq_lens = torch.tensor(self.lengths, dtype=torch.int32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.stats = torch.zeros(oda.ODA_STATS_LEN, dtype=torch.int64, device="cuda")
        self.ws = torch.zeros(oda.oda_decode_workspace_size(self.B, hkv, hq), dtype=torch.uint8,
                              device="cuda")
        self.kv = oda.make_kv(self.kc, self.vc, self.bt, self.seq_lens, self.status, self.stats)
        self.snapshot()
        self.qbits = oda_synth.bf16_bits(self.q)
        self.knew_bits = oda_synth.bf16_bits(self.k_new)
        self.vnew_bits = oda_synth.bf16_bits(self.v_new)

    def snapshot(self):
        """Host copy of the cache as it is now (the oracle reads this copy)."""
        self.kbits = oda_synth.bf16_bits(self.kc)
        self.vbits = oda_synth.bf16_bits(self.vc)
        self.bt_h = self.bt.cpu().numpy()

    def out_buffers(self, fill=float("nan"), dtype=torch.float32):
        out = torch.full((self.B, self.hq, 128), fill, dtype=dtype, device="cuda")
        lse = torch.full((self.B, self.hq), fill, dtype=torch.float32, device="cuda")
        return out, lse

    def oracle(self, positions_of, commit=False, seqs=None):
        """fp64 attention for every sequence b in `seqs` over positions_of(b, t)."""
        out = np.zeros((self.B, self.hq, 128))
        lse = np.zeros((self.B, self.hq))
        for b in (range(self.B) if seqs is None else seqs):
            t = self.lengths[b] - 1
            pos = np.asarray(positions_of(b, t), dtype=np.int64)
            ks, vs = [], []
            for g in range(self.hkv):
                kr = O.paged_rows(self.kbits, self.bt_h[b], pos, g)
                vr = O.paged_rows(self.vbits, self.bt_h[b], pos, g)
                if commit and pos.size and pos[-1] == t:
                    kr[-1] = O.widen_bf16(self.knew_bits[b, g])
                    vr[-1] = O.widen_bf16(self.vnew_bits[b, g])
                ks.append(kr)
                vs.append(vr)
            out[b], lse[b] = O.decode_attention(O.widen_bf16(self.qbits[b]), ks, vs, SCALE)
        return out, lse

    def slot_bits(self, cache_bits, b, t):
        """bits of position t of sequence b in a host cache copy: [Hkv][128]."""
        return cache_bits[self.bt_h[b, t // 16], :, t % 16, :]
