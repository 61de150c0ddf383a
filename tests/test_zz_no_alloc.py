"""oda_decode_full_noalloc: the Full decode for callers that cannot allocate device memory
(its split partials and merge tickets live in a device array inside liboda instead of a
caller workspace). Called twice in a row through the C ABI, it must give what the
workspace entry point gives on the same inputs, within the decode tolerance. This file is
collected last so that a stop-at-first-failure run has already run every other test."""
import math

import numpy as np
import pytest
import torch

from oda_cases import Case, assert_attn_close, assert_lse_close
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def test_noalloc_full_matches_workspace_entry_point_twice():
    c = Case([1, 17, 300, 5000, 40_000], hq=32, hkv=8, seed=123)
    gate = torch.tensor([1, 1, 0, 1, 1], dtype=torch.int32, device="cuda")
    ref, ref_lse = c.out_buffers(fill=3.0)
    oda.oda_decode_full(c.kv, c.q, 1 / math.sqrt(128), ref, c.ws, gate=gate, lse=ref_lse)
    torch.cuda.synchronize()
    for _ in range(2):
        out, lse = c.out_buffers(fill=3.0)
        oda.oda_decode_full_noalloc(c.kv, c.q, 1 / math.sqrt(128), out, gate=gate, lse=lse)
        torch.cuda.synchronize()
        assert int(c.status.item()) == 0
        assert_attn_close(out.cpu().numpy(), ref.cpu().numpy(), "noalloc")
        assert_lse_close(lse.cpu().numpy(), ref_lse.cpu().numpy())
        assert torch.all(out[2] == 3.0)                       # gated off: untouched


def test_noalloc_rejects_batches_beyond_its_scratch():
    c = Case([10], hq=32, hkv=8, seed=124)
    big = oda.make_kv(c.kc, c.vc, c.bt.repeat(1024, 1).contiguous(),
                      c.seq_lens.repeat(1024).contiguous())
    out = torch.zeros(1024, 32, 128, dtype=torch.float32, device="cuda")
    q = c.q.repeat(1024, 1, 1).contiguous()
    with pytest.raises(oda.OdaError, match="WORKSPACE_TOO_SMALL"):
        oda.oda_decode_full_noalloc(big, q, 1 / math.sqrt(128), out)
    assert np.all(out.cpu().numpy() == 0)
