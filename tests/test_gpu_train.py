"""The recall head's training objective on the GPU (oda_recall_loss_grad) against the oracle's
loss and gradient: q within 1e-3, the loss within 1e-4 relative, and every gradient entry
within 1e-4 of the largest gradient magnitude of its tensor (fp32 sums of up to 3 * 4096
products against fp64). Shapes cover the 16-head hidden size with the bench's batch, ragged
batches and row counts that end mid-slab and mid-block, bf16 h_local, residuals on both
sides of the Huber knee, and bitwise determinism."""
import numpy as np
import pytest
import torch

import oda_synth
from oda_cases import Q_TOL
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import build as B
from sparse_kv_recall_b200 import oda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    B.build()
    oda.load()


def _case(batch, hidden, mlp, std, seed, bf16=False):
    g = torch.Generator().manual_seed(seed)
    hp, em, hl = (torch.randn(batch, hidden, generator=g) for _ in range(3))
    if bf16:
        hl = hl.to(torch.bfloat16)
    w1 = torch.randn(3 * hidden, mlp, generator=g) * std
    b1 = torch.randn(mlp, generator=g) * std
    w2 = torch.randn(mlp, generator=g) * std
    wl = oda_synth.Workload(name="train", layers=1, batch=batch, num_q_heads=16, num_kv_heads=8,
                            prefill=1, steps=1, seed=seed)
    gain = oda_synth.make_gains(wl, 0)
    gain[::3] += 4.0                   # some steps that clearly gain from Full
    return hp, em, hl, w1, b1, w2, 0.05, gain


def _run(hp, em, hl, w1, b1, w2, b2, gain, lam, ws=None):
    dev = "cuda"
    batch, hidden = hp.shape
    mlp = w1.shape[1]
    args = [t.to(dev) for t in (hp, em, hl, w1, b1, w2)]
    if ws is None:
        ws = torch.zeros(oda.oda_recall_train_workspace_size(batch, hidden, mlp),
                         dtype=torch.uint8, device=dev)
    loss = torch.full((1,), float("nan"), device=dev)
    db2 = torch.full((1,), float("nan"), device=dev)
    dw1 = torch.full_like(args[3], float("nan"))
    db1 = torch.full_like(args[4], float("nan"))
    dw2 = torch.full_like(args[5], float("nan"))
    q = torch.full((batch,), float("nan"), device=dev)
    oda.oda_recall_loss_grad(*args, b2, gain.to(dev), lam, ws, loss, dw1, db1, dw2, db2, q_out=q)
    torch.cuda.synchronize()
    return q, loss, dw1, db1, dw2, db2


def _close(got, ref, what):
    got = got.double().cpu().numpy()
    scale = max(np.abs(ref).max(), 1e-6)
    d = np.abs(got - ref).max()
    assert d <= 1e-4 * scale, "%s: max|d| = %g of %g" % (what, d, scale)


@pytest.mark.parametrize("batch,hidden,mlp,std,bf16", [
    (8, 2048, 256, 0.02, False),       # the 16-head hidden size, the bench's batch
    (8, 2048, 256, 0.3, True),         # large residuals: both Huber branches, bf16 h_local
    (1, 100, 128, 0.2, False),         # 300 rows: slabs and row blocks end ragged
    (13, 700, 192, 0.1, False),        # batch not a multiple of 8
])
def test_loss_and_gradient_match_oracle(batch, hidden, mlp, std, bf16):
    hp, em, hl, w1, b1, w2, b2, gain = _case(batch, hidden, mlp, std, seed=batch * 7 + mlp, bf16=bf16)
    lam = 0.5
    q, loss, dw1, db1, dw2, db2 = _run(hp, em, hl, w1, b1, w2, b2, gain, lam)
    ref = O.recall_loss_grad(hp.double().numpy(), em.double().numpy(), hl.double().numpy(),
                             w1.double().numpy(), b1.double().numpy(), w2.double().numpy(), b2,
                             gain.double().numpy(), lam)
    rloss, rq, rdw1, rdb1, rdw2, rdb2 = ref
    assert np.abs(q.cpu().numpy() - rq).max() <= Q_TOL
    assert abs(loss.item() - rloss) <= 1e-4 * max(abs(rloss), 1e-3)
    _close(dw1, rdw1, "dW1")
    _close(db1, rdb1, "db1")
    _close(dw2, rdw2, "dw2")
    assert abs(db2.item() - rdb2) <= 1e-5
    if std == 0.02:
        r = rq - O.signed_log_target(gain.double().numpy(), lam)
        assert (np.abs(r) > 1).any() and (np.abs(r) < 1).any()     # both Huber branches


def test_gradient_is_deterministic_and_workspace_reusable():
    case = _case(8, 2048, 256, 0.05, seed=3)
    ws = torch.zeros(oda.oda_recall_train_workspace_size(8, 2048, 256), dtype=torch.uint8,
                     device="cuda")
    a = _run(*case, lam=0.2, ws=ws)
    b = _run(*case, lam=0.2, ws=ws)      # the ticket was left zero: the same ws serves again
    c = _run(*case, lam=0.2)
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y) and torch.equal(x, z)
