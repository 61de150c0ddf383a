"""The tensor-core page scores' operand mapping, checked on the CPU: the registers each lane
loads for `mma.sync m16n8k16` (16-byte chunks tig + 4j of tokens gid and gid + 8; k-step
2j + h takes words 2h and 2h + 1) are placed where the PTX fragment layout of that
instruction puts them, and the eight k-steps must add up to K q^T exactly. This pins the k
order the kernel relies on (every dim once, the same dim for A and B at each k index)
without a GPU; the GPU parity tests check the kernel itself."""
import numpy as np
import pytest


def _words(row_chunk):
    """8 consecutive elements (one 16-byte chunk) as 4 words of (low, high) elements."""
    return [(row_chunk[2 * w], row_chunk[2 * w + 1]) for w in range(4)]


def _emulate(K, q, G):
    """C[16][8] accumulated over the kernel's eight k-steps from per-lane registers placed by
    the m16n8k16 fragment layout (a0/a1: rows gid/gid+8, cols 2tig+i; a2/a3: cols 2tig+8+i;
    b0: rows 2tig+i, col gid; b1: rows 2tig+8+i; i = low/high element)."""
    C = np.zeros((16, 8))
    for j in range(4):
        for h in range(2):
            A = np.full((16, 16), np.nan)
            B = np.full((16, 8), np.nan)
            for lane in range(32):
                gid, tig = lane >> 2, lane & 3
                cols = slice(8 * (tig + 4 * j), 8 * (tig + 4 * j) + 8)
                ka, kb = _words(K[gid, cols]), _words(K[gid + 8, cols])
                qw = _words(q[gid, cols]) if gid < G else [(0.0, 0.0)] * 4
                a = [ka[2 * h], kb[2 * h], ka[2 * h + 1], kb[2 * h + 1]]
                for i in range(2):
                    A[gid, 2 * tig + i] = a[0][i]
                    A[gid + 8, 2 * tig + i] = a[1][i]
                    A[gid, 2 * tig + 8 + i] = a[2][i]
                    A[gid + 8, 2 * tig + 8 + i] = a[3][i]
                    B[2 * tig + i, gid] = qw[2 * h][i]
                    B[2 * tig + 8 + i, gid] = qw[2 * h + 1][i]
            assert not np.isnan(A).any() and not np.isnan(B).any()  # every slot filled once
            C += A @ B
    return C


@pytest.mark.parametrize("G", [2, 4])
def test_fragment_k_order_reproduces_scores(G):
    r = np.random.default_rng(G)
    K = r.integers(-8, 9, size=(16, 128)).astype(np.float64)  # small integers: exact sums
    q = r.integers(-8, 9, size=(8, 128)).astype(np.float64)
    C = _emulate(K, q, G)
    assert np.array_equal(C[:, :G], K @ q[:G].T)
    assert np.array_equal(C[:, G:], np.zeros((16, 8 - G)))


def test_each_dim_feeds_exactly_one_k_index():
    """Over the eight k-steps the lanes' words cover dims 0..127 once each, and for every
    (k-step, k index) A and B take the same dim."""
    seen = {}
    for j in range(4):
        for h in range(2):
            for tig in range(4):
                base = 8 * (tig + 4 * j) + 4 * h  # words 2h, 2h + 1 of the chunk: 4 dims
                for kk, dim in ((2 * tig, base), (2 * tig + 1, base + 1),
                                (2 * tig + 8, base + 2), (2 * tig + 9, base + 3)):
                    assert (2 * j + h, kk) not in seen
                    seen[(2 * j + h, kk)] = dim
    assert sorted(seen.values()) == list(range(128))
