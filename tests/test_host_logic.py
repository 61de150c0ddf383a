"""Host-side logic of the product, on CPU: DA keep-page lists against the oracle's visible
sets, and the synthetic input recipe's structure."""
import numpy as np
import pytest

import oda_synth
from oracle import oda_oracle as O
from sparse_kv_recall_b200 import da


def _check(mode, t, off):
    keep = da.keep_pages(mode, t, off)
    assert np.all(np.diff(keep) > 0) and keep[0] >= 0 and keep[-1] <= t // 16
    got = O.keep_positions(t, keep)
    assert np.array_equal(got, O.da_mode_positions(mode, t, off)), (mode, t, off)


@pytest.mark.parametrize("mode", [da.GLOBAL, da.FOCUS, da.LOCAL])
def test_keep_pages_match_oracle_sets(mode):
    r = np.random.default_rng(mode)
    for t in list(range(0, 70)) + [2047, 2048, 4095, 4096, 34815, 34816, 40000, 100_003]:
        for _ in range(3):
            off = int(r.integers(0, max(1, t + 1 - 34816) + 1))
            _check(mode, t, off)
    t = 1_048_576 + 100
    _check(mode, t, 500_000)
    _check(mode, t, 0)
    _check(mode, t, t + 1 - 34816)


def test_keep_lists_padding_and_counts():
    draws = [oda_synth.DaDraw(mode=0, focus_offset=0), oda_synth.DaDraw(mode=2, focus_offset=0)]
    keep, counts = da.keep_lists(draws, [100, 10_000], max_keep=700)
    assert counts.tolist() == [7, 10_000 // 16 - (10_000 - 4095) // 16 + 1]
    assert keep[0, :7].tolist() == list(range(7)) and np.all(keep[0, 7:] == -1)
    with pytest.raises(ValueError):
        da.keep_lists(draws, [100, 100_000], max_keep=10)


def test_da_mode_draws_follow_recipe():
    w = oda_synth.WORKLOADS["da-1m-b2"]
    counts = np.zeros(3)
    for step in range(400):
        for d in oda_synth.draw_da_modes(w, step, [w.prefill + step] * 2):
            counts[d.mode] += 1
            assert 0 <= d.focus_offset <= w.prefill + step + 1 - 34816
    frac = counts / counts.sum()
    assert np.allclose(frac, [0.2, 0.5, 0.3], atol=0.04)


def test_layout_is_a_permutation_of_pages():
    w = oda_synth.Workload(name="t", layers=1, batch=3, num_q_heads=4, num_kv_heads=2, prefill=50,
                           steps=1, seed=5)
    lay = oda_synth.make_layout(w, extra_tokens=20, lengths=[1, 17, 300], spare_pages=3)
    bt = lay.block_table.numpy()
    used = bt[bt >= 0]
    assert sorted(used.tolist()) == sorted(set(used.tolist()))
    assert lay.num_blocks == 2 + 3 + 20 + 3
    assert [int((row >= 0).sum()) for row in bt] == [2, 3, 20]
    lens = oda_synth.prefill_lengths(oda_synth.WORKLOADS["qwen3-8b-ragged-b16"])
    assert len(lens) == 16 and min(lens) >= 8192 and max(lens) <= 65536
