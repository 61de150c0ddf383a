"""The decode kernel's visibility plan (oda_plan.cuh, compiled for the host) against the
oracle's set definitions, bit-exact, without a GPU: Local, Full, Keep, the device-compiled
Declarative-Attention modes and context-parallel shards, over many positions and
parameters. Each listed page must be ascending and resolved through the page table."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import oda_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def probe():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    exe = os.path.join(ROOT, "_build", "plan_probe")
    cmd = [nvcc, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I",
           os.path.join(ROOT, "sparse_kv_recall_b200", "csrc"), os.path.join(HERE, "plan_probe.cu"),
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True)

    def run(cases):
        text = "\n".join(" ".join(str(x) for x in c) for c in cases) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True)
        res = []
        for line in out.stdout.splitlines():
            assert line != "bad", "plan listed a page out of order or unresolved"
            f = [int(x) for x in line.split()]
            res.append((f[0], f[1], np.array(f[2:], dtype=np.int64)))
        assert len(res) == len(cases)
        return res
    return run


T_GRID = list(range(0, 70)) + [255, 256, 257, 1023, 2047, 2048, 2051, 4095, 4100, 40_000, 131_072]


def test_local_and_full(probe):
    cases, want = [], []
    for t in T_GRID:
        for s in (0, 1, 4, 16, 17):
            for w in (1, 2, 16, 17, 64, 2048):
                cases.append(("L", t, s, w))
                want.append(O.local_positions(t, s, w))
        cases.append(("F", t))
        want.append(O.full_positions(t))
    for (err, _, got), ref in zip(probe(cases), want):
        assert err == 0 and np.array_equal(got, ref)


def test_keep_lists(probe):
    r = np.random.default_rng(5)
    cases, want = [], []
    for t in [0, 15, 16, 100, 1000, 5000]:
        last = t // 16
        for _ in range(20):
            k = np.sort(r.choice(last + 1, size=r.integers(0, last + 2), replace=False))
            cases.append(("K", t, len(k)) + tuple(int(x) for x in k))
            want.append(O.keep_positions(t, k))
    for (err, _, got), ref in zip(probe(cases), want):
        assert err == 0 and np.array_equal(got, ref)


def test_da_modes_compiled_on_device_match_regions(probe):
    r = np.random.default_rng(6)
    cases, want = [], []
    for t in [0, 3, 16, 100, 2047, 5000, 40_000, 131_071]:
        for mode in (0, 1, 2):
            for _ in range(12 if mode == 1 else 1):
                off = int(r.integers(0, t + 40))
                fl, rc, ll = int(r.choice([1, 16, 100, 32768])), int(r.choice([1, 17, 2048])), \
                    int(r.choice([1, 33, 4096]))
                cases.append(("D", t, mode, off, fl, rc, ll))
                want.append(O.da_mode_positions(mode, t, off, focus_len=fl, recent=rc,
                                                local_len=ll))
    for (err, _, got), ref in zip(probe(cases), want):
        assert err == 0 and np.array_equal(got, ref)


def test_da_bad_mode_and_offset_make_the_sequence_empty(probe):
    res = probe([("D", 100, 3, 0, 16, 16, 16), ("D", 100, 1, -1, 16, 16, 16),
                 ("D", 100, -1, 0, 16, 16, 16)])
    for err, npages, got in res:
        assert err == 5 and npages == 0 and got.size == 0     # ODA_DEV_BAD_DA


def test_shards_partition_full(probe):
    cases, want, groups = [], [], []
    for t in [0, 15, 16, 17, 300, 4096, 50_001]:
        for parts in (1, 2, 3, 8):
            # page-aligned, roughly equal cuts of 0..capacity, the last one open-ended
            cap = (t // 16 + 1) * 16
            cuts = [((cap * i // parts) // 16) * 16 for i in range(parts)] + [1 << 30]
            g = []
            for lo, hi in zip(cuts, cuts[1:]):
                if hi <= lo:
                    continue
                cases.append(("S", t, lo, hi))
                want.append(O.shard_positions(t, lo, hi))
                g.append(len(cases) - 1)
            groups.append((t, g))
    res = probe(cases)
    for (err, _, got), ref in zip(res, want):
        assert err == 0 and np.array_equal(got, ref)
    for t, g in groups:                                  # the shards tile 0..t exactly once
        allp = np.concatenate([res[i][2] for i in g])
        assert np.array_equal(np.sort(allp), O.full_positions(t))
