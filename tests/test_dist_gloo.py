"""The multi-GPU plumbing of bench.py on CPU ranks (gloo, world size 2): each rank runs its
own replica with its own seeded sequences, timing is the max over ranks, throughput the sum
of every rank's tokens, and there is no collective on the data path."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import oda_synth
    d = bench.Dist(world)
    try:
        ms = d.max(10.0 + rank)                       # slowest rank decides the time
        tokens = d.sum(4.0)                           # every rank's tokens count
        w = oda_synth.scaled(oda_synth.WORKLOADS["qwen3-1.7b-16k-b8"], seed=1235 + 1000 * rank)
        g = torch.Generator().manual_seed(0)
        first = oda_synth.make_step_inputs(oda_synth.scaled(w, layers=1, batch=1), 0).q_local[0]
        d.barrier()
        out[rank] = (ms, tokens, float(first.float().sum()), g.initial_seed())
    finally:
        d.close()


def test_two_replicas_over_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 11.0
    assert res[0][1] == res[1][1] == 8.0
    assert res[0][2] != res[1][2]                     # different sequences on each rank


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "1")
    d = bench.Dist(1)
    d.rank = 1
    args = type("A", (), {"workload": "pr1-ref-4k", "steps": 1, "warmup": 3})()
    assert bench.run_reference(args, d) is None


def test_clock_sampler_without_nvidia_smi_is_reported():
    import bench
    c = bench.ClockSampler(0)
    c.proc = None
    assert c.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_profiled_bytes_follow_committed_summaries(tmp_path, monkeypatch):
    """bench.py reads the DRAM bytes of the step's kernels from the committed ncu summaries,
    and only while the kernel sources they were taken on are unchanged."""
    import bench
    full = bench.profiled_traffic(131073)
    assert full is not None and 1.0 <= full / (131073 * 8 * 512) < 1.05
    step = bench.profiled_step_bytes(28, 2.0, 131073)
    local = float(bench._profile_fields(bench.LOCAL_PROFILE)["dram_bytes_per_launch"])
    recall = float(bench._profile_fields(bench.RECALL_PROFILE,
                                         bench.RECALL_SOURCES)["dram_bytes_per_launch"])
    assert step == 28 * local + recall + 2.0 * full
    stale = tmp_path / "stale.md"
    stale.write_text(open(bench.LOCAL_PROFILE).read().replace(
        bench.kernel_source_hash(), "0000000000000000"))
    monkeypatch.setattr(bench, "LOCAL_PROFILE", str(stale))
    assert bench.profiled_step_bytes(28, 2.0, 131073) is None
