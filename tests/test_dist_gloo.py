"""The multi-GPU plumbing of bench.py on CPU ranks (gloo, world size 2): each rank runs its
own replica with its own seeded sequences, timing is the max over ranks, throughput the sum
of every rank's tokens, and there is no collective on the data path."""
import json
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


def test_profiled_bytes_follow_committed_captures(tmp_path, monkeypatch):
    """bench.py reads the DRAM bytes of the step's kernels from the JSON its --ncu-summary
    writes from an ncu capture, by step mode, and only while the kernel sources it was taken
    on are unchanged; the summary is read back from a raw CSV export the way ncu writes it."""
    import bench
    csv = tmp_path / "raw.csv"
    csv.write_text(
        '"ID","Process ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum",'
        '"gpu__time_duration.sum"\n'
        '"","","","Mbyte","Mbyte","usecond"\n'
        '"0","1","void oda::local_chain_kernel<2>(oda::LocalChainParams)","200.5","1.5","40"\n'
        '"1","1","void oda::full_chain_kernel<2>(oda::FullChainParams)","1,080","8","200"\n'
        '"2","1","void oda::full_chain_kernel<2>(oda::FullChainParams)","1,082","8","202"\n'
        '"3","1","void oda::cluster_decode_kernel<2>(oda::DecodeParams)","8.5","0.5","6"\n'
        '"4","1","void oda::recall_kernel(oda::RecallParams)","6.3","0.1","4"\n')
    paths = {k: tmp_path / (k + ".json") for k in bench.PROFILES}
    info = bench.ncu_summary(str(csv), "full_chain_kernel", str(paths["full_chain"]),
                             {"tokens_per_layer": 131073, "layers_per_launch": 2})
    assert info["launches_captured"] == 2
    assert info["dram_bytes_per_launch"] == 1089e6
    assert abs(info["gpu_time_s_per_launch_under_ncu"] - 201e-6) < 1e-12
    bench.ncu_summary(str(csv), "local_chain_kernel", str(paths["local_chain"]),
                      {"layers_per_launch": 28})
    bench.ncu_summary(str(csv), "cluster_decode_kernel", str(paths["local_cluster"]),
                      {"layers_per_launch": 1})
    bench.ncu_summary(str(csv), "recall_kernel", str(paths["recall"]), {})
    monkeypatch.setattr(bench, "PROFILES", {k: str(v) for k, v in paths.items()})
    per = 1089e6 / (131073 * 2)
    assert abs(bench.profiled_traffic(131073, 28) - per * 131073 * 28) < 1.0
    step = bench.profiled_step_bytes("persistent", 28, 0.5, 131073)
    assert abs(step - (202e6 * 28 / 28 + 0.5 * per * 131073 * 28)) < 1.0
    step = bench.profiled_step_bytes("full-persistent", 28, 0.5, 131073)
    assert abs(step - (9e6 * 28 + 6.4e6 + 0.5 * per * 131073 * 28)) < 1.0
    assert bench.profiled_step_bytes("per-layer", 28, 0.5, 131073) is None   # no capture
    stale = json.load(open(paths["full_chain"]))
    stale["source_sha"] = "0000000000000000"
    json.dump(stale, open(paths["full_chain"], "w"))
    assert bench.profiled_traffic(131073, 28) is None
    assert bench.profiled_step_bytes("full-persistent", 28, 0.5, 131073) is None


def test_bench_step_kernel_modes_match_the_library():
    import bench
    from sparse_kv_recall_b200 import oda
    assert bench.STEP_KERNELS == {"full-persistent": oda.ODA_STEP_FULL_PERSISTENT,
                                  "per-layer": oda.ODA_STEP_PER_LAYER,
                                  "persistent": oda.ODA_STEP_PERSISTENT}
