"""The benchmark's multi-process logic on CPU: two gloo ranks take the
maximum of their times and count the whole job's tokens; the reference arm
runs on rank 0 only.  No GPU is involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) ms for the timed steps and 10 (r + 1) ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 * (rank + 1)], dist, torch.device("cpu"))
        value = bench.job_throughput(world, 64 * 23, 10, got[0])
        ref = bench.run_reference(None, rank, world) if rank != 0 else "rank0"
        out.put((rank, got, value, ref))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value, ref in res:
        assert got == [2.0, 20.0]  # both ranks see the slowest rank's times
        assert value == pytest.approx(2 * 64 * 23 * 10 / 2e-3)  # all ranks' tokens over the max time
    assert res[1][3] is None  # the reference arm does no work off rank 0


def test_single_process_is_identity():
    assert bench.max_over_ranks([3, 4.5], None, torch.device("cpu")) == [3.0, 4.5]
    assert bench.job_throughput(1, 10, 5, 1000.0) == pytest.approx(50.0)


def test_reference_arm_line(monkeypatch):
    import oracle
    oracle.build()
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--workload", "nano_layer_t16",
                                     "--steps", "1", "--warmup", "0"])
    args = bench.parse_args()
    line = bench.run_reference(args, 0, 1)
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1


def test_captured_traffic_lookup():
    """roofline.traffic comes from the committed capture table only for a
    listed (workload, T, kernel) whose sources hash to the recorded value."""
    import hashlib
    import json
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    assert entries
    for e in entries:
        h = hashlib.sha256()
        for src in e["sources"]:
            with open(os.path.join(bench.ROOT, src), "rb") as f:
                h.update(f.read())
        got = bench.captured_traffic(e["workload"], e["T"], e["kernel"])
        assert got == (e["read"] + e["write"] if h.hexdigest() == e["sha256"] else None)
    assert bench.captured_traffic("nano_decode_stack", 64, "no_such_kernel") is None
    assert bench.captured_traffic("no_such_workload", 64, entries[0]["kernel"]) is None


def test_streaming_kernel_names_follow_the_library_selection():
    import workloads
    assert bench.streaming_kernel_names(workloads.NANO, 64) == ("experts_w13_tma_kernel", "experts_w2_tma_kernel")
    assert bench.streaming_kernel_names(workloads.LARGE, 32) == ("experts_w13_tma_kernel", "experts_w2_tma_kernel")
    # the tcgen05 gate/up kernel from 12 picks per routed expert on the large-batch sequence
    assert bench.streaming_kernel_names(workloads.LARGE, 200) == ("experts_w13_tma_kernel", "experts_w2_tma_kernel")
    assert bench.streaming_kernel_names(workloads.LARGE, 512) == ("experts_w13_tc8_kernel", "experts_w2_tma_kernel")
    small = workloads.LayerShape(H=384, E=8, K=2, I=128, Is=128, routed_scaling=1.0)
    assert bench.streaming_kernel_names(small, 100) == ("experts_w13_bulk_kernel", "experts_w2_kernel")
    odd = workloads.LayerShape(H=1152, E=8, K=2, I=768, Is=256, routed_scaling=1.0)
    assert bench.streaming_kernel_names(odd, 100) == ("experts_w13_kernel", "experts_w2_tma_kernel")


def test_clock_sampler_summary_from_nvml_samples():
    s = bench.ClockSampler(0)
    s.samples = [(1965.0, 1965.0, 0), (1900.0, 1965.0, 0x4), (1950.0, 1965.0, 0)]
    got = s.summary()
    assert got == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    s.samples = [(1200.0, 1965.0, 0x8 | 0x40)]
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.ClockSampler(0).summary()["samples"] == 0
