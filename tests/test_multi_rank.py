"""bench.py's multi-rank logic on CPU with the gloo backend (world size 2):
disjoint channel shards, distinct seeds, max-over-ranks timing and the
whole-job throughput computed from it."""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    shard = bench.rank_shard(2, rank, world)
    # each rank reports its own timings; every rank must see the max
    mine = [10.0 + rank, 5.0 - rank, 1.5 * (rank + 1)]
    got = bench.max_over_ranks(mine, dist, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"shard": shard, "max": got}, f)


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    shards = [r["shard"] for r in res]
    assert shards[0]["seed"] != shards[1]["seed"]
    assert shards[0]["channel_end"] == shards[1]["channel_begin"]      # disjoint, adjacent slices
    assert res[0]["max"] == res[1]["max"] == [11.0, 5.0, 3.0]


def test_job_throughput_is_total_over_slowest():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 3 steps x 1000 elements in 2 ms (the slower rank) -> 3e6 elements/s
    assert bench.job_throughput(1000, 2, 3, 2.0) == pytest.approx(3.0e6)
    assert bench.max_over_ranks([1, 2]) == [1.0, 2.0]


def test_recorded_traffic_follows_the_convolution_sources(tmp_path, monkeypatch):
    """The roofline's DRAM traffic is reported only while the hash of the
    convolution's sources matches the one the counters were taken with."""
    import bench
    good = tmp_path / "traffic.txt"
    good.write_text(f"kernel_source_sha256_16: {bench.kernel_source_hash(3)}\n"
                    "dram_bytes_per_launch_full_size: 123456\n")
    monkeypatch.setitem(bench.TRAFFIC_FILES, 3, str(good))
    assert bench.recorded_traffic(3) == 123456.0
    stale = tmp_path / "stale.txt"
    stale.write_text("kernel_source_sha256_16: 0000000000000000\ndram_bytes_per_launch_full_size: 1\n")
    monkeypatch.setitem(bench.TRAFFIC_FILES, 3, str(stale))
    assert bench.recorded_traffic(3) is None
    assert bench.recorded_traffic(1) is None     # no capture recorded for that workload
    # each workload's hash covers the sources of its own convolution kernel
    assert bench.kernel_source_hash(3) != bench.kernel_source_hash(2)
    assert bench.kernel_source_hash(2) == bench.kernel_source_hash(5)


def test_launch_counts_and_reference_sample_sizes():
    """Launches per forward step as the library issues them, and the
    reference arm's per-step sample (about 1e9 multiply-adds of direct sum)."""
    import bench
    import s4inputs
    C = s4inputs.CONFIGS
    assert [bench.launches_per_step(C[k]) for k in (1, 2, 3, 4, 5)] == [2, 2, 3, 4, 3]
    assert [bench.reference_chunk(C[k]) for k in (1, 2, 3, 4, 5)] == [4, 7, 1, 1, 1]


def test_algorithmic_units_of_the_workloads():
    """Per-step units behind the roofline: 8 B per element of u and y plus
    16 B per (h, t) of spectrum for the convolution; 40 FLOP per (channel,
    frequency < L/2, mode pair) for the Cauchy sums; 4 per (channel, k, mode)
    for the Vandermonde product."""
    import bench
    import s4inputs
    a = bench.algorithmic(s4inputs.CONFIGS[2])
    assert a["elements"] == 16 * 256 * 4096
    assert a["conv_bytes"] == 8 * 16 * 256 * 4096 + 16 * 256 * 4096
    assert a["kernel_flop"] == 40 * 256 * 2048 * 32
    a5 = bench.algorithmic(s4inputs.CONFIGS[5])
    assert a5["kernel_flop"] == 4 * 1024 * 8192 * 32


def test_peak_file_is_read_or_falls_back(tmp_path, monkeypatch):
    """The HBM peak comes from MEASURED_PEAKS.json when it holds a usable
    copy bandwidth (plain or {"value": ...}), and falls back, labelled as
    such, when the file is missing, malformed or lacks the figure."""
    import json
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = tmp_path / "MEASURED_PEAKS.json"
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, bench.NOMINAL_SM_MHZ, "fallback")
    f.write_text(json.dumps({"hbm_gbs": 6541.8, "bf16_tflops": 1643.0}))
    assert bench.peaks() == (6541.8, bench.NOMINAL_SM_MHZ, "measured")
    f.write_text(json.dumps({"hbm_gbs": {"value": 6000.0}, "sm_max_mhz": 1900}))
    assert bench.peaks() == (6000.0, 1900.0, "measured")
    for bad in ("not json", json.dumps({"bf16_tflops": 1643.0}), json.dumps({"hbm_gbs": "n/a"}), json.dumps([1, 2])):
        f.write_text(bad)
        assert bench.peaks()[2] == "fallback"


def test_torch_formulation_of_the_kernel_matches_the_oracle():
    """The bench's context timing of the pages' formulation (torch complex64
    Cauchy sums, Woodbury, 2/(1+z), irfft) computes the kernel the oracle
    does: on the CPU, at the small workload, every output within the
    parity bound."""
    import numpy as np
    import torch
    import bench
    import s4inputs
    from oracle import workloads
    inp = s4inputs.make_inputs(1)
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])) for k in ("Lambda", "P", "Q", "B", "C", "log_dt")}
    K = bench.torch_dplr_kernel(torch, d, inp["L"], chunk=3).numpy()
    Kr = workloads.dplr_kernel(inp)
    err = max(np.abs(K[h] - Kr[h]).max() / np.abs(Kr[h]).max() for h in range(inp["H"]))
    assert err <= 1e-4, err
