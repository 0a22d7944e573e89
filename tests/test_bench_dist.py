"""Host-side logic of the multi-process benchmark on CPU: two gloo ranks agree on the
slowest rank's time and the whole-job aggregate (weak scaling, no data-path collective)."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    from datetime import timedelta

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    assert bench.dist_env() == (world, rank, rank)
    bench.barrier()
    slow = bench.max_over_ranks(10.0 + 5.0 * rank)  # rank 1 is the slow one
    value = bench.aggregate_value(world, head_tokens=1000, steps=4, total_ms_max=slow)
    out[rank] = (slow, value)
    bench.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    # 2 ranks x 1000 head-tokens x 4 steps in the slowest rank's 15 ms
    assert out[0][1] == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_value(1, 100, 10, 1000.0) == pytest.approx(1000.0)


def test_algorithmic_bytes_match_the_per_token_table():
    import bench
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    gdn = wl.workload("gdn_bf16")
    assert bench.algorithmic_bytes(gdn) == gdn.head_tokens * 1048
    kda = wl.workload("kda_bf16")
    assert bench.algorithmic_bytes(kda) == kda.head_tokens * 1556
    long = wl.workload("gdn_long_t4096")
    assert bench.algorithmic_bytes(long) == long.head_tokens * 1064


def test_vla_accounting_matches_the_per_token_table():
    import bench
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    for d, per_token, flops in ((32, 640, 1.23e4), (96, 1920, 1.11e5)):
        w = wl.workload(f"vla_fp32_d{d}")
        # per head-token: q, k, v, u in and out out (fp32); the d x d end states once per head
        assert bench.algorithmic_bytes(w, with_state_out=False) == w.head_tokens * per_token
        assert bench.algorithmic_bytes(w) == w.head_tokens * per_token + w.B * w.H * 2 * d * d * 4
        assert bench.algorithmic_flops(w) / w.head_tokens == pytest.approx(flops, rel=0.01)


def test_decode_accounting_is_the_state_round_trip_plus_one_token():
    import bench
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    w = wl.workload("gdn_decode_bf16")
    assert w.decode and w.T == 1
    # per head and step: the fp32 state read and written (2 * 128 * 128 * 4), q, k, v in and
    # out out (bf16, 4 * 128 * 2), beta and the scalar gate (fp32)
    assert bench.algorithmic_bytes(w) == w.B * w.H * (2 * 128 * 128 * 4 + 4 * 128 * 2 + 4 + 4)
    # the resident state alone is larger than the 126 MiB L2
    assert w.B * w.H * w.dv * w.dk * 4 > 126 * 2**20


def test_cpu_baseline_runs_whole_passes_up_to_the_target_time(oracle):
    import re

    import bench
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    w = wl.workload("gdn_bf16", B=1, H=2, T=256)
    r = bench.cpu_baseline(wl.generate_dr(w, 0), target_s=1.0)
    m = re.search(r"(?:(\d+) passes over )?(\d+) of 2 heads x all 256 tokens .* ([\d.]+) s\)", r["sample"])
    assert m, r["sample"]
    passes = int(m.group(1) or 1)
    # either the target time was reached or the pass cap (100) stopped it
    assert float(m.group(3)) >= 0.95 or passes == 100
    assert r["kind"] == "oracle" and r["cores"] >= 1 and r["value"] > 0


def test_every_per_config_workload_is_accounted():
    # the benchmark's configuration list names real workloads, each with positive algorithmic
    # bytes and FLOPs, and the headline is one of them
    import bench
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    assert bench.DEFAULT_WORKLOAD in bench.PER_CONFIG
    for name in bench.PER_CONFIG:
        w = wl.workload(name)
        assert bench.algorithmic_bytes(w) > 0 and bench.algorithmic_flops(w) > 0, name
        nsets, flush = bench.rotation(bench.algorithmic_bytes(w))
        assert 1 <= nsets <= 4
        cfg = bench.workload_config(w, 1)
        assert cfg["workload"] == name and cfg["B"] * cfg["H"] * cfg["T"] == w.head_tokens
