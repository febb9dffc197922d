"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The forward pass shards into independent heads, so ranks share no data; the
only cross-rank step is the timing reduction (max over ranks) and the
whole-job throughput computed from it.
"""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        assert bench.dist_env() == (rank, rank, world)
        # rank r "took" 10 + r milliseconds: everyone must see the slowest
        t = bench.reduce_max(10.0 + rank, dev)
        bench.barrier(dev)
        value = bench.job_value(100.0, world, t / 1e3)
        out[rank] = (t, value)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_reduce_max_and_job_value_over_gloo(world):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert sorted(out.keys()) == list(range(world))
    for rank in range(world):
        t, value = out[rank]
        assert t == 10.0 + (world - 1)
        assert value == pytest.approx(100.0 * world / (t / 1e3))


def test_single_process_helpers_are_identity():
    dev = torch.device("cpu")
    assert bench.reduce_max(3.5, dev) == 3.5
    bench.barrier(dev)  # no process group: no-op
    assert bench.job_value(10.0, 1, 2.0) == 5.0


def test_work_model_matches_the_flop_formula():
    from structured_sub_quadratic_b200.inputs import WORKLOADS
    wl = WORKLOADS["480p"]
    # 2 N d [(2T+1) c1 b2 + 2T c2 b1] per head, 12 heads
    assert bench.alg_flops(wl) == 12 * 2 * 4680 * 128 * (3 * 52 + 2 * 90)
    assert bench.alg_bytes(wl) == 12 * 4 * 4680 * 128 * 2
    fl, by = bench.kernel_work("tc_l_output", wl)
    assert fl == 12 * 4680 * 90 * 128 * 4 and by > 0


def test_reference_arm_times_the_oracle_on_the_host(capsys):
    """bench.py --impl reference: the float64 oracle on the host cores, one JSON line."""
    import json
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                       "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("argv", [["--workload", "vit", "--layout", "w,fh"],
                                  ["--warmup", "2"]])
def test_bench_rejects_invalid_options(argv):
    with pytest.raises(SystemExit):
        bench.main(argv)


def test_roofline_uses_algorithmic_work_not_intermediates():
    """The roofline of a kernel divides its share of the method's own work (Q/K/V/O
    bytes, or its FLOPs) by its event time; Kt/Y intermediates are not counted."""
    from structured_sub_quadratic_b200.inputs import WORKLOADS
    peaks = {"hbm_gbs": 6458.1, "bf16_tflops": 1672.0, "bf16_tflops_sustained": 1408.0}
    wl = WORKLOADS["480p"]
    # R-update at 480p: K and V read once, 2 * 12 * 4680 * 128 * 2 bytes, HBM bound
    r = bench.roofline_for("tc_r_update", 0.0230128, 1, wl, peaks, "measured", 29064192.0)
    kv = 2 * 12 * 4680 * 128 * 2
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == kv
    assert r["frac"] == pytest.approx(kv / 23.0128e-6 / 1e9 / 6458.1)
    assert r["frac"] == pytest.approx(0.1935, abs=1e-3)
    assert r["traffic_over_algorithmic"] == pytest.approx(29064192.0 / kv)
    # output kernel at 720p: 4 |p| b1 c2 d FLOPs per (g, i, p), tensor bound, sustained peak
    wl = WORKLOADS["720p"]
    r = bench.roofline_for("tc_l_output", 1.1126, 1, wl, peaks, "measured", None)
    fl = 12 * 75600 * 945 * 2 * 128 * 4
    assert r["bound"] == "tensor" and r["algorithmic_flops"] == fl
    assert r["frac"] == pytest.approx(fl / 1.1126e-3 / 1e12 / 1408.0)
    assert r["traffic_over_algorithmic"] is None
