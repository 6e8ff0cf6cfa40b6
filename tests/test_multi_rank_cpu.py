"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): replicas get distinct
seeded inputs, per-rank times reduce to their max, and the whole-job rate counts every
rank's units over the slowest rank's time.  No data-path collective exists to test: the
units are independent."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth_inputs as si


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(1.5 + rank)
        seed = bench.replica_seed(1003, rank)
        x = torch.from_numpy(si.normal(seed, si.Q, (64,)))
        gathered = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out[rank] = (t, bool(torch.equal(gathered[0], gathered[1])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_replicas():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5
    assert res[0][1] is False  # the two replicas' inputs differ


def test_aggregate_rate_counts_all_ranks():
    assert bench.aggregate_rate(1e12, 4, 1000.0) == pytest.approx(4e12)
    assert bench.aggregate_rate(2.0, 1, 2.0) == pytest.approx(1000.0)


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_json_line_has_no_nan():
    """Phases left out with --only report null (NaN is not JSON)."""
    import json
    line = {"value": float("nan"), "nested": {"x": [1.0, float("nan")], "y": "s"}, "z": 2}
    out = json.dumps(bench._nan_to_null(line), allow_nan=False)
    assert json.loads(out) == {"value": None, "nested": {"x": [1.0, None], "y": "s"}, "z": 2}


def test_paged_workload_bytes_follow_lengths():
    w = bench.PAGED
    lens = bench.paged_lengths(w["seed"])
    assert len(lens) == w["B"] and lens.min() >= w["len_lo"] and lens.max() <= w["len_hi"]
    assert bench.paged_kv_bytes(lens) == 2.0 * lens.sum() * w["Hkv"] * w["d"] * 2


def test_varlen_flops_match_the_closed_form():
    """Causal varlen forward FLOPs: sum over sequences of 4 Hq L^2 d / 2, which for Hq = 32,
    d = 128 is 8192 L^2 per sequence; the backward counts 2.5 times that."""
    lens = bench.varlen_lengths(bench.VARLEN["seed"])
    assert len(lens) == bench.VARLEN["nseq"]
    assert lens.min() >= bench.VARLEN["len_lo"] and lens.max() <= bench.VARLEN["len_hi"]
    assert bench.varlen_flops(lens) == float(sum(8192 * int(L) * int(L) for L in lens))
    assert bench.varlen_flops([5]) == 4 * 32 * 25 * 128 / 2


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON line with
    the contract's keys; a rank other than 0 prints nothing and exits 0."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
           "--cpu-seconds", "1"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300,
                         env={**os.environ, "RANK": "0", "WORLD_SIZE": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "TFLOP/s" and j["higher_is_better"] is True
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"] == {"value": j["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    other = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300,
                           env={**os.environ, "RANK": "1", "WORLD_SIZE": "2"})
    assert other.returncode == 0 and not other.stdout.strip()
