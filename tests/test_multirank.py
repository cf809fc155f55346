"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The layer shards by (batch, head) with no exchange step.  By default the heads
of one layer are split into contiguous ranges, one per GPU (strong scaling);
--shard replicas runs one independent layer per GPU (weak scaling).  The only
cross-rank operations are the barrier, the max-over-ranks of the step timings
and the sum of the ranks' work.  These tests run that logic as real gloo
ranks, check that the head partition reassembles the one-rank layer, and
launch the reference arm through torchrun."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import svg_inputs as si  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings that differ in every slot
        mine = [10.0 + rank, 5.0 - rank, 1.0 + 0.5 * rank]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        work = bench.sum_over_ranks([1.0e12 * (rank + 1), 3.0], world, torch.device("cpu"))
        wl = si.WORKLOADS["cogvideox"]
        value, tok, ms = bench.aggregate(work[0], got[0], 4, world * wl.B * wl.N)
        dist.barrier()
        results[rank] = {"max": got, "sum": work, "value": value, "tokens": tok, "ms": ms,
                         "seed": bench.rank_seed(wl, rank)}
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    r0, r1 = results[0], results[1]
    assert r0["max"] == r1["max"] == [11.0, 5.0, 1.5]
    assert r0["sum"] == r1["sum"] == [3.0e12, 6.0]
    # whole-job value: both ranks' work over the slowest rank's step time
    assert r0["ms"] == pytest.approx(11.0 / 4)
    assert r0["value"] == pytest.approx(3.0e12 / (11.0 / 4 * 1e-3) / 1e12)
    assert r0["tokens"] == pytest.approx(2 * 17550 / (11.0 / 4 * 1e-3))
    assert r0["value"] == r1["value"]
    # independent inputs per rank
    assert r0["seed"] != r1["seed"]


def test_single_rank_passthrough():
    assert bench.max_over_ranks([3, 2.5], 1, None) == [3.0, 2.5]
    assert bench.sum_over_ranks([3, 2.5], 1, None) == [3.0, 2.5]
    v, t, ms = bench.aggregate(1.0e12, 20.0, 10, 100)
    assert ms == 2.0 and v == pytest.approx(500.0) and t == pytest.approx(5.0e4)


def test_head_shards_partition_the_layer():
    # every head on exactly one rank, contiguous ranges in rank order, sizes
    # within one of each other (H not divisible by the rank count included)
    for H in (1, 2, 3, 7, 24, 40, 48):
        for world in range(1, min(H, 8) + 1):
            shards = [bench.shard_heads(H, world, r) for r in range(world)]
            assert [h for s in shards for h in s] == list(range(H)), (H, world)
            sizes = [len(s) for s in shards]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
            assert sizes == sorted(sizes, reverse=True)
    assert bench.shard_heads(24, 5, 0) == range(0, 5) and bench.shard_heads(24, 5, 4) == range(20, 24)


def _shard_layer_main(rank, world, port, results):
    """One rank of a head-sharded layer: draw only this rank's heads, run the
    oracle layer on them, and gather (heads, o, mode, mse) on every rank."""
    import datetime

    import torch.distributed as dist
    from oracle import svg_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        wl = si.small("hunyuan720").scaled("shard-test", H=3)
        heads = bench.shard_heads(wl.H, world, rank)
        q, k, v, _ = si.generate(wl, seed=wl.seed, heads=heads)
        idx = si.sample_queries(wl)
        o, mode, mse = O.svg_layer(*(si.as_float64(t) for t in (q, k, v)), idx, wl.F, wl.P,
                                   wl.width)
        got = [None] * world
        dist.all_gather_object(got, (heads.start, heads.stop, o, mode, mse))
        if rank == 0:
            results["parts"] = got
    finally:
        dist.destroy_process_group()


def test_head_sharded_layer_reassembles_gloo():
    """World size 2 over a 3-head layer (uneven split): the ranks' outputs,
    modes and errors, put back in head order, equal the one-rank layer."""
    from oracle import svg_oracle as O
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_shard_layer_main, args=(world, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    parts = results["parts"]
    assert [(p[0], p[1]) for p in parts] == [(0, 2), (2, 3)]
    wl = si.small("hunyuan720").scaled("shard-test", H=3)
    q, k, v, _ = si.generate(wl)
    o, mode, mse = O.svg_layer(*(si.as_float64(t) for t in (q, k, v)), si.sample_queries(wl),
                               wl.F, wl.P, wl.width)
    np.testing.assert_array_equal(np.concatenate([p[2] for p in parts], axis=1), o)
    np.testing.assert_array_equal(np.concatenate([p[3] for p in parts]), mode)
    np.testing.assert_array_equal(np.concatenate([p[4] for p in parts]), mse)
    assert set(mode.tolist()) == {0, 1}  # both kinds of heads occur


def test_rank_inputs_differ():
    wl = si.small("cogvideox")
    a = si.generate(wl, seed=bench.rank_seed(wl, 0))[0]
    b = si.generate(wl, seed=bench.rank_seed(wl, 1))[0]
    assert a.shape == b.shape and (a != b).any()


def test_reference_arm_under_torchrun_prints_once():
    """torchrun with 2 ranks: rank 0 alone runs the oracle and prints one JSON
    line carrying the contract's keys; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--cpu-budget", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "hunyuan720"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0


def test_traffic_tracks_kernel_sources(monkeypatch):
    """DRAM traffic is reported only for the kernel sources it was measured on."""
    rec = bench.ATTN_TRAFFIC["hunyuan720"]
    monkeypatch.setattr(bench, "attn_sources_sha256", lambda: rec["sha256"])
    assert bench.attn_traffic("hunyuan720") == rec["bytes"]
    assert bench.attn_traffic("wan480") is None
    monkeypatch.setattr(bench, "attn_sources_sha256", lambda: "0" * 64)
    assert bench.attn_traffic("hunyuan720") is None


def test_host_chunk_divides_the_heads():
    for bh, want in ((24, 4), (40, 4), (48, 4), (7, 1), (6, 3), (3, 3), (1, 1), (12, 4)):
        assert bench.host_chunk(bh) == want
        assert bh % bench.host_chunk(bh) == 0


def test_recorded_traffic_matches_the_sources():
    """The recorded capture belongs to the attention sources in the tree."""
    for name in ("hunyuan720", "wan720"):
        assert bench.attn_traffic(name) == bench.ATTN_TRAFFIC[name]["bytes"]


def test_effective_flops_count_the_element_mask():
    # the metric's work 4 d sum(kept pairs): kept pairs equal the number of
    # (query, key) elements the oracle's block mask keeps, ragged tiles
    # counted by their valid rows and columns
    from oracle import svg_oracle as O
    for name in ("cogvideox", "hunyuan720"):
        wl = si.small(name)
        for kind in (O.MODE_SPATIAL, O.MODE_TEMPORAL, O.MODE_DENSE):
            ip, ix = O.geometric_block_lists(kind, wl.F, wl.P, wl.width, wl.N)
            want = int(O.block_mask_from_lists(ip, ix, wl.N).sum())
            assert bench.kept_pairs(ip, ix, wl.N) == want
    ip, ix = O.geometric_block_lists(O.MODE_DENSE, 1, 300, 0, 300)
    assert bench.kept_pairs(ip, ix, 300) == 300 * 300


def test_clock_samples_summary():
    # nvidia-smi rows: index, clocks.sm, clocks.max.sm, power.draw, active mask,
    # hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    lines = ["0, 1965, 1965, 612.3, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
             "0, 1950, 1965, 998.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
             "0, 1890, 1965, 1001.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
             "garbage line\n"]
    got = bench.parse_clock_samples(lines)
    assert got["sm_mhz"] == 1950 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["reasons"] == ["sw_power_cap"]
    hot = lines[:1] + ["0, 1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n"]
    assert bench.parse_clock_samples(hot)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_samples([])["reasons"] == ["no samples"]
