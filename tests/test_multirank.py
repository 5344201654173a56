"""The N > 1 host path of bench.py with two gloo ranks on CPU: rank
environment, the max-over-ranks timing reduction every rank takes part in,
and the reference arm that runs on rank 0 only."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.rank_env()
        # per-rank "timed region" lengths; every rank must see the slowest
        got = bench.max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
        got2 = bench.max_over_ranks(7.0 - rank, w, torch.device("cpu"))
        dist.barrier()
        out[rank] = (r, w, lr, got, got2)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == (0, 2, 0, 15.0, 7.0)
    assert res[1] == (1, 2, 1, 15.0, 7.0)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun every rank but 0 exits 0 without work and prints nothing."""
    sys.path.insert(0, ROOT)
    import bench
    called = []
    monkeypatch.setattr(bench, "bench_reference", lambda args, wl: called.append(wl.name))
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
    assert called == [] and capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
    assert called == ["large_bf16_n32768"]


def test_bench_rank_plans_cover_the_layer_once():
    """bench.py --gpus N: the ranks' query-block ranges cover every query block
    of the layer exactly once (one sequence: zig-zag pairs; varlen batch:
    whole sequences), and their rows and causal pairs add up to the layer's."""
    sys.path.insert(0, ROOT)
    import bench
    from cross_model_attention_block_b200 import synth
    for name in ("large_bf16_n32768", "mid_bf16_n8192", "varlen_paged_64seq"):
        wl = synth.workloads()[name]
        nqb = sum((L + wl.B - 1) // wl.B for L in wl.lengths)
        full_rows, full_pairs = bench.plan_units(wl, [(0, nqb)])
        assert full_rows == wl.ntok
        assert full_pairs == sum(L * (L + 1) // 2 for L in wl.lengths)
        for world in (1, 2, 4, 8):
            plans = [bench.rank_plan(wl, r, world) for r in range(world)]
            blocks = sorted(g for p in plans for a, b in p for g in range(a, b))
            assert blocks == list(range(nqb)), (name, world)
            units = [bench.plan_units(wl, p) for p in plans]
            assert sum(u[0] for u in units) == full_rows
            assert sum(u[1] for u in units) == full_pairs


def test_bench_layer_jobs():
    """bench.py's layers per rank: one-layer workloads run sender 0 and its
    receiver; the multi-receiver workload runs all 8 sender layers and all
    6 + 4 receiver layers at N = 1, and at N > 1 the ranks' sender layers
    cover the 8 once, each receiver layer on the rank of its sender layer."""
    sys.path.insert(0, ROOT)
    import bench
    from cross_model_attention_block_b200 import synth
    w2 = synth.workloads()["large_bf16_n32768"]
    assert bench.layer_jobs(w2, 0, 1) == ([0], [(0, 0, 0)])
    assert bench.layer_jobs(w2, 1, 4) == ([0], [(0, 0, 0)])
    w3 = synth.workloads()["multi_receiver_n16384"]
    s, r = bench.layer_jobs(w3, 0, 1)
    assert s == list(range(8)) and len(r) == 10
    assert all(w3.receivers[rr][2][l] == src for rr, l, src in r)
    for world in (2, 4, 8):
        all_s, all_r = [], []
        for rank in range(world):
            s, r = bench.layer_jobs(w3, rank, world)
            assert all(src in s for _, _, src in r)
            all_s += s
            all_r += [(rr, l) for rr, l, _ in r]
        assert sorted(all_s) == list(range(8))
        assert sorted(all_r) == sorted((rr, l) for rr, (_, n, _) in enumerate(w3.receivers)
                                       for l in range(n))
