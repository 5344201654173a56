"""Work partitions across ranks (host logic, CPU): every unit is assigned to
exactly one rank, the cost spread stays within the stated bounds, and two
gloo ranks that each compute their own share cover the work exactly once."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from cross_model_attention_block_b200 import partition as part
from cross_model_attention_block_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _blocks(ranges):
    return [q for a, b in ranges for q in range(a, b)]


@pytest.mark.parametrize("nqb", [1, 2, 3, 7, 8, 64, 255, 256])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_covers_every_query_block_once(nqb, world):
    seen = []
    costs = []
    for r in range(world):
        rg = part.zigzag_ranges(nqb, world, r)
        assert all(a < b for a, b in rg)
        assert all(rg[i][1] < rg[i + 1][0] for i in range(len(rg) - 1))  # disjoint, merged
        assert len(rg) <= 2
        seen += _blocks(rg)
        costs.append(part.ranges_cost(rg))
    assert sorted(seen) == list(range(nqb))
    # runs differ by at most one pair (nqb + 1 units); the middle block of an
    # odd nqb adds at most nqb // 2 + 1 more
    assert max(costs) - min(costs) <= (nqb + 1) + (nqb // 2 + 1)


def test_zigzag_is_exactly_balanced_on_the_32k_workload():
    w = synth.workloads()["large_bf16_n32768"]
    nqb = w.lengths[0] // w.B
    for world in (2, 4, 8):
        costs = {part.ranges_cost(part.zigzag_ranges(nqb, world, r)) for r in range(world)}
        assert costs == {nqb * (nqb + 1) // 2 // world}
    assert part.zigzag_ranges(256, 8, 0) == [(0, 16), (240, 256)]
    assert part.zigzag_ranges(256, 8, 7) == [(112, 144)]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_sequences_balanced_by_causal_cost(world):
    w = synth.workloads()["varlen_paged_64seq"]
    shares = [part.balance_sequences(w.lengths, world, r) for r in range(world)]
    assert sorted(i for s in shares for i in s) == list(range(len(w.lengths)))
    loads = [sum(part.sequence_cost(w.lengths[i]) for i in s) for s in shares]
    # greedy longest-first: the spread is at most the largest single cost
    assert max(loads) - min(loads) <= max(part.sequence_cost(L) for L in w.lengths)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_layers_keep_receivers_with_their_sender_cache(world):
    w = synth.workloads()["multi_receiver_n16384"]
    senders, readers = [], []
    for r in range(world):
        s, rl = part.layer_split(w.sender_layers, w.receivers, world, r)
        senders += s
        readers += rl
        for rec, layer in rl:
            assert w.receivers[rec][2][layer] in s  # co-located with its cache
    assert sorted(senders) == list(range(w.sender_layers))
    want = sorted((r, l) for r, (_, n, _) in enumerate(w.receivers) for l in range(n))
    assert sorted(readers) == want


def test_lpt_rejects_no_ranks():
    with pytest.raises(ValueError):
        part.lpt([1, 2], 0)
    with pytest.raises(ValueError):
        part.zigzag_ranges(8, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime
    from cross_model_attention_block_b200 import partition as pt
    from cross_model_attention_block_b200 import synth as sy
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w2 = sy.workloads()["large_bf16_n32768"]
        w4 = sy.workloads()["varlen_paged_64seq"]
        mine = (pt.zigzag_ranges(w2.lengths[0] // w2.B, world, rank),
                pt.balance_sequences(w4.lengths, world, rank))
        got = [None] * world
        dist.all_gather_object(got, mine)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_cover_the_work_once():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]                      # every rank sees the same split
    blocks = sorted(q for rg, _ in res[0] for a, b in rg for q in range(a, b))
    assert blocks == list(range(256))
    seqs = sorted(i for _, s in res[0] for i in s)
    assert seqs == list(range(64))
