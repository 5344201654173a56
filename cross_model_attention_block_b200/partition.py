"""Work partitions of the hot path over the ranks of one node (host logic).

Every unit of the path is independent (MapFlow article, 163.com, section on the
three system components: block statistics, selection and extraction per
query block; the fused kernel per query row; one sender state per layer), so
ranks share no data-path collective; a partition only decides which units a
rank runs.  Three partitions, one per workload shape:

* one long sequence: query blocks in zig-zag pairs (qb, nqb-1-qb).  Causal
  cost grows with the query block (a row of query block qb reads qb+1 key
  blocks), so every pair costs nqb+1 block units; each rank takes a
  contiguous run of pairs, i.e. one front range and one back range of global
  query blocks, which the *_range entry points take directly;
* one sender state read by several receivers: whole sender layers, each with
  the receiver layers that read it (so a cache never leaves the GPU that
  built it), balanced by cost;
* a packed varlen batch: whole sequences, balanced by causal cost ~ L^2.

Balancing uses the greedy longest-processing-time rule: units in decreasing
cost, each to the currently lightest rank (ties to the lower rank).
"""
from __future__ import annotations


def zigzag_ranges(nqb: int, world: int, rank: int):
    """Global query-block ranges [(begin, end), ...] of `rank` among `world`
    ranks for one sequence of nqb query blocks (ascending, disjoint, merged
    when adjacent).  Pair p = (p, nqb-1-p); pairs are split into contiguous
    runs of near-equal length; with nqb odd the middle block goes to the rank
    whose run ends at the middle (the last rank)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    npairs = nqb // 2
    a = npairs * rank // world
    b = npairs * (rank + 1) // world
    ranges = []
    if b > a:
        ranges.append((a, b))
    back_lo, back_hi = nqb - b, nqb - a
    if rank == world - 1 and nqb % 2 == 1:
        back_lo -= 1                      # the middle block nqb // 2
    if back_hi > back_lo:
        if ranges and ranges[-1][1] == back_lo:
            ranges[-1] = (ranges[-1][0], back_hi)
        else:
            ranges.append((back_lo, back_hi))
    return ranges


def query_block_cost(qb: int) -> int:
    """Causal cost of query block qb of a sequence, in key blocks read."""
    return qb + 1


def ranges_cost(ranges) -> int:
    return sum(query_block_cost(q) for a, b in ranges for q in range(a, b))


def lpt(costs, world: int):
    """Greedy longest-processing-time assignment: unit indices per rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0] * world
    out = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        out[r].append(i)
        load[r] += costs[i]
    return [sorted(x) for x in out]


def sequence_cost(L: int) -> int:
    """Causal (query, key) pairs of a sequence of L tokens."""
    return L * (L + 1) // 2


def balance_sequences(lengths, world: int, rank: int):
    """Indices of the sequences of a packed batch that `rank` runs."""
    return lpt([sequence_cost(int(L)) for L in lengths], world)[rank]


def layer_split(sender_layers: int, receivers, world: int, rank: int,
                compress_cost: float = 1.0, mapped_cost: float = 1.0):
    """(sender layers, [(receiver, layer), ...]) that `rank` runs.

    receivers: [(name, n_layers, layer_table)], layer_table[l] = the sender
    layer receiver layer l reads.  A sender layer costs compress_cost plus
    mapped_cost per receiver layer reading it; the receiver layers go with
    their sender layer."""
    readers = [[] for _ in range(sender_layers)]
    for r, (_, n, table) in enumerate(receivers):
        for l in range(n):
            readers[table[l]].append((r, l))
    costs = [compress_cost + mapped_cost * len(readers[s]) for s in range(sender_layers)]
    mine = lpt(costs, world)[rank]
    return mine, sorted(rl for s in mine for rl in readers[s])
