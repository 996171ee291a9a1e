"""CPU model of the decode kernel's work partition and merge protocol (host logic, no GPU).

The kernel cuts U = heads * units_per_head units into W contiguous worker ranges
[floor(U x / W), floor(U (x+1) / W)), W <= U.  A worker writes a head's output directly when its
range covers the whole head; otherwise it writes a partial into slot 0 (its first head) or 1 (its
last head) and takes a ticket; the worker drawing ticket (workers touching the head - 1) merges the
partials of workers worker_of(head start) .. worker_of(head end - 1), reading slot 0 of a worker
whose range starts inside the head and slot 1 otherwise.  This model replays that arithmetic with
every arrival order and checks each head is produced exactly once from exactly the partials that
were written.
"""
import itertools
import random


def start(x, U, W):
    return U * x // W


def worker_of(u, U, W):
    return ((u + 1) * W + U - 1) // U - 1


def segments(x, U, W, uph):
    """(head, seg_a, seg_b) of worker x, in order."""
    ub, ue = start(x, U, W), start(x + 1, U, W)
    out = []
    u = ub
    while u < ue:
        h = u // uph
        b = min(ue, (h + 1) * uph)
        out.append((h, u, b))
        u = b
    return out


def replay(heads, uph, W, order_seed):
    U = heads * uph
    assert W <= U
    written = {}          # (worker, slot) -> head
    direct = {}           # head -> count of direct writes
    arrivals = []         # (worker, head) partial arrivals
    for x in range(W):
        ub, ue = start(x, U, W), start(x + 1, U, W)
        assert ub < ue, "every worker owns a unit"
        assert worker_of(ub, U, W) == x and worker_of(ue - 1, U, W) == x
        for (h, a, b) in segments(x, U, W, uph):
            if a == h * uph and b == (h + 1) * uph:
                direct[h] = direct.get(h, 0) + 1
                continue
            slot = 0 if a == ub else 1
            assert (x, slot) not in written
            written[(x, slot)] = h
            arrivals.append((x, h))
    random.Random(order_seed).shuffle(arrivals)
    tickets = {}
    merged = {}
    for (x, h) in arrivals:
        t = tickets.get(h, 0)
        tickets[h] = t + 1
        wf, wl = worker_of(h * uph, U, W), worker_of((h + 1) * uph - 1, U, W)
        if t == wl - wf:
            reads = []
            for y in range(wf, wl + 1):
                sy = 0 if start(y, U, W) >= h * uph else 1
                assert written.get((y, sy)) == h, (h, y, sy)
                reads.append((y, sy))
            merged[h] = merged.get(h, 0) + 1
            assert len(reads) == sum(1 for v in written.values() if v == h)
    for h in range(heads):
        assert direct.get(h, 0) + merged.get(h, 0) == 1, (h, direct.get(h), merged.get(h))
        assert not (direct.get(h) and any(v == h for v in written.values()))


def test_partition_and_merge_many_shapes():
    rng = random.Random(1)
    shapes = [(1, 1, 1), (1, 15, 15), (4, 15, 60), (4, 15, 7), (2048, 71, 1776), (256, 39, 1776),
              (128, 263, 1776), (128, 263, 1184), (3, 5, 14), (7, 3, 20), (1, 1000, 999)]
    for _ in range(200):
        heads = rng.randint(1, 60)
        uph = rng.randint(1, 40)
        W = rng.randint(1, heads * uph)
        shapes.append((heads, uph, W))
    for i, (heads, uph, W) in enumerate(shapes):
        replay(heads, uph, min(W, heads * uph), order_seed=i)


def test_worker_of_is_the_owner():
    for U, W in itertools.product([1, 2, 7, 60, 1000, 12345], [1, 3, 4, 59, 60, 999]):
        if W > U:
            continue
        for u in list(range(min(U, 200))) + [U - 1]:
            x = worker_of(u, U, W)
            assert start(x, U, W) <= u < start(x + 1, U, W)
