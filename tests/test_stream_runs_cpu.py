"""Model check of the attention kernel's stream-mode schedule (CPU only).

In stream mode a CTA walks the Q tiles of its heads (u = CTA, CTA + grid, ...)
two at a time across head boundaries; consecutive rounds whose two tiles share
a head form a run, which loads the head's K/V blocks once when they fit the
ring (`carry`).  This mirrors the cursor and run flags of ``next_round`` in
``csrc/attn_kernel.cuh`` and checks what the kernel's barrier protocol relies
on: a run starts with ``first`` and ends with ``last`` inside one head, every
K/V event loaded is released exactly once, and every tile of the CTA's heads is
visited exactly once.
"""
import itertools

import pytest


def stream_rounds(num_units, nq, grid, cta):
    u, tq = cta, 0
    out = []
    while u < num_units:
        ub, tb = u, tq + 1
        if tb == nq:
            ub, tb = u + grid, 0
        nslots = 2 if ub < num_units else 1
        if nslots == 1:
            ub, tb = u, tq
        shared = ub == u
        t0 = tq
        first = not (shared and nslots == 2 and t0 >= 2)
        last = not (shared and nslots == 2 and t0 + 3 < nq)
        out.append(dict(u=u, ub=ub, t0=t0, t1=tb, nslots=nslots, shared=shared,
                        first=first, last=last))
        u, tq = ub, tb + 1
        if nslots == 1 or tq == nq:
            u = num_units if nslots == 1 else ub + grid
            tq = 0
    return out


def check_cta(num_units, nq, grid, nb, ring, cta):
    carry = nb <= ring
    loaded = released = 0
    run_head = None
    tiles = []
    for x in stream_rounds(num_units, nq, grid, cta):
        tiles.append((x["u"], x["t0"]))
        if x["nslots"] == 2:
            tiles.append((x["ub"], x["t1"]))
        events = nb * (1 if x["shared"] else 2)
        if carry and x["shared"]:
            if x["first"]:
                assert run_head is None
                run_head = x["u"]
                loaded += events
            else:
                assert run_head == x["u"], "a run continues in another head"
            if x["last"]:
                released += events
                run_head = None
        else:
            assert run_head is None, "a run left open before a streamed round"
            loaded += events
            released += events
    assert run_head is None
    assert loaded == released
    heads = sorted({h for h, _ in tiles})
    assert sorted(tiles) == sorted((h, t) for h in heads for t in range(nq))


@pytest.mark.parametrize("nq", [3, 5, 7, 9])
def test_stream_runs_are_consistent(nq):
    for num_units, grid, nb, ring in itertools.product([1, 2, 7, 148, 149, 300, 4096],
                                                       [1, 2, 5, 148], [2, 5, 9], [4, 5, 6]):
        if grid > num_units:
            continue
        for cta in range(grid):
            check_cta(num_units, nq, grid, nb, ring, cta)


def test_runs_at_the_bench_shape():
    # 577 tokens: 5 tiles per head; a CTA's rounds alternate runs of two rounds
    # (tiles 0-1, 2-3 or 1-2, 3-4) with rounds that pair two heads.
    rounds = stream_rounds(4096, 5, 148, 0)
    shared_runs = sum(1 for x in rounds if x["shared"] and x["first"] and not x["last"])
    assert shared_runs >= 20
    assert all(x["first"] and x["last"] for x in rounds if not x["shared"])
