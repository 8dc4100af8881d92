"""The attention forward's work schedule, checked on the CPU through the C ABI
(ag_attn_fwd_schedule runs the library's own host-side planner; no GPU).

The unit of work is a pair of 16-position query blocks of one batch item
over its n_kt = ceil(L/128) key tiles.  Whatever the schedule, every pair
must be computed exactly once over every key tile, and no cluster may get
more than the planner's bound.
"""
import ctypes
import math

import pytest

I = ctypes.c_int


@pytest.fixture(scope="module")
def lib():
    import long_context_genomics_b200 as ag

    return ag.lib


def schedule(lib, B, L, pairs, with_scratch=0):
    out = [I() for _ in range(6)]
    wb, fb = (I * 129)(), (I * 129)()
    st = lib.ag_attn_fwd_schedule(ctypes.c_int64(B), ctypes.c_int64(L), pairs, with_scratch,
                                  *[ctypes.byref(x) for x in out], wb, fb)
    assert st == 0, st
    sched, clusters, tail, whole, n_whole, split_at = (x.value for x in out)
    return dict(sched=sched, clusters=clusters, tail=tail, whole=whole, n_whole=n_whole,
                split_at=split_at, wb=list(wb), fb=list(fb))


def sizes(B, L):
    nb = -(-L // 16)
    return B * ((nb + 1) // 2), -(-L // 128)


CASES = [(1, 1), (1, 16), (1, 512), (1, 1040), (1, 2048), (3, 400), (1, 4096), (1, 6144),
         (1, 8192), (2, 8192), (1, 10000), (2, 2064), (4, 8192), (1, 65536)]


@pytest.mark.parametrize("B,L", CASES)
@pytest.mark.parametrize("pairs", [74, 66, 13, 1])
def test_no_scratch_schedule_covers_every_step_once(lib, B, L, pairs):
    """Whole pairs and first pieces in the first launch, second pieces in the
    second: every (pair, key tile) step exactly once."""
    s = schedule(lib, B, L, pairs)
    items, n_kt = sizes(B, L)
    assert s["sched"] == 1
    cl, tail, nw, a = s["clusters"], s["tail"], s["n_whole"], s["split_at"]
    assert 1 <= cl <= min(pairs, 128) and 0 <= tail <= min(pairs, 128)
    wb, fb = s["wb"], s["fb"]
    assert wb[0] == 0 and fb[0] == 0
    assert all(wb[c] <= wb[c + 1] and fb[c] <= fb[c + 1] for c in range(cl))
    assert wb[cl] == nw and fb[cl] == items - nw == tail
    if tail:
        assert 0 < a < n_kt
    steps = [0] * (items * n_kt)
    for c in range(cl):
        for item in range(wb[c], wb[c + 1]):
            for j in range(n_kt):
                steps[item * n_kt + j] += 1
        for sp in range(fb[c], fb[c + 1]):
            for j in range(a):
                steps[(nw + sp) * n_kt + j] += 1
    for c in range(tail):  # second launch: one second piece per cluster
        for j in range(a, n_kt):
            steps[(nw + c) * n_kt + j] += 1
    assert all(v == 1 for v in steps)


SEG_COST = 5   # the planner's cost of one segment, in key-tile steps
TAIL_COST = 4  # and of the second launch's start


@pytest.mark.parametrize("B,L", CASES)
def test_no_scratch_schedule_is_never_worse_than_whole_pairs(lib, B, L):
    """Two phases are chosen only when their critical path (first launch's
    busiest cluster plus the second piece, every segment counted SEG_COST
    steps longer) beats whole pairs."""
    items, n_kt = sizes(B, L)
    s = schedule(lib, B, L, 74)
    whole_cost = math.ceil(items / 74) * (n_kt + SEG_COST)
    cl, wb, fb, a = s["clusters"], s["wb"], s["fb"], s["split_at"]
    first = max((wb[c + 1] - wb[c]) * (n_kt + SEG_COST) + (fb[c + 1] - fb[c]) * (a + SEG_COST)
                for c in range(cl))
    cost = first + (n_kt - a + SEG_COST + TAIL_COST if s["tail"] else 0)
    assert cost <= whole_cost
    if not s["tail"]:
        assert first == whole_cost


def test_full_context_schedule_on_a_b200(lib):
    """L = 8192, B = 1 on 74 SM pairs: 256 pairs do not divide over 74, so
    whole pairs would cost 4 x 64 = 256 key-tile steps on the busiest pair;
    the two-phase schedule costs 192 + 34 (the ideal is 16384 / 74 = 221.4),
    with at most 4 segments on a cluster of the first launch."""
    s = schedule(lib, 1, 8192, 74)
    assert s["tail"] == 74 and s["split_at"] == 30 and s["n_whole"] == 182
    loads = [(s["wb"][c + 1] - s["wb"][c]) * 64 + (s["fb"][c + 1] - s["fb"][c]) * 30
             for c in range(s["clusters"])]
    segs = [(s["wb"][c + 1] - s["wb"][c]) + (s["fb"][c + 1] - s["fb"][c])
            for c in range(s["clusters"])]
    assert max(loads) == 192 and max(segs) == 4
    # L = 4096: 128 pairs of 32 steps; cutting them would add segments that
    # cost more than they balance, so whole pairs (2 per cluster).
    s1 = schedule(lib, 1, 4096, 74)
    assert s1["tail"] == 0 and s1["clusters"] == 74
    # The nine-layer stack's B = 2 divides almost evenly (512 / 74 = 6.92): whole pairs.
    s2 = schedule(lib, 2, 8192, 74)
    assert s2["tail"] == 0 and s2["clusters"] == 74


@pytest.mark.parametrize("B,L", [(1, 512), (1, 1024), (1, 8192), (2, 8192), (3, 400)])
def test_range_schedule_of_the_noalloc_entry_point(lib, B, L):
    """ag_attn_fwd_noalloc's range schedule: contiguous runs of steps, one per
    cluster, rounded to whole pairs only when that costs the busiest cluster
    less than half a pair."""
    items, n_kt = sizes(B, L)
    s = schedule(lib, B, L, 74, with_scratch=1)
    assert s["sched"] == 0
    assert 1 <= s["clusters"] <= 74
    if s["whole"]:
        assert math.ceil(items / s["clusters"]) - items / s["clusters"] <= 0.5
    else:
        assert s["clusters"] == min(74, items * n_kt)


def test_schedule_argument_checks(lib):
    wb, fb = (I * 129)(), (I * 129)()
    outs = [I() for _ in range(6)]
    ptrs = [ctypes.byref(x) for x in outs]
    assert lib.ag_attn_fwd_schedule(1, 512, 74, 0, *ptrs, None, fb) == 1   # AG_ERR_NULL
    assert lib.ag_attn_fwd_schedule(1, 512, 0, 0, *ptrs, wb, fb) == 2     # AG_ERR_SHAPE
    assert lib.ag_attn_fwd_schedule(0, 512, 74, 0, *ptrs, wb, fb) == 2
    assert lib.ag_attn_fwd_schedule(1, 70000, 74, 0, *ptrs, wb, fb) == 4  # AG_ERR_UNSUPPORTED
