"""The split rule as the host restates it (`bench.split_pieces`, which `bench.py` uses to
report the split partials a step moves): a worked example, and the invariants every split
must keep on random lengths — every page in exactly one piece, each worker's pieces in
sequence order and contiguous, at most its first and last piece shared with another
worker, and whole sequences when the lengths are nearly uniform and fit one per worker.
"""
import random

import pytest

import bench

PAGE = 64


def _lens(pages):
    return [n * PAGE for n in pages]


def test_worked_example():
    # pages 10, 3, 0, 20 with a piece cost of 6 units: units 16, 9, 0, 26 = 51 over three
    # workers, q = ceil(51 / 3) = 17 rounded up to 20.  Sequence 0's pages sit at units
    # [6, 16), sequence 1's at [22, 25), sequence 3's at [31, 51).
    plan = bench.split_pieces(_lens([10, 3, 0, 20]), workers=3, piece_cost=6, whole_slack=-1)
    assert plan == [[(0, 0, 10)], [(1, 0, 3), (3, 0, 9)], [(3, 9, 20)]]


def test_zero_piece_cost_is_the_split_by_pages():
    plan = bench.split_pieces(_lens([10, 3, 0, 20]), workers=3, piece_cost=0, whole_slack=-1)
    # 33 pages, q = 11 rounded up to 12
    assert plan == [[(0, 0, 10), (1, 0, 2)], [(1, 2, 3), (3, 0, 11)], [(3, 11, 20)]]


def test_headline_runs_whole():
    plan = bench.split_pieces([8192] * 64, workers=74)
    assert plan == [[(b, 0, 128)] for b in range(64)]
    assert bench.split_partial_bytes([8192] * 64, 128, 74) == 0


@pytest.mark.parametrize("seed", range(40))
def test_invariants_on_random_lengths(seed):
    rng = random.Random(seed)
    b_n = rng.choice([1, 3, 16, 64, 200])
    workers = rng.choice([1, 2, 7, 74, 148])
    cost = rng.choice([0, 1, 6, 12])
    lens = [rng.choice([0, 1, 63, 64, 65, 4096, rng.randint(0, 20000)]) for _ in range(b_n)]
    pages = [(t + PAGE - 1) // PAGE for t in lens]
    plan = bench.split_pieces(lens, workers, piece_cost=cost, whole_slack=-1)
    assert len(plan) <= workers
    seen = {}
    for w, pieces in enumerate(plan):
        assert [b for b, _, _ in pieces] == sorted({b for b, _, _ in pieces})
        for k, (b, lo, hi) in enumerate(pieces):
            assert 0 <= lo < hi <= pages[b]
            if 0 < k < len(pieces) - 1:
                assert (lo, hi) == (0, pages[b])  # a middle piece is a whole sequence
            for p in range(lo, hi):
                assert (b, p) not in seen
                seen[(b, p)] = w
    assert len(seen) == sum(pages)
    for b, n in enumerate(pages):
        holders = sorted({seen[(b, p)] for p in range(n)})
        assert holders == list(range(holders[0], holders[-1] + 1)) if n else holders == []
