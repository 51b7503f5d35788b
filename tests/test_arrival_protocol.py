"""The split-K attention merge protocol ("the last chunk task to arrive
merges"), executed over every interleaving of its events on tiny cases by
oracle/arrival.py: the rules the kernel and the host follow pass, and each
planted mistake -- a wrong merge threshold, a missing release or acquire
half of the arrival atomic, a host that counts the arrivals of a step
wrongly -- is caught."""
import time

import pytest

from oracle import arrival as ar


# positions whose steps have 1, 2 and 3 non-empty chunks with 3 splits (32
# positions per chunk at least), a short step again, then longer ones
POSITIONS = [5, 40, 70, 12, 100, 200]


def test_arrival_counts_follow_the_chunk_rule():
    assert [ar.arrivals(p, 3) for p in POSITIONS] == [0, 2, 3, 0, 3, 3]
    assert ar.chunk_len(201, 3) == 67 and ar.chunk_len(64, 3) == 32
    assert ar.arrivals(2047, 4) == 4 and ar.arrivals(31, 4) == 0


def test_the_protocol_as_built_is_safe_in_every_order():
    t0 = time.time()
    assert ar.check(ar.Protocol(), POSITIONS, 3) is None
    assert ar.check(ar.Protocol(), [40, 70, 100, 130], 4) is None
    assert time.time() - t0 < 60


@pytest.mark.parametrize("proto,what", [
    (ar.Protocol(threshold=0), "0 tasks merged"),
    (ar.Protocol(threshold=-2), "earlier step"),
    (ar.Protocol(release=False), "earlier step"),
    (ar.Protocol(acquire=False), "earlier step"),
    (ar.Protocol(base_rule="splits"), "0 tasks merged"),
    (ar.Protocol(base_rule="always"), "tasks merged"),
])
def test_planted_mistakes_are_caught(proto, what):
    bad = ar.check(proto, POSITIONS, 3)
    assert bad is not None, proto
    assert what in bad[1], bad
