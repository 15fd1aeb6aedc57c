"""Model check of the sequential scan kernel's hand-off protocol (CPU only).

The sequential kernels (``csrc/scan_rec.cu``) split a CTA into recurrence warps
and I/O warps that hand tiles to each other through ``kTileStages`` shared-
memory stages and named hardware barriers: the producer of a tile executes
``bar.arrive`` and the consumer ``bar.sync``, and a barrier completes when all
of the CTA's threads have arrived (arrivals and syncs both count). There are
no spin loops and nothing polls memory, so the protocol's correctness is a
property of the order of these barrier operations alone. Race detectors are
not available for these kernels here, so this test replays the protocol --
the same per-chunk sequence of barrier operations and tile accesses as the
kernel's two roles -- under many random interleavings of the warps and checks:

* no deadlock: every warp reaches the end;
* every tile read sees the chunk it expects, fully written by all of its
  writers, and no writer overwrites a stage before all of its readers have
  finished with the chunk it holds;
* no barrier is left with arrivals pending when the warps exit.

It also plants protocol mistakes and checks that each one is caught, so the
checker itself is known to detect the failures it claims to rule out.

The model abstracts the warps' work to "begin/end access of tile (kind,
stage)" events; a barrier counts threads exactly as the hardware does
(``count`` threads per phase; a warp contributes 32).
"""
import random

import pytest

TILE_STAGES = 3   # kTileStages in csrc/scan_rec.cu

# The kernel's protocol has two barriers per tile stage s:
#   F(s): the I/O warps have widened the chunk now in stage s (its step and B/C
#         tiles are ready); the recurrence warps sync on it before each chunk;
#   D(s): the recurrence warps are done with the chunk in stage s (its readout
#         partials are ready); the I/O warps sync on it before finishing it.
# The "stage is free again" conditions need no barrier of their own, because
# the I/O warps widen chunk c only after finishing chunk c - S + 1 ... c - S's
# readout (program order), and the recurrence warps finish chunk c before it
# is overwritten: the I/O warps' sync on D(s) for chunk c precedes their
# widening of chunk c + S. PROTOCOL = "fd" checks that; PROTOCOL = "four" is
# the earlier protocol with separate "empty" barriers XE(s) and YE(s).


def rec_warp(n, mut, S, protocol="fd"):
    """One recurrence warp's operations for a sequence of n chunks."""
    for c in range(n):
        s = c % S
        yield ("sync", ("XF", s))
        if protocol == "four" and c >= S and mut != "no_ye_wait":
            yield ("sync", ("YE", s))
        yield ("begin_read", ("X", s), c)
        yield ("begin_write", ("Y", s), c)
        if mut == "yf_before_write":
            yield ("arrive", ("YF", s))
        yield ("end_read", ("X", s), c)
        yield ("end_write", ("Y", s), c)
        if protocol == "four" and (c + S < n or mut == "xe_always"):
            yield ("arrive", ("XE", s))
        if mut != "yf_before_write":
            yield ("arrive", ("YF", s))


def io_warp(n, mut, S, protocol="fd"):
    """One I/O warp's operations: widen chunk c, then finish chunk c - (S - 1)."""
    lag = S - 1 if mut != "finish_lag_s" else S
    for c in range(n):
        s = c % S
        if protocol == "four" and c >= S and mut != "no_xe_wait":
            yield ("sync", ("XE", s))
        if mut == "xf_before_write":
            yield ("arrive", ("XF", s))
        yield ("begin_write", ("X", s), c)
        yield ("end_write", ("X", s), c)
        if mut != "xf_before_write":
            yield ("arrive", ("XF", s))
        j = c - lag
        if j >= 0:
            sf = (j + 1) % S if mut == "finish_wrong_stage" else j % S
            yield ("sync", ("YF", sf))
            yield ("begin_read", ("Y", sf), j)
            yield ("end_read", ("Y", sf), j)
            if protocol == "four" and (j + S < n or (mut == "ye_one_extra" and j + S == n)):
                yield ("arrive", ("YE", sf))
    for j in range(max(n - lag, 0), n):
        sf = j % S
        yield ("sync", ("YF", sf))
        yield ("begin_read", ("Y", sf), j)
        yield ("end_read", ("Y", sf), j)


class Violation(Exception):
    pass


def simulate(n, rec_warps, io_warps, mut=None, stages=TILE_STAGES, seed=0, bias=0.0, protocol="fd"):
    """Run one random interleaving; raise Violation on a protocol error."""
    rng = random.Random(seed)
    S = stages
    procs = [("rec", i, rec_warp(n, mut, S, protocol)) for i in range(rec_warps)] + \
            [("io", i, io_warp(n, mut, S, protocol)) for i in range(io_warps)]
    total = 32 * (rec_warps + io_warps)
    count = {}        # barrier -> threads arrived in the current phase
    waiting = {}      # barrier -> set of blocked process indices
    blocked = set()
    pending = [None] * len(procs)   # next operation of each process
    done = [False] * len(procs)
    writers = {"X": io_warps, "Y": rec_warps}   # warps that write one chunk of a tile
    readers = {"X": rec_warps, "Y": io_warps}
    content = {}      # (kind, stage) -> chunk whose writes have begun
    written = {}      # (kind, stage, chunk) -> writers finished
    reads_done = {}   # (kind, stage, chunk) -> readers finished
    active_r = {}     # (kind, stage) -> readers in progress
    active_w = {}

    def arrive(b, who, block):
        count[b] = count.get(b, 0) + 32
        if block:
            waiting.setdefault(b, set()).add(who)
            blocked.add(who)
        if count[b] == total:
            count[b] = 0
            for w in waiting.pop(b, set()):
                blocked.discard(w)
        elif count[b] > total:  # pragma: no cover - cannot happen with resets
            raise Violation(f"barrier {b} over-arrived")

    def step(i):
        op = pending[i]
        pending[i] = None
        kind = op[0]
        if kind in ("sync", "arrive"):
            arrive(op[1], i, kind == "sync")
            return
        tile, c = op[1], op[2]
        k = tile[0]
        if kind == "begin_write":
            prev = content.get(tile)
            if prev is not None and prev != c:
                if reads_done.get((k, tile[1], prev), 0) < readers[k] or active_r.get(tile, 0):
                    raise Violation(f"{tile} overwritten with chunk {c} before chunk {prev} was read")
            content[tile] = c
            active_w[tile] = active_w.get(tile, 0) + 1
        elif kind == "end_write":
            active_w[tile] -= 1
            written[(k, tile[1], c)] = written.get((k, tile[1], c), 0) + 1
        elif kind == "begin_read":
            if content.get(tile) != c or written.get((k, tile[1], c), 0) < writers[k] or active_w.get(tile, 0):
                raise Violation(f"{tile} read for chunk {c} before it was written")
            active_r[tile] = active_r.get(tile, 0) + 1
        elif kind == "end_read":
            active_r[tile] -= 1
            reads_done[(k, tile[1], c)] = reads_done.get((k, tile[1], c), 0) + 1

    last = None
    while True:
        for i, (_, _, gen) in enumerate(procs):
            if pending[i] is None and not done[i]:
                try:
                    pending[i] = next(gen)
                except StopIteration:
                    done[i] = True
        runnable = [i for i in range(len(procs)) if not done[i] and i not in blocked]
        if not runnable:
            if all(done):
                break
            raise Violation("deadlock")
        # optionally keep running the same warp (lets one role run far ahead)
        i = last if (last in runnable and rng.random() < bias) else rng.choice(runnable)
        last = i
        step(i)
    left = {b: v for b, v in count.items() if v}
    if left:
        raise Violation(f"barriers left with pending arrivals: {left}")


def check_protocol(mut=None, stages=TILE_STAGES, rec_warps=4, io_warps=2, schedules=60, protocol="fd"):
    for n in range(1, 14):
        for k in range(schedules):
            simulate(n, rec_warps, io_warps, mut=mut, stages=stages, seed=1000 * n + k, bias=(k % 4) * 0.3,
                     protocol=protocol)


@pytest.mark.parametrize("io_warps", [2, 4])
@pytest.mark.parametrize("protocol", ["fd", "four"])
def test_protocol_holds(io_warps, protocol):
    """The kernel's protocol (and the earlier four-barrier one), for 1 to 13
    chunks, random interleavings (some biased so that one role runs far ahead
    of the other)."""
    check_protocol(io_warps=io_warps, protocol=protocol)


@pytest.mark.parametrize("mut", ["xf_before_write", "yf_before_write", "finish_wrong_stage", "finish_lag_s"])
def test_planted_mistakes_are_caught(mut):
    """Mistakes in the two-barrier protocol; finishing S chunks behind instead
    of S - 1 lets the I/O warps overwrite a step tile still being read."""
    with pytest.raises(Violation):
        check_protocol(mut=mut)


@pytest.mark.parametrize("mut", ["no_ye_wait", "no_xe_wait", "xe_always", "ye_one_extra"])
def test_planted_mistakes_four_barrier_protocol(mut):
    with pytest.raises(Violation):
        check_protocol(mut=mut, protocol="four")


def test_two_stages():
    """The same protocol with two stages (the I/O warps then finish one chunk
    behind instead of two) is also consistent."""
    check_protocol(stages=2)


@pytest.mark.parametrize("io_warps", [2, 4])
def test_four_stages(io_warps):
    """Four stages (the I/O warps finishing three chunks behind), as the
    kernel's static bound on named barriers allows, with 2 or 4 I/O warps."""
    check_protocol(stages=4, io_warps=io_warps)
