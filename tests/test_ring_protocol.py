"""The shared-memory ring protocol of the bulk-copy kernels (the W8A8 GEMV and the T <= 8 lm_head), modelled
on the host.

A producer issues one copy per unit into stage i mod nst after the stage's previous unit was released; a copy
lands some time later and completes the stage's full barrier; consumer warp i mod ncons waits on that barrier
with a parity test, reads the stage and releases it.  A parity wait only tells the current phase's parity, so a
waiter two phases ahead of the copies passes early and reads another unit's data.  The kernels avoid this by
giving each stage a single owner warp (nst a multiple of ncons).  This model checks the rule under random
schedules, and shows that the round-robin sharing it replaced (10 stages, 8 warps) does pass early.
"""
import random

import pytest


def _run(nst: int, ncons: int, units: int, rng: random.Random) -> bool:
    """One random schedule; True if some consumer passed its wait before its unit's copy had landed."""
    full_done = [0] * nst      # completed phases of each full barrier
    empty_done = [0] * nst     # completed phases of each empty barrier (one arrival each)
    data = [None] * nst        # the unit whose bytes sit in the stage
    in_flight = []             # (stage, unit) copies issued, not landed
    issued = 0
    nxt = list(range(ncons))   # next unit of each consumer warp
    early = False
    while True:
        moves = []
        if issued < units:
            s = issued % nst
            if issued < nst or empty_done[s] >= issued // nst:
                moves.append(("issue",))
        if in_flight:
            moves.append(("land", rng.randrange(len(in_flight))))
        for c in range(ncons):
            i = nxt[c]
            if i < units:
                s, par = i % nst, (i // nst) & 1
                if (full_done[s] & 1) != par:   # try_wait.parity succeeds
                    moves.append(("consume", c))
        if not moves:
            return early
        mv = rng.choice(moves)
        if mv[0] == "issue":
            in_flight.append((issued % nst, issued))
            issued += 1
        elif mv[0] == "land":
            s, u = in_flight.pop(mv[1])
            data[s] = u
            full_done[s] += 1
        else:
            c = mv[1]
            i = nxt[c]
            s = i % nst
            if full_done[s] < i // nst + 1 or data[s] != i:
                early = True
                return early
            empty_done[s] += 1
            nxt[c] += ncons


@pytest.mark.parametrize("nst,ncons", [(8, 8), (10, 5), (7, 7), (5, 5), (3, 3), (8, 4)])
def test_single_owner_stages_never_pass_early(nst, ncons):
    rng = random.Random(1000 * nst + ncons)
    for _ in range(300):
        assert not _run(nst, ncons, units=4 * nst + 3, rng=rng)


def test_round_robin_sharing_passes_early():
    rng = random.Random(7)
    assert any(_run(10, 8, units=60, rng=rng) for _ in range(300))


def test_the_kernels_keep_the_rule():
    import os
    import re
    root = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "weight_quantized_expert_b200",
                        "csrc")
    w8 = open(os.path.join(root, "w8a8.cu")).read()
    assert "p.nst -= p.nst % p.ncons;" in w8          # the GEMV rounds its stage count to the consumer count
    lm = open(os.path.join(root, "lm_head.cu")).read()
    m = re.search(r"constexpr int RNST = (\d+);", lm)
    assert m and "constexpr int RNC = 2 * RNST;" in lm   # the lm_head pairs own one stage each
