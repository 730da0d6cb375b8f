"""Host model of the fp16 S-stream's barrier schedule (stream_h16.cu).

One CTA of the kernel runs four roles that meet only at mbarriers:
  the S producer   fills S slot s % NSS once the split warps released stage s - NSS;
  the X producer   fills X slot s % NSX once the MMAs of stage s - NSX are done;
  the MMA issuer   runs stage s from A slot s % NT and X slot s % NSX into
                   accumulator set (s / 2) % NT, after the split warps folded
                   that set's previous pair (at the first stage of a pair);
  the split warps  read S slot s % NSS and release it, write A slot s % NT once
                   the MMAs of stage s - NT are done, and at the start of each
                   pair (and after the last stage) fold the previous pair's set.

The model plays these roles in random interleavings and checks that every
schedule finishes (no deadlock), that no wait could mistake an older phase
for the one it waits on (parity aliasing: an mbarrier wait tells phases apart
by parity only), and that no slot or accumulator set is overwritten before
its reader is done.  The ring sizes are read from the kernel source, so a
change there is checked here.  Two planted faults (a missing wait before
the split warps overwrite an A slot, too few completion barriers) must be
caught.  The MMA issuer's wait for a folded accumulator set turns out to be
implied by the stage order (the split warps fold pair g - 2 before they
write the A operand of stage 2g); the model shows that too.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "symmetric_nmf_clustering_b200", "csrc",
                   "stream_h16.cu")


def ring_sizes():
    text = open(SRC).read()
    out = {}
    for name in ("H16_NSS", "H16_NSX", "H16_NT", "H16_NDONE"):
        m = re.search(r"constexpr int %s = (\d+);" % name, text)
        assert m, name
        out[name] = int(m.group(1))
    return out


class Aliasing(AssertionError):
    pass


class Hazard(AssertionError):
    pass


class Barrier:
    def __init__(self, arrivals):
        self.arrivals = arrivals
        self.pending = arrivals
        self.completed = 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.arrivals

    def passed(self, j):
        """A parity wait for completion j (0-based) of this barrier."""
        if self.completed >= j + 2:
            raise Aliasing(f"completion {j} awaited after {self.completed} completions")
        return self.completed > j


def play(ksteps, rings, rnd, fold_wait=True, a_wait=True):
    NSS, NSX, NT, NDONE = rings["H16_NSS"], rings["H16_NSX"], rings["H16_NT"], rings["H16_NDONE"]
    sfull = [Barrier(1) for _ in range(NSS)]
    sempty = [Barrier(1) for _ in range(NSS)]
    xfull = [Barrier(1) for _ in range(NSX)]
    tfull = [Barrier(1) for _ in range(NT)]
    dempty = [Barrier(1) for _ in range(NT)]
    done = [Barrier(1) for _ in range(NDONE)]
    pos = {"s": 0, "x": 0, "mma": 0, "split": 0, "phase": 0}
    s_slot = [None] * NSS       # stage held by each S slot
    x_slot = [None] * NSX
    a_slot = [None] * NT
    d_set = [None] * NT         # pair accumulating in each set
    folded, mma_done = set(), set()

    def s_producer():
        s = pos["s"]
        if s >= ksteps or (s >= NSS and not sempty[s % NSS].passed((s - NSS) // NSS)):
            return False
        if s_slot[s % NSS] is not None:
            raise Hazard(f"S slot refilled with stage {s} before stage {s_slot[s % NSS]} was read")
        s_slot[s % NSS] = s
        sfull[s % NSS].arrive()
        pos["s"] += 1
        return True

    def x_producer():
        s = pos["x"]
        if s >= ksteps or (s >= NSX and not done[(s - NSX) % NDONE].passed((s - NSX) // NDONE)):
            return False
        prev = x_slot[s % NSX]
        if prev is not None and prev not in mma_done:
            raise Hazard(f"X slot refilled with stage {s} under the MMAs of stage {prev}")
        x_slot[s % NSX] = s
        xfull[s % NSX].arrive()
        pos["x"] += 1
        return True

    def mma():
        s = pos["mma"]
        if s >= ksteps:
            return False
        g, first = s // 2, s % 2 == 0
        if not tfull[s % NT].passed(s // NT) or not xfull[s % NSX].passed(s // NSX):
            return False
        if fold_wait and first and g >= NT and not dempty[g % NT].passed(g // NT - 1):
            return False
        if a_slot[s % NT] != s or x_slot[s % NSX] != s:
            raise Hazard(f"MMA of stage {s} read operands of another stage")
        if first:
            prev = d_set[g % NT]
            if prev is not None and prev not in folded:
                raise Hazard(f"pair {g} overwrote the unfolded accumulator of pair {prev}")
            d_set[g % NT] = g
        mma_done.add(s)
        done[s % NDONE].arrive()
        pos["mma"] += 1
        return True

    def fold(s_last):
        g = s_last // 2
        if not done[s_last % NDONE].passed(s_last // NDONE):
            return False
        if d_set[g % NT] != g or any(t not in mma_done for t in range(2 * g, s_last + 1)):
            raise Hazard(f"pair {g} folded before its MMAs were done")
        folded.add(g)
        dempty[g % NT].arrive()
        return True

    def split():
        s, ph = pos["split"], pos["phase"]
        if s == ksteps:
            if ph == 0 and ksteps > 0:
                if not fold(ksteps - 1):
                    return False
                pos["phase"] = 1
                return True
            return False
        if ph == 0:                     # read the stage of S, release the slot
            if not sfull[s % NSS].passed(s // NSS):
                return False
            if s_slot[s % NSS] != s:
                raise Hazard(f"split warps read stage {s_slot[s % NSS]} for stage {s}")
            s_slot[s % NSS] = None
            sempty[s % NSS].arrive()
        elif ph == 1:                   # write A once the MMAs of stage s - NT are done
            if a_wait and s >= NT and not done[(s - NT) % NDONE].passed((s - NT) // NDONE):
                return False
            prev = a_slot[s % NT]
            if prev is not None and prev not in mma_done:
                raise Hazard(f"A slot overwritten with stage {s} under the MMAs of stage {prev}")
            a_slot[s % NT] = s
            tfull[s % NT].arrive()
        else:                           # at the start of a pair, fold the previous one
            if s >= 2 and s % 2 == 0 and not fold(s - 1):
                return False
        pos["phase"] = (ph + 1) % 3
        if pos["phase"] == 0:
            pos["split"] += 1
        return True

    roles = [s_producer, x_producer, mma, split]
    while True:
        rnd.shuffle(roles)
        if not any(role() for role in roles):
            break
    finished = (pos["mma"] == ksteps and pos["split"] == ksteps and
                folded == {t // 2 for t in range(ksteps)})
    return finished


def test_ring_sizes_meet_the_kernel_static_assert():
    r = ring_sizes()
    assert r["H16_NDONE"] > r["H16_NSX"] and r["H16_NDONE"] > r["H16_NT"]
    assert r["H16_NDONE"] % r["H16_NSX"] == 0 and r["H16_NDONE"] % r["H16_NT"] == 0


@pytest.mark.parametrize("ksteps", list(range(0, 14)) + [31])
def test_every_schedule_finishes_without_aliasing_or_hazard(ksteps):
    rings = ring_sizes()
    rnd = random.Random(ksteps)
    for _ in range(200):
        assert play(ksteps, rings, rnd)


def test_model_catches_a_missing_a_slot_wait():
    rings = ring_sizes()
    rnd = random.Random(1)
    with pytest.raises(Hazard):
        for _ in range(500):
            play(12, rings, rnd, a_wait=False)


def test_fold_wait_is_implied_by_the_stage_order():
    rings = ring_sizes()
    rnd = random.Random(3)
    for ksteps in range(0, 14):
        for _ in range(100):
            assert play(ksteps, rings, rnd, fold_wait=False)


def test_model_catches_too_few_completion_barriers():
    # with as many completion barriers as X slots, a waiter can fall two
    # phases behind (or a slot be refilled early)
    rings = dict(ring_sizes())
    rings["H16_NDONE"] = 1
    rnd = random.Random(2)
    with pytest.raises((Aliasing, Hazard)):
        for _ in range(500):
            play(12, rings, rnd)
