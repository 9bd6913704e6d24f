"""CPU model check of the few-token decode kernel's weight ring (decode_multi.cu).

One CTA, one layer, random interleavings of the producer (fills items in
order, refilling a slot once its previous item is consumed) and the compute
warps:

* gate/up items: one unit each, cut into k-group chunks (two in the kernel); the CTA's
  chunks go round-robin to all warps, and the last chunk of a unit to finish
  frees its slot;
* down items: batches of units; units go round-robin to all warps, the warp
  that finishes an item's last unit frees the slot;
* before waiting on a slot, a unit's warp waits until every earlier item of
  that slot is consumed, so the fill parity it waits on names its own item;
* every warp finishes its gate/up units before any down unit starts (the
  kernel's barrier and its grid-wide h exchange).

mbarriers are modelled with their phase-parity semantics (a wait on parity P
passes once the phase with parity P has completed, i.e. while the current
phase parity differs from P).  The check: every run finishes, and every
consumer reads the fill it expects.  Two planted mistakes show the check is
not vacuous: without the wait on the slot's earlier items a unit reads an
older fill (or the run stalls), a slot freed by the first unit of an item
instead of the last lets the producer overwrite units still being read, and
a gate/up slot freed by the first chunk of a unit does the same.
"""
import random

import pytest


class MBar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def try_wait(self, parity):
        return (self.phase & 1) != parity


class Stale(AssertionError):
    pass


def gu_parts(n_gu, nkg, NW, nch=2):
    """Per warp, its (unit, chunks of that unit) list in processing order: unit q is cut into nch
    k-group chunks and the CTA's chunk c goes to warp c % NW."""
    plan = [[] for _ in range(NW)]
    for ch in range(n_gu * nch):
        plan[ch % NW].append((ch // nch, nch))
    return plan


def run(nslot, n_gu, n_dn, dps, NW=12, seed=0, gate_on_earlier=True, free_on_last=True, nkg=40,
        gu_free_on_last=True, nch=2):
    rnd = random.Random(seed)
    full = [MBar(1) for _ in range(nslot)]
    empty = [MBar(1) for _ in range(nslot)]
    ccnt, icnt = [0] * nslot, [0] * nslot
    n_dn_items = (n_dn + dps - 1) // dps
    n_items = n_gu + n_dn_items
    content = [None] * nslot           # item in the slot
    reading = [0] * nslot              # units of the slot's item still being read
    prod = {"q": 0, "fpar": 0, "filled": 0}

    def slot(a):
        return a % nslot, (a // nslot) & 1, a // nslot

    plan = gu_parts(n_gu, nkg, NW, nch)
    pcnt = {}
    warps = [{"ph": "gu", "j": 0, "u": w, "busy": None} for w in range(NW)]
    for _ in range(400000):
        actors = (["p"] if prod["q"] < n_items else []) + [w for w in range(NW) if warps[w]["ph"] != "done"]
        if not actors:
            return True
        rnd.shuffle(actors)
        moved = False
        for a in actors:
            if a == "p":
                q = prod["q"]
                s, _, _ = slot(q)
                if (prod["filled"] >> s) & 1 and not empty[s].try_wait(((prod["fpar"] >> s) & 1) ^ 1):
                    continue
                if reading[s]:
                    raise Stale(f"slot {s} refilled while {reading[s]} unit(s) still read it")
                content[s] = q
                full[s].arrive()
                prod["fpar"] ^= 1 << s
                prod["filled"] |= 1 << s
                prod["q"] += 1
                moved = True
                break
            ws = warps[a]
            if ws["ph"] == "gu":
                if ws["busy"] is not None:            # finish the part being read
                    s, q, nparts = ws["busy"]
                    reading[s] -= 1
                    pcnt[q] = pcnt.get(q, 0) + 1
                    # planted mistake: the first chunk of a unit to finish frees the slot
                    if pcnt[q] == (nparts if gu_free_on_last else 1):
                        ccnt[s] += 1
                        empty[s].arrive()
                    ws["busy"] = None
                    ws["j"] += 1
                    moved = True
                    break
                if ws["j"] >= len(plan[a]):
                    ws["ph"] = "wait"
                    moved = True
                    break
                q, nparts = plan[a][ws["j"]]
                s, par, fill = slot(q)
                if gate_on_earlier and ccnt[s] < fill:
                    continue
                if not full[s].try_wait(par):
                    continue
                if content[s] != q:
                    raise Stale(f"gate/up unit {q} read slot {s} holding item {content[s]}")
                reading[s] += 1
                ws["busy"] = (s, q, nparts)
                moved = True
                break
            if ws["ph"] == "wait":
                if all(w["ph"] != "gu" for w in warps):
                    ws["ph"] = "dn"
                    moved = True
                    break
                continue
            if ws["ph"] == "dn":
                if ws["busy"] is not None:            # finish the unit being read
                    s, it, cnt = ws["busy"]
                    reading[s] -= 1
                    icnt[s] += 1
                    if free_on_last and icnt[s] == cnt:
                        icnt[s] = 0
                        ccnt[s] += 1
                        empty[s].arrive()
                    ws["busy"] = None
                    ws["u"] += NW
                    moved = True
                    break
                u = ws["u"]
                if u >= n_dn:
                    ws["ph"] = "done"
                    moved = True
                    break
                it = u // dps
                cnt = min(dps, n_dn - it * dps)
                s, par, fill = slot(n_gu + it)
                if gate_on_earlier and ccnt[s] < fill:
                    continue
                if not full[s].try_wait(par):
                    continue
                if content[s] != n_gu + it:
                    raise Stale(f"down item {it} read slot {s} holding item {content[s]}")
                reading[s] += 1
                if not free_on_last and u % dps == 0:   # planted: the first unit frees the slot
                    ccnt[s] += 1
                    empty[s].arrive()
                ws["busy"] = (s, it, cnt)
                moved = True
                break
        if not moved:
            return False
    return False


CASES = [(5, 32, 81, 5), (5, 33, 81, 5), (7, 8, 20, 5), (5, 8, 4, 5), (8, 21, 52, 5),
         (5, 10, 90, 5), (2, 4, 30, 5), (3, 1, 13, 4), (5, 8, 60, 1), (6, 3, 70, 2),
         (8, 7, 19, 5), (5, 36, 88, 5), (4, 13, 40, 5), (2, 2, 5, 5)]


@pytest.mark.parametrize("n_gu", [1, 2, 5, 7, 8, 11, 12, 13, 24, 35])
def test_gate_up_chunks_cover_every_step_once(n_gu):
    """The kernel's chunk bounds kb = j nkg / GU_CH, ke = (j + 1) nkg / GU_CH tile every unit's k groups."""
    for nch in (2, 4):
        for nkg in (4, 5, 40, 48):
            steps = []
            for j in range(nch):
                steps += list(range(j * nkg // nch, (j + 1) * nkg // nch))
            assert steps == list(range(nkg))
        plan = gu_parts(n_gu, 40, 12, nch)
        assert sorted(q for w in plan for q, _ in w) == sorted(q for q in range(n_gu) for _ in range(nch))


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("nch", [2, 4])
def test_ring_protocol_completes_and_reads_the_right_fill(case, nch):
    for seed in range(25):
        assert run(*case, seed=seed, nch=nch)


def test_planted_no_wait_on_earlier_items_is_caught():
    caught = 0
    for seed in range(25):
        try:
            # one-unit items: a warp's next unit is twelve items on, past a whole turn of the ring
            ok = run(5, 8, 60, 1, seed=seed, gate_on_earlier=False)
        except Stale:
            ok = False
        caught += not ok
    assert caught > 0


def test_planted_gate_up_slot_freed_by_first_chunk_is_caught():
    caught = 0
    for seed in range(25):
        try:
            ok = run(5, 7, 20, 5, seed=seed, gu_free_on_last=False)
        except (Stale, AssertionError):
            ok = False
        caught += not ok
    assert caught > 0


def test_planted_slot_freed_by_first_unit_is_caught():
    caught = 0
    for seed in range(25):
        try:
            ok = run(5, 8, 40, 5, seed=seed, free_on_last=False)
        except Stale:
            ok = False
        caught += not ok
    assert caught > 0
