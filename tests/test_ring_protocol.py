"""Model check, on the CPU, of the single-token kernel's weight ring.

One producer lane fills nslot shared-memory slots with a layer's items: the
CTA's gate/up tiles first, then its down batches.  Items past the ring reuse
the slot of a gate/up tile of the same layer once every gate/up warp has
arrived on that slot's "empty" barrier.  Consumers wait on a slot's "full"
barrier with the parity that the item's position in the ring gives.  The
compute warps pass a CTA barrier between gate/up and down and another at the
end of the layer; a layer's first fills wait for their "route" arrival, made
after the previous layer's end.  The host plan admits a shape only when the
gate/up tiles fit the ring and so do the down batches, so an item past the
ring always replaces a gate/up tile.

An mbarrier wait is modelled by its parity test: a wait for parity P passes
once the barrier's completed phase count k has (k & 1) != P, so a fresh
barrier passes a wait for parity 1 at once.  A random scheduler interleaves the
producer, the compute warps and the landing of the copies in flight.  Checked:
each item is read from its slot while that slot holds it (never before its copy
lands, never after a refill), the producer reuses a slot only after every
gate/up warp is done with it, and no schedule deadlocks.  Two planted mistakes
(the wrong empty phase, no barrier after gate/up) are caught.
"""
import random


def ring_slot(s0, p0, q, nslot):
    """Slot of item q of a layer whose first item sits in slot s0 (fill parity p0)."""
    sq, par = s0 + q, p0
    while sq >= nslot:
        sq -= nslot
        par ^= 1
    return sq, par


def run(nslot, layers, gw, nw, per_slot, rng, empty_parity_flip=0, skip_gate_up_barrier=False):
    """One kernel's worth of layers; layers = [(gate/up items, down units)].
    nw compute warps, the first gw of which compute every gate/up item; down
    units go per_slot to a ring item and to warps w, w + nw, ...  The two
    arguments after rng plant a mistake: the other phase of the empty barrier
    in the producer, or no CTA barrier between gate/up and down."""
    full = [0] * nslot          # completed fill phases per slot
    empty = [0] * nslot         # completed "every gate/up warp is done" phases per slot
    content = [None] * nslot    # item whose copy has landed in the slot
    landing = []                # copies issued but not landed: (slot, item)
    gu_cnt = [0] * nslot        # gate/up items the producer issued into each slot
    arrivals = {}               # (slot, empty phase) -> gate/up warps that arrived
    route = [0]                 # layers whose "route" arrival the compute warps made

    def items(n_gu, n_dn):
        return n_gu + (n_dn + per_slot - 1) // per_slot

    def producer():
        s0, p0 = 0, 0
        for l, (n_gu, n_dn) in enumerate(layers):
            yield ("wait_route", l)
            n_items = items(n_gu, n_dn)
            for q in range(n_items):
                s, _ = ring_slot(s0, p0, q, nslot)
                if q >= nslot:   # the slot's previous item is a gate/up tile of this layer
                    yield ("wait_empty", s, ((gu_cnt[s] & 1) ^ 1) ^ empty_parity_flip)
                yield ("issue", s, (l, q))
                if q < n_gu:
                    gu_cnt[s] += 1
            s0, p0 = ring_slot(s0, p0, n_items, nslot)

    def compute_warp(w):
        s0, p0 = 0, 0
        for l, (n_gu, n_dn) in enumerate(layers):
            if w == 0:
                yield ("arrive_route", l)   # the experts are chosen; the producer may start
            if w < gw:
                for q in range(n_gu):
                    s, par = ring_slot(s0, p0, q, nslot)
                    yield ("wait_full", s, par, (l, q))
                    yield ("read", s, (l, q))
                    yield ("arrive_empty", s)
            if not skip_gate_up_barrier:
                yield ("barrier", (l, "gate/up done"))
            for nl in range(w, n_dn, nw):
                q = n_gu + nl // per_slot
                s, par = ring_slot(s0, p0, q, nslot)
                yield ("wait_full", s, par, (l, q))
                yield ("read", s, (l, q))
            yield ("barrier", (l, "layer done"))
            s0, p0 = ring_slot(s0, p0, items(n_gu, n_dn), nslot)

    agents = [producer()] + [compute_warp(w) for w in range(nw)]
    pending = [next(a, None) for a in agents]

    def can_run(st):
        if st[0] == "wait_route":
            return route[0] > st[1]
        if st[0] == "wait_empty":
            return (empty[st[1]] & 1) != st[2]
        if st[0] == "wait_full":
            return (full[st[1]] & 1) != st[2]
        if st[0] == "barrier":   # every compute warp has reached it
            return all(p == st for p in pending[1:])
        return True

    while any(p is not None for p in pending) or landing:
        ready = [i for i, p in enumerate(pending) if p is not None and can_run(p)]
        if landing and (not ready or rng.random() < 0.3):
            s, item = landing.pop(rng.randrange(len(landing)))   # copies land in any order
            content[s] = item
            full[s] += 1
            continue
        assert ready, f"deadlock: pending {pending}"
        i = rng.choice(ready)
        st = pending[i]
        if st[0] == "barrier":   # all compute warps leave it together
            for j in range(1, len(agents)):
                pending[j] = next(agents[j], None)
            continue
        if st[0] == "arrive_route":
            route[0] += 1
        elif st[0] == "wait_empty":
            s = st[1]
            assert empty[s] == gu_cnt[s], f"slot {s} reused after {empty[s]} of {gu_cnt[s]} gate/up items"
        elif st[0] == "issue":
            s = st[1]
            assert all(ls != s for ls, _ in landing), f"slot {s} refilled while a copy is in flight"
            landing.append((s, st[2]))
        elif st[0] == "wait_full":
            s, item = st[1], st[3]
            assert content[s] == item, f"wait on slot {s} passed holding {content[s]}, wanted {item}"
        elif st[0] == "read":
            s, item = st[1], st[2]
            assert content[s] == item and all(ls != s for ls, _ in landing), \
                f"slot {s} read for {item} while it holds {content[s]} or is being refilled"
        elif st[0] == "arrive_empty":
            key = (st[1], empty[st[1]])
            arrivals.setdefault(key, set()).add(i)
            if len(arrivals[key]) == gw:
                empty[st[1]] += 1
        pending[i] = next(agents[i], None)


def random_plan(rng):
    """A ring and a layer sequence that the host plan admits: a layer's gate/up
    tiles fit the ring, and so do its down batches."""
    nslot, per_slot = rng.randint(2, 8), rng.randint(1, 3)
    layers = []
    for _ in range(rng.randint(1, 5)):
        layers.append((rng.randint(0, nslot), rng.randint(0, nslot * per_slot)))
    return nslot, per_slot, layers


def test_ring_items_reach_their_consumers():
    rng = random.Random(2024)
    for _ in range(400):
        nslot, per_slot, layers = random_plan(rng)
        nw = rng.randint(1, 5)
        run(nslot, layers, gw=rng.randint(1, nw), nw=nw, per_slot=per_slot, rng=rng)


def _caught(rng, **mistake):
    caught = 0
    for _ in range(200):
        nslot, per_slot = rng.randint(2, 6), rng.randint(1, 2)
        layers = [(nslot, nslot * per_slot)] * 2   # every layer overflows the ring
        nw = rng.randint(2, 4)
        try:
            run(nslot, layers, gw=rng.randint(1, nw), nw=nw, per_slot=per_slot, rng=rng, **mistake)
        except AssertionError:
            caught += 1
    return caught


def test_wrong_empty_parity_would_be_caught():
    """The checker is not vacuous: a producer that waits on the other phase of
    the empty barrier refills slots that gate/up warps still read."""
    assert _caught(random.Random(99), empty_parity_flip=1) > 0


def test_down_waits_rely_on_the_gate_up_barrier():
    """A down item in a slot's second fill of a layer waits for parity 1; without
    the CTA barrier after gate/up that wait can pass on the slot's fresh phase,
    before even its gate/up copy has landed."""
    assert _caught(random.Random(5), skip_gate_up_barrier=True) > 0
