"""Model check, on the CPU, of the tensor-core grouped GEMM's pipeline.

Agents, as in the kernel:
  * B producers and A loaders each fill the stage ring (S stages) for every
    k block of every item.  A loaders wait on a stage's "empty" barrier, then
    write it; B producers request a k block's raw codes first (into their own
    buffers, not the stage), then decode the previous k block into its stage
    and publish it, and only then wait on "empty" for the stage of the k block
    just requested (the stage it decodes into next).  Both publish a stage on
    its "full" barrier one k block late and flush the last stage at the end of
    each item.  For an item of a
    cached expert the B producers instead issue one bulk copy of the stage
    image, completing on the stage's "cbar" barrier, and arrive on "full" at
    once; the MMA issuer waits on both.
  * The MMA issuer.  For an item with one or two M=128 accumulators (na) it
    waits until the epilogue has released the TMEM slots it will use: a ring
    of two slots, u counting slot uses, slot u & 1, phase u >> 1.  For each k
    block it waits on "full", issues the MMAs and commits to "empty".  At the
    end of the item it commits to "acc_full" of each slot used.
  * The tensor pipe.  It completes the issued MMAs and commits in order; a
    commit arrives once every earlier MMA has completed.
  * The epilogue.  For each accumulator it waits on "acc_full", reads the slot
    and arrives on "acc_empty".

An mbarrier wait for parity P passes once the barrier's completed phase count
k has (k & 1) != P.  A random scheduler interleaves all of them.  Checked: no
stage is rewritten while an MMA still reads it; an MMA reads a complete stage
of its own k block; no slot is written while the epilogue reads it; the
epilogue reads a finished accumulator of the right item; nothing deadlocks.
"""
import random


def run(items, nk, S, rng, mistake=None, cached=None):
    cached = cached or [False] * len(items)
    full = [0] * S             # completed phases
    empty = [0] * S
    cbar = [0] * S
    acc_full = [0, 0]
    acc_empty = [0, 0]
    full_arrivals = [0] * S    # arrivals in the current phase (2 producer agents)
    stage = [dict(B=None, A=None) for _ in range(S)]   # published content per part
    writing = [set() for _ in range(S)]                 # parts being written now
    reading = [0] * S          # MMAs in flight that read the stage
    slot_item = [None, None]   # (item, accumulator) the slot's MMAs are for
    slot_mma = [0, 0]          # MMAs in flight that write the slot
    slot_done = [None, None]   # (item, accumulator) whose MMAs have all completed
    slot_reading = [False, False]
    pipe = []                  # tensor pipe queue: ("mma", stage, slots) or ("commit", barrier)
    copies = []                # bulk copies in flight: (stage, k block)

    def producer(part):
        it, pending = 0, None
        for i, na in enumerate(items):
            if part == "B" and cached[i]:
                for kb in range(nk):
                    s = it % S
                    yield ("wait", ("empty", s), ((it // S) & 1) ^ 1)
                    yield ("bulk", s, (i, kb))
                    yield ("publish_now", s)
                    it += 1
                continue
            for kb in range(nk):
                s = it % S
                par = ((it // S) & 1) ^ (0 if mistake == "producer_parity" else 1)
                if part == "A":
                    yield ("wait", ("empty", s), par)
                    yield ("write", part, s, (i, kb))
                    if pending is not None:
                        yield ("publish", part, pending)
                else:
                    if pending is not None:   # decode the previous k block into its stage
                        yield ("write", part, pending[0], pending[1])
                        yield ("publish", part, pending)
                    yield ("wait", ("empty", s), par)
                pending = (s, (i, kb))
                it += 1
            if part == "B":
                yield ("write", part, pending[0], pending[1])
            yield ("publish", part, pending)
            pending = None

    def mma():
        it, u = 0, 0
        cpar = [0] * S
        for i, na in enumerate(items):
            for a in range(na):
                par = (((u + a) >> 1) & 1) ^ (0 if mistake == "acc_empty_parity" else 1)
                yield ("wait", ("acc_empty", (u + a) & 1), par)
            slots = [(u + a) & 1 for a in range(na)]
            yield ("claim", slots, i)
            for kb in range(nk):
                s = it % S
                yield ("wait", ("full", s), (it // S) & 1)
                if cached[i] and mistake != "skip_cbar":
                    yield ("wait", ("cbar", s), cpar[s])
                if cached[i]:
                    cpar[s] ^= 1
                yield ("issue", s, (i, kb), slots)
                yield ("commit", ("empty", s))
                it += 1
            for sl in slots:
                yield ("commit", ("acc_full", sl))
            u += na

    def epilogue():
        u = 0
        for i, na in enumerate(items):
            for a in range(na):
                sl = u & 1
                yield ("wait", ("acc_full", sl), (u >> 1) & 1)
                if mistake == "release_before_read":
                    yield ("release", sl)
                    yield ("read", sl, (i, a))
                else:
                    yield ("read", sl, (i, a))
                    yield ("release", sl)
                u += 1

    bars = {"full": full, "empty": empty, "acc_full": acc_full, "acc_empty": acc_empty, "cbar": cbar}
    agents = [producer("B"), producer("A"), mma(), epilogue()]
    pending_step = [next(a, None) for a in agents]
    done_reading = set()

    def can_run(st):
        if st[0] == "wait":
            (name, idx), par = st[1], st[2]
            return (bars[name][idx] & 1) != par
        return True

    def complete(entry):
        if entry[0] == "mma":
            _, s, slots = entry
            reading[s] -= 1
            for sl in slots:
                slot_mma[sl] -= 1
        else:
            name, idx = entry[1]
            bars[name][idx] += 1
            if name == "acc_full":
                slot_done[idx] = slot_item[idx]

    while any(p is not None for p in pending_step) or pipe or copies:
        ready = [j for j, p in enumerate(pending_step) if p is not None and can_run(p)]
        if copies and (not ready or rng.random() < 0.3):
            s, blk = copies.pop(rng.randrange(len(copies)))   # a stage image lands
            writing[s].discard("B")
            stage[s]["B"] = blk
            cbar[s] += 1
            continue
        if pipe and (not ready or rng.random() < 0.35):
            complete(pipe.pop(0))
            continue
        assert ready, f"deadlock: {pending_step}"
        j = rng.choice(ready)
        st = pending_step[j]
        kind = st[0]
        if kind == "write":
            _, part, s, blk = st
            assert reading[s] == 0, f"stage {s} rewritten for {blk} while an MMA reads it"
            writing[s].add(part)
            stage[s][part] = None
        elif kind == "bulk":
            _, s, blk = st
            assert reading[s] == 0, f"stage {s} rewritten for {blk} while an MMA reads it"
            assert all(cs != s for cs, _ in copies), f"stage {s} copied into twice at once"
            writing[s].add("B")
            stage[s]["B"] = None
            copies.append((s, blk))
        elif kind == "publish_now":
            s = st[1]
            full_arrivals[s] += 1
            if full_arrivals[s] == 2:
                full_arrivals[s] = 0
                full[s] += 1
        elif kind == "publish":
            _, part, (s, blk) = st
            writing[s].discard(part)
            stage[s][part] = blk
            full_arrivals[s] += 1
            if full_arrivals[s] == 2:
                full_arrivals[s] = 0
                full[s] += 1
        elif kind == "claim":
            _, slots, i = st
            for a, sl in enumerate(slots):
                assert not slot_reading[sl], f"slot {sl} claimed for item {i} while the epilogue reads it"
                slot_item[sl] = (i, a)
                slot_done[sl] = None
        elif kind == "issue":
            _, s, blk, slots = st
            assert stage[s]["A"] == blk and stage[s]["B"] == blk and not writing[s], \
                f"MMA on stage {s} for {blk}: stage holds {stage[s]}"
            for sl in slots:
                assert not slot_reading[sl], f"slot {sl} written while the epilogue reads it"
                slot_mma[sl] += 1
            reading[s] += 1
            pipe.append(("mma", s, slots))
        elif kind == "commit":
            pipe.append(("commit", st[1]))
        elif kind == "read":
            _, sl, acc = st
            assert slot_done[sl] == acc and slot_mma[sl] == 0, \
                f"epilogue read slot {sl} for {acc}: holds {slot_item[sl]}, finished {slot_done[sl]}"
            done_reading.add(acc)
        elif kind == "release":
            acc_empty[st[1]] += 1
        pending_step[j] = next(agents[j], None)
        # the epilogue holds a slot while its next step reads it, and (in the kernel's order)
        # after the read until it releases the slot
        nxt = pending_step[3]
        slot_reading[0] = slot_reading[1] = False
        if nxt is not None and (nxt[0] == "read" or (nxt[0] == "release" and mistake != "release_before_read")):
            slot_reading[nxt[1]] = True
    assert len(done_reading) == sum(items)


def random_case(rng):
    items = [rng.choice([1, 2]) for _ in range(rng.randint(1, 6))]
    return items, rng.randint(1, 4), rng.randint(2, 4)


def test_pipeline_never_overwrites_and_never_deadlocks():
    rng = random.Random(31)
    for _ in range(500):
        items, nk, S = random_case(rng)
        run(items, nk, S, rng)


def test_pipeline_with_cached_stage_images():
    rng = random.Random(37)
    for _ in range(500):
        items, nk, S = random_case(rng)
        run(items, nk, S, rng, cached=[rng.random() < 0.5 for _ in items])


def test_mma_that_skips_the_image_barrier_would_be_caught():
    rng = random.Random(41)
    caught = 0
    for _ in range(300):
        items, nk, S = random_case(rng)
        try:
            run(items, nk, S, rng, mistake="skip_cbar", cached=[True] * len(items))
        except AssertionError:
            caught += 1
    assert caught > 0


def _caught(mistake, seed):
    rng = random.Random(seed)
    caught = 0
    for _ in range(300):
        items, nk, S = random_case(rng)
        try:
            run(items, nk, S, rng, mistake=mistake)
        except AssertionError:
            caught += 1
    return caught


def test_wrong_slot_release_parity_would_be_caught():
    assert _caught("acc_empty_parity", 1) > 0


def test_releasing_a_slot_before_reading_it_would_be_caught():
    assert _caught("release_before_read", 2) > 0


def test_wrong_stage_empty_parity_would_be_caught():
    assert _caught("producer_parity", 3) > 0
