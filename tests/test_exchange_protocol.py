"""Model check, on the CPU, of the single-token kernel's cross-CTA exchange
protocol: three arrival counters (logits, h, output parts), each exchange an
add per CTA followed by a wait for the counter to reach the grid size; CTA 0
zeroes the NEXT exchange's counter just before it arrives at the current one,
so the counters never need epochs.

Every CTA runs the kernel's sequence of steps (over several launches, the
counters persisting between them); a random scheduler interleaves the CTAs'
steps one at a time.  Checked: no schedule deadlocks, and whenever a wait
passes, every CTA has made its arrival for that same exchange (a wait can
neither pass early on a stale count nor miss its count because of a zeroing).
"""
import random

LOGITS, H, Y = 0, 1, 2


def cta_steps(cta, launches, layers):
    """The kernel's exchange steps for one CTA, in program order.  Launches on
    one stream are ordered: every CTA of a launch ends before the next starts
    ("end" steps form that boundary)."""
    for n in range(launches):
        if n > 0:
            yield ("end", n - 1)
        for l in range(layers):
            if l > 0:
                yield ("wait", Y, (n, l - 1, Y))
            for kind in (LOGITS, H):
                if cta == 0:
                    yield ("zero", (kind + 1) % 3)
                yield ("arrive", kind, (n, l, kind))
                yield ("wait", kind, (n, l, kind))
            if cta == 0:
                yield ("zero", (Y + 1) % 3)
            yield ("arrive", Y, (n, l, Y))
        if cta == 0:   # the last layer's output is read by CTA 0 only
            yield ("wait", Y, (n, layers - 1, Y))


def _can_run(step, cnt, G, pending):
    if step[0] == "wait":
        return cnt[step[1]] >= G
    if step[0] == "end":   # launch boundary: every CTA has finished that launch
        return all(p is not None and p[0] == "end" for p in pending)
    return True


def run_schedule(G, launches, layers, rng):
    cnt = [0, 0, 0]
    arrived = {}                       # exchange instance -> CTAs that arrived
    progs = [cta_steps(c, launches, layers) for c in range(G)]
    pending = [next(p, None) for p in progs]
    while any(s is not None for s in pending):
        ready = [c for c in range(G) if pending[c] is not None and _can_run(pending[c], cnt, G, pending)]
        assert ready, f"deadlock with counters {cnt} and pending {pending}"
        c = rng.choice(ready)
        step = pending[c]
        if step[0] == "zero":
            cnt[step[1]] = 0
        elif step[0] == "arrive":
            cnt[step[1]] += 1
            arrived.setdefault(step[2], set()).add(c)
        elif step[0] == "wait":
            assert arrived.get(step[2], set()) == set(range(G)), \
                f"CTA {c} passed the wait of {step[2]} before every CTA arrived"
        elif step[0] == "end":   # the next launch starts for every CTA at once
            for o in range(G):
                pending[o] = next(progs[o], None)
            continue
        pending[c] = next(progs[c], None)


def test_counter_exchanges_never_pass_early_and_never_deadlock():
    rng = random.Random(12345)
    for trial in range(400):
        G = rng.choice([2, 3, 5, 8])
        run_schedule(G, launches=rng.choice([1, 2, 3]), layers=rng.choice([1, 2, 4]), rng=rng)


def test_zeroing_the_current_counter_instead_would_be_caught():
    """The checker is not vacuous: a protocol that zeroes the counter it is about
    to arrive at (instead of the next one) loses arrivals and deadlocks."""
    def bad_steps(cta, launches, layers):
        for step in cta_steps(cta, launches, layers):
            if step[0] == "zero":
                yield ("zero", (step[1] + 2) % 3)   # the current exchange's counter
            else:
                yield step

    rng = random.Random(7)
    caught = 0
    for trial in range(200):
        G = 4
        cnt = [0, 0, 0]
        progs = [bad_steps(c, 2, 3) for c in range(G)]
        pending = [next(p, None) for p in progs]
        arrived = {}
        failed = False
        while any(s is not None for s in pending):
            ready = [c for c in range(G) if pending[c] is not None and _can_run(pending[c], cnt, G, pending)]
            if not ready:
                failed = True
                break
            c = rng.choice(ready)
            step = pending[c]
            if step[0] == "zero":
                cnt[step[1]] = 0
            elif step[0] == "arrive":
                cnt[step[1]] += 1
                arrived.setdefault(step[2], set()).add(c)
            elif step[0] == "wait" and arrived.get(step[2], set()) != set(range(G)):
                failed = True
                break
            elif step[0] == "end":
                for o in range(G):
                    pending[o] = next(progs[o], None)
                continue
            pending[c] = next(progs[c], None)
        caught += failed
    assert caught > 0
