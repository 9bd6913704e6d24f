"""Model check, on the CPU, of the few-token decode kernel's cross-CTA exchanges.

The router logits and h are tagged words: a CTA stores its share as (tag,
value) in one 64-bit store, layer l of a launch carrying tag tag0 + l, and a
reader re-reads until every word it needs carries the tag it expects.  The
layer output goes through fp32 atomics and an arrival counter, cleared by the
host before every launch.  The host advances tag0 by the launch's layer count;
every buffer is reused every layer and across launches.  (The same model with
the output as plain parts behind a counter — "plain" below — shows that the
planted ordering mistake on an output buffer is caught.)

Every CTA runs its kernel's sequence of steps over several launches; a random
scheduler interleaves the CTAs' steps one at a time (a read or a counter wait
is a step that can only run once satisfied).  Checked: no schedule deadlocks;
every word a reader accepts was written for the layer and launch it wants (no
stale word passes for a new one); and no CTA overwrites a word that some CTA
still has to read.  Planted mistakes show the check is not vacuous: one tag for
every layer of a launch, a tag base the host does not advance (one-layer
calls), and a layer's output written before the CTA has read that layer's
logits (so before it knows every CTA has read the previous output).
"""
import random

import pytest


class Stale(AssertionError):
    pass


def steps(kind, cta, launches, L):   # kind: "multi" (the kernel) or "plain" (planted-mistake harness)
    """A CTA's exchange steps in program order: ("w", buf, layer) stores the CTA's words of buf,
    ("r", buf, layer) reads every CTA's words of buf (tagged buffers: once their tags are right;
    plain buffers: after the counter wait), ("arrive"/"wait", buf, layer) a counter, ("end",) the
    launch boundary (stream order)."""
    for n in range(launches):
        if n > 0:
            yield ("end",)
        for l in range(L):
            if l > 0:
                yield ("wait", "y", l - 1)
                if kind == "plain":
                    yield ("r", "y", l - 1)
            yield ("w", "logits", l)
            yield ("r", "logits", l)
            yield ("w", "h", l)
            if kind == "plain":
                yield ("arrive", "h", l)
                yield ("wait", "h", l)
            yield ("r", "h", l)
            if kind == "plain":
                yield ("w", "y", l)
            yield ("arrive", "y", l)
        if kind == "multi" or cta == 0:   # who reads the last layer's output
            yield ("wait", "y", L - 1)
            if kind == "plain":
                yield ("r", "y", L - 1)


def run(kind="plain", G=4, launches=3, L=3, seed=0, tag_per_layer=True, advance_base=True,
        early_output=False):
    rnd = random.Random(seed)
    progs = [list(steps(kind, c, launches, L)) for c in range(G)]
    if early_output:
        # planted: CTA 1 stores each layer's output words before it has read that layer's logits
        p = progs[1]
        for i in range(len(p)):
            if p[i][0] == "w" and p[i][1] == "y":
                j = max(k for k in range(i) if p[k][0] == "r" and p[k][1] == "logits")
                p.insert(j, p.pop(i))
    pc = [0] * G
    launch = [0] * G
    words = {b: [None] * G for b in ("logits", "h", "y")}   # (tag, launch, layer) per CTA's share
    tagged = {"logits"} | ({"h"} if kind == "multi" else set())
    # readers that still have to read each (buf, launch, layer)
    owed = {}

    def tag(n, l):
        b = 1 + (n * L if advance_base else 0)
        return b + (l if tag_per_layer else 0)

    def readers(buf, n, l):
        if buf == "y" and l == L - 1:
            return {0} if kind == "plain" else set()
        return set(range(G))

    cnt = {}
    ended = [set() for _ in range(launches)]
    for _ in range(200000):
        live = [c for c in range(G) if pc[c] < len(progs[c])]
        if not live:
            return True
        rnd.shuffle(live)
        moved = False
        for c in live:
            st = progs[c][pc[c]]
            n = launch[c]
            if st[0] == "end":
                ended[n].add(c)
                if len(ended[n]) < G:
                    continue   # stream order: the next launch starts after every CTA ended
                launch[c] += 1
            elif st[0] == "w":
                _, buf, l = st
                old = words[buf][c]
                if old is not None:
                    left = owed.get((buf,) + old[1:], set())
                    if left:
                        raise Stale(f"CTA {c} overwrote {buf} of launch {old[1]} layer {old[2]} "
                                    f"that CTAs {sorted(left)} still read")
                words[buf][c] = (tag(n, l), n, l)
                owed.setdefault((buf, n, l), set(readers(buf, n, l)))
            elif st[0] == "r":
                _, buf, l = st
                want = tag(n, l)
                if buf in tagged and any(w is None or w[0] != want for w in words[buf]):
                    continue
                for w in words[buf]:
                    if (w[1], w[2]) != (n, l):
                        raise Stale(f"CTA {c} accepted {buf} of launch {w[1]} layer {w[2]} for launch {n} "
                                    f"layer {l}")
                owed.setdefault((buf, n, l), set(readers(buf, n, l))).discard(c)
            elif st[0] == "arrive":
                cnt[(n,) + st[1:]] = cnt.get((n,) + st[1:], 0) + 1
            elif st[0] == "wait":
                if cnt.get((n,) + st[1:], 0) < G:
                    continue
            pc[c] += 1
            moved = True
            break
        if not moved:
            return False
    return False


@pytest.mark.parametrize("kind", ["multi", "plain"])
@pytest.mark.parametrize("G,L", [(1, 3), (2, 1), (3, 3), (5, 2)])
def test_tagged_exchanges_complete_and_read_the_right_layer(kind, G, L):
    for seed in range(40):
        assert run(kind, G=G, L=L, seed=seed)


def _caught(L=3, **kw):
    n = 0
    for seed in range(40):
        try:
            ok = run(G=3, L=L, seed=seed, **kw)
        except Stale:
            ok = False
        n += not ok
    return n


def test_planted_one_tag_for_every_layer_is_caught():
    assert _caught(tag_per_layer=False) > 0


def test_planted_tag_base_not_advanced_is_caught():
    # one-layer calls (moe_forward): every launch would reuse the same tag
    assert _caught(L=1, advance_base=False) > 0


def test_planted_output_before_the_layers_logits_is_caught():
    assert _caught(early_output=True) > 0
