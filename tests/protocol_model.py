"""Executable models of the barrier protocols of the tensor-core kernels
(race detection on the CPU).

Each model replays one CTA's roles -- TMA producers, MMA-issuing threads,
softmax warpgroups -- as coroutines under random interleavings, with:

* mbarriers of exact phase / parity semantics: an arrival count and a
  transaction-byte count per phase; ``try_wait.parity(P)`` succeeds once the
  most recently completed phase has parity P;
* TMA copies that land at random later times (``complete_tx``);
* one in-order queue of MMAs and commits per issuing thread; the queues of
  different threads drain in arbitrary interleaving (a superset of what one
  tensor pipe can do), and a commit arrives when its queue reaches it, i.e.
  after every earlier MMA of that thread.

The data each step reads or overwrites (ring stages, score / P buffers in
TMEM, the output accumulator) is tracked, and every hazard -- a stage
refilled before its last reader ran, P overwritten before P V read it, O
touched while a P V may still run, a wait that can never complete -- raises
``Hazard``. The kernels modelled: ``attn::pf::prefill_kernel`` (dense mode:
two ping-pong query tiles, K ring of 2, V ring of 3, three release
barriers; in the paged mode the tile holding the last key landing on its own
barrier and cleared past the length before its stage counts as full),
``attn::mla::mla_decode_kernel`` (two issuing threads taking
even and odd tiles, each ring stage filled in a score-only group and a value
group with their own producers and releases, the Q staging in ring stage 1,
the tail clearing) and ``attn::dec::decode_split_kernel``
(persistent over units, one ring for K then V tiles, two P slots, the
8-bit path's converter warps between an 8-bit ring and the ring). ``bug``
plants one protocol mistake, so that tests can show a model catches it.
"""
from __future__ import annotations

import random


class Hazard(AssertionError):
    pass


def check(cond, *what):
    if not cond:
        raise Hazard(what)


class Bar:
    """An mbarrier: expected arrivals per phase, pending transaction bytes."""

    def __init__(self, name: str, count: int):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        check(self.pending >= 0, "extra arrival", self.name)
        self._advance()

    def expect_tx(self, n: int):
        self.tx += n

    def complete_tx(self, n: int):
        self.tx -= n
        self._advance()

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def test(self, parity: int) -> bool:
        return (self.phase & 1) != parity


class Sim:
    def __init__(self, seed: int):
        self.rng = random.Random(seed)
        self.bars: dict[str, Bar] = {}
        self.loads: list = []
        self.queues: dict[str, list] = {}

    def bar(self, name: str, count: int):
        self.bars[name] = Bar(name, count)

    def wait(self, name: str, parity: int):
        while not self.bars[name].test(parity):
            yield

    def load(self, bar: str, on_land):
        """A TMA copy completing `bar` (expect_tx + arrive by the issuer)."""
        b = self.bars[bar]
        b.expect_tx(1)
        b.arrive()
        self.loads.append((bar, on_land))

    def mma(self, thread: str, fn):
        self.queues.setdefault(thread, []).append(("mma", fn))

    def commit(self, thread: str, bar: str):
        self.queues.setdefault(thread, []).append(("commit", bar))

    def run(self, roles, limit: int = 400000):
        alive = list(roles)
        steps = 0
        while alive or self.loads or any(self.queues.values()):
            steps += 1
            check(steps < limit, "no progress: a wait can never complete")
            c = self.rng.random()
            if c < 0.15 and self.loads:
                bar, on_land = self.loads.pop(self.rng.randrange(len(self.loads)))
                on_land()
                self.bars[bar].complete_tx(1)
                continue
            if c < 0.40:
                busy = [k for k, q in self.queues.items() if q]
                if busy:
                    kind, x = self.queues[self.rng.choice(busy)].pop(0)
                    if kind == "mma":
                        x()
                    else:
                        self.bars[x].arrive()
                    continue
            if not alive:
                continue
            r = self.rng.choice(alive)
            try:
                next(r)
            except StopIteration:
                alive.remove(r)


# ---------------------------------------------------------------------------
# attn::pf::prefill_kernel (dense mode)
# ---------------------------------------------------------------------------
KSTAGE, VSTAGE, NREL = 2, 3, 3
PREFILL_BUGS = ("k_release_early", "v_release_early", "s_before_pv", "no_v_wait", "no_q_rot_wait",
                "tail_lands_on_v_full")


def prefill(nt: tuple[int, int], seed: int, rescale_p: float, bug: str | None = None, rope: bool = False,
            paged_tail: bool = False):
    """Tile t visits key tiles 0 .. nt[t]-1 (the second tile may have one
    more, as consecutive position blocks do, or none). With `rope`, each
    softmax warpgroup first rotates its Q tile in place (after Q lands) and
    the MMA thread waits for that before the tile's first score MMAs."""
    sim = Sim(seed)
    nmax = max(nt)
    sim.bar("q_full", 1)
    for s in range(KSTAGE):
        sim.bar(f"k_full{s}", 1)
    for s in range(VSTAGE):
        sim.bar(f"v_full{s}", 1)
    for i in range(NREL):
        sim.bar(f"rel{i}", 1)
    for t in range(2):
        sim.bar(f"s_full{t}", 1)
        sim.bar(f"p_full{t}", 1)
        sim.bar(f"o_done{t}", 1)
        sim.bar(f"q_rot{t}", 1)
    sim.bar("mma_done", 1)
    sim.bar("v_tail", 1)
    cleared = set()
    qst = {"landed": False, "rotated": set()}
    kst, vst = {}, {}
    s_done, pv_done, sbuf, pbuf = set(), set(), {}, {}

    def producer_k():
        if nt[0] or nt[1]:
            sim.load("q_full", lambda: qst.__setitem__("landed", True))
        for j in range(nmax):
            s = j % KSTAGE
            if j >= KSTAGE:
                it = max(0, j - KSTAGE - (2 if bug == "k_release_early" else 1))
                yield from sim.wait(f"rel{it % NREL}", (it // NREL) & 1)
                # K tile j - KSTAGE was last read by the S MMAs issued in iteration j - KSTAGE - 1
                for t in range(2):
                    check(j - KSTAGE >= nt[t] or (t, j - KSTAGE) in s_done, "K stage refilled early", j)
            sim.load(f"k_full{s}", lambda s=s, j=j: kst.__setitem__(s, j))
            yield

    def producer_v():
        for j in range(nmax):
            s = j % VSTAGE
            if j >= VSTAGE:
                it = j - VSTAGE - (1 if bug == "v_release_early" else 0)
                if it >= 0:
                    yield from sim.wait(f"rel{it % NREL}", (it // NREL) & 1)
                for t in range(2):
                    check(j - VSTAGE >= nt[t] or (t, j - VSTAGE) in pv_done, "V stage refilled early", j)
            if paged_tail and j == nmax - 1 and bug != "tail_lands_on_v_full":
                # the tile holding the last key lands on v_tail; its rows past
                # the length are cleared before v_full of the stage completes
                sim.load("v_tail", lambda s=s, j=j: vst.__setitem__(s, j))
            else:
                sim.load(f"v_full{s}", lambda s=s, j=j: vst.__setitem__(s, j))
            yield
        if paged_tail and nmax > 0:
            st = (nmax - 1) % VSTAGE
            if bug == "tail_lands_on_v_full":
                yield from sim.wait(f"v_full{st}", ((nmax - 1) // VSTAGE) & 1)
            else:
                yield from sim.wait("v_tail", 0)
            check(vst.get(st) == nmax - 1, "tail cleared before it landed")
            cleared.add(nmax - 1)
            if bug != "tail_lands_on_v_full":
                sim.bars[f"v_full{st}"].arrive()

    def issue_s(t, j):
        def ex():
            check(kst.get(j % KSTAGE) == j, "S reads the wrong K tile", t, j)
            check(qst["landed"] and (not rope or t in qst["rotated"]), "S reads an unready Q tile", t, j)
            check(pbuf.get(t) is None or (t, pbuf[t]) in pv_done, "S overwrote an unread P", t, j)
            sbuf[t] = j
            s_done.add((t, j))
        sim.mma("mma", ex)
        sim.commit("mma", f"s_full{t}")

    def issue_pv(t, j):
        yield from sim.wait(f"p_full{t}", j & 1)
        def ex():
            check(pbuf.get(t) == j, "P V reads the wrong P", t, j)
            check(vst.get(j % VSTAGE) == j, "P V reads the wrong V tile", t, j)
            check(not paged_tail or j != nmax - 1 or j in cleared, "P V reads an uncleared tail tile", t, j)
            pv_done.add((t, j))
        sim.mma("mma", ex)
        if j == nt[t] - 1:
            sim.commit("mma", f"o_done{t}")

    def mma():
        yield from sim.wait("q_full", 0)
        if nmax > 0:
            yield from sim.wait("k_full0", 0)
            for t in range(2):
                if nt[t] > 0:
                    if rope and bug != "no_q_rot_wait":
                        yield from sim.wait(f"q_rot{t}", 0)
                    issue_s(t, 0)
        for j in range(nmax):
            if bug != "no_v_wait":
                yield from sim.wait(f"v_full{j % VSTAGE}", (j // VSTAGE) & 1)
            if j + 1 < nmax:
                yield from sim.wait(f"k_full{(j + 1) % KSTAGE}", ((j + 1) // KSTAGE) & 1)
            for t in range(2):
                if j >= nt[t]:
                    continue
                if bug == "s_before_pv" and j + 1 < nt[t]:
                    issue_s(t, j + 1)
                    yield from issue_pv(t, j)
                    continue
                yield from issue_pv(t, j)
                if j + 1 < nt[t]:
                    issue_s(t, j + 1)
            sim.commit("mma", f"rel{j % NREL}")
            yield
        sim.commit("mma", "mma_done")
        yield from sim.wait("mma_done", 0)

    def softmax(t):
        if rope and nt[t] > 0:
            yield from sim.wait("q_full", 0)
            check(qst["landed"], "Q rotated before it landed", t)
            qst["rotated"].add(t)
            sim.bars[f"q_rot{t}"].arrive()
        for j in range(nt[t]):
            yield from sim.wait(f"s_full{t}", j & 1)
            check(sbuf.get(t) == j, "softmax reads the wrong S", t, j)
            if j > 0 and sim.rng.random() < rescale_p:
                # O stable: S of tile j was committed after P V of tile j-1
                check((t, j - 1) in pv_done, "O rescaled while a P V may run", t, j)
            pbuf[t] = j
            sim.bars[f"p_full{t}"].arrive()
            yield
        if nt[t] > 0:
            yield from sim.wait(f"o_done{t}", 0)
            check(all((t, j) in pv_done for j in range(nt[t])), "epilogue before the last P V", t)

    sim.run([producer_k(), producer_v(), mma(), softmax(0), softmax(1)])
    check(len(pv_done) == nt[0] + nt[1], "P V missing")


# ---------------------------------------------------------------------------
# attn::mla::mla_decode_kernel
# ---------------------------------------------------------------------------
# A ring stage is filled in two groups: A (the boxes only the score MMAs read),
# freed when the tile's score MMAs complete, and B (this CTA's value boxes),
# freed when its P.V completes; each group has its own producer thread.
MLA_BUGS = ("kv_empty_parity", "no_qt_ready", "no_qt_ready_b", "no_tail_ready", "no_group_wait", "pv_unordered",
            "a_release_early")


def mla(nt: int, tail_partial: bool, seed: int, rescale_p: float, bug: str | None = None):
    sim = Sim(seed)
    for n in ("q_full", "qt_ready", "tail_ready", "o_done"):
        sim.bar(n, 1)
    for s in range(2):
        for g in range(2):
            sim.bar(f"kv_empty{s}_{g}", 1)
            sim.bar(f"kv_full{s}_{g}", 1)
    for i in range(2):
        for n in ("s_full", "p_full", "pv_done", "s_done"):
            sim.bar(f"{n}{i}", 1)
    stage = {(s, g): None for s in range(2) for g in range(2)}
    stage[(1, 0)] = stage[(1, 1)] = "Q"      # Q columns 0-255 staged over both groups of ring stage 1
    st = dict(q_copied=False, tail_cleared=False)
    scores_done, pv_done, sbuf, pbuf = set(), set(), {}, {}

    def producer(g):
        if g == 0:
            sim.load("q_full", lambda: None)
        for j in range(nt):
            s = j % 2
            if j == 1 and not (bug == "no_qt_ready" and g == 0) and not (bug == "no_qt_ready_b" and g == 1):
                yield from sim.wait("qt_ready", 0)
            if j >= 2:
                par = ((j // 2) + (0 if bug == "kv_empty_parity" else 1)) & 1
                yield from sim.wait(f"kv_empty{s}_{g}", par)
                if g == 0:
                    check((j - 2) in scores_done, "group A refilled before its score MMAs completed", j)
                else:
                    check((j - 2) in pv_done, "group B refilled before its P V completed", j)
            check(stage[(s, g)] != "Q" or st["q_copied"], "Q staging overwritten before the copy", j, g)
            sim.load(f"kv_full{s}_{g}", lambda s=s, g=g, j=j: stage.__setitem__((s, g), j))
            yield
        if g == 1 and nt > 0 and tail_partial:  # value rows past the length cleared in the last tile
            s = (nt - 1) % 2
            yield from sim.wait(f"kv_full{s}_1", ((nt - 1) // 2) & 1)
            check(stage[(s, 1)] == nt - 1, "tail cleared before its tile landed")
            st["tail_cleared"] = True
            sim.bars["tail_ready"].arrive()

    def qcopy():
        if nt > 0:
            yield from sim.wait("q_full", 0)
            st["q_copied"] = True
            sim.bars["qt_ready"].arrive()

    def issuer(par):
        if nt <= par:
            return
        th = f"mma{par}"
        yield from sim.wait("q_full", 0)
        yield from sim.wait("qt_ready", 0)
        for j in range(par, nt, 2):
            s, ph = j % 2, (j // 2) & 1
            yield from sim.wait(f"kv_full{s}_0", ph)
            if bug == "a_release_early":
                sim.commit(th, f"kv_empty{s}_0")
            for g in range(2):
                if g == 1:
                    if bug != "no_group_wait":
                        yield from sim.wait(f"kv_full{s}_1", ph)
                    if j == nt - 1 and tail_partial and bug != "no_tail_ready":
                        yield from sim.wait("tail_ready", 0)
                def ex(j=j, s=s, g=g):
                    check(stage[(s, g)] == j, "score MMA reads the wrong tile", j, g)
                    check(g == 0 or not (j == nt - 1 and tail_partial) or st["tail_cleared"],
                          "tail read before cleared", j)
                    check(g > 0 or pbuf.get(j & 1) is None or pbuf[j & 1] in pv_done, "S overwrote an unread P", j)
                    if g == 1:
                        sbuf[j & 1] = j
                        scores_done.add(j)
                sim.mma(th, ex)
            if bug != "a_release_early":
                sim.commit(th, f"kv_empty{s}_0")
            sim.commit(th, f"s_full{j & 1}")
            yield from sim.wait(f"p_full{j & 1}", (j >> 1) & 1)
            if j > 0 and bug != "pv_unordered":
                yield from sim.wait(f"pv_done{par ^ 1}", ((j - 1) >> 1) & 1)
            def pv(j=j, s=s):
                check(pbuf.get(j & 1) == j, "P V reads the wrong P", j)
                check(stage[(s, 1)] == j, "P V reads the wrong tile", j)
                check(j == 0 or (j - 1) in pv_done, "O accumulated out of order", j)
                pv_done.add(j)
            sim.mma(th, pv)
            sim.commit(th, f"kv_empty{s}_1")
            sim.commit(th, f"pv_done{par}")
            if j == nt - 1:
                sim.commit(th, "o_done")
            yield
        sim.commit(th, f"s_done{par}")
        yield from sim.wait(f"s_done{par}", 0)

    def softmax():
        for j in range(nt):
            yield from sim.wait(f"s_full{j & 1}", (j >> 1) & 1)
            check(sbuf.get(j & 1) == j, "softmax reads the wrong S", j)
            if j > 0 and sim.rng.random() < rescale_p:
                yield from sim.wait(f"pv_done{(j - 1) & 1}", ((j - 1) >> 1) & 1)
                check((j - 1) in pv_done, "O rescaled while a P V may run", j)
            pbuf[j & 1] = j
            sim.bars[f"p_full{j & 1}"].arrive()
            yield
        if nt > 0:
            yield from sim.wait("o_done", 0)
            check(pv_done == set(range(nt)), "epilogue before the last P V")

    sim.run([producer(0), producer(1), qcopy(), issuer(0), issuer(1), softmax()])
    check(pv_done == set(range(nt)), "P V missing")


# ---------------------------------------------------------------------------
# attn::dec::decode_split_kernel (persistent: a CTA walks several units)
# ---------------------------------------------------------------------------
DEC_NSTAGE, DEC_NSTAGE8 = 2, 2
DECODE_BUGS = ("q_reload_early", "empty_parity", "p_slot_parity", "no_p_wait", "conv_no_empty_wait")


def decode(units: list[int], seed: int, fp8: bool = False, bug: str | None = None):
    """One CTA's units in order; unit n holds units[n] key tiles. A unit
    streams its K tiles (score MMAs into TMEM), then its V tiles (P V into
    the output accumulator), through one ring; on the 8-bit path the tiles
    land in an 8-bit ring and converter warps widen them into the ring."""
    sim = Sim(seed)
    NS, NS8 = DEC_NSTAGE, DEC_NSTAGE8
    for n in ("q_full", "q_empty", "q_conv", "s_full", "o_full", "mma_done"):
        sim.bar(n, 1)
    for s in range(NS):
        sim.bar(f"full{s}", 1)
        sim.bar(f"empty{s}", 1)
    for s in range(NS8):
        sim.bar(f"full8_{s}", 1)
        sim.bar(f"empty8_{s}", 1)
    for x in range(2):
        sim.bar(f"p_full{x}", 1)
        sim.bar(f"p_empty{x}", 1)
    st = dict(q=None, qconv=None)
    ring, ring8, sread, pslot = {}, {}, set(), {}
    s_tiles, s_exec, pv_exec, o_read, ring_used, ring8_used = {}, set(), set(), set(), {}, {}

    def tiles(n):           # (unit, tile index within the unit's 2 * units[n] ring tiles)
        return [(n, j) for j in range(2 * units[n])]

    def producer():
        t = 0
        for n in range(len(units)):
            if n > 0 and bug != "q_reload_early":
                yield from sim.wait("q_empty", (n - 1) & 1)
            sim.load("q_full", lambda n=n: st.__setitem__("q", n))
            for tile in tiles(n):
                if fp8:
                    s8 = t % NS8
                    yield from sim.wait(f"empty8_{s8}", ((t // NS8) & 1) ^ 1)
                    check(ring8.get(s8) is None or ring8_used.get(s8) == ring8[s8], "8-bit stage refilled early", tile)
                    sim.load(f"full8_{s8}", lambda s8=s8, tile=tile: ring8.__setitem__(s8, tile))
                else:
                    s = t % NS
                    par = ((t // NS) & 1) ^ (0 if bug == "empty_parity" else 1)
                    yield from sim.wait(f"empty{s}", par)
                    check(ring.get(s) is None or ring_used.get(s) == ring[s], "ring stage refilled early", tile)
                    sim.load(f"full{s}", lambda s=s, tile=tile: ring.__setitem__(s, tile))
                t += 1
                yield

    def converter():
        t = 0
        for n in range(len(units)):
            yield from sim.wait("q_full", n & 1)
            check(st["q"] == n, "converter reads the wrong Q", n)
            st["qconv"] = n
            sim.bars["q_conv"].arrive()
            for tile in tiles(n):
                s8, s = t % NS8, t % NS
                yield from sim.wait(f"full8_{s8}", (t // NS8) & 1)
                if bug != "conv_no_empty_wait":
                    yield from sim.wait(f"empty{s}", ((t // NS) & 1) ^ 1)
                check(ring8.get(s8) == tile, "converter reads the wrong 8-bit tile", tile)
                check(ring.get(s) is None or ring_used.get(s) == ring[s], "ring stage overwritten early", tile)
                ring[s] = tile
                ring8_used[s8] = tile
                sim.bars[f"full{s}"].arrive()
                sim.bars[f"empty8_{s8}"].arrive()
                t += 1
                yield

    def mma():
        t = pc = 0
        for n, nt in enumerate(units):
            yield from sim.wait("q_conv" if fp8 else "q_full", n & 1)
            for j in range(nt):
                g = t + j
                s = g % NS
                yield from sim.wait(f"full{s}", (g // NS) & 1)
                def ex(n=n, j=j, s=s):
                    check(ring.get(s) == (n, j), "score MMA reads the wrong K tile", n, j)
                    check(st["q"] == n and (not fp8 or st["qconv"] == n), "score MMA reads the wrong Q", n)
                    check(n == 0 or j >= units[n - 1] or (n - 1, j) in sread, "S overwritten while being read", n, j)
                    ring_used[s] = (n, j)
                    s_tiles[j] = n
                    s_exec.add((n, j))
                sim.mma("mma", ex)
                sim.commit("mma", f"empty{s}")
            sim.commit("mma", "q_empty")
            sim.commit("mma", "s_full")
            t += nt
            for j in range(nt):
                g = t + j
                s = g % NS
                yield from sim.wait(f"full{s}", (g // NS) & 1)
                if bug != "no_p_wait":
                    yield from sim.wait(f"p_full{pc & 1}", (pc >> 1) & 1)
                def pv(n=n, j=j, s=s, x=pc & 1, nt=nt):
                    check(ring.get(s) == (n, nt + j), "P V reads the wrong V tile", n, j)
                    check(pslot.get(x) == (n, j), "P V reads the wrong P", n, j)
                    check(j > 0 or n == 0 or (n - 1) in o_read, "O overwritten before it was read", n)
                    check(j == 0 or (n, j - 1) in pv_exec, "O accumulated out of order", n, j)
                    ring_used[s] = (n, nt + j)
                    pv_exec.add((n, j))
                sim.mma("mma", pv)
                sim.commit("mma", f"empty{s}")
                sim.commit("mma", f"p_empty{pc & 1}")
                pc += 1
            sim.commit("mma", "o_full")
            t += nt
            yield
        sim.commit("mma", "mma_done")
        yield from sim.wait("mma_done", 0)

    def softmax():
        pc = 0
        for n, nt in enumerate(units):
            yield from sim.wait("s_full", n & 1)
            check(all(s_tiles.get(j) == n for j in range(nt)), "softmax reads S of another unit", n)
            for j in range(nt):
                check(s_tiles.get(j) == n, "S tile overwritten during pass 2", n, j)
                sread.add((n, j))
                par = ((pc >> 1) & 1) ^ (0 if bug == "p_slot_parity" else 1)
                yield from sim.wait(f"p_empty{pc & 1}", par)
                prev = pslot.get(pc & 1)
                check(prev is None or prev in pv_exec, "P slot overwritten before P V read it", n, j)
                pslot[pc & 1] = (n, j)
                sim.bars[f"p_full{pc & 1}"].arrive()
                pc += 1
                yield
            yield from sim.wait("o_full", n & 1)
            check(all((n, j) in pv_exec for j in range(nt)), "output read before the last P V", n)
            o_read.add(n)

    roles = [producer(), mma(), softmax()] + ([converter()] if fp8 else [])
    sim.run(roles)
    check(len(pv_exec) == sum(units), "P V missing")
