"""A model of the split-KV decode kernel's barrier protocol, run under random interleavings (CPU).

The kernel (csrc/decode.cuh, one CTA) has a TMA producer streaming 16-key stages into a ring of
NST slots, two table warps that take alternate stages and write each stage's correction cos/sin
table into that slot's table area, and consumer warps (two per kv head) that read every stage. They
meet on three barriers per slot, all waited on by phase parity:
- full[slot]: the stage's bytes landed (the producer's expect_tx, completed by the copy);
- tbl[slot]: the slot's table is written (one arrive per table-warp lane; here one per warp);
- empty[slot]: every consumer warp is done with the slot (one arrive per consumer warp).
Consumers wait for tbl only on stages that hold long-range keys. The model replays each actor's
program in a random order and checks that
- no wait passes on the wrong phase (a parity alias: the barrier ran two phases ahead),
- no copy lands in a slot a consumer still reads, and no table is rewritten while a consumer reads it,
- every program finishes (no deadlock),
for splits of various lengths and band positions (stages before, across and after local_from)."""
import random

import pytest

NST = 5  # stages in the ring


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        self._flip()

    def expect(self, n):
        self.tx += n
        self.pending -= 1
        self._flip()

    def complete_tx(self, n):
        self.tx -= n
        self._flip()

    def _flip(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def run_decode_protocol(nstage, long_stages, n_cons, rnd, skip_table_empty_wait=False):
    """long_stages: set of stage indices that hold long-range keys (their consumers wait for tbl)."""
    full = [Bar(1) for _ in range(NST)]
    tbl = [Bar(1) for _ in range(NST)]  # the model's table warp arrives once for its 32 lanes
    empty = [Bar(n_cons) for _ in range(NST)]
    landed = []  # copies in flight: (slot, stage)
    readers = [0] * NST  # consumer warps reading a slot's K/V and table
    table_of = [-1] * NST  # stage whose table the slot holds
    data_of = [-1] * NST  # stage whose K/V the slot holds

    prod = [("stage", s) for s in range(nstage)]
    tables = {cw: [("tstage", s) for s in range(cw, nstage, 2)] for cw in (0, 1)}
    cons = {c: [("cstage", s) for s in range(nstage)] for c in range(n_cons)}
    progs = {"prod": prod, **{f"tbl{cw}": p for cw, p in tables.items()}, **{f"c{c}": p for c, p in cons.items()}}
    pc = {k: 0 for k in progs}
    # per consumer, the sub-step within a stage: 0 = waiting for the stage, 1 = reading it
    sub = {c: 0 for c in range(n_cons)}

    def step_prod():
        s = progs["prod"][pc["prod"]][1]
        st = s % NST
        if s >= NST:
            if not empty[st].passed(((s // NST) - 1) & 1):
                return False
            assert empty[st].phase == s // NST, "empty parity alias (producer)"
        full[st].expect(1)
        landed.append((st, s))
        return True

    def step_land():
        st, s = landed.pop(rnd.randrange(len(landed)))
        assert readers[st] == 0, "a copy landed in a slot a consumer still reads"
        data_of[st] = s
        full[st].complete_tx(1)
        return True

    def step_table(cw):
        s = progs[f"tbl{cw}"][pc[f"tbl{cw}"]][1]
        st = s % NST
        if s >= NST and not skip_table_empty_wait:
            if not empty[st].passed(((s // NST) - 1) & 1):
                return False
            assert empty[st].phase == s // NST, "empty parity alias (table warp)"
        if s in long_stages:
            assert readers[st] == 0, "a table was rewritten while a consumer reads it"
            table_of[st] = s
        tbl[st].arrive()
        return True

    def step_consumer(c):
        s = progs[f"c{c}"][pc[f"c{c}"]][1]
        st = s % NST
        if sub[c] == 0:
            if not full[st].passed((s // NST) & 1):
                return False
            assert full[st].phase == s // NST + 1, "full parity alias"
            if s in long_stages:
                if not tbl[st].passed((s // NST) & 1):
                    return False
                assert tbl[st].phase == s // NST + 1, "tbl parity alias"
                assert table_of[st] == s, "consumer read a table of another stage"
            assert data_of[st] == s, "consumer read K/V of another stage"
            readers[st] += 1
            sub[c] = 1
            return None  # progressed, stage not finished
        readers[st] -= 1
        empty[st].arrive()
        sub[c] = 0
        return True

    while True:
        acts = []
        if pc["prod"] < len(progs["prod"]):
            acts.append(("prod", step_prod))
        if landed:
            acts.append(("land", step_land))
        for cw in (0, 1):
            if pc[f"tbl{cw}"] < len(progs[f"tbl{cw}"]):
                acts.append((f"tbl{cw}", lambda cw=cw: step_table(cw)))
        for c in range(n_cons):
            if pc[f"c{c}"] < len(progs[f"c{c}"]):
                acts.append((f"c{c}", lambda c=c: step_consumer(c)))
        if not acts:
            return True
        rnd.shuffle(acts)
        for name, fn in acts:
            r = fn()
            if r is None:
                break
            if r:
                if name in pc:
                    pc[name] += 1
                break
        else:
            raise AssertionError(f"deadlock at {pc}")


# (stages in the split, first local stage or None when every stage is long, consumer warps)
CASES = [(1, None, 8), (4, None, 8), (5, None, 8), (6, None, 8), (23, None, 8), (23, 17, 8), (23, 0, 8),
         (40, 25, 4), (111, 100, 8), (7, 3, 2)]


@pytest.mark.parametrize("nstage,first_local,n_cons", CASES)
def test_decode_protocol_completes_without_aliasing(nstage, first_local, n_cons):
    rnd = random.Random(nstage * 7 + (first_local or 0) + n_cons)
    # stages before the band edge hold long-range keys; the band-edge stage holds both
    edge = nstage if first_local is None else first_local
    long_stages = set(range(min(edge + 1, nstage)))
    for _ in range(20):
        assert run_decode_protocol(nstage, long_stages, n_cons, rnd) is True


def test_model_catches_a_table_warp_that_skips_the_empty_wait():
    # planted mistake: a table warp rewrites a slot's table without waiting for its consumers
    rnd = random.Random(5)
    caught = 0
    for _ in range(200):
        try:
            run_decode_protocol(30, set(range(30)), 8, rnd, skip_table_empty_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0
