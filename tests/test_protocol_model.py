"""A model of the ping-pong prefill kernel's barrier protocol, run under random interleavings (CPU).

The kernel (csrc/prefill_tc2.cuh) has five actors per CTA: a TMA producer, the MMA issuer, the
tensor pipe that executes the issued MMAs in order, and two softmax groups (tiles A and B). They
meet on mbarriers that are waited on by phase parity. The model replays each actor's program
step by step in a random order and checks that
- no actor ever passes a parity wait on the wrong phase (a parity alias: the barrier ran two
  phases ahead of the waiter),
- the producer never overwrites Q while a QK^T that reads it is pending,
- every program finishes (no deadlock),
for the visit schedules of every kernel kind: plain, bifocal (long visits, Q reload, local visits),
sliding window (long visits skipped), and query tiles at offsets that are not tile multiples
(chunked prefill). The schedule below restates the kernel's tile classification.
"""
import random

import pytest

BM = BN = 128
NSLOT = 4  # K/V ring slots: two per visit (K, then V)


def schedule(i0, n_kt, w0, kind):
    """Visit counts of one query tile starting at absolute row i0 with n_kt key tiles."""
    if kind == "plain":
        return dict(n_long=0, n_loc=n_kt)
    A = (i0 - (BN - 1) - w0) // BN        # tiles t <= A: every pair long-range
    C = (i0 + (BM - 1) - w0) // BN + 1    # tiles t >= C: every pair local
    n_lf = min(max(A + 1, 0), n_kt)
    n_b = max(min(C, n_kt) - n_lf, 0)
    n_bl = n_b if w0 > 0 else 0
    n_of = n_kt - n_lf - n_b
    if kind == "window":
        return dict(n_long=0, n_loc=n_bl + n_of)
    return dict(n_long=n_lf + n_b, n_loc=n_bl + n_of)


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

    def passed(self, parity):  # try_wait.parity: true once the phase with this parity completed
        return (self.phase & 1) != parity


def softmax_prog(x, nv, rnd):
    """One softmax group's steps: per visit it waits for S, then sends P in two halves (p_lo, then
    p_ready) by one of the kernel's three routes, chosen at random per visit:
    - fast: both halves against the current reference, no wait on O;
    - rare: the first half is sent, then the second half needs a new reference, so O is rescaled
      once the first half's P.V has run (o_lo) and before the second half is sent;
    - exact: both halves computed before either is sent; O is rescaled once the previous visit's
      P.V has run (o_done).
    After the last visit the epilogue waits for the last P.V."""
    prog = []
    for v in range(nv):
        prog.append(("wait_s", x, v))
        route = rnd.choice(("fast", "rare", "exact"))
        if route == "fast":
            prog += [("arrive_lo", x), ("arrive_hi", x)]
        elif route == "rare":
            prog += [("arrive_lo", x), ("wait_olo", x, v), ("rescale", x), ("arrive_hi", x)]
        else:
            if v >= 1:
                prog += [("wait_o", x, v - 1), ("rescale", x)]
            prog += [("arrive_lo", x), ("arrive_hi", x)]
    if nv:
        prog.append(("wait_o", x, nv - 1))
    return prog


def softmax_step(st, x, s_full, p_lo, p_ready, o_lo, o_done, pipe, skip_olo_wait=False):
    """One softmax step of softmax_prog; False while it has to wait."""
    if st[0] == "wait_s":
        if not s_full[x].passed(st[2] & 1):
            return False
        assert s_full[x].phase == st[2] + 1, "S parity alias"
    elif st[0] == "wait_o":
        if not o_done[x].passed(st[2] & 1):
            return False
        assert o_done[x].phase >= st[2] + 1, "O parity alias"
    elif st[0] == "wait_olo":
        if skip_olo_wait:
            return True
        if not o_lo[x].passed(st[2] & 1):
            return False
        assert o_lo[x].phase == st[2] + 1, "o_lo parity alias"
    elif st[0] == "rescale":
        assert not any(e[0] in ("o_lo", "o_done") and e[1] == x for e in pipe), "O rescaled while a P.V into it runs"
    elif st[0] == "arrive_lo":
        for _ in range(4):
            p_lo[x].arrive()
    else:
        for _ in range(4):
            p_ready[x].arrive()
    return True


def run_protocol(sch, rnd, skip_q_free_wait=False, skip_olo_wait=False):
    nv = sch["n_long"] + sch["n_loc"]
    has_long, has_orig = sch["n_long"] > 0, sch["n_loc"] > 0
    reload_q = has_long and has_orig
    v_sw = sch["n_long"]
    full = [Bar(1) for _ in range(NSLOT)]
    empty = [Bar(1) for _ in range(NSLOT)]
    s_full, p_ready, o_done = [Bar(1), Bar(1)], [Bar(4), Bar(4)], [Bar(1), Bar(1)]
    p_lo, o_lo = [Bar(4), Bar(4)], [Bar(1), Bar(1)]
    q_full, q_free = Bar(1), Bar(1)
    tma, pipe = [], []
    state = {"q_readers": 0}

    prod = [("loadq",)]
    n = 0
    for v in range(nv):
        if reload_q and v == v_sw:
            prod += ([] if skip_q_free_wait else [("wait", q_free, 0)]) + [("loadq",)]
        for _ in range(2):
            prod.append(("fill", n))
            n += 1

    mma = [("wait", q_full, 0), ("wait", full[0], 0), ("qk", 0), ("qk", 1), ("commit", empty[0])]
    if reload_q and v_sw == 1:
        mma.append(("commit", q_free))
    for v in range(nv):
        vs = (2 * v + 1) % NSLOT
        mma += [("wait", p_lo[0], v & 1), ("wait", full[vs], ((2 * v + 1) // NSLOT) & 1), ("pvlo", 0),
                ("wait", p_ready[0], v & 1), ("pvhi", 0)]
        more = v + 1 < nv
        if more:
            if reload_q and v + 1 == v_sw:
                mma.append(("wait", q_full, 1))
            k2 = (2 * (v + 1)) % NSLOT
            mma += [("wait", full[k2], ((2 * (v + 1)) // NSLOT) & 1), ("qk", 0)]
        mma += [("wait", p_lo[1], v & 1), ("pvlo", 1), ("wait", p_ready[1], v & 1), ("pvhi", 1),
                ("commit", empty[vs])]
        if more:
            mma += [("qk", 1), ("commit", empty[(2 * (v + 1)) % NSLOT])]
            if reload_q and v + 2 == v_sw:
                mma.append(("commit", q_free))

    progs = {"prod": prod, "mma": mma, "smA": softmax_prog(0, nv, rnd), "smB": softmax_prog(1, nv, rnd)}
    pc = {k: 0 for k in progs}

    def step_prod():
        st = progs["prod"][pc["prod"]]
        if st[0] == "loadq":
            assert state["q_readers"] == 0, "Q overwritten while a QK^T reads it"
            q_full.expect(1)
            tma.append(q_full)
        elif st[0] == "wait":
            if not st[1].passed(st[2]):
                return False
        else:
            k = st[1]
            s, use = k % NSLOT, k // NSLOT
            if use > 0:
                if not empty[s].passed((use - 1) & 1):
                    return False
                assert empty[s].phase == use, "empty-slot parity alias"
            full[s].expect(1)
            tma.append(full[s])
        return True

    def step_mma():
        st = progs["mma"][pc["mma"]]
        if st[0] == "wait":
            return st[1].passed(st[2])
        if st[0] == "qk":
            state["q_readers"] += 1
            pipe.append(("s_full", st[1]))
        elif st[0] == "pvlo":
            pipe.append(("o_lo", st[1]))
        elif st[0] == "pvhi":
            pipe.append(("o_done", st[1]))
        else:
            pipe.append(("bar", st[1]))
        return True

    def step_tensor():
        kind, arg = pipe.pop(0)
        if kind == "s_full":
            state["q_readers"] -= 1
            s_full[arg].arrive()
        elif kind == "o_done":
            o_done[arg].arrive()
        elif kind == "o_lo":
            o_lo[arg].arrive()
        else:
            arg.arrive()
        return True

    def step_softmax(name, x):
        return softmax_step(progs[name][pc[name]], x, s_full, p_lo, p_ready, o_lo, o_done, pipe, skip_olo_wait)

    def actors():
        out = []
        if pc["prod"] < len(progs["prod"]):
            out.append(("prod", step_prod))
        if tma:
            out.append(("tma", lambda: (tma.pop(rnd.randrange(len(tma))).complete_tx(1), True)[1]))
        if pc["mma"] < len(progs["mma"]):
            out.append(("mma", step_mma))
        if pipe:
            out.append(("tensor", step_tensor))
        for name, x in (("smA", 0), ("smB", 1)):
            if pc[name] < len(progs[name]):
                out.append((name, lambda name=name, x=x: step_softmax(name, x)))
        return out

    while True:
        acts = actors()
        if not acts:
            return True
        rnd.shuffle(acts)
        for name, fn in acts:
            if fn():
                if name in pc:
                    pc[name] += 1
                break
        else:
            raise AssertionError(f"deadlock at {pc}")


CASES = [
    # (L queries, q_off, w0, kind)
    (1100, 0, 300, "bifocal"), (4096, 0, 0, "bifocal"), (4096, 0, 1, "bifocal"), (3000, 0, 5000, "bifocal"),
    (8192, 0, 127, "bifocal"), (8192, 0, 128, "bifocal"), (2048, 0, 0, "plain"),
    (2048, 0, 512, "window"), (2048, 0, 1000, "window"), (4096, 0, 129, "window"),
    (300, 1000, 100, "bifocal"), (333, 777, 50, "bifocal"), (300, 1024, 64, "window"),
]


@pytest.mark.parametrize("Lq,q_off,w0,kind", CASES)
def test_protocol_completes_without_aliasing(Lq, q_off, w0, kind):
    rnd = random.Random(Lq * 31 + q_off + w0)
    n_qt = (Lq + BM - 1) // BM
    for qt in range(n_qt):
        i0 = q_off + qt * BM
        n_kt = (min(i0 + BM, q_off + Lq) + BN - 1) // BN
        sch = schedule(i0, n_kt, w0, kind)
        for _ in range(2):
            assert run_protocol(sch, rnd) is True


def test_model_catches_a_missing_q_free_wait():
    # planted protocol mistake: the producer reloads Q without waiting for q_free, so in some
    # interleavings the original-RoPE Q lands while a long-range QK^T still reads the old one
    sch = schedule(2048, 17, 300, "bifocal")
    assert sch["n_long"] > 0 and sch["n_loc"] > 0
    rnd = random.Random(7)
    caught = 0
    for _ in range(200):
        try:
            run_protocol(sch, rnd, skip_q_free_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0


# ---------------------------------------------------------------- fused-load form
NK3, NV2 = 3, 2  # fused form: K ring (raw tile lands, transform warps rotate it in place) and V ring


def run_protocol_fused(sch, rnd, skip_kraw_wait=False, skip_olo_wait=False):
    """The fused form's protocol: the TMA producer brings raw Q, raw K tiles (ring of three) and V
    tiles (ring of two); the transform warps rotate Q and each K tile in place once its raw bytes
    have landed; the MMA issuer, tensor pipe and softmax groups are those of the other form, with
    K and V on their own rings. Checks as run_protocol, plus: a raw tile never lands in a slot a
    pending MMA reads, and the transform never touches a slot before its raw bytes have landed."""
    nv = sch["n_long"] + sch["n_loc"]
    has_long, has_orig = sch["n_long"] > 0, sch["n_loc"] > 0
    reload_q = has_long and has_orig
    v_sw = sch["n_long"]
    kraw = [Bar(1) for _ in range(NK3)]
    kfull = [Bar(1) for _ in range(NK3)]
    kempty = [Bar(1) for _ in range(NK3)]
    vfull = [Bar(1) for _ in range(NV2)]
    vempty = [Bar(1) for _ in range(NV2)]
    s_full, p_ready, o_done = [Bar(1), Bar(1)], [Bar(4), Bar(4)], [Bar(1), Bar(1)]
    p_lo, o_lo = [Bar(4), Bar(4)], [Bar(1), Bar(1)]
    q_raw, q_full, q_free = Bar(1), Bar(1), Bar(1)
    tma, pipe = [], []
    state = {"q_readers": 0, "k_readers": [0] * NK3, "v_readers": [0] * NV2, "k_landed": [0] * NK3}

    # The producer issues K two visits ahead of V (step u: K(u), then V(u - 2)), so a K fill never
    # waits behind a V slot; the raw Q reload goes out once q_free has completed: tried at step
    # v_sw, waited for at step v_sw + 1 (after V(v_sw - 1), which the MMA needs to get there).
    prod = [("loadq",)]
    for u in range(nv + 2):
        if u < nv:
            prod.append(("kfill", u))
        if 2 <= u < nv + 2:
            prod.append(("vfill", u - 2))
        if reload_q and u == v_sw:
            prod.append(("tryq",))
        if reload_q and u == v_sw + 1:
            prod.append(("waitq",))

    xf = [("wait", q_raw, 0), ("rotq",), ("arrive", q_full)]
    for v in range(nv):
        if not skip_kraw_wait:
            xf.append(("wait", kraw[v % NK3], (v // NK3) & 1))
        xf += [("rotk", v), ("arrive", kfull[v % NK3])]
        if reload_q and v == v_sw:  # K(v_sw) first, then the reloaded Q
            xf += [("wait", q_raw, 1), ("rotq",), ("arrive", q_full)]

    mma = [("wait", q_full, 0), ("wait", kfull[0], 0), ("qk", 0, 0), ("qk", 1, 0), ("commit", kempty[0])]
    if reload_q and v_sw == 1:
        mma.append(("commit", q_free))
    for v in range(nv):
        mma += [("wait", p_lo[0], v & 1), ("wait", vfull[v % NV2], (v // NV2) & 1), ("pvlo", 0, v),
                ("wait", p_ready[0], v & 1), ("pvhi", 0, v)]
        more = v + 1 < nv
        if more:
            if reload_q and v + 1 == v_sw:
                mma.append(("wait", q_full, 1))
            mma += [("wait", kfull[(v + 1) % NK3], ((v + 1) // NK3) & 1), ("qk", 0, v + 1)]
        mma += [("wait", p_lo[1], v & 1), ("pvlo", 1, v), ("wait", p_ready[1], v & 1), ("pvhi", 1, v),
                ("commit", vempty[v % NV2])]
        if more:
            mma += [("qk", 1, v + 1), ("commit", kempty[(v + 1) % NK3])]
            if reload_q and v + 2 == v_sw:
                mma.append(("commit", q_free))

    progs = {"prod": prod, "xf": xf, "mma": mma, "smA": softmax_prog(0, nv, rnd), "smB": softmax_prog(1, nv, rnd)}
    pc = {k: 0 for k in progs}

    def land(kind, arg):
        def go():
            if kind == "k":
                assert state["k_readers"][arg[0]] == 0, "raw K landed in a slot a QK^T still reads"
                state["k_landed"][arg[0]] = arg[1] + 1
            elif kind == "v":
                assert state["v_readers"][arg] == 0, "V landed in a slot a PV still reads"
            elif kind == "q":
                assert state["q_readers"] == 0, "raw Q landed while a QK^T reads Q"
            arg_bar.complete_tx(1)
        arg_bar = {"k": lambda: kraw[arg[0]], "v": lambda: vfull[arg], "q": lambda: q_raw}[kind]()
        return go

    def step_prod():
        st = progs["prod"][pc["prod"]]
        if st[0] == "loadq":
            q_raw.expect(1)
            tma.append(land("q", None))
        elif st[0] == "tryq":
            if q_free.passed(0) and not state.get("q_reloaded"):
                state["q_reloaded"] = True
                q_raw.expect(1)
                tma.append(land("q", None))
        elif st[0] == "waitq":
            if not state.get("q_reloaded"):
                if not q_free.passed(0):
                    return False
                state["q_reloaded"] = True
                q_raw.expect(1)
                tma.append(land("q", None))
        elif st[0] == "wait":
            return st[1].passed(st[2])
        elif st[0] == "kfill":
            v = st[1]
            s, use = v % NK3, v // NK3
            if use > 0:
                if not kempty[s].passed((use - 1) & 1):
                    return False
                assert kempty[s].phase == use, "K empty-slot parity alias"
            kraw[s].expect(1)
            tma.append(land("k", (s, v)))
        else:
            v = st[1]
            s, use = v % NV2, v // NV2
            if use > 0:
                if not vempty[s].passed((use - 1) & 1):
                    return False
                assert vempty[s].phase == use, "V empty-slot parity alias"
            vfull[s].expect(1)
            tma.append(land("v", s))
        return True

    def step_xf():
        st = progs["xf"][pc["xf"]]
        if st[0] == "wait":
            return st[1].passed(st[2])
        if st[0] == "rotq":
            assert state["q_readers"] == 0, "Q rotated while a QK^T reads it"
        elif st[0] == "rotk":
            v = st[1]
            assert state["k_landed"][v % NK3] == v + 1, "K slot rotated before its raw tile landed"
            assert state["k_readers"][v % NK3] == 0, "K slot rotated while a QK^T reads it"
        else:
            st[1].arrive()
        return True

    def step_mma():
        st = progs["mma"][pc["mma"]]
        if st[0] == "wait":
            return st[1].passed(st[2])
        if st[0] == "qk":
            state["q_readers"] += 1
            state["k_readers"][st[2] % NK3] += 1
            pipe.append(("s_full", st[1], st[2]))
        elif st[0] in ("pvlo", "pvhi"):
            state["v_readers"][st[2] % NV2] += 1
            pipe.append(("o_lo" if st[0] == "pvlo" else "o_done", st[1], st[2]))
        else:
            pipe.append(("bar", st[1], None))
        return True

    def step_tensor():
        kind, arg, v = pipe.pop(0)
        if kind == "s_full":
            state["q_readers"] -= 1
            state["k_readers"][v % NK3] -= 1
            s_full[arg].arrive()
        elif kind in ("o_lo", "o_done"):
            state["v_readers"][v % NV2] -= 1
            (o_lo if kind == "o_lo" else o_done)[arg].arrive()
        else:
            arg.arrive()
        return True

    def step_softmax(name, x):
        return softmax_step(progs[name][pc[name]], x, s_full, p_lo, p_ready, o_lo, o_done, pipe, skip_olo_wait)

    def actors():
        out = []
        for name, fn in (("prod", step_prod), ("xf", step_xf), ("mma", step_mma)):
            if pc[name] < len(progs[name]):
                out.append((name, fn))
        if tma:
            out.append(("tma", lambda: (tma.pop(rnd.randrange(len(tma)))(), True)[1]))
        if pipe:
            out.append(("tensor", step_tensor))
        for name, x in (("smA", 0), ("smB", 1)):
            if pc[name] < len(progs[name]):
                out.append((name, lambda name=name, x=x: step_softmax(name, x)))
        return out

    while True:
        acts = actors()
        if not acts:
            return True
        rnd.shuffle(acts)
        for name, fn in acts:
            if fn():
                if name in pc:
                    pc[name] += 1
                break
        else:
            raise AssertionError(f"deadlock at {pc}")


@pytest.mark.parametrize("Lq,q_off,w0,kind", CASES)
def test_fused_protocol_completes_without_aliasing(Lq, q_off, w0, kind):
    rnd = random.Random(Lq * 17 + q_off + w0)
    n_qt = (Lq + BM - 1) // BM
    for qt in range(n_qt):
        i0 = q_off + qt * BM
        n_kt = (min(i0 + BM, q_off + Lq) + BN - 1) // BN
        sch = schedule(i0, n_kt, w0, kind)
        for _ in range(2):
            assert run_protocol_fused(sch, rnd) is True


def test_fused_model_catches_a_missing_raw_wait():
    # planted mistake: the transform warps rotate a K slot without waiting for its raw tile
    sch = schedule(2048, 17, 300, "bifocal")
    rnd = random.Random(11)
    caught = 0
    for _ in range(100):
        try:
            run_protocol_fused(sch, rnd, skip_kraw_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0


def test_model_catches_a_rescale_before_the_first_half_ran():
    # planted mistake: the rare route rescales O without waiting for the first half's P.V
    sch = schedule(2048, 17, 300, "bifocal")
    rnd = random.Random(13)
    caught = 0
    for _ in range(200):
        try:
            run_protocol(sch, rnd, skip_olo_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0
    caught = 0
    for _ in range(200):
        try:
            run_protocol_fused(sch, rnd, skip_olo_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0
