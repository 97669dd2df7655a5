"""The barrier protocols of the persistent and ring-buffered kernels (quantiser, pooled top-k, linear branch,
block-64 flash, W8A8 GEMM), on the CPU.

Each kernel role (a producer thread, an MMA-issuing thread, a warp of
converters or of the epilogue) is written out as its sequence of steps in
program order: barrier waits and arrivals, and the begin / end of each access
to a shared buffer (a shared-memory stage or operand buffer, a TMEM
accumulator).  Asynchronous work is placed where its completion is signalled:
a bulk copy writes its stage until the arrival on the stage's full barrier, an
MMA reads its operands and writes its accumulator until its commit arrives.
A random scheduler then runs the roles in arbitrary interleavings and checks:

  - no deadlock;
  - every parity wait is sound: a wait for completion k of a barrier (parity
    k % 2) must find the barrier at k or k + 1 completions whenever the role
    stands at it, because the hardware only compares parities (k - 1 would let
    it through early, k + 2 would hold it for good);
  - no role writes a buffer while another still reads it (or writes it for a
    different item), and every read finds the item it expects, completely
    written.

The role programs follow the kernels in csrc/k_linear.cu (linear_kv_kernel,
linear_apply_kernel, linear_sum_kernel), csrc/k_flash64.cu (one slot of
flash64_kernel), csrc/k_w8a8.cu (w8a8_gemm_kernel) and csrc/k_prologue.cu
(quant_kernel) and csrc/k_topk.cu (pool_topk16_kernel's chunk ring), whose
block barriers are modelled as one barrier phase per use that every warp or
thread arrives at and waits for: the same loop structure, stage and phase
arithmetic, barrier counts and arrival points.
"""
import random
from collections import defaultdict

import pytest


class Violation(AssertionError):
    pass


class Buffers:
    """Multi-reader buffers with item tags; writers of one tag may overlap."""

    def __init__(self):
        self.readers = defaultdict(int)
        self.writers = defaultdict(int)
        self.wtag = {}
        self.content = {}

    def wbeg(self, b, tag, who):
        if self.readers[b]:
            raise Violation(f"{who} writes {b} ({tag}) while it is read")
        if self.writers[b] and self.wtag[b] != tag:
            raise Violation(f"{who} writes {b} ({tag}) while {self.wtag[b]} is being written")
        self.writers[b] += 1
        self.wtag[b] = tag
        self.content[b] = None

    def wend(self, b):
        self.writers[b] -= 1
        if self.writers[b] == 0:
            self.content[b] = self.wtag[b]

    def rbeg(self, b, tag, who):
        if self.writers[b] or self.content.get(b) != tag:
            raise Violation(f"{who} reads {b} expecting {tag}, holds {self.content.get(b)} "
                            f"({self.writers[b]} writers)")
        self.readers[b] += 1

    def rend(self, b):
        self.readers[b] -= 1


def simulate(programs, counts, seed):
    """programs: role -> list of steps; counts: barrier -> arrivals per phase."""
    rng = random.Random(seed)
    pc = {r: 0 for r in programs}
    done = defaultdict(int)
    arrivals = defaultdict(int)
    buf = Buffers()

    def check_waits():
        for r, prog in programs.items():
            if pc[r] < len(prog) and prog[pc[r]][0] == "wait":
                _, b, k = prog[pc[r]]
                c = done[b]
                if c >= k + 2:
                    raise Violation(f"{r} waits for completion {k} of {b}, which has {c}: parity alias")
                if c < k and (k - c) % 2 == 1:
                    raise Violation(f"{r} waits for completion {k} of {b}, which has {c}: passes early")

    while True:
        check_waits()
        ready = []
        for r, prog in programs.items():
            if pc[r] >= len(prog):
                continue
            st = prog[pc[r]]
            if st[0] != "wait" or done[st[1]] >= st[2] + 1:
                ready.append(r)
        if not ready:
            left = {r: programs[r][pc[r]] for r in programs if pc[r] < len(programs[r])}
            if left:
                raise Violation(f"deadlock: {left}")
            return
        r = rng.choice(ready)
        st = programs[r][pc[r]]
        op = st[0]
        if op == "arrive":
            b = st[1]
            arrivals[b] += 1
            if arrivals[b] == counts[b]:
                arrivals[b] = 0
                done[b] += 1
        elif op == "wbeg":
            buf.wbeg(st[1], st[2], r)
        elif op == "wend":
            buf.wend(st[1])
        elif op == "rbeg":
            buf.rbeg(st[1], st[2], r)
        elif op == "rend":
            buf.rend(st[1])
        pc[r] += 1


# --------------------------------------------------------------- linear_kv --
def linear_kv_programs(nitems, chunks, J=4, stages=3, ops=2, nconv=8, nepi=8):
    """Single accumulator set (4 blocks per item use all 512 TMEM columns)."""
    P, C = {}, defaultdict(lambda: 1)
    U = nitems * J * chunks
    prod = []
    for u in range(U):
        s = u % stages
        if u >= stages:
            prod.append(("wait", ("raw_empty", s), u // stages - 1))
        prod += [("wbeg", ("raw", s), u), ("wend", ("raw", s)), ("arrive", ("raw_full", s))]
    P["producer"] = prod
    for w in range(nconv):
        cv, u, zi = [], 0, 0
        for it in range(nitems):
            for jj in range(J):
                for c in range(chunks):
                    s, b = u % stages, u % ops
                    cv.append(("wait", ("raw_full", s), u // stages))
                    if u >= ops:
                        cv.append(("wait", ("op_empty", b), u // ops - 1))
                    cv += [("rbeg", ("raw", s), u), ("wbeg", ("op", b, w), u), ("wend", ("op", b, w)),
                           ("rend", ("raw", s)), ("arrive", ("op_full", b)), ("arrive", ("raw_empty", s))]
                    u += 1
                cv += [("wbeg", ("zred", zi & 1, w), zi), ("wend", ("zred", zi & 1, w)),
                       ("arrive", ("z_ready", zi & 1)), ("wait", ("z_ready", zi & 1), zi >> 1)]
                if w < nconv // 2:  # threads ct < 128 add the 16 row slots
                    cv += [("rbeg", ("zred", zi & 1, x), zi) for x in range(nconv)]
                    cv += [("rend", ("zred", zi & 1, x)) for x in range(nconv)]
                zi += 1
        P[f"conv{w}"] = cv
    mma, u = [], 0
    for it in range(nitems):
        if it > 0:
            mma.append(("wait", ("acc_empty",), it - 1))
        for jj in range(J):
            for c in range(chunks):
                b = u % ops
                mma.append(("wait", ("op_full", b), u // ops))
                mma += [("rbeg", ("op", b, w), u) for w in range(nconv)]
                if c == 0:
                    mma.append(("wbeg", ("acc", jj), it))
                mma += [("rend", ("op", b, w)) for w in range(nconv)]
                mma.append(("arrive", ("op_empty", b)))
                u += 1
        mma += [("wend", ("acc", jj)) for jj in range(J)] + [("arrive", ("acc_full",))]
    P["mma"] = mma
    for e in range(nepi):
        ep = []
        for it in range(nitems):
            ep.append(("wait", ("acc_full",), it))
            ep += [("rbeg", ("acc", jj), it) for jj in range(J)]
            ep += [("rend", ("acc", jj)) for jj in range(J)] + [("arrive", ("acc_empty",))]
        P[f"epi{e}"] = ep
    for s in range(stages):
        C[("raw_empty", s)] = nconv
    for b in range(ops):
        C[("op_full", b)] = nconv
    C[("z_ready", 0)] = C[("z_ready", 1)] = nconv
    C[("acc_empty",)] = nepi
    return P, C


# ------------------------------------------------------------ linear_apply --
def linear_apply_programs(nitems, nrow=4):
    """Two groups of row warps alternate items; group g = item % 2 owns stage g
    (q rows -> phi(Q) -> O_l -> y staging in one region, H images and Z rows)
    and TMEM columns g (num, y).  Region parts: one per row warp; phi(Q) and
    O_l rows of a warp land in every part, its raw rows and its staging in its
    own part."""
    P, C = {}, defaultdict(lambda: 1)
    parts = range(nrow)
    hq = [("wbeg", ("W",), 0), ("wend", ("W",)), ("arrive", ("w_full",))]
    qq = []
    for k in range(nitems):
        g, u = k & 1, k >> 1
        if k >= 2:
            hq.append(("wait", ("h_empty", g), u - 1))
            qq.append(("wait", ("empty", g), u - 1))
        hq += [("wbeg", ("H", g), k), ("wbeg", ("Z", g), k), ("wend", ("H", g)), ("wend", ("Z", g)),
               ("arrive", ("full", g))]
        qq += [("wbeg", ("Q", g, p), (k, "q")) for p in parts] + [("wend", ("Q", g, p)) for p in parts]
        qq.append(("arrive", ("full", g)))
    P["hprod"], P["qprod"] = hq, qq
    m1, m2 = [], [("wait", ("w_full",), 0)]
    for k in range(nitems):
        g, u = k & 1, k >> 1
        m1.append(("wait", ("a_full", g), u))
        m1 += [("rbeg", ("Q", g, p), (k, "a")) for p in parts] + [("rbeg", ("H", g), k), ("wbeg", ("num", g), k)]
        m1 += [("rend", ("Q", g, p)) for p in parts] + [("rend", ("H", g)), ("wend", ("num", g))]
        m1 += [("arrive", ("num_full", g)), ("arrive", ("h_empty", g))]
        m2.append(("wait", ("o_full", g), u))
        m2 += [("rbeg", ("Q", g, p), (k, "o")) for p in parts] + [("rbeg", ("W",), 0), ("wbeg", ("y", g), k)]
        m2 += [("rend", ("Q", g, p)) for p in parts] + [("rend", ("W",)), ("wend", ("y", g))]
        m2.append(("arrive", ("y_full", g)))
    P["mma1"], P["mma2"] = m1, m2
    for grp in range(2):
        for w in range(nrow):
            rw = []
            for k in range(grp, nitems, 2):
                g, u = grp, k >> 1
                rw += [("wait", ("full", g), u), ("rbeg", ("Q", g, w), (k, "q")), ("rend", ("Q", g, w)),
                       ("arrive", ("qread", g)), ("wait", ("qread", g), u), ("rbeg", ("Z", g), k)]
                rw += [("wbeg", ("Q", g, p), (k, "a")) for p in parts] + [("wend", ("Q", g, p)) for p in parts]
                rw += [("rend", ("Z", g)), ("arrive", ("a_full", g)), ("wait", ("num_full", g), u),
                       ("rbeg", ("num", g), k)]
                rw += [("wbeg", ("Q", g, p), (k, "o")) for p in parts] + [("wend", ("Q", g, p)) for p in parts]
                rw += [("rend", ("num", g)), ("arrive", ("o_full", g)), ("wait", ("y_full", g), u),
                       ("rbeg", ("y", g), k), ("rend", ("y", g)),
                       ("wbeg", ("Q", g, w), (k, "y")), ("wend", ("Q", g, w)),
                       ("rbeg", ("Q", g, w), (k, "y")), ("rend", ("Q", g, w)), ("arrive", ("empty", g))]
            P[f"row{grp}.{w}"] = rw
    for g in range(2):
        C[("full", g)] = 2
        C[("empty", g)] = C[("qread", g)] = C[("a_full", g)] = C[("o_full", g)] = nrow
    return P, C


# -------------------------------------------------------------- linear_sum --
def linear_sum_programs(ntiles, nbt, stages=3, nawarps=8):
    """The K-stage ring continues across tiles; one accumulator set (both M
    tiles, 512 columns); the A warps also run the epilogue."""
    P, C = {}, defaultdict(lambda: 1)
    prod, g = [], 0
    for T in range(ntiles):
        for kt in range(nbt):
            s = g % stages
            if g >= stages:
                prod.append(("wait", ("empty", s), g // stages - 1))
            prod += [("wbeg", ("B", s), g), ("wend", ("B", s)), ("arrive", ("b_full", s))]
            g += 1
    P["bprod"] = prod
    mma, g = [], 0
    for T in range(ntiles):
        if T > 0:
            mma.append(("wait", ("acc_empty",), T - 1))
        for kt in range(nbt):
            s = g % stages
            mma += [("wait", ("a_full", s), g // stages), ("wait", ("b_full", s), g // stages)]
            mma += [("rbeg", ("A", s, w), g) for w in range(nawarps)] + [("rbeg", ("B", s), g)]
            if kt == 0:
                mma.append(("wbeg", ("D",), T))
            mma += [("rend", ("A", s, w)) for w in range(nawarps)] + [("rend", ("B", s)), ("arrive", ("empty", s))]
            g += 1
        mma += [("wend", ("D",)), ("arrive", ("acc_full",))]
    P["mma"] = mma
    for w in range(nawarps):
        aw, g = [], 0
        for T in range(ntiles):
            for kt in range(nbt):
                s = g % stages
                if g >= stages:
                    aw.append(("wait", ("empty", s), g // stages - 1))
                aw += [("wbeg", ("A", s, w), g), ("wend", ("A", s, w)), ("arrive", ("a_full", s))]
                g += 1
            aw += [("wait", ("acc_full",), T), ("rbeg", ("D",), T), ("rend", ("D",)), ("arrive", ("acc_empty",))]
        P[f"aw{w}"] = aw
    for s in range(stages):
        C[("a_full", s)] = nawarps
    C[("acc_empty",)] = nawarps
    return P, C


@pytest.mark.parametrize("nitems,chunks", [(1, 1), (2, 1), (3, 2), (5, 1)])
def test_linear_kv_protocol(nitems, chunks):
    P, C = linear_kv_programs(nitems, chunks)
    for seed in range(40):
        simulate(P, C, seed)


@pytest.mark.parametrize("nitems", [1, 2, 3, 4, 7])
def test_linear_apply_protocol(nitems):
    P, C = linear_apply_programs(nitems)
    for seed in range(60):
        simulate(P, C, seed)


@pytest.mark.parametrize("ntiles,nbt", [(1, 1), (1, 4), (2, 2), (3, 5), (4, 1)])
def test_linear_sum_protocol(ntiles, nbt):
    P, C = linear_sum_programs(ntiles, nbt)
    for seed in range(40):
        simulate(P, C, seed)


# The checker itself: each of these planted protocol mistakes must be caught.
def _drop_step(P, role, pred):
    prog = P[role]
    i = next(i for i, st in enumerate(prog) if pred(st))
    P[role] = prog[:i] + prog[i + 1:]


def _caught(P, C, seeds=200):
    for seed in range(seeds):
        try:
            simulate(P, C, seed)
        except Violation:
            return True
    return False


def test_checker_catches_a_missing_empty_wait():
    # the producer refills stage 0 without waiting for the converters
    P, C = linear_kv_programs(2, 1)
    _drop_step(P, "producer", lambda st: st[0] == "wait")
    assert _caught(P, C)


def test_checker_catches_a_missing_qread_barrier():
    # a row warp writes phi(Q) over rows another warp may still be reading
    P, C = linear_apply_programs(2)
    for grp in range(2):
        for w in range(4):
            P[f"row{grp}.{w}"] = [st for st in P[f"row{grp}.{w}"] if st[1][0] != "qread"]
    assert _caught(P, C)


def test_checker_catches_an_early_h_refill():
    # the H producer refills a stage without waiting for the first MMA
    P, C = linear_apply_programs(4)
    P["hprod"] = [st for st in P["hprod"] if not (st[0] == "wait" and st[1][0] == "h_empty")]
    assert _caught(P, C)


def test_checker_catches_a_wrong_arrival_count():
    # one A warp fewer counted on a_full: the MMA may read a stage being written
    P, C = linear_sum_programs(2, 3)
    for s in range(3):
        C[("a_full", s)] = 7
    assert _caught(P, C)


def test_checker_catches_a_parity_alias():
    # a waiter two phases behind: wait for completion 0 placed after the role
    # could only get there once completion 2 happened
    P = {"a": [("arrive", ("x",)), ("arrive", ("x",)), ("arrive", ("x",)), ("arrive", ("y",))],
         "b": [("wait", ("y",), 0), ("wait", ("x",), 0)]}
    C = defaultdict(lambda: 1)
    with pytest.raises(Violation, match="alias"):
        simulate(P, C, 0)


# ---------------------------------------------------------------- flash64 --
def flash64_programs(nitems, nsteps, rescale, nsoft=4):
    """One slot of the block-64 flash kernel (the two slots share nothing but
    the CTA).  Buffers: Q tiles (2), K and V stages (2), step metadata (4),
    S (TMEM), P~ (2, a part per softmax warp), O (TMEM, a part per softmax
    warp's lanes).  rescale(gs) says whether the softmax rescales O at step gs
    (data-dependent in the kernel; only where s > 0)."""
    P, C = {}, defaultdict(lambda: 1)
    W = range(nsoft)
    total = nitems * nsteps
    kp, vp, gs = [], [], 0
    for ui in range(nitems):
        qb = ui & 1
        if ui >= 2:
            kp.append(("wait", ("q_empty", qb), (ui >> 1) - 1))
        kp += [("wbeg", ("Q", qb), ui), ("wend", ("Q", qb)), ("arrive", ("q_full", qb))]
        for s in range(nsteps):
            st, ms = gs & 1, gs & 3
            for prog, nm in ((kp, "K"), (vp, "V")):
                if gs >= 2:
                    prog.append(("wait", (nm.lower() + "_empty", st), (gs >> 1) - 1))
                prog += [("wbeg", (nm, st), gs), ("wend", (nm, st)), ("arrive", (nm.lower() + "_full", st))]
            if gs >= 4:
                kp.append(("wait", ("m_empty", ms), (gs >> 2) - 1))
            kp += [("wbeg", ("meta", ms), gs), ("wend", ("meta", ms)), ("arrive", ("m_full", ms))]
            gs += 1
    P["kprod"], P["vprod"] = kp, vp
    mma = []
    for gs in range(total + 1):
        if gs < total:
            ui, s = divmod(gs, nsteps)
            qb, st = ui & 1, gs & 1
            if s == 0:
                mma.append(("wait", ("q_full", qb), ui >> 1))
            mma.append(("wait", ("k_full", st), gs >> 1))
            if gs > 0:
                mma.append(("wait", ("s_free",), gs - 1))
            mma += [("rbeg", ("Q", qb), ui), ("rbeg", ("K", st), gs)] + [("wbeg", ("S", w), gs) for w in W]
            mma += [("rend", ("Q", qb)), ("rend", ("K", st))] + [("wend", ("S", w)) for w in W]
            mma += [("arrive", ("s_full",)), ("arrive", ("k_empty", st))]
            if s == nsteps - 1:
                mma.append(("arrive", ("q_empty", qb)))
        if gs > 0:
            gp = gs - 1
            b = st = gp & 1
            mma += [("wait", ("v_full", st), gp >> 1), ("wait", ("p_full", b), gp >> 1)]
            mma += [("rbeg", ("Pt", b, w), gp) for w in W] + [("rbeg", ("V", st), gp)]
            mma += [("wbeg", ("O", w), gp) for w in W]
            mma += [("rend", ("Pt", b, w)) for w in W] + [("rend", ("V", st))] + [("wend", ("O", w)) for w in W]
            mma += [("arrive", ("o_done",)), ("arrive", ("p_empty", b)), ("arrive", ("v_empty", st))]
    mma.append(("arrive", ("fin",)))
    P["mma"] = mma
    for w in W:
        sm, gs = [], 0
        for ui in range(nitems):
            for s in range(nsteps):
                b = gs & 1
                sm += [("wait", ("m_full", gs & 3), gs >> 2), ("rbeg", ("meta", gs & 3), gs),
                       ("rend", ("meta", gs & 3)), ("arrive", ("m_empty", gs & 3))]
                if gs >= 2:
                    sm.append(("wait", ("p_empty", b), (gs >> 1) - 1))
                sm += [("wait", ("s_full",), gs), ("rbeg", ("S", w), gs), ("rend", ("S", w)), ("arrive", ("s_free",)),
                       ("wbeg", ("Pt", b, w), gs), ("wend", ("Pt", b, w))]
                if s > 0 and rescale(gs):
                    sm += [("wait", ("o_done",), gs - 1), ("wbeg", ("O", w), ("r", gs)), ("wend", ("O", w))]
                sm.append(("arrive", ("p_full", b)))
                gs += 1
            # epilogue: the last PV of the item complete (p_empty of its parity)
            sm += [("wait", ("p_empty", (gs - 1) & 1), (gs - 1) >> 1), ("rbeg", ("O", w), gs - 1), ("rend", ("O", w))]
        P[f"soft{w}"] = sm
    for x in range(4):
        C[("m_empty", x)] = nsoft
    for b in range(2):
        C[("p_full", b)] = nsoft
    C[("s_free",)] = nsoft
    return P, C


@pytest.mark.parametrize("nitems,nsteps", [(1, 1), (1, 3), (2, 1), (2, 2), (3, 3), (4, 2), (2, 5)])
def test_flash64_protocol(nitems, nsteps):
    for seed in range(60):
        pick = random.Random(1000 + seed)
        flags = {gs: pick.random() < 0.5 for gs in range(nitems * nsteps)}
        P, C = flash64_programs(nitems, nsteps, lambda gs: flags[gs])
        simulate(P, C, seed)


def test_checker_catches_the_epilogue_waiting_on_o_done():
    # The epilogue's wait for the last PV taken on o_done instead of p_empty:
    # o_done may have completed PV(gs-2), PV(gs-1), both or neither, so a
    # parity wait on it can alias.
    hits = 0
    for seed in range(300):
        pick = random.Random(seed)
        flags = {gs: pick.random() < 0.2 for gs in range(3 * 3)}
        P, C = flash64_programs(3, 3, lambda gs: flags[gs])
        for w in range(4):
            P[f"soft{w}"] = [("wait", ("o_done",), st[2] * 2 + (st[1][1])) if st[0] == "wait" and st[1][0] == "p_empty"
                             and i + 1 < len(P[f"soft{w}"]) and P[f"soft{w}"][i + 1][0] == "rbeg"
                             and P[f"soft{w}"][i + 1][1][0] == "O" else st for i, st in enumerate(P[f"soft{w}"])]
        try:
            simulate(P, C, seed)
        except Violation:
            hits += 1
    assert hits > 0


# ------------------------------------------------------------------ w8a8 --
def w8a8_programs(ntiles, nk, stages=6, accs=4, nepi=8):
    """w8a8_gemm_kernel: a K-step ring and four TMEM accumulators, both
    counted over all tiles of the CTA; every K block's INT32 product is read
    by the eight promotion warps before its accumulator is reused."""
    P, C = {}, defaultdict(lambda: 1)
    n = ntiles * nk
    prod = []
    for it in range(n):
        st = it % stages
        if it >= stages:
            prod.append(("wait", ("empty", st), it // stages - 1))
        prod += [("wbeg", ("AB", st), it), ("wend", ("AB", st)), ("arrive", ("full", st))]
    P["producer"] = prod
    mma = []
    for it in range(n):
        st, b = it % stages, it % accs
        mma.append(("wait", ("full", st), it // stages))
        if it >= accs:
            mma.append(("wait", ("acc_empty", b), it // accs - 1))
        mma += [("rbeg", ("AB", st), it), ("wbeg", ("acc", b), it), ("rend", ("AB", st)), ("wend", ("acc", b)),
                ("arrive", ("empty", st)), ("arrive", ("acc_full", b))]
    mma.append(("arrive", ("fin",)))
    P["mma"] = mma
    for e in range(nepi):
        ep = []
        for it in range(n):
            b = it % accs
            ep += [("wait", ("acc_full", b), it // accs), ("rbeg", ("acc", b), it), ("rend", ("acc", b)),
                   ("arrive", ("acc_empty", b))]
        P[f"promo{e}"] = ep
    for b in range(accs):
        C[("acc_empty", b)] = nepi
    return P, C


@pytest.mark.parametrize("ntiles,nk", [(1, 1), (1, 7), (2, 3), (3, 40), (5, 2)])
def test_w8a8_gemm_protocol(ntiles, nk):
    P, C = w8a8_programs(ntiles, nk)
    for seed in range(30):
        simulate(P, C, seed)


# ------------------------------------------------------------------ quant --
def quant_programs(ntiles, q_tok, nwarps=4, stages=3):
    """quant_kernel: thread 0 (in warp 0) keeps a 3-stage ring of bulk copies
    of the Q, K, V rows one tile ahead per stage; block barriers (one phase
    per use, all warps) order the reads of a stage before its refill and the
    reuse of the tile images, partial sums and per-warp maxima across tiles."""
    P, C = {}, defaultdict(lambda: 1)
    for w in range(nwarps):
        pr = []
        issued = 0
        if w == 0:
            while issued < min(stages, ntiles):
                st = issued % stages
                pr += [("wbeg", ("stage", st), issued), ("wend", ("stage", st)), ("arrive", ("full", st))]
                issued += 1
        for j in range(ntiles):
            st = j % stages
            pr += [("wait", ("full", st), j // stages), ("arrive", ("A", j)), ("wait", ("A", j), 0),
                   ("rbeg", ("stage", st), j), ("wbeg", ("img", 2), j), ("wend", ("img", 2)),
                   ("rend", ("stage", st)), ("wbeg", ("red", w), j), ("wend", ("red", w)),
                   ("arrive", ("B", j)), ("wait", ("B", j), 0)]
            if w == 0 and issued < ntiles:  # refill the stage just read
                pr += [("wbeg", ("stage", issued % stages), issued), ("wend", ("stage", issued % stages)),
                       ("arrive", ("full", issued % stages))]
                issued += 1
            pr += [("rbeg", ("red", x), j) for x in range(nwarps)] + [("rend", ("red", x)) for x in range(nwarps)]
            if q_tok:
                pr += [("wbeg", ("rowmax", w), j), ("wend", ("rowmax", w)), ("arrive", ("R", j)), ("wait", ("R", j), 0)]
                pr += [("rbeg", ("rowmax", x), j) for x in range(nwarps)] + [("rend", ("rowmax", x)) for x in range(nwarps)]
            pr += [("wbeg", ("img", 0), j), ("wend", ("img", 0)), ("wbeg", ("psum", w), j), ("wend", ("psum", w)),
                   ("arrive", ("C", j)), ("wait", ("C", j), 0)]
            pr += [("rbeg", ("psum", x), j) for x in range(nwarps)] + [("rend", ("psum", x)) for x in range(nwarps)]
            pr += [("rbeg", ("img", x), j) for x in (0, 2)] + [("rend", ("img", x)) for x in (0, 2)]
        P[f"warp{w}"] = pr
    for j in range(ntiles):
        for b in ("A", "B", "R", "C"):
            C[(b, j)] = nwarps
    return P, C


@pytest.mark.parametrize("ntiles,q_tok", [(1, 0), (2, 1), (3, 0), (4, 1), (7, 0), (8, 1)])
def test_quant_ring_protocol(ntiles, q_tok):
    P, C = quant_programs(ntiles, q_tok)
    for seed in range(40):
        simulate(P, C, seed)


def test_checker_catches_a_refill_before_the_barrier():
    # thread 0 refilling the stage before every warp has passed barrier B
    P, C = quant_programs(4, 0)
    prog = P["warp0"]
    i = next(i for i, st in enumerate(prog) if st == ("arrive", ("B", 0)))
    k = next(i for i, st in enumerate(prog) if st[0] == "wbeg" and st[1] == ("stage", 0) and st[2] == 3)
    refill = prog[k:k + 3]
    P["warp0"] = prog[:i] + refill + prog[i:k] + prog[k + 3:]
    assert _caught(P, C)


# --------------------------------------------------------------- pool_topk --
def pool_topk16_programs(nchunk, nthreads=4, nbuf=3):
    """pool_topk16_kernel phase 1: every thread copies its share of kbar chunk
    c into buffer c % 3 with cp.async (one commit group per chunk), two chunks
    ahead; cp.async.wait_group<2> (or <1>, <0> at the tail) retires its own
    groups up to chunk c, a block barrier publishes them, the chunk is scored,
    and a second barrier ends every read of the buffer before it is refilled.
    A thread's copy of chunk c is 'being written' from its issue until the
    wait that retires its group."""
    P, C = {}, defaultdict(lambda: 1)
    for t in range(nthreads):
        pr, pending = [], []

        def issue(c):
            pr.append(("wbeg", ("kb", c % nbuf, t), c))
            pending.append(c)

        def wait_group(n):  # all but the n most recent of this thread's groups complete
            while len(pending) > n:
                c = pending.pop(0)
                pr.append(("wend", ("kb", c % nbuf, t)))

        issue(0)
        if nchunk > 1:
            issue(1)
        for c in range(nchunk):
            if c + 2 < nchunk:
                issue(c + 2)
                wait_group(2)
            elif c + 1 < nchunk:
                wait_group(1)
            else:
                wait_group(0)
            pr += [("arrive", ("S1", c)), ("wait", ("S1", c), 0)]
            pr += [("rbeg", ("kb", c % nbuf, x), c) for x in range(nthreads)]
            pr += [("rend", ("kb", c % nbuf, x)) for x in range(nthreads)]
            pr += [("wbeg", ("psc", t), c), ("wend", ("psc", t)), ("arrive", ("S2", c)), ("wait", ("S2", c), 0)]
            pr += [("rbeg", ("psc", x), c) for x in range(nthreads)] + [("rend", ("psc", x)) for x in range(nthreads)]
        P[f"t{t}"] = pr
    for c in range(nchunk):
        C[("S1", c)] = C[("S2", c)] = nthreads
    return P, C


@pytest.mark.parametrize("nchunk", [1, 2, 3, 4, 7, 19])
def test_pool_topk16_ring_protocol(nchunk):
    P, C = pool_topk16_programs(nchunk)
    for seed in range(40):
        simulate(P, C, seed)


def test_checker_catches_a_two_buffer_ring_two_chunks_ahead():
    # two buffers with the same two-chunk lookahead: chunk c + 2 overwrites the buffer still being scored
    P, C = pool_topk16_programs(5, nbuf=2)
    assert _caught(P, C)
