"""The multi-stream enqueue orders of the preparation and of the quantizer, replayed on the CPU.

`csrc/prepare.cu` factors A = L L^T and builds Xt = (L^-1)^T panel by panel on four
streams (c: the diagonal blocks, o: L21 and the next block column, t: trailing
updates, s: the inverse), ordered only by event records and waits.  This module
restates both enqueue loops, `panel_loop` (128-wide panels) and `panel_loop_deferred`
(128-wide panels inside 512-wide outer panels), launch by launch, with the regions of
each buffer that every launch reads and writes, and checks three things:

* no race: every two launches on different streams that touch overlapping regions,
  one of them writing, are ordered by a chain of stream order and event waits (the
  happens-before closure of the enqueue sequence, with CUDA's rule that a wait refers
  to the event's latest record at the time of the wait, and a wait on an event never
  recorded is a no-op);
* exactness: running the launches in enqueue order in fp64, with the same region
  arithmetic, gives (L^-1)^T of the input to rounding;
* sensitivity: removing any one of the load-bearing waits is reported as a race.

Four waits of the C++ loops are implied by the others plus stream order, so removing one
alone leaves no race: the panel stream's waits for a ring slot's previous trailing update
and inverse (panel_loop; the previous panel's wait for the trailing update and the diagonal
launch's wait for the inverse reach them first), its wait for the previous outer panel's
bulk update (panel_loop_deferred; the in-panel waits for the trailing stream reach it), and
the inverse stream's wait for the outer panel's L21 (its per-panel L21 waits reach it).
They stay in the C++ so that every launch states its own inputs.

The quantizer's two streams (`csrc/quantize.cu`, super_block_loop) are replayed the same
way at the end of the module; there every wait is load-bearing, and the blocked order
must give the codes of the unblocked column loop.

The restatement must change with the C++ loops: it is a model of them, not derived
from them.  The GPU tests check the result of the real enqueue against the oracle.
"""
import numpy as np
import pytest

PB, SPB, NBUF, NSUP = 128, 512, 3, 3
NLI = 3 * (SPB // PB)


class Sim:
    """Launches on named streams, event records and waits, and their happens-before order."""

    def __init__(self, skip=()):
        self.ops = []          # (stream, reads, writes, fn, name)
        self.deps = []         # per op: the ops it follows directly
        self.last = {}         # stream -> its last op
        self.events = {}       # event -> the op its latest record follows (None: nothing yet)
        self.pending = {}      # stream -> ops waited for since its last op
        self.skip = set(skip)

    def record(self, ev, strm):
        self.events[ev] = self.last.get(strm)

    def wait(self, strm, ev, label=None):
        if label is not None and label in self.skip:
            return
        d = self.events.get(ev)
        if d is not None:
            self.pending.setdefault(strm, set()).add(d)

    def op(self, strm, reads, writes, fn, name):
        deps = set(self.pending.pop(strm, set()))
        if strm in self.last:
            deps.add(self.last[strm])
        self.ops.append((strm, reads, writes, fn, name))
        self.deps.append(deps)
        self.last[strm] = len(self.ops) - 1

    def races(self):
        hb = []
        for d in self.deps:
            m = 0
            for j in d:
                m |= hb[j] | (1 << j)
            hb.append(m)

        def ov(a, b):
            return a[0] == b[0] and a[1] < b[2] and b[1] < a[2] and a[3] < b[4] and b[3] < a[4]

        found = []
        for i, (_, ri, wi, _, ni) in enumerate(self.ops):
            for j in range(i):
                if (hb[i] >> j) & 1:
                    continue
                _, rj, wj, _, nj = self.ops[j]
                if any(ov(a, b) for a in wi for b in wj + rj) or any(ov(a, b) for a in ri for b in wj):
                    found.append((nj, ni))
        return found

    def run(self):
        for op in self.ops:
            op[3]()


def R(buf, r0, r1, c0, c1):
    """Rows [r0, r1) and columns [c0, c1) of a buffer."""
    return (buf, r0, r1, c0, c1)


def _spd(n, seed):
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((n, n + 20))
    return G @ G.T / n + 0.1 * np.eye(n)


def _potrf(sim, A, LI, k0, nb, b, b1, kp):
    """potrf_inv_kernel: the previous panel's term of the diagonal block, then its
    factor's inverse T into LI[b] (zero past nb)."""
    def fn():
        D = np.tril(A[k0:k0 + nb, k0:k0 + nb])
        D = D + np.tril(D, -1).T
        if kp >= 0:
            Lk = A[k0:k0 + nb, kp:kp + PB] @ LI[b1].T
            D = D - Lk @ Lk.T
        T = np.zeros((PB, PB))
        T[:nb, :nb] = np.linalg.inv(np.linalg.cholesky(D))
        LI[b][:] = T
    reads = [R("A", k0, k0 + nb, k0, k0 + nb)]
    if kp >= 0:
        reads += [R("A", k0, k0 + nb, kp, kp + PB), R("LI", b1, b1 + 1, 0, 1)]
    sim.op("c", reads, [R("LI", b, b + 1, 0, 1)], fn, f"potrf{k0}")


def model_panel_loop(n, skip=(), seed=0):
    """panel_loop: per panel k, the ring slot b = k mod NBUF holds L21 (Lr) and T_k (LI)."""
    A0 = _spd(n, seed)
    A = A0.copy()
    Xt = np.zeros((n, n))
    Phi, XP, XQ = np.zeros((n, PB)), np.zeros((n, PB)), np.zeros((n, PB))
    Lr = [np.full((n, PB), np.nan) for _ in range(NBUF)]
    LI = [np.full((PB, PB), np.nan) for _ in range(NBUF)]
    sim = Sim(skip)
    c, o, t, s = "c", "o", "t", "s"
    for panel, k0 in enumerate(range(0, n, PB)):
        nb, rest = min(PB, n - k0), n - min(n, k0 + PB)
        b, b1, b2 = panel % NBUF, (panel - 1) % NBUF, (panel - 2) % NBUF
        # ---- the diagonal block ----
        if panel >= 2:
            sim.wait(c, ("next", b2), "c_next")
            sim.wait(c, ("trail", b2), "c_trail")
        if panel >= NBUF:
            sim.wait(c, ("done", b), "c_done")
        _potrf(sim, A, LI, k0, nb, b, b1, k0 - PB if panel > 0 else -1)
        sim.record(("diag", b), c)
        if rest > 0:
            # ---- L21 and the next block column ----
            sim.wait(o, ("diag", b), "o_diag")
            if panel >= NBUF:
                sim.wait(o, ("trail", b), "o_trail_slot")
                sim.wait(o, ("done", b), "o_done_slot")
            if panel == 0:
                def fn(nb=nb, rest=rest):
                    Phi[:rest, :nb] = A[nb:nb + rest, :nb]
                sim.op(o, [R("A", nb, n, 0, nb)], [R("Phi", 0, n, 0, PB)], fn, "split0")

            def fn(nb=nb, rest=rest, b=b):
                Lr[b][:rest, :nb] = Phi[:rest, :nb] @ LI[b][:nb, :nb].T
            sim.op(o, [R("Phi", 0, n, 0, PB), R("LI", b, b + 1, 0, 1)], [R(("L", b), 0, n, 0, PB)], fn,
                   f"l21_{k0}")
            sim.record(("l21", b), o)
            nb2 = min(PB, rest)
            if rest > nb2:
                if panel >= 1:
                    sim.wait(o, ("trail", b1), "o_trail_prev")
                r2, c1 = k0 + nb + nb2, k0 + nb

                def fn(nb=nb, nb2=nb2, r2=r2, c1=c1, b=b, rest=rest):
                    A[r2:n, c1:c1 + nb2] -= Lr[b][nb2:rest, :nb] @ Lr[b][:nb2, :nb].T
                    Phi[:n - r2, :nb2] = A[r2:n, c1:c1 + nb2]
                sim.op(o, [R(("L", b), 0, n, 0, PB), R("A", r2, n, c1, c1 + nb2)],
                       [R("A", r2, n, c1, c1 + nb2), R("Phi", 0, n, 0, PB)], fn, f"next{k0}")
                sim.record(("next", b), o)
                # ---- the trailing update of blocks >= k + 2 ----
                sim.wait(t, ("l21", b), "t_l21")

                def fn(nb=nb, nb2=nb2, r2=r2, b=b, rest=rest):
                    L2 = Lr[b][nb2:rest, :nb]
                    A[r2:n, r2:n] -= L2 @ L2.T
                sim.op(t, [R(("L", b), 0, n, 0, PB), R("A", r2, n, r2, n)], [R("A", r2, n, r2, n)], fn,
                       f"trail{k0}")
                sim.record(("trail", b), t)
        # ---- the inverse's block column k ----
        sim.wait(s, ("diag", b), "s_diag")

        def fn(k0=k0, nb=nb, b=b):
            Xt[k0:k0 + nb, k0:k0 + nb] = LI[b][:nb, :nb].T
            XQ[k0:k0 + nb, :] = LI[b][:, :nb].T
        sim.op(s, [R("LI", b, b + 1, 0, 1)], [R("Xt", k0, k0 + nb, k0, k0 + nb), R("XQ", k0, k0 + nb, 0, PB)],
               fn, f"xtdiag{k0}")
        if k0 > 0:
            def fn(k0=k0, nb=nb, b=b):
                XP[:k0, :nb] = Xt[:k0, k0:k0 + nb]
                Xt[:k0, k0:k0 + nb] = XP[:k0, :nb] @ LI[b][:nb, :nb].T
                XQ[:k0, :nb] = Xt[:k0, k0:k0 + nb]
            sim.op(s, [R("Xt", 0, k0, k0, k0 + nb), R("LI", b, b + 1, 0, 1)],
                   [R("Xt", 0, k0, k0, k0 + nb), R("XP", 0, n, 0, PB), R("XQ", 0, k0, 0, PB)], fn, f"xtcol{k0}")
        if rest > 0:
            sim.wait(s, ("l21", b), "s_l21")

            def fn(k0=k0, nb=nb, b=b, rest=rest):
                Xt[:k0 + nb, k0 + nb:] -= XQ[:k0 + nb, :nb] @ Lr[b][:rest, :nb].T
            sim.op(s, [R("XQ", 0, k0 + nb, 0, PB), R(("L", b), 0, n, 0, PB), R("Xt", 0, k0 + nb, k0 + nb, n)],
                   [R("Xt", 0, k0 + nb, k0 + nb, n)], fn, f"xtrest{k0}")
        sim.record(("done", b), s)
    return sim, A0, Xt


def model_panel_loop_deferred(n, skip=(), seed=0):
    """panel_loop_deferred: per outer panel S (slot sb = S mod NSUP) the L21 of its four
    panels in Sh[sb] and the finished Xt columns in SX; T_k in the ring LI[k mod NLI]."""
    A0 = _spd(n, seed)
    A = A0.copy()
    Xt = np.zeros((n, n))
    Phi, XP = np.zeros((n, PB)), np.zeros((n, PB))
    Sh = [np.full((n, SPB), np.nan) for _ in range(NSUP)]
    SX = np.full((n, SPB), np.nan)
    LI = [np.full((PB, PB), np.nan) for _ in range(NLI)]
    sim = Sim(skip)
    c, o, t, s = "c", "o", "t", "s"
    for S, s0 in enumerate(range(0, n, SPB)):
        se, sb = min(n, s0 + SPB), S % NSUP
        Lb = Sh[sb]
        for k0 in range(s0, se, PB):
            p, j = k0 // PB, (k0 - s0) // PB
            nb, rest = min(PB, n - k0), n - min(n, k0 + PB)
            b, b1, b2 = p % NLI, (p - 1) % NLI, (p - 2) % NLI
            cj = PB * j
            if j == 0 and S > 0:
                sim.wait(c, ("col", sb), "c_col")
            if j >= 2:
                sim.wait(c, ("next", b2), "c_next")
                sim.wait(c, ("trail", b2), "c_trail")
            if p >= NLI:
                sim.wait(c, ("done", b), "c_done")
            _potrf(sim, A, LI, k0, nb, b, b1, k0 - PB if j > 0 else -1)
            sim.record(("diag", b), c)
            if rest > 0:
                sim.wait(o, ("diag", b), "o_diag")
                if j == 0 and S >= NSUP:
                    sim.wait(o, ("bulk", sb), "o_bulk_slot")
                    sim.wait(o, ("inv", sb), "o_inv_slot")
                if p == 0:
                    def fn(nb=nb, rest=rest):
                        Phi[:rest, :nb] = A[nb:nb + rest, :nb]
                    sim.op(o, [R("A", nb, n, 0, nb)], [R("Phi", 0, n, 0, PB)], fn, "split0")

                def fn(k0=k0, nb=nb, rest=rest, b=b, cj=cj, Lb=Lb):
                    Lb[k0 + nb:n, cj:cj + nb] = Phi[:rest, :nb] @ LI[b][:nb, :nb].T
                sim.op(o, [R("Phi", 0, n, 0, PB), R("LI", b, b + 1, 0, 1)], [R(("S", sb), k0 + nb, n, cj, cj + PB)],
                       fn, f"l21_{k0}")
                sim.record(("l21", b), o)
                nb2 = min(PB, rest)
                if k0 + nb < se and rest > nb2:
                    if j >= 1:
                        sim.wait(o, ("trail", b1), "o_trail_prev")
                    r2, c1 = k0 + nb + nb2, k0 + nb

                    def fn(nb=nb, nb2=nb2, r2=r2, c1=c1, cj=cj, Lb=Lb):
                        A[r2:n, c1:c1 + nb2] -= Lb[r2:n, cj:cj + nb] @ Lb[c1:c1 + nb2, cj:cj + nb].T
                        Phi[:n - r2, :nb2] = A[r2:n, c1:c1 + nb2]
                    sim.op(o, [R(("S", sb), c1, n, cj, cj + PB), R("A", r2, n, c1, c1 + nb2)],
                           [R("A", r2, n, c1, c1 + nb2), R("Phi", 0, n, 0, PB)], fn, f"next{k0}")
                sim.record(("next", b), o)
                # the outer panel's columns beyond the next block column
                c0 = k0 + 2 * PB
                if c0 < se:
                    sim.wait(t, ("l21", b), "t_l21")

                    def fn(c0=c0, cj=cj, nb=nb, se=se, Lb=Lb):
                        A[c0:n, c0:se] -= Lb[c0:n, cj:cj + nb] @ Lb[c0:se, cj:cj + nb].T
                    sim.op(t, [R(("S", sb), c0, n, cj, cj + PB), R("A", c0, n, c0, se)], [R("A", c0, n, c0, se)],
                           fn, f"trail{k0}")
                sim.record(("trail", b), t)
            # ---- the inverse's block column p ----
            sim.wait(s, ("diag", b), "s_diag")

            def fn(k0=k0, nb=nb, b=b, cj=cj):
                Xt[k0:k0 + nb, k0:k0 + nb] = LI[b][:nb, :nb].T
                SX[k0:k0 + nb, cj:cj + PB] = LI[b][:, :nb].T
            sim.op(s, [R("LI", b, b + 1, 0, 1)], [R("Xt", k0, k0 + nb, k0, k0 + nb), R("SX", k0, k0 + nb, cj, cj + PB)],
                   fn, f"xtdiag{k0}")
            if k0 > 0:
                def fn(k0=k0, nb=nb, b=b, cj=cj):
                    XP[:k0, :nb] = Xt[:k0, k0:k0 + nb]
                    Xt[:k0, k0:k0 + nb] = XP[:k0, :nb] @ LI[b][:nb, :nb].T
                    SX[:k0, cj:cj + PB] = 0.0
                    SX[:k0, cj:cj + nb] = Xt[:k0, k0:k0 + nb]
                sim.op(s, [R("Xt", 0, k0, k0, k0 + nb), R("LI", b, b + 1, 0, 1)],
                       [R("Xt", 0, k0, k0, k0 + nb), R("XP", 0, n, 0, PB), R("SX", 0, k0, cj, cj + PB)], fn,
                       f"xtcol{k0}")
            if se > k0 + nb:
                def fn(k0=k0, nb=nb, cj=cj, se=se):
                    SX[k0 + nb:se, cj:cj + PB] = 0.0
                sim.op(s, [], [R("SX", k0 + nb, se, cj, cj + PB)], fn, f"zero{k0}")
            if rest > 0:
                sim.wait(s, ("l21", b), "s_l21")
                c1 = k0 + nb
                if c1 < se:
                    def fn(k0=k0, nb=nb, c1=c1, cj=cj, se=se, Lb=Lb):
                        Xt[:k0 + nb, c1:se] -= SX[:k0 + nb, cj:cj + nb] @ Lb[c1:se, cj:cj + nb].T
                    sim.op(s, [R("SX", 0, k0 + nb, cj, cj + PB), R(("S", sb), c1, se, cj, cj + PB),
                               R("Xt", 0, k0 + nb, c1, se)], [R("Xt", 0, k0 + nb, c1, se)], fn, f"xtin{k0}")
            sim.record(("done", b), s)
        if se >= n:
            break
        # ---- the outer panel's bulk updates (K = se - s0) ----
        se2, K, sn = min(n, se + SPB), se - s0, (S + 1) % NSUP
        sim.record(("lsup", sb), o)
        if S >= 1:
            sim.wait(o, ("bulk", (S - 1) % NSUP), "o_bulk_prev")

        def fn(se=se, se2=se2, K=K, Lb=Lb):
            A[se:n, se:se2] -= Lb[se:n, :K] @ Lb[se:se2, :K].T
            nbn = min(PB, n - se)
            if n - se - nbn > 0:
                Phi[:n - se - nbn, :nbn] = A[se + nbn:n, se:se + nbn]
        sim.op(o, [R(("S", sb), se, n, 0, SPB), R("A", se, n, se, se2)],
               [R("A", se, n, se, se2), R("Phi", 0, n, 0, PB)], fn, f"col{se}")
        sim.record(("col", sn), o)
        sim.wait(t, ("lsup", sb), "t_lsup")
        if se2 < n:
            def fn(se2=se2, K=K, Lb=Lb):
                A[se2:n, se2:n] -= Lb[se2:n, :K] @ Lb[se2:n, :K].T
            sim.op(t, [R(("S", sb), se2, n, 0, SPB), R("A", se2, n, se2, n)], [R("A", se2, n, se2, n)], fn,
                   f"bulk{se}")
        sim.record(("bulk", sb), t)
        sim.wait(s, ("lsup", sb), "s_lsup")

        def fn(se=se, K=K, Lb=Lb):
            Xt[:se, se:n] -= SX[:se, :K] @ Lb[se:n, :K].T
        sim.op(s, [R("SX", 0, se, 0, SPB), R(("S", sb), se, n, 0, SPB), R("Xt", 0, se, se, n)],
               [R("Xt", 0, se, se, n)], fn, f"binv{se}")
        sim.record(("inv", sb), s)
    return sim, A0, Xt


def _check(model, n, skip=()):
    sim, A0, Xt = model(n, skip)
    races = sim.races()
    sim.run()
    ref = np.linalg.inv(np.linalg.cholesky(A0)).T
    err = np.max(np.abs(np.triu(Xt) - ref)) / np.max(np.abs(ref))
    return races, err


# panel counts from one to 24, ragged last panels, every ring slot reused
@pytest.mark.parametrize("n", [128, 200, 300, 640, 1000, 1700, 3000])
def test_panel_loop_is_race_free_and_exact(n):
    races, err = _check(model_panel_loop, n)
    assert races == [], races[:4]
    assert err < 1e-12


# several outer panels, partial last ones, the outer-panel ring reused
@pytest.mark.parametrize("n", [256, 640, 1100, 1600, 2600])
def test_deferred_loop_is_race_free_and_exact(n):
    races, err = _check(model_panel_loop_deferred, n)
    assert races == [], races[:4]
    assert err < 1e-12


# each load-bearing wait, removed alone, leaves a race the check reports
@pytest.mark.parametrize("label", ["c_next", "c_trail", "c_done", "o_diag", "o_trail_prev", "t_l21", "s_diag",
                                   "s_l21"])
def test_panel_loop_missing_wait_is_reported(label):
    races, _ = _check(model_panel_loop, 1700, skip=(label,))
    assert races, label


@pytest.mark.parametrize("label", ["c_col", "c_next", "c_trail", "c_done", "o_diag", "o_trail_prev", "t_l21",
                                   "t_lsup", "s_diag", "s_l21"])
def test_deferred_loop_missing_wait_is_reported(label):
    races, _ = _check(model_panel_loop_deferred, 2600, skip=(label,))
    assert races, label


# the four implied waits: removing one alone leaves the order race-free
@pytest.mark.parametrize("model,label", [(model_panel_loop, "o_trail_slot"), (model_panel_loop, "o_done_slot"),
                                         (model_panel_loop_deferred, "o_bulk_prev"),
                                         (model_panel_loop_deferred, "s_lsup")])
def test_implied_waits(model, label):
    races, err = _check(model, 2600 if model is model_panel_loop_deferred else 1700, skip=(label,))
    assert races == [] and err < 1e-12


# ---------------------------------------------------------------------------
# The quantizer's two streams (`csrc/quantize.cu`, super_block_loop): per super-block
# of SBK = 512 columns, on the high-priority stream the sweep (its columns, the scaled
# errors E[b]) and the update of the next super-block's columns (near); on the other
# stream the operand B[b] = U[super-block, later columns]^T and the update of all
# columns after that (far).  E and B are double buffers (b = super-block mod 2).
# The sweep is modelled by GPTQ's column step without the group machinery: round the
# column, its error over the pivot, the update of the block's later columns; the
# whole order must then equal the unblocked column loop.
# ---------------------------------------------------------------------------
SBK = 512


def model_super_block_loop(out, n, skip=(), seed=0):
    rng = np.random.default_rng(seed)
    W0 = rng.standard_normal((out, n)) * 4.0
    U = np.triu(rng.standard_normal((n, n)) * 0.02, 1) + np.diag(1.0 + rng.random(n))
    Wf = W0.copy()
    codes = np.full((out, n), np.nan)
    E = [np.full((out, SBK), np.nan) for _ in range(2)]
    B = [np.full((n, SBK), np.nan) for _ in range(2)]
    sim = Sim(skip)
    hi, lo = "hi", "lo"
    S = -(-n // SBK)

    def operand(sb):
        b0, be, bb = sb * SBK, sb * SBK + SBK, sb & 1

        def fn():
            B[bb][:n - be, :] = U[b0:be, be:n].T
        sim.op(lo, [], [R(("B", bb), 0, n, 0, SBK)], fn, f"operand{sb}")
        sim.record(("opnd", bb), lo)

    for sb in range(min(2, S - 1)):
        operand(sb)
    for sb in range(S):
        b, s0 = sb & 1, sb * SBK
        se = min(n, s0 + SBK)

        def fn(b=b, s0=s0, se=se):
            for j in range(s0, se):
                q = np.round(Wf[:, j])
                codes[:, j] = q
                e = (Wf[:, j] - q) / U[j, j]
                E[b][:, j - s0] = e
                Wf[:, j + 1:se] -= np.outer(e, U[j, j + 1:se])
        sim.op(hi, [R("W", 0, out, s0, se)], [R("W", 0, out, s0, se), R(("E", b), 0, out, 0, SBK),
                                              R("codes", 0, out, s0, se)], fn, f"sweep{sb}")
        if se >= n:
            break
        kn = min(SBK, n - se)
        sim.record("swept", hi)
        sim.wait(hi, ("opnd", b), "hi_opnd")
        if sb > 0:
            sim.wait(hi, "far", "hi_far")

        def fn(b=b, se=se, kn=kn):
            Wf[:, se:se + kn] -= E[b] @ B[b][:kn].T
        sim.op(hi, [R(("E", b), 0, out, 0, SBK), R(("B", b), 0, kn, 0, SBK), R("W", 0, out, se, se + kn)],
               [R("W", 0, out, se, se + kn)], fn, f"near{sb}")
        sim.record("near", hi)
        if n - se > kn:
            sim.wait(lo, "swept", "lo_swept")

            def fn(b=b, se=se, kn=kn):
                Wf[:, se + kn:] -= E[b] @ B[b][kn:n - se].T
            sim.op(lo, [R(("E", b), 0, out, 0, SBK), R(("B", b), kn, n - se, 0, SBK), R("W", 0, out, se + kn, n)],
                   [R("W", 0, out, se + kn, n)], fn, f"far{sb}")
        sim.record("far", lo)
        if sb + 2 < S - 1:
            sim.wait(lo, "near", "lo_near")
            operand(sb + 2)
    return sim, W0, U, codes


def _check_quantizer(out, n, skip=()):
    sim, W0, U, codes = model_super_block_loop(out, n, skip)
    races = sim.races()
    sim.run()
    W = W0.copy()
    ref = np.empty_like(W)
    for j in range(n):                      # the unblocked column loop
        q = np.round(W[:, j])
        ref[:, j] = q
        e = (W[:, j] - q) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
    return races, np.array_equal(codes, ref)


# one super-block, two, and several with a ragged last one (every buffer reused)
@pytest.mark.parametrize("n", [300, 1024, 1800, 2600])
def test_quantizer_streams_are_race_free_and_match_the_column_loop(n):
    races, same = _check_quantizer(8, n)
    assert races == [], races[:4]
    assert same


@pytest.mark.parametrize("label", ["hi_opnd", "hi_far", "lo_swept", "lo_near"])
def test_quantizer_missing_wait_is_reported(label):
    races, _ = _check_quantizer(8, 2600, skip=(label,))
    assert races, label
