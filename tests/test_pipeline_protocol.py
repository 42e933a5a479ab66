"""Model check of the prefill kernel's mbarrier protocol on the CPU.

The roles of one CTA of attn_fwd_fp4_kernel (TMA producer, MMA issuer, the
softmax warps) are replayed as cooperative processes.  The model carries:
- mbarriers with arrival counts and phase parity;
- TMA copies that complete asynchronously;
- tensor-core MMAs that complete in issue order;
- tcgen05.commit arrivals once every earlier MMA has completed.

A random scheduler interleaves the processes, and every wait is a parity wait
exactly as the kernel issues it.  The checks are:
- every wait returns only after the phase it is meant to see has completed
  (a parity wait that returns one lap early is the bug class this test
  guards against);
- every shared buffer (S in TMEM, P-hat in shared memory, O) is read and
  overwritten in the right order;
- every schedule finishes, so there is no deadlock.

The waits, counts and parities below restate the kernel's; keep them in step
with csrc/attn_fwd.cu.
"""
import random

import pytest


class ProtocolError(AssertionError):
    pass


BLOCKED = "blocked"


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1

    def parity_ready(self, parity):
        # mbarrier.try_wait.parity: true once the phase of that parity completed,
        # i.e. while the current (incomplete) phase has the other parity
        return (self.phase & 1) != parity


class Sim:
    def __init__(self, nkt, NS, NSB, NH, rng, fused_q=False, relax_lag=None, two_issuers=False, kv_one=True,
                 qbias=False):
        self.nkt, self.NS, self.NSB, self.NH, self.rng = nkt, NS, NSB, NH, rng
        # a warp that does not rescale O in tile j waits for PV_{j - relax_lag},
        # or for no product at all (None: the kernel with one MMA-issuing
        # thread, where the S_j wait covers PV_{j-2}); 1 waits for the
        # previous product on every tile
        self.relax_lag = relax_lag
        # two MMA-issuing threads: S and PV products complete in two
        # independent orders
        self.two_issuers = two_issuers
        # one barrier per K/V stage that completes when both copies landed
        # (the kernel's default), or one barrier per copy
        self.kv_one = kv_one
        # the Q-Mean score terms ride on the K/V barrier; the softmax warps
        # wait for it before reading them (and the TMA reloads a stage only
        # after PV of its previous tile)
        self.qbias = qbias
        self.bias_stage = [None] * NS
        self.W = 4 * NH
        self.fused_q = fused_q
        B = Barrier
        # the Q tile comes from one tensor copy, or (fused path) from every
        # softmax warp quantizing its rows, one arrival each
        self.bars = {"QFULL": B("QFULL", self.W if fused_q else 1)}
        # row-max exchange: one barrier per TMEM lane quadrant, the two warps
        # that share its rows arrive once per tile
        for q in range(4):
            self.bars[f"XM{q}"] = B(f"XM{q}", 2)
        self.q_rows_written = set()
        for s in range(NS):
            for n in ("KFULL", "KEMPTY", "VFULL", "VEMPTY"):
                self.bars[f"{n}{s}"] = B(f"{n}{s}", 1)
            self.bars[f"KVFULL{s}"] = B(f"KVFULL{s}", 2)
        for s in range(NSB):
            self.bars[f"SFULL{s}"] = B(f"SFULL{s}", 1)
            self.bars[f"SEMPTY{s}"] = B(f"SEMPTY{s}", self.W)
        for s in range(2):
            self.bars[f"PFULL{s}"] = B(f"PFULL{s}", self.W)
            self.bars[f"PEMPTY{s}"] = B(f"PEMPTY{s}", 1)
        # shared state with tags
        self.s_buf = [None] * NSB          # tile held by each S buffer
        self.s_readers = [set() for _ in range(NSB)]
        self.p_buf = [dict() for _ in range(2)]   # warp -> tile written
        self.k_stage = [None] * NS
        self.v_stage = [None] * NS
        self.xm = [dict(), dict()]
        self.pv_done = -1                  # last PV completed
        self.pv_started = -1               # last PV begun
        self.mma_queue = []                # in-order async tensor-core work (one issuer)
        self.pv_queue = []                 # PV products of a second issuer
        self.copies = []                   # pending TMA copies

    # -------------------------------------------------------------- waits ---
    def wait(self, bar, parity, min_phase):
        """Generator step: block until the parity wait returns, then check that
        the phase this wait means (min_phase completions) has happened."""
        b = self.bars[bar]
        while not b.parity_ready(parity):
            yield BLOCKED
        if b.phase < min_phase:
            raise ProtocolError(f"{bar}: parity wait returned at phase {b.phase}, needs >= {min_phase}")

    # -------------------------------------------------------------- roles ---
    def tma(self):
        for j in range(self.nkt):
            st, ph = j % self.NS, (j // self.NS) & 1
            yield from self.wait(f"KEMPTY{st}", ph ^ 1, j // self.NS)
            self.copies.append(("K", st, j))
            yield from self.wait(f"VEMPTY{st}", ph ^ 1, j // self.NS)
            self.copies.append(("V", st, j))

    def mma(self):
        yield from self.wait("QFULL", 0, 1)
        if self.fused_q and len(self.q_rows_written) != self.W:
            raise ProtocolError(f"QK^T issued with Q-hat rows of {sorted(self.q_rows_written)} written")

        def issue_s(j):
            st, sb = j % self.NS, j % self.NSB
            full = "KVFULL" if self.kv_one else "KFULL"
            yield from self.wait(f"{full}{st}", (j // self.NS) & 1, j // self.NS + 1)
            yield from self.wait(f"SEMPTY{sb}", ((j // self.NSB) & 1) ^ 1, j // self.NSB)
            self.mma_queue.append(("S", j, [f"SFULL{sb}", f"KEMPTY{st}"]))

        def issue_pv(j):
            st, pb = j % self.NS, j & 1
            # V_j first (its scale copy goes ahead of the wait for P-hat_j)
            if not self.kv_one:
                yield from self.wait(f"VFULL{st}", (j // self.NS) & 1, j // self.NS + 1)
            elif self.two_issuers:
                yield from self.wait(f"KVFULL{st}", (j // self.NS) & 1, j // self.NS + 1)
            yield from self.wait(f"PFULL{pb}", (j >> 1) & 1, (j >> 1) + 1)
            (self.pv_queue if self.two_issuers else self.mma_queue).append(("PV", j, [f"VEMPTY{st}", f"PEMPTY{pb}"]))

        if self.nkt > 0:
            yield from issue_s(0)
        for j in range(self.nkt):
            if j + 1 < self.nkt:
                yield from issue_s(j + 1)
            yield from issue_pv(j)
        # (the kernel's K-scale copy on even tiles only and the normalizer
        # fused into the PV MMA change no barrier)

    def softmax(self, w):
        if self.fused_q:
            # quantize this warp's share of the Q tile, then arrive
            yield "work"
            self.q_rows_written.add(w)
            self.bars["QFULL"].arrive()
        for j in range(self.nkt):
            sb, pb = j % self.NSB, j & 1
            yield from self.wait(f"SFULL{sb}", (j // self.NSB) & 1, j // self.NSB + 1)
            if self.s_buf[sb] != j:
                raise ProtocolError(f"warp {w} read S buffer {sb} holding tile {self.s_buf[sb]} for tile {j}")
            self.s_readers[sb].add(w)
            self.bars[f"SEMPTY{sb}"].arrive()
            if self.qbias:
                st = j % self.NS
                yield from self.wait(f"KVFULL{st}", (j // self.NS) & 1, j // self.NS + 1)
                if self.v_stage[st] != j:
                    raise ProtocolError(f"warp {w} read the score terms of stage {st} holding {self.v_stage[st]}")
            if self.NH == 2:
                self.xm[j & 1][w] = j
                self.bars[f"XM{w & 3}"].arrive()
                yield from self.wait(f"XM{w & 3}", j & 1, j + 1)
                partner = w ^ 4
                if self.xm[j & 1].get(partner) != j:
                    raise ProtocolError(f"warp {w} read the row max of tile {self.xm[j & 1].get(partner)} for {j}")
            # the warp's rescale vote comes first; a rescaling warp waits for
            # the previous product PV_{j-1} (which also covers the P-hat
            # buffer's last reader PV_{j-2}: commits complete in order), any
            # other warp for PV_{j-relax_lag} only
            rescale = j > 0 and self.rng.random() < 0.5
            jw = j - 1 if rescale else (j - self.relax_lag if self.relax_lag is not None else -1)
            if jw >= 0:
                yield from self.wait(f"PEMPTY{jw & 1}", (jw >> 1) & 1, (jw >> 1) + 1)
            if self.pv_done < j - 2:
                raise ProtocolError(f"warp {w} overwrote P-hat buffer {pb} before PV_{j - 2} retired")
            self.p_buf[pb][w] = j
            if rescale:
                if self.pv_done < j - 1 or self.pv_started >= j:
                    raise ProtocolError(f"warp {w} rescaled O for tile {j} with PV_{self.pv_done} done, "
                                        f"PV_{self.pv_started} started")
            self.bars[f"PFULL{pb}"].arrive()
        yield from self.epilogue(w)

    def epilogue(self, w):
        # O is final once the last PV retired
        if self.nkt > 0:
            jl = self.nkt - 1
            yield from self.wait(f"PEMPTY{jl & 1}", (jl >> 1) & 1, (jl >> 1) + 1)
            self.check_o(w)

    def check_o(self, w):
        if self.pv_done != self.nkt - 1:
            raise ProtocolError(f"warp {w} read O with PV_{self.pv_done} of {self.nkt - 1} done")

    # ------------------------------------------------------ async engines ---
    def step_async(self):
        """One asynchronous event, if any: a TMA copy lands, or the next MMA in
        issue order completes and its commits arrive."""
        events = []
        if self.copies:
            events.append("copy")
        if self.mma_queue:
            events.append("mma")
        if self.pv_queue:
            events.append("pv")
        if not events:
            return False
        ev = self.rng.choice(events)
        if ev == "copy":
            kind, st, j = self.copies.pop(self.rng.randrange(len(self.copies)))
            (self.k_stage if kind == "K" else self.v_stage)[st] = j
            self.bars[f"KVFULL{st}" if self.kv_one else f"{kind}FULL{st}"].arrive()
            return True
        kind, j, commits = (self.mma_queue if ev == "mma" else self.pv_queue).pop(0)
        if kind == "S":
            sb = j % self.NSB
            if self.k_stage[j % self.NS] != j:
                raise ProtocolError(f"S_{j} read K stage holding tile {self.k_stage[j % self.NS]}")
            if self.s_buf[sb] is not None and len(self.s_readers[sb]) != self.W:
                raise ProtocolError(f"S_{j} overwrote buffer {sb} before every warp read tile {self.s_buf[sb]}")
            self.s_buf[sb], self.s_readers[sb] = j, set()
        else:
            pb = j & 1
            if set(self.p_buf[pb].values()) != {j} or len(self.p_buf[pb]) != self.W:
                raise ProtocolError(f"PV_{j} read P-hat buffer {pb} holding {self.p_buf[pb]}")
            if self.v_stage[j % self.NS] != j:
                raise ProtocolError(f"PV_{j} read V stage holding tile {self.v_stage[j % self.NS]}")
            self.pv_started = j
            self.pv_done = j
        for c in commits:
            self.bars[c].arrive()
        return True

    def run(self):
        if not self.fused_q:
            self.bars["QFULL"].arrive()    # the Q tile (its copy lands before anything else matters)
        live = [self.tma(), self.mma()] + [self.softmax(w) for w in range(self.W)]
        idle = 0
        while live or self.mma_queue or self.pv_queue or self.copies:
            progressed = self.rng.random() < 0.5 and self.step_async()
            self.rng.shuffle(live)
            finished = []
            for p in live[: self.rng.randint(1, len(live))] if live else []:
                try:
                    if next(p) != BLOCKED:
                        progressed = True
                except StopIteration:
                    finished.append(p)
                    progressed = True
            live = [p for p in live if p not in finished]
            if progressed or self.step_async():
                idle = 0
            else:
                idle += 1
                if idle > 500:
                    raise ProtocolError("deadlock: every role waits and no copy or MMA is in flight")
        return True


@pytest.mark.parametrize("NH,NS,NSB", [(1, 3, 1), (2, 3, 1), (2, 3, 2), (2, 2, 2), (1, 2, 1)])
@pytest.mark.parametrize("nkt", [1, 2, 3, 5, 9])
@pytest.mark.parametrize("relax_lag,kv_one", [(None, True), (1, True), (None, False)])
def test_prefill_protocol_random_schedules(NH, NS, NSB, nkt, relax_lag, kv_one):
    for seed in range(40):
        Sim(nkt, NS, NSB, NH, random.Random(1000 * nkt + seed), relax_lag=relax_lag, kv_one=kv_one).run()


@pytest.mark.parametrize("NH,NSB", [(1, 1), (2, 2)])
@pytest.mark.parametrize("nkt", [1, 3, 7])
def test_q_mean_terms_protocol(NH, NSB, nkt):
    """The Q-Mean score terms travel with V on the stage's single K/V
    barrier; a softmax warp reads stage j % NS only while it holds tile j."""
    for seed in range(40):
        Sim(nkt, 3, NSB, NH, random.Random(5000 * nkt + seed), qbias=True).run()


@pytest.mark.parametrize("nkt", [2, 5, 9])
def test_two_issuers_wait_for_the_buffer_reader(nkt):
    """With S and PV issued by two threads, nothing orders S_j after
    PV_{j-2}: the kernel then waits for PV_{j-2} in tiles without a rescale."""
    for seed in range(40):
        Sim(nkt, 3, 1, 1, random.Random(3000 * nkt + seed), relax_lag=2, two_issuers=True).run()


@pytest.mark.parametrize("kw", [dict(relax_lag=3), dict(relax_lag=None, two_issuers=True)])
def test_model_catches_a_missing_buffer_wait(kw):
    # (the K/V barrier layout does not matter here)
    """Waiting for PV_{j-3} in tiles without a rescale, or for nothing when
    two threads issue the products, lets a warp overwrite the P-hat buffer
    that PV_{j-2} may still read (or parity-wait on a phase two laps back):
    the model must flag it."""
    caught = 0
    for seed in range(200):
        try:
            Sim(7, 3, 1, 1, random.Random(seed), **kw).run()
        except ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("NH,NS,NSB", [(1, 3, 1), (2, 3, 2), (2, 2, 2)])
@pytest.mark.parametrize("nkt", [1, 2, 5])
def test_fused_q_protocol_random_schedules(NH, NS, NSB, nkt):
    """The fused path: the softmax warps write Q-hat before their first wait;
    QK^T must not start before every warp's rows are written."""
    for seed in range(40):
        Sim(nkt, NS, NSB, NH, random.Random(7000 * nkt + seed), fused_q=True).run()


def test_model_catches_a_short_q_barrier():
    """A Q barrier that completes after one arrival lets QK^T start before
    the other warps have written their rows: the model must flag it."""
    caught = 0
    for seed in range(100):
        sim = Sim(3, 3, 1, 1, random.Random(seed), fused_q=True)
        sim.bars["QFULL"] = Barrier("QFULL", 1)
        try:
            sim.run()
        except ProtocolError:
            caught += 1
    assert caught > 0


def test_model_catches_a_one_lap_early_epilogue():
    """The model must flag the bug class it guards: an epilogue that waits on
    a barrier only the rescaling tiles await (so it can lag two phases) and
    parity-waits for the last phase."""

    class Buggy(Sim):
        def __init__(self, *a):
            super().__init__(*a)
            self.bars["ORDY"] = Barrier("ORDY", 1)

        def step_async(self):
            if self.mma_queue and self.mma_queue[0][0] == "PV":
                self.mma_queue[0][2].append("ORDY")
            return super().step_async()

        def epilogue(self, w):
            # the old epilogue: a parity wait on a barrier that lags when the
            # last tiles needed no rescale
            jl = self.nkt - 1
            b = self.bars["ORDY"]
            while not b.parity_ready(jl & 1):
                yield BLOCKED
            self.check_o(w)

    caught = 0
    for seed in range(200):
        sim = Buggy(6, 3, 1, 1, random.Random(seed))
        sim.rng = random.Random(seed)
        try:
            sim.run()
        except ProtocolError:
            caught += 1
    assert caught > 0
