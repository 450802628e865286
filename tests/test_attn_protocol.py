"""Executable model of the attention kernel's barrier protocol (CPU).

The persistent attention kernel (csrc/attn.cu) coordinates its roles only
through mbarriers: a unit ring filled by a claimer lane, Q/K/V buffers loaded
by TMA, S/P/O in tensor memory, and the epilogue's staged output. A protocol
mistake there shows up on the GPU as a hang or as a buffer overwritten while
still in use. This model replays each role's sequence of waits, arrivals,
copies and MMA commits as in the kernel, for paired (two query tiles with
their own key/value streams) and 128-row (both halves share each key/value
tile) units, and runs them under random interleavings, with TMA copies
completing in any order and each issuer's MMAs completing in issue order.
Paired units may be split: both query halves hold the same query rows and
walk the two halves of one key list; the second half publishes its row
maxima and sums and hands its Q buffer back, and the first half reads the
second half's O, combines and stores.
It checks that:
- every wait targets the phase the kernel means (its parity never aliases a
  phase two away, in either direction) and that no run deadlocks;
- no buffer is written while a reader still needs it and no reader sees a
  buffer before it is filled.
Mistakes planted in copies of the model are caught, so the checks have teeth.
The softmax warpgroups are one agent each (their 128 arrivals count as one).
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_fvattn_b200", "csrc", "attn.cu")


def kernel_constant(name):
    return int(re.search(rf"constexpr int {name} = (\d+);", open(SRC).read()).group(1))


# ring depths as the kernel declares them
SLOTS, NK, NV = kernel_constant("kUnitSlots"), kernel_constant("kNK"), kernel_constant("kNV")
# roles that take every unit from the ring, in warps: the Q/K and V producers,
# the QK and PV issuers, and the 8 softmax warps
RING_CONSUMER_WARPS = 4 + 8


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.phase = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending > self.count:
            raise ProtocolError(f"{self.name}: more arrivals than its count")
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1

    def ready(self, k):
        """Would a parity wait for the completion of phase k return now?"""
        if self.phase >= k + 2:
            raise ProtocolError(f"{self.name}: wait for phase {k} lapped (now {self.phase}), parity aliases")
        if self.phase == k - 1:
            raise ProtocolError(f"{self.name}: wait for phase {k} would pass early on phase {k - 2}'s parity")
        return self.phase == k + 1


class Model:
    def __init__(self, units, paired, mutation=None):
        self.units = list(units)
        self.paired = paired
        self.mut = mutation
        B = Barrier
        self.b = {
            "QFull": [B("QFull0"), B("QFull1")], "QEmpty": [B("QEmpty0"), B("QEmpty1")],
            "KFull": [B(f"KFull{i}") for i in range(NK)], "KEmpty": [B(f"KEmpty{i}") for i in range(NK)],
            "VFull": [B(f"VFull{i}") for i in range(NV)], "VEmpty": [B(f"VEmpty{i}") for i in range(NV)],
            "SFull": [B("SFull0"), B("SFull1")], "SFree": B("SFree"),
            "PFull": [B("PFull0"), B("PFull1")], "PFree": [B("PFree0"), B("PFree1")],
            "OFull": [B("OFull0"), B("OFull1")], "OEmpty": [B("OEmpty0"), B("OEmpty1")],
            "UFull": [B(f"UFull{i}") for i in range(SLOTS)],
            "UEmpty": [B(f"UEmpty{i}", 6) for i in range(SLOTS)],   # producer, V, QK, PV, 2 softmax
            "Taken": B("Taken"),
            "Comb": B("Comb"),
            "OStaged": [B("OStaged0"), B("OStaged1")],
        }
        self.slots = [None] * SLOTS
        self.next_unit = 0
        # buffer states
        self.Q = ["free", "free"]
        self.K = ["free"] * NK
        self.V = ["free"] * NV
        self.S = "free"          # free -> writing -> full(h) -> free
        self.P = ["free", "free"]
        self.O = ["free", "free"]  # free -> acc -> complete -> free
        self.comb = "free"         # the second half's row maxima and sums of a split unit
        self.qk_inflight = [0, 0]
        self.combs = 0            # split units combined so far (the first half's Comb waits)
        self.async_tma = []       # (callback) completing in any order
        self.fifo = {"qk": [], "pv": [], "st0": [], "st1": []}

    # ---- helpers
    def need(self, cond, msg):
        if not cond:
            raise ProtocolError(msg)

    def tiles(self, u, h):
        """Key tiles of half h: paired, its own count; otherwise the unit's
        count for half 0 and, if the unit has a second half, for half 1."""
        if self.paired:
            return u[h]
        return u[0] if (h == 0 or u[1] > 0) else 0

    # ---- roles (generators yielding ("wait", barrier, phase) or ("arrive", barrier))
    def claimer(self):
        n = 0
        while True:
            if n > 0:
                k = n - 1 if self.mut != "claim_early" else n
                yield ("wait", self.b["Taken"], k)
            if n >= SLOTS:
                yield ("wait", self.b["UEmpty"][n % SLOTS], n // SLOTS - 1)
            u = self.units[self.next_unit] if self.next_unit < len(self.units) else None
            self.next_unit += 1
            self.slots[n % SLOTS] = u
            yield ("arrive", self.b["UFull"][n % SLOTS])
            if u is None:
                return
            n += 1

    def take(self, n):
        slot = n % SLOTS
        yield ("wait", self.b["UFull"][slot], n // SLOTS)
        u = self.slots[slot]
        yield ("arrive", self.b["UEmpty"][slot])
        return u

    def load(self, kind, idx, bar):
        buf = getattr(self, kind)
        self.need(buf[idx] == "free", f"{kind}[{idx}] loaded while in use ({buf[idx]})")
        buf[idx] = "loading"

        def done():
            buf[idx] = "ready"
            bar.arrive()
        self.async_tma.append(done)

    def producer(self):
        """Q and K loads, in the kernel's order. Paired: both Q tiles, then the
        key tiles. Otherwise a unit's first NK key tiles go to ring slots last
        filled by the previous unit, so they are issued before the unit's Q
        loads wait for the previous epilogues (mutation k_ahead: one more,
        whose slot frees only after this unit's own first product)."""
        kc, qloads, n = 0, [0, 0], 0
        early = NK + 1 if self.mut == "k_ahead" else NK
        while True:
            u = yield from self.take(n)
            if u is None:
                return

            def load_q(h):
                if qloads[h] > 0 and self.mut != "no_q_wait":
                    yield ("wait", self.b["QEmpty"][h], qloads[h] - 1)
                self.load("Q", h, self.b["QFull"][h])
                qloads[h] += 1

            def load_k():
                nonlocal kc
                ks = kc % NK
                if kc >= NK and self.mut != "no_kempty":
                    yield ("wait", self.b["KEmpty"][ks], kc // NK - 1)
                self.load("K", ks, self.b["KFull"][ks])
                kc += 1

            if self.paired:
                for h in (0, 1):
                    if u[h]:
                        yield from load_q(h)
                for r in range(max(u[0], u[1])):
                    for h in (0, 1):
                        if r < u[h]:
                            yield from load_k()
            else:
                q_issued = False
                for k in range(u[0]):
                    if not q_issued and k == early:
                        for h in (0, 1):
                            if self.tiles(u, h):
                                yield from load_q(h)
                        q_issued = True
                    yield from load_k()
                if not q_issued:
                    for h in (0, 1):
                        if self.tiles(u, h):
                            yield from load_q(h)
            if self.mut != "no_taken":
                yield ("arrive", self.b["Taken"])
            n += 1

    def vproducer(self):
        vc, n = 0, 0
        while True:
            u = yield from self.take(n)
            if u is None:
                return
            nk = max(u[0], u[1]) if self.paired else u[0]
            for r in range(nk):
                for h in ((0, 1) if self.paired else (0,)):
                    if self.paired and r >= u[h]:
                        continue
                    vs = vc % NV
                    if vc >= NV:
                        yield ("wait", self.b["VEmpty"][vs], vc // NV - 1)
                    self.load("V", vs, self.b["VFull"][vs])
                    vc += 1
            n += 1

    def qk_issuer(self):
        kc, qk, qwait, n = 0, 0, [0, 0], 0
        halves_of = lambda u: (0, 1) if (self.paired or u[1] > 0) else (0,)
        while True:
            u = yield from self.take(n)
            if u is None:
                return
            if not self.paired:
                for h in halves_of(u):
                    yield ("wait", self.b["QFull"][h], qwait[h])
                    qwait[h] += 1
            nk = max(u[0], u[1]) if self.paired else u[0]
            for r in range(nk):
                hs = [h for h in (0, 1) if r < u[h]] if self.paired else list(halves_of(u))
                if not self.paired:
                    ks = kc % NK
                    yield ("wait", self.b["KFull"][ks], kc // NK)
                for h in hs:
                    if self.paired:
                        if r == 0:
                            yield ("wait", self.b["QFull"][h], qwait[h])
                            qwait[h] += 1
                        ks = kc % NK
                        yield ("wait", self.b["KFull"][ks], kc // NK)
                    if qk > 0 and self.mut != "no_sfree":
                        yield ("wait", self.b["SFree"], qk - 1)
                    self.need(self.Q[h] == "ready", f"QK reads Q[{h}] in state {self.Q[h]}")
                    self.need(self.K[ks] == "ready", f"QK reads K[{ks}] in state {self.K[ks]}")
                    self.need(self.S == "free", f"QK overwrites S in state {self.S}")
                    self.S = "writing"
                    self.qk_inflight[h] += 1

                    def qk_done(h=h):
                        self.S = ("full", h)
                        self.qk_inflight[h] -= 1
                        self.b["SFull"][h].arrive()
                    self.fifo["qk"].append(qk_done)
                    qk += 1
                    if self.paired:
                        self.fifo["qk"].append(self._free_k(ks))
                        kc += 1
                if not self.paired:
                    self.fifo["qk"].append(self._free_k(ks))
                    kc += 1
            n += 1

    def _free_k(self, ks):
        def f():
            self.K[ks] = "free"
            self.b["KEmpty"][ks].arrive()
        return f

    def pv_issuer(self):
        vc, pf, oe, o_pend, n = 0, [0, 0], [0, 0], [False, False], 0
        halves_of = lambda u: (0, 1) if (self.paired or u[1] > 0) else (0,)
        while True:
            u = yield from self.take(n)
            if u is None:
                return
            nk = max(u[0], u[1]) if self.paired else u[0]
            for r in range(nk):
                hs = [h for h in (0, 1) if r < u[h]] if self.paired else list(halves_of(u))
                if not self.paired:
                    vs = vc % NV
                    yield ("wait", self.b["VFull"][vs], vc // NV)
                for h in hs:
                    if self.paired:
                        vs = vc % NV
                        yield ("wait", self.b["VFull"][vs], vc // NV)
                    yield ("wait", self.b["PFull"][h], pf[h])
                    pf[h] += 1
                    if r == 0 and o_pend[h] and self.mut != "no_o_free":
                        yield ("wait", self.b["OEmpty"][h], oe[h])
                        oe[h] += 1
                        o_pend[h] = False
                    self.need(self.V[vs] == "ready", f"PV reads V[{vs}] in state {self.V[vs]}")
                    self.need(self.P[h] == "full", f"PV reads P[{h}] in state {self.P[h]}")
                    if r == 0:
                        self.need(self.O[h] == "free", f"PV starts O[{h}] in state {self.O[h]}")
                        self.O[h] = "acc"
                    last = r == (u[h] if self.paired else u[0]) - 1

                    def pv_done(h=h, last=last):
                        self.P[h] = "free"
                        self.b["PFree"][h].arrive()
                        if last:
                            self.O[h] = "complete"
                            self.b["OFull"][h].arrive()
                    self.fifo["pv"].append(pv_done)
                    if last:
                        o_pend[h] = True
                    if self.paired:
                        self.fifo["pv"].append(self._free_v(vs))
                        vc += 1
                if not self.paired:
                    self.fifo["pv"].append(self._free_v(vs))
                    vc += 1
            n += 1

    def _free_v(self, vs):
        def f():
            self.V[vs] = "free"
            self.b["VEmpty"][vs].arrive()
        return f

    def softmax(self, h):
        sf, pw, of, n = 0, 0, 0, 0
        staged = 0                # epilogues of this half that staged and stored a tile
        while True:
            u = yield from self.take(n)
            n += 1
            if u is None:
                return
            nt = self.tiles(u, h)
            if nt == 0:
                continue
            for r in range(nt):
                yield ("wait", self.b["SFull"][h], sf)
                sf += 1
                self.need(self.S == ("full", h), f"softmax {h} reads S in state {self.S}")
                self.S = "free"
                yield ("arrive", self.b["SFree"])
                if pw > 0 and self.mut != "no_pfree":
                    yield ("wait", self.b["PFree"][h], pw - 1)
                self.need(self.P[h] == "free", f"softmax {h} overwrites P[{h}] in state {self.P[h]}")
                self.P[h] = "full"
                yield ("arrive", self.b["PFull"][h])
                pw += 1
            split = self.paired and len(u) > 2 and u[2]
            if split and h == 1:
                # second half of a split unit: O_1 complete, row maxima and sums
                # published, Q[1] handed back; O_1 is read by the first half
                yield ("wait", self.b["OFull"][1], of)
                of += 1
                self.need(self.O[1] == "complete", f"split half 1 ends with O in state {self.O[1]}")
                self.need(self.comb == "free", f"split half 1 overwrites the combine data ({self.comb})")
                self.comb = "written"
                yield ("arrive", self.b["Comb"])
                self.need(self.Q[1] == "ready" and self.qk_inflight[1] == 0,
                          f"split half 1 hands back Q[1] in state {self.Q[1]} with {self.qk_inflight[1]} QK in flight")
                self.Q[1] = "free"
                yield ("arrive", self.b["QEmpty"][1])
                continue
            # epilogue: O read, staged in Q[h], stored, Q[h] handed back
            yield ("wait", self.b["OFull"][h], of)
            of += 1
            self.need(self.O[h] == "complete", f"epilogue {h} reads O in state {self.O[h]}")
            if split and u[1] > 0:
                # combine: the second half's maxima and sums, then its O
                yield ("wait", self.b["Comb"], self.combs)
                self.combs += 1
                self.need(self.comb == "written", f"combine reads the second half's data in state {self.comb}")
                self.need(self.O[1] == "complete", f"combine reads O[1] in state {self.O[1]}")
                self.comb = "free"
                self.O[1] = "free"
                if self.mut != "no_comb_release":
                    yield ("arrive", self.b["OEmpty"][1])
            self.O[h] = "free"
            yield ("arrive", self.b["OEmpty"][h])
            self.need(self.Q[h] == "ready" and self.qk_inflight[h] == 0,
                      f"epilogue {h} stages into Q[{h}] in state {self.Q[h]} with {self.qk_inflight[h]} QK in flight")
            self.Q[h] = "staged"
            st = self.fifo[f"st{h}"]

            def read_done(h=h):
                self.Q[h] = "stored"
            st.append(read_done)
            if self.mut == "early_q_release":
                yield ("arrive", self.b["QEmpty"][h])   # before the stores have read the tile
            # all rows staged: the storing thread waits for this epilogue's phase
            yield ("arrive", self.b["OStaged"][h])
            yield ("wait", self.b["OStaged"][h], (of - 1) if self.mut == "staged_phase_from_of" else staged)
            staged += 1
            yield ("drain", f"st{h}")
            self.need(self.Q[h] == "stored", f"Q[{h}] handed back in state {self.Q[h]}")
            self.Q[h] = "free"
            if self.mut != "early_q_release":
                yield ("arrive", self.b["QEmpty"][h])

    # ---- scheduler
    def run(self, rng, max_steps=200000):
        agents = {"claimer": self.claimer(), "producer": self.producer(), "vproducer": self.vproducer(),
                  "qk": self.qk_issuer(), "pv": self.pv_issuer(), "sm0": self.softmax(0), "sm1": self.softmax(1)}
        pending = {name: None for name in agents}
        done = set()

        def advance(name):
            try:
                pending[name] = next(agents[name])
            except StopIteration:
                done.add(name)
                pending[name] = None

        for name in agents:
            advance(name)
        for _ in range(max_steps):
            choices = []
            for name, act in pending.items():
                if name in done:
                    continue
                kind = act[0]
                if kind == "arrive" or (kind == "wait" and act[1].ready(act[2])) or \
                        (kind == "drain" and not self.fifo[act[1]]):
                    choices.append(("agent", name))
            choices += [("tma", i) for i in range(len(self.async_tma))]
            choices += [("fifo", q) for q, items in self.fifo.items() if items]
            if not choices:
                if len(done) == len(agents):
                    return
                raise ProtocolError("deadlock: " + ", ".join(
                    f"{n} waits on {pending[n][1].name if pending[n][0] == 'wait' else pending[n][1]}"
                    for n in agents if n not in done))
            kind, what = rng.choice(choices)
            if kind == "agent":
                act = pending[what]
                if act[0] == "arrive":
                    act[1].arrive()
                advance(what)
            elif kind == "tma":
                self.async_tma.pop(what)()
            else:
                self.fifo[what].pop(0)()
        raise ProtocolError("no progress within the step limit")


def random_units(rng, paired, n, split_share=0.0):
    units = []
    for _ in range(n):
        if paired:
            a = rng.randint(1, 4)
            b = rng.choice([0] + [rng.randint(1, 4)] * 5)   # an empty second tile now and then
            if rng.random() < split_share:
                # split: the key list's tiles divided, the first half takes the larger part
                t = rng.randint(1, 8)
                a, b = (t + 1) // 2, t // 2
                units.append((a, b, 1))
                continue
            units.append((a, b))
        else:
            units.append((rng.randint(1, 5), rng.choice([0, 1, 1, 1])))  # (key tiles, has a second half)
    return units


@pytest.mark.parametrize("paired", [True, False])
def test_protocol_has_no_deadlock_or_hazard(paired):
    rng = random.Random(1234 + paired)
    for trial in range(150):
        Model(random_units(rng, paired, rng.randint(1, 14)), paired).run(rng)


@pytest.mark.parametrize("share", [0.5, 1.0])
def test_split_units_have_no_deadlock_or_hazard(share):
    rng = random.Random(4321 + int(share * 10))
    for trial in range(200):
        Model(random_units(rng, True, rng.randint(1, 14), share), True).run(rng)


def test_staged_phase_counts_only_stored_epilogues():
    # the second half of a split unit completes O_1 without staging a tile, so
    # the storing thread's wait must count staged epilogues, not O completions
    rng = random.Random(13)
    caught = False
    for trial in range(300):
        try:
            Model(random_units(rng, True, rng.randint(2, 12), 0.6), True, "staged_phase_from_of").run(rng)
        except ProtocolError:
            caught = True
            break
    assert caught


def test_split_units_need_the_combine_release():
    # the first half of a split unit must hand O_1 back once it has combined,
    # or the next product into O_1 waits forever
    rng = random.Random(11)
    caught = False
    for trial in range(300):
        try:
            Model(random_units(rng, True, rng.randint(2, 12), 0.7), True, "no_comb_release").run(rng)
        except ProtocolError:
            caught = True
            break
    assert caught


@pytest.mark.parametrize("mutation", ["no_q_wait", "no_sfree", "no_pfree", "early_q_release", "no_kempty",
                                      "claim_early", "no_taken"])
def test_planted_protocol_mistakes_are_caught(mutation):
    rng = random.Random(99)
    caught = False
    for trial in range(300):
        try:
            Model(random_units(rng, True, rng.randint(2, 12)), True, mutation).run(rng)
        except ProtocolError:
            caught = True
            break
    assert caught, mutation


def test_key_loads_ahead_of_q_are_bounded_by_the_ring():
    # One more early key tile than the ring holds waits for this unit's own
    # first product, which needs the Q load queued behind it: a deadlock.
    rng = random.Random(7)
    caught = False
    for trial in range(300):
        try:
            Model(random_units(rng, False, rng.randint(2, 12)), False, "k_ahead").run(rng)
        except ProtocolError:
            caught = True
            break
    assert caught


def test_o_free_wait_is_implied_by_p_order():
    # The PV issuer waits for the epilogue to have read O_h before the next
    # unit's first product into O_h. The model shows that wait never binds:
    # that product needs P_h of the next unit, which the same softmax
    # warpgroup writes only after its epilogue -- and with split units, where
    # the first half reads O_1, the PV issuer reaches O_1's next product only
    # after the first half's, whose P comes after the combine. The kernel
    # keeps the wait as a guard.
    rng = random.Random(7)
    for trial in range(200):
        paired = bool(trial & 1)
        share = 0.6 if (paired and trial % 4 == 1) else 0.0
        Model(random_units(rng, paired, rng.randint(1, 14), share), paired, "no_o_free").run(rng)


def test_unit_ring_consumer_count_matches_the_roles():
    # the unit slots are freed after this many arrivals; each role above
    # (a softmax warpgroup as 4 warps) arrives once per unit
    assert kernel_constant("kUnitConsumers") == RING_CONSUMER_WARPS
