"""The barrier protocol of the chunked tensor-core multi-token kernel
(csrc/gdn_decode_chunk.cu), restated as a model and run under randomised schedules on the
host.

One CTA walks its (sequence, k-head) groups; a group's v-heads are its units. Four agents
share the CTA's buffers:
  * the producers (warps 4-11, one agent: their named barriers keep them together) fill
    the group operand tiles X and Z (double-buffered) and the unit buffers (v, the solve's
    coefficients, z; double-buffered), and emit each unit's gated RMSNorm from o; their raw
    rows arrive by cp.async in committed groups (a group's q|k rows, a head's v rows into
    the staging area that aliases the group scratch, a head's z rows into its unit buffer)
    that land at some later time, and at the latest when a wait_group asks for them;
  * the consumers (warps 0-3, one agent) take each unit's state tile from the copy ring
    into TMEM chunk by chunk, issue the first GEMM once the tile is in, solve, write o, issue
    the update, and store the new state while the next unit's tile goes in; thread 64 among
    them issues the bulk copy of the next unit's chunk q once chunk q has been read;
  * the bulk-copy engine lands a copy at some later time and completes its ring barrier;
  * the tensor core runs each issuing thread's MMAs and commits in order, at some later time.
An mbarrier wait with parity P passes when the barrier's completed-phase count has the
other parity, exactly as the hardware decides it, so a parity formula off by one phase
shows up as a premature pass (caught by the data checks) or a deadlock.

Checked for every schedule: no deadlock; no buffer (ring chunk, operand tile, unit buffer,
TMEM column block) rewritten before its reader is done with it, asynchronous readers
included; every read sees the data meant for it (ring chunks by the state tile they hold:
pool slot and v-head; staged rows by their group or head), no v rows landing in the scratch
while a group phase uses it; every unit's outputs emitted once and its state stored once; no
copy or MMA left in flight at the end; each group's and unit's rows staged once (the
look-ahead always right). Each planted protocol mistake must be caught by some schedule.

The abort paths too: at a random moment one blocked wait gives up, as a wait bounded by the
cycle counter would; every wait after it sees the abort flag, each role leaves by the
kernel's own path (the producers after their copies have landed; the consumers after the MMA
batches of either GEMM they issued and the state copies in flight have completed) and the
model checks that nothing is still in flight when the CTA frees its TMEM and leaves.
Dropping the consumers' wait for the first GEMM on that path must be caught."""
import collections
import random

import pytest

RING = CHUNKS = 4


class Deadlock(Exception):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.arrivals, self.phases = count, 0, 0

    def arrive(self):
        self.arrivals += 1
        if self.arrivals == self.count:
            self.arrivals = 0
            self.phases += 1

    def passes(self, parity):
        return (self.phases & 1) != parity


class CTA:
    def __init__(self, cta, grid, valid, slot, Hk, G, spec=False, mistake=None):
        self.cta, self.grid, self.ngroups = cta, grid, len(valid)
        self.valid, self.slot, self.Hk, self.G, self.spec, self.mistake = valid, slot, Hk, G, spec, mistake
        self.bars = {f"ring_full{s}": Bar(1) for s in range(RING)}
        for b in range(2):
            for name in ("grp_full", "grp_empty", "unit_full", "unit_empty"):
                self.bars[f"{name}{b}"] = Bar(1)
        self.bars["mma"] = Bar(1)
        self.bars["g1"] = Bar(2)  # committed by the two threads that issue the first GEMM
        self.fifo = {0: collections.deque(), 32: collections.deque()}
        self.tma = []
        self.ring = [dict(tile=None, read=True, inflight=False) for _ in range(RING)]
        self.xz = [dict(tag=None, x_out=0, x_done=0, z_out=0, z_done=0) for _ in range(2)]
        self.unit = [dict(v=None, o=None, z=None) for _ in range(2)]
        self.a_tag, self.a_out = [None] * CHUNKS, [0] * CHUNKS  # S0 high/low parts in TMEM
        self.d2 = [None] * CHUNKS  # (kind, unit), kind "init" (gamma S0) or "upd" (new state)
        self.d2_stored = [True] * CHUNKS
        self.d1_done, self.d1_read = collections.Counter(), -1
        self.y_tag, self.y_out = None, 0
        self.p_keys, self.c_keys = [], []
        self.emitted, self.stored = collections.Counter(), collections.Counter()
        self.group_stagings, self.unit_stagings = collections.Counter(), collections.Counter()
        self.abort = False   # the CTA's abort flag (a wait gave up)
        self.graw = None
        self.uraw = None   # the head whose v rows are in the staging area
        self.cp = []       # committed cp.async groups in commit order: [kind, landing action, landed]

    def tile(self, g, j):
        return (self.slot[g], (g % self.Hk) * self.G + j)

    # ---- producer-side data actions
    def copy(self, kind, action):
        self.cp.append([kind, action, False])

    def cp_in_flight(self):
        return [c for c in self.cp if not c[2]]

    def land_group(self, c):
        c[1]()
        c[2] = True

    def cp_wait(self, keep):
        """cp.async.wait_group keep: every committed group but the `keep` most recently
        committed ones (landed or not) has landed."""
        for c in self.cp[:len(self.cp) - keep]:
            if not c[2]:
                self.land_group(c)

    def stage_group(self, g):
        self.group_stagings[g] += 1
        self.copy("group", lambda: setattr(self, "graw", g))

    def conv_group(self, g):
        assert self.graw == g, "conv of a group whose rows are not staged"
        assert not any(c[0] == "v" for c in self.cp_in_flight()), "v rows landing in the scratch during the group phase"

    def stage_v(self, h):
        self.uraw = None
        self.copy("v", lambda: setattr(self, "uraw", h))

    def conv_v(self, h):
        assert self.uraw == h, "v conv of a head whose rows have not landed"

    def write_group(self, gb, li):
        b = self.xz[gb]
        assert b["x_out"] == 0 and b["z_out"] == 0, "operand tile rewritten under a running MMA"
        if b["tag"] is not None:
            assert b["x_done"] == 2 * CHUNKS * self.G, "operand tile rewritten before every first-GEMM MMA read it"
            assert b["z_done"] == (0 if self.spec else self.G), "key tile rewritten before every update read it"
        b.update(tag=li, x_done=0, z_done=0)

    def stage_z(self, b, u):
        self.unit_stagings[u] += 1
        prev = self.unit[b]["z"]
        assert prev is None or self.emitted[self.p_keys[prev]], "z rows overwritten before their unit was emitted"
        self.unit[b]["z"] = None  # (in flight)
        self.copy("z", lambda: self.unit[b].__setitem__("z", u))

    def write_unit(self, b, u):
        prev = self.unit[b]["v"]
        assert prev is None or self.emitted[self.p_keys[prev]], "unit buffer overwritten before its unit was emitted"
        self.unit[b].update(v=u, o=None)

    def emit(self, b, u):
        assert self.unit[b]["o"] == u and self.unit[b]["z"] == u, "emitted a unit whose o or z is not there"
        self.emitted[self.p_keys[u]] += 1

    # ---- consumer-side data actions
    def read_unit(self, b, u):
        assert self.unit[b]["v"] == u and self.unit[b]["o"] is None, "consumers read a unit the producers did not write"

    def write_o(self, b, u):
        assert self.unit[b]["v"] == u
        self.unit[b]["o"] = u

    def tma_issue(self, q, tile):
        r = self.ring[q]
        assert r["read"] and not r["inflight"], "state chunk copied over a ring buffer still in use"
        r.update(inflight=True, read=False)
        self.tma.append((q, tile))

    def take_chunk(self, s, q, tile, u):
        assert s == q, "a unit's chunk q not in ring buffer q"
        r = self.ring[s]
        assert not r["inflight"] and not r["read"] and r["tile"] == tile, f"ring holds {r['tile']}, expected {tile}"
        r["read"] = True
        assert self.a_out[q] == 0, "S0 parts in TMEM rewritten under a running first GEMM"
        self.a_tag[q] = u
        if not self.spec:
            assert self.d2_stored[q], "accumulator chunk overwritten before its state was stored"
            self.d2[q], self.d2_stored[q] = ("init", u), False

    def store_chunk(self, q, u):
        assert self.d2[q] == ("upd", u) and not self.d2_stored[q], f"stored {self.d2[q]} as unit {u}'s state"
        self.d2_stored[q] = True
        self.stored[self.c_keys[u]] += 1

    def gemm1(self, q, u, gb, li):
        for t in (0, 32):
            assert self.xz[gb]["tag"] == li and self.a_tag[q] == u
            if q == 0:
                assert self.d1_read == u - 1, "first GEMM overwrites partial sums not yet read"
            self.xz[gb]["x_out"] += 1
            self.a_out[q] += 1
            self.fifo[t].append(("gemm1", q, u, gb, li))
            if q == CHUNKS - 1:
                self.fifo[t].append(("commit", "g1"))

    def read_d1(self, u):
        assert self.d1_done[u] == 2 * CHUNKS, "partial sums read before the first GEMM completed"
        self.d1_read = u

    def write_y(self, u):
        assert self.y_out == 0, "update operand rewritten under a running update"
        self.y_tag = u

    def gemm2(self, u, gb, li):
        assert self.xz[gb]["tag"] == li and self.y_tag == u and all(d == ("init", u) for d in self.d2)
        self.xz[gb]["z_out"] += 1
        self.y_out += 1
        self.fifo[0].append(("gemm2", u, gb, li))
        self.fifo[0].append(("commit", "mma"))

    # ---- asynchronous completions
    def complete(self, op):
        if op[0] == "commit":
            self.bars[op[1]].arrive()
        elif op[0] == "gemm1":
            _, q, u, gb, li = op
            assert self.xz[gb]["tag"] == li and self.a_tag[q] == u, "first GEMM operands changed while it ran"
            self.xz[gb]["x_out"] -= 1
            self.xz[gb]["x_done"] += 1
            self.a_out[q] -= 1
            self.d1_done[u] += 1
        else:
            _, u, gb, li = op
            assert self.xz[gb]["tag"] == li and self.y_tag == u and all(d == ("init", u) for d in self.d2), \
                "update operands changed while it ran"
            self.xz[gb]["z_out"] -= 1
            self.xz[gb]["z_done"] += 1
            self.y_out -= 1
            self.d2 = [("upd", u)] * CHUNKS

    def land_copy(self, k):
        self.land_group(self.cp_in_flight()[k])

    def land(self, k):
        q, tile = self.tma.pop(k)
        self.ring[q].update(tile=tile, inflight=False, read=False)
        self.bars[f"ring_full{q}"].arrive()

    # ---- the two roles, in the kernel's order. A wait yields ("w", barrier, parity) and gets
    # back whether it passed (False once the abort flag is set, or when it times out); a
    # bounded wait of an abort path yields ("b", barrier, parity) and waits for the phase.
    def producer(self):
        Hk, G, grid, ng = self.Hk, self.G, self.grid, self.ngroups
        li = hu = 0
        emitted = gstaged = -1
        stop = False
        for g in range(self.cta, ng, grid):
            gn = g + grid
            if not self.valid[g]:
                continue
            gb, hk = li & 1, g % Hk
            ok = True
            if li >= 2:
                ok = yield ("w", f"grp_empty{gb}", ((li >> 1) - 1) & 1)
            if not (ok and not self.abort):  # the producers agree, and leave together
                self.abort |= not ok
                break
            if gstaged != g:
                self.stage_group(g)
                gstaged = g
            self.cp_wait(0)
            self.conv_group(g)
            g2 = gn  # the next group this CTA runs: its rows into the staging buffer just read
            if g2 < ng and not self.valid[g2]:
                g2 += grid
                while g2 < ng and not self.valid[g2]:
                    g2 += grid
            if g2 < ng:
                self.stage_group(g2)
                gstaged = g2
            self.write_group(gb, li)
            self.bars[f"grp_full{gb}"].arrive()
            li += 1
            for j in range(G):
                hb, h = hu & 1, hk * G + j
                self.p_keys.append((g, h))
                ok = True
                if hu >= 2 and self.mistake != "no_unit_empty_wait":
                    par = (hu >> 1) & 1 if self.mistake == "unit_empty_parity" else ((hu >> 1) - 1) & 1
                    ok = yield ("w", f"unit_empty{hb}", par)
                if not (ok and not self.abort):
                    self.abort |= not ok
                    stop = True
                    break
                if j == 0:
                    self.stage_v(h)
                if hu >= 2 and emitted < hu - 2:
                    self.emit(hb, hu - 2)
                    emitted = hu - 2
                if j == 0:
                    self.stage_z(hb, hu)
                self.cp_wait(2 if self.mistake == "wait_keeps_two" else 1)
                self.conv_v(h)
                self.write_unit(hb, hu)
                if j + 1 < G:  # the staging area is free: the next head's v rows
                    self.stage_v(h + 1)
                self.bars[f"unit_full{hb}"].arrive()
                if j + 1 < G:  # the next head's buffer: its previous unit leaves, its z rows start
                    nb = (hu + 1) & 1
                    ok2 = True
                    if hu >= 1:
                        ok2 = yield ("w", f"unit_empty{nb}", ((hu - 1) >> 1) & 1)
                    if not (ok2 and not self.abort):
                        self.abort |= not ok2
                        stop = True
                        break
                    if hu >= 1 and emitted < hu - 1:
                        self.emit(nb, hu - 1)
                        emitted = hu - 1
                    self.stage_z(nb, hu + 1)
                hu += 1
            if stop:
                break
        if self.mistake != "drain_without_wait":
            self.cp_wait(0)
        if not self.abort:
            for u in range(emitted + 1, hu):  # the last units' outputs
                got = yield ("w", f"unit_empty{u & 1}", (u >> 1) & 1)
                if not (got and not self.abort):
                    self.abort |= not got
                    break
                self.emit(u & 1, u)
        self.cp_wait(0)  # no copy of this thread lands after the CTA has left

    def consumer(self):
        Hk, G, grid, ng = self.Hk, self.G, self.grid, self.ngroups
        li = hu = chunk = issued = g1_seen = mma_seen = mma_issued = g1_commits = 0
        pend = None
        ok = True

        def next_group(frm):
            gg = frm
            while gg < ng and not self.valid[gg]:
                gg += grid
            return gg

        g0 = next_group(self.cta)
        if g0 < ng:
            for q in range(CHUNKS):
                self.tma_issue(q, self.tile(g0, 0))
                issued += 1
        for g in range(self.cta, ng, grid):
            gn = g + grid
            if not self.valid[g]:
                continue
            gb, hk = li & 1, g % Hk
            got = yield ("w", f"grp_full{gb}", (li >> 1) & 1)
            if not (got and not self.abort):
                ok = False
                break
            for j in range(G):
                hb, h = hu & 1, hk * G + j
                self.c_keys.append((g, h))
                if j + 1 >= G:  # the copier's next tile: the next group's first head
                    g2 = gn
                    if g2 < ng and not self.valid[g2] and self.mistake != "copier_no_skip":
                        g2 = next_group(gn + grid)
                    nt = self.tile(g2, 0) if g2 < ng else None
                else:
                    nt = self.tile(g, j + 1)
                w = yield ("w", f"unit_full{hb}", (hu >> 1) & 1)
                if w:
                    self.read_unit(hb, hu)
                for q in range(CHUNKS):
                    s = chunk % RING
                    if w:
                        w = yield ("w", f"ring_full{s}", (chunk // RING) & 1)
                    if self.mistake == "copy_before_read" and nt is not None:
                        self.tma_issue(q, nt)
                        issued += 1
                    if pend is not None:
                        self.store_chunk(q, pend)
                    if w:
                        self.take_chunk(s, q, self.tile(g, j), hu)
                    if not (w and not self.abort):  # the chunk's barrier
                        ok = False
                        break
                    chunk += 1
                    if nt is not None and self.mistake != "copy_before_read":  # after the chunk's barrier
                        self.tma_issue(q, nt)
                        issued += 1
                if not ok:
                    break
                for q in range(CHUNKS):  # the first GEMM once the whole tile is in (threads 0 and 32)
                    self.gemm1(q, hu, gb, li)
                g1_commits += 1
                pend = None
                w = yield ("w", "g1", g1_seen & 1)
                if w:
                    g1_seen += 1
                    self.read_d1(hu)
                    self.write_o(hb, hu)
                    if not self.spec:
                        self.write_y(hu)
                if not (w and not self.abort):
                    ok = False
                    break
                if not self.spec:
                    self.gemm2(hu, gb, li)
                    mma_issued += 1
                self.bars[f"unit_empty{hb}"].arrive()
                if not self.spec:
                    if self.mistake != "no_mma_wait":
                        w = yield ("w", "mma", mma_seen & 1)
                        if w:
                            mma_seen += 1
                    pend = hu
                if not (w and not self.abort):
                    ok = False
                    break
                hu += 1
            if not ok:
                break
            self.bars[f"grp_empty{gb}"].arrive()
            li += 1
        if ok and pend is not None:
            for q in range(CHUNKS):
                self.store_chunk(q, pend)
        if not ok:  # what was issued completes before TMEM is freed and the CTA leaves
            self.abort = True
            if g1_commits > g1_seen and self.mistake != "no_first_gemm_drain":
                yield ("b", "g1", g1_seen & 1)
            if mma_issued > mma_seen:
                yield ("b", "mma", mma_seen & 1)
            for v in range(chunk, issued):
                yield ("b", f"ring_full{v % RING}", (v // RING) & 1)
        self.issued, self.chunks = issued, chunk

    # ---- the scheduler
    def run(self, rng, policy, timeout_rate=0.0):
        """timeout_rate: the chance per step that one blocked wait gives up (once per run)."""
        agents = {"P": self.producer(), "C": self.consumer()}
        waits, resume = {}, {}
        for name in list(agents):
            self._step(agents, waits, resume, name)
        timed_out = False
        for _ in range(1_000_000):
            def can_go(n):
                kind, bar, par = waits[n]
                return self.bars[bar].passes(par) or (kind == "w" and self.abort)
            ready = [("agent", n) for n in agents if can_go(n)]
            pending = ([("fifo", t) for t in (0, 32) if self.fifo[t]] + [("tma", k) for k in range(len(self.tma))] +
                       [("cp", k) for k in range(len(self.cp_in_flight()))])
            blocked = [n for n in agents if waits[n][0] == "w" and not can_go(n)]
            if timeout_rate and not timed_out and blocked and rng.random() < timeout_rate:
                n = rng.choice(blocked)  # this wait gives up: its agent sees False and sets the abort flag
                timed_out = True
                resume[n] = False
                self._step(agents, waits, resume, n)
                continue
            if not agents:  # every role has left: the CTA frees its TMEM and leaves now
                break
            if not ready and not pending:
                raise Deadlock({n: waits[n] for n in agents})
            if policy == "late_copies":  # copies land only when a wait needs them or nothing else runs
                pool = ready + [e for e in pending if e[0] != "cp"] or pending
            elif policy == "agents_first" and ready:
                pool = ready
            elif policy == "async_first" and pending:
                pool = pending
            else:
                pool = ready + pending
            kind, which = rng.choice(pool)
            if kind == "agent":
                bar_kind, bar, par = waits[which]
                resume[which] = self.bars[bar].passes(par)
                self._step(agents, waits, resume, which)
            elif kind == "fifo":
                self.complete(self.fifo[which].popleft())
            elif kind == "cp":
                self.land_copy(which)
            else:
                self.land(which)
        else:
            raise AssertionError("the model did not finish")

    @staticmethod
    def _step(agents, waits, resume, name):
        try:
            waits[name] = agents[name].send(resume.pop(name, None))
        except StopIteration:
            del agents[name]
            waits.pop(name, None)

    def check_end(self):
        assert not self.tma and not self.fifo[0] and not self.fifo[32] and not self.cp_in_flight(), \
            "work in flight when the CTA frees its TMEM and leaves"
        if self.abort:
            return
        assert self.p_keys == self.c_keys, "producers and consumers ran different units"
        assert self.issued == self.chunks, "state chunks copied that no unit took"
        for key in self.p_keys:
            assert self.emitted[key] == 1, key
            assert self.stored[key] == (0 if self.spec else CHUNKS), key
        assert all(c == 1 for c in self.group_stagings.values())
        assert sorted(self.unit_stagings) == list(range(len(self.p_keys)))
        assert all(c == 1 for c in self.unit_stagings.values())


def launch_with_timeout(B, Hk, G, grid, bad_seqs=(), spec=False, mistake=None, seed=0, policy="random",
                        rate=0.05):
    """All CTAs of one launch, one wait of each giving up at a random moment; returns how many
    CTAs took their abort paths."""
    ngroups = B * Hk
    valid = [g // Hk not in bad_seqs for g in range(ngroups)]
    slot = [(7 * (g // Hk) + 3) % 1000 for g in range(ngroups)]
    aborted = 0
    for cta in range(min(grid, ngroups)):
        m = CTA(cta, grid, valid, slot, Hk, G, spec, mistake)
        m.run(random.Random(1000 * seed + cta), policy, timeout_rate=rate)
        m.check_end()
        aborted += m.abort
    return aborted


def launch(B, Hk, G, grid, bad_seqs=(), spec=False, mistake=None, seed=0, policy="random"):
    """All CTAs of one launch, each run to its end under its own random schedule; returns the
    units covered. A sequence in bad_seqs has a bad slot or no tokens: every role skips it."""
    ngroups = B * Hk
    valid = [g // Hk not in bad_seqs for g in range(ngroups)]
    slot = [(7 * (g // Hk) + 3) % 1000 for g in range(ngroups)]
    units = collections.Counter()
    for cta in range(min(grid, ngroups)):
        m = CTA(cta, grid, valid, slot, Hk, G, spec, mistake)
        m.run(random.Random(1000 * seed + cta), policy)
        m.check_end()
        units.update(m.p_keys)
    want = collections.Counter((g, (g % Hk) * G + j) for g in range(ngroups) if valid[g] for j in range(G))
    assert units == want
    return units


SCENARIOS = [
    # B   Hk  G  grid  bad sequences
    (1, 1, 1, 1, ()),
    (6, 1, 1, 2, ()),             # three one-unit groups per CTA
    (3, 2, 4, 2, ()),
    (4, 2, 8, 3, (1,)),
    (9, 1, 2, 2, (0, 2, 3, 4)),   # invalid first group and a run of invalid groups
    (5, 3, 3, 4, (4,)),           # invalid last groups
    (7, 2, 1, 3, (1, 2, 6)),
    (2, 1, 3, 4, ()),             # more CTAs than groups
]
POLICIES = ["random", "agents_first", "async_first", "late_copies"]


@pytest.mark.parametrize("spec", [False, True], ids=["decode", "verify"])
@pytest.mark.parametrize("scenario", SCENARIOS, ids=lambda s: f"B{s[0]}_Hk{s[1]}_G{s[2]}_grid{s[3]}_bad{len(s[4])}")
def test_pipeline_protocol_under_random_schedules(scenario, spec):
    B, Hk, G, grid, bad = scenario
    for policy in POLICIES:
        for seed in range(8 if policy == "random" else 3):
            launch(B, Hk, G, grid, bad, spec=spec, seed=seed, policy=policy)


@pytest.mark.parametrize("mistake", ["no_unit_empty_wait", "unit_empty_parity", "copier_no_skip",
                                     "copy_before_read", "no_mma_wait", "wait_keeps_two", "drain_without_wait"])
def test_planted_protocol_mistakes_are_caught(mistake):
    caught = 0
    for scenario in SCENARIOS:
        B, Hk, G, grid, bad = scenario
        for policy in POLICIES:
            for seed in range(4):
                try:
                    launch(B, Hk, G, grid, bad, mistake=mistake, seed=seed, policy=policy)
                except (AssertionError, Deadlock):
                    caught += 1
    assert caught > 0, mistake


@pytest.mark.parametrize("spec", [False, True], ids=["decode", "verify"])
def test_abort_paths_leave_nothing_in_flight(spec):
    aborted = 0
    for B, Hk, G, grid, bad in SCENARIOS:
        for policy in POLICIES:
            for seed in range(6):
                for rate in (0.02, 0.2):
                    aborted += launch_with_timeout(B, Hk, G, grid, bad, spec=spec, seed=seed, policy=policy, rate=rate)
    assert aborted > 100  # the abort paths were taken, from many points


def test_abort_without_the_first_gemm_drain_is_caught():
    caught = 0
    for B, Hk, G, grid, bad in SCENARIOS:
        for policy in POLICIES:
            for seed in range(6):
                try:
                    launch_with_timeout(B, Hk, G, grid, bad, mistake="no_first_gemm_drain", seed=seed, policy=policy,
                                        rate=0.2)
                except (AssertionError, Deadlock):
                    caught += 1
    assert caught > 0
