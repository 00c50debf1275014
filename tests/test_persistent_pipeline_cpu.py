"""The barrier protocol of the persistent single-token kernel (csrc/gdn_decode_persistent.cu),
restated as a model and run under randomised schedules on the host.

A launch is ncl clusters of G CTAs (one per v-head of a k-head). In every CTA:
  * the loader takes unit v's group (fixed units cid + v ncl; later ones, under the dynamic
    schedule, from a counter shared by all clusters: the cluster's rank 0 takes the group of
    unit v + 1 once unit v's copies are out and relays it to every CTA of the cluster through
    a ring of kRing entries, by st.async completing on the receiver's ring barrier), waits
    for stage v % NSTAGE to be free, arms its full barrier (state tile and z) and conv barrier
    and issues the copies; after the last group it posts one end marker per consumer team;
  * the finishers (the first finisher warp and the others, which meet it at two named
    barriers per unit) wait for the conv inputs, send this CTA's raw q/k share of the unit to
    buffer v % QB of every CTA of the cluster (st.async, completing on that CTA's q/k
    barrier) and keep v; the first warp then arms its own q/k barrier, waits for every share,
    arrives on the full barrier and publishes the norms and gates (pub barrier);
  * the consumer teams take units in turn: the stage's previous unit released (empty
    barrier), full barrier, the tile and the q/k buffer, pub barrier, the update, then the
    empty barrier.
mbarriers are modelled with the hardware's arrival and transaction counts (a phase completes
when both reach zero; bytes may land before they are expected) and waits with its parity
rule. Copies and st.async deliveries land at random later times.

Checked for every schedule: no deadlock; every stage, q/k buffer and ring entry holds the
unit (or group) its reader expects when it is read, and nothing is written into it while a
reader still uses it; the CTAs of a cluster walk the same groups; every group of the launch
is processed by exactly one cluster and each of its units once; the dynamic counters end at
zero. The q/k buffers (QB = NSTAGE + 2) and the relay ring (kRing = 16 against at most
NSTAGE + 1 entries outstanding) are the two bounds the kernel's argument rests on; planted
mistakes, among them one q/k buffer fewer and a ring of NSTAGE entries, must be caught.

With two teams over three stages a stage's successive units belong to different teams; a
team that waited on the full barrier straight away could be two phases ahead of it (the
stage's previous unit not yet complete, its tile still landing) and pass at once. The
consumers therefore first wait for the stage's previous unit to be released; without that
wait ("no_stage_release_wait") the model finds such schedules."""
import collections
import random

import pytest

END = -1


class Deadlock(Exception):
    pass


class MBar:
    """An mbarrier: expected arrivals per phase, pending arrivals and transaction bytes."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phases = count, count, 0, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        assert self.pending > 0
        self.tx += expect_tx
        self.pending -= 1
        self._check()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._check()

    def passes(self, parity):
        return (self.phases & 1) != parity


class Launch:
    def __init__(self, ngroups, ncl, G, nstage, valid, dyn=True, nteams=2, fixed=2, ring=16, qb=None,
                 mistake=None):
        self.ngroups, self.ncl, self.G, self.NSTAGE, self.valid = ngroups, ncl, G, nstage, valid
        self.dyn, self.NTEAMS, self.F, self.kRing = dyn, nteams, fixed, ring
        self.QB = qb if qb is not None else nstage + 2
        self.mistake = mistake
        self.sched = [0, 0]  # the shared counter and the count of loaders done
        self.async_events = []
        self.ctas = [[CTA(self, c, r) for r in range(G)] for c in range(ncl)]

    def post(self, kind, fn):
        self.async_events.append((kind, fn))

    def agents(self):
        out = []
        for cl in self.ctas:
            for cta in cl:
                out += cta.agents()
        return out

    def run(self, rng, policy):
        agents = {id(a): a for a in self.agents()}
        conds = {}
        for k in list(agents):
            self._step(agents, conds, k)
        for _ in range(2_000_000):
            ready = [("agent", k) for k in agents if conds[k]()]
            pending = [("async", i) for i in range(len(self.async_events))]
            if not ready and not pending:
                if agents:
                    raise Deadlock(f"{len(agents)} agents blocked")
                return
            if policy == "agents_first" and ready:
                pool = ready
            elif policy == "async_first" and pending:
                pool = pending
            elif policy == "late_async":
                pool = ready or pending
            elif policy == "newest_async":  # later copies land before earlier ones
                pool = ready + pending[-1:]
            else:
                pool = ready + pending
            kind, which = rng.choice(pool)
            if kind == "agent":
                self._step(agents, conds, which)
            else:
                self.async_events.pop(which)[1]()
        raise AssertionError("the model did not finish")

    @staticmethod
    def _step(agents, conds, k):
        try:
            conds[k] = next(agents[k])
        except StopIteration:
            del agents[k]
            conds.pop(k, None)

    def check_end(self):
        done = collections.Counter()
        for cl in self.ctas:
            seqs = [cta.groups for cta in cl]
            assert all(s == seqs[0] for s in seqs), "the CTAs of a cluster walked different groups"
            for cta in cl:
                assert sorted(cta.consumed) == list(range(len(cta.groups))), "a unit not consumed exactly once"
            done.update(seqs[0])
        assert done == collections.Counter(range(self.ngroups)), "a group not processed exactly once"
        if self.dyn:
            assert self.sched == [0, 0], "the dynamic counters do not end at zero"


class CTA:
    def __init__(self, launch, c, r):
        L = launch
        self.L, self.c, self.r = L, c, r
        ns, qb = L.NSTAGE, L.QB
        self.full = [MBar(2) for _ in range(ns)]
        self.empty = [MBar(1) for _ in range(ns)]  # (a team's warps arrive together)
        self.cbar = [MBar(1) for _ in range(ns)]
        self.pub = [MBar(1) for _ in range(ns)]
        self.qkbar = [MBar(1) for _ in range(qb)]
        self.rbar = [MBar(1) for _ in range(L.kRing)]
        self.si = [None] * ns          # the stage's group (END: end marker)
        self.tile = [None] * ns        # the unit whose state tile has landed
        self.conv = [None] * ns        # the unit whose conv inputs have landed
        self.vsb = [None] * ns         # the unit whose v values the finishers wrote
        self.qk = [[None] * L.G for _ in range(qb)]  # per buffer, per sending rank: the unit
        self.qk_readers = [set() for _ in range(qb)]  # units whose consumers still read the buffer
        self.ring = [None] * L.kRing   # (entry, group)
        self.ring_read = [True] * L.kRing
        self.groups = []               # the group of each unit, as the loader took them
        self.consumed = []
        self.fin_gen = [0, 0]          # named-barrier generations of the two finisher agents

    def peers(self):
        return self.L.ctas[self.c]

    def agents(self):
        return [self.loader(), self.finisher_first(), self.finisher_rest()] + \
               [self.consumer(t) for t in range(self.L.NTEAMS)]

    # ---------------------------------------------------------------- loader
    def loader(self):
        L, ns = self.L, self.L.NSTAGE
        cid = self.c
        ring_size = L.NSTAGE if L.mistake == "small_ring" else L.kRing

        def relay(v, val):  # rank 0: the group of unit v >= F to every CTA of the cluster
            e = v - L.F
            for peer in self.peers():
                def deliver(peer=peer, e=e, val=val):
                    slot = e % ring_size
                    assert peer.ring_read[slot], "relay overwrote a ring entry not yet read"
                    peer.ring[slot] = (e, val)
                    peer.ring_read[slot] = False
                    peer.rbar[slot].complete_tx(4)
                L.post("relay", deliver)

        def receive(v):
            if not L.dyn or v < L.F:
                g = cid + v * L.ncl
            else:
                e = v - L.F
                slot = e % ring_size
                self.rbar[slot].arrive(expect_tx=4)
                par = (e // ring_size) & 1
                yield lambda: self.rbar[slot].passes(par)
                ent = self.ring[slot]
                assert ent is not None and ent[0] == e, "ring entry of another unit"
                self.ring_read[slot] = True
                g = ent[1]
            return g if g < L.ngroups else END

        g_next = yield from receive(0)
        v = 0
        while True:
            g = g_next
            if g == END:  # one end marker per consumer team
                for e in range(1 if L.mistake == "one_end_marker" else L.NTEAMS):
                    ve = v + e
                    s = ve % ns
                    if ve >= ns:
                        par = ((ve // ns) - 1) & 1
                        yield lambda s=s, par=par: self.empty[s].passes(par)
                    self.si[s] = END
                    self.cbar[s].arrive()
                    self.full[s].arrive()
                    self.full[s].arrive()
                break
            s = v % ns
            if v >= ns:
                par = ((v // ns) - 1) & 1 if L.mistake != "empty_parity" else (v // ns) & 1
                yield lambda s=s, par=par: self.empty[s].passes(par)
            self.groups.append(g)
            self.si[s] = g
            ok = L.valid[g]
            if ok:
                self.full[s].arrive(expect_tx=1)
                self.cbar[s].arrive(expect_tx=1)

                def land_conv(s=s, v=v):
                    self.conv[s] = v
                    self.cbar[s].complete_tx(1)

                def land_tile(s=s, v=v):
                    self.tile[s] = v
                    self.full[s].complete_tx(1)
                self.conv[s] = self.tile[s] = None  # (being overwritten)
                L.post("copy", land_conv)
                L.post("copy", land_tile)
            else:
                self.full[s].arrive()
                self.cbar[s].arrive()
            if L.dyn and v + 1 >= L.F and self.r == 0:
                val = L.F * L.ncl + L.sched[0]
                L.sched[0] += 1
                relay(v + 1, val)
            g_next = yield from receive(v + 1)
            v += 1
        if L.dyn:
            L.sched[1] += 1
            if L.sched[1] == L.ncl * L.G:
                L.sched[0] = L.sched[1] = 0

    # ---------------------------------------------------------------- finishers
    def fin_barrier(self, me):
        """One named-barrier meeting of the two finisher agents."""
        self.fin_gen[me] += 1
        k = self.fin_gen[me]
        other = 1 - me
        yield lambda: self.fin_gen[other] >= k

    def finisher_rest(self):
        """The finisher warps after the first: the conv, the sends, then the next unit."""
        ns, qb = self.L.NSTAGE, self.L.QB
        v = 0
        while True:
            s = v % ns
            par = (v // ns) & 1
            yield lambda s=s, par=par: self.cbar[s].passes(par)
            yield from self.fin_barrier(1)
            if self.si[s] == END:
                return
            yield from self.fin_barrier(1)  # every finisher's v values are written
            v += 1

    def finisher_first(self):
        L, ns, qb = self.L, self.L.NSTAGE, self.L.QB
        v = 0
        while True:
            s, q = v % ns, v % qb
            par = (v // ns) & 1
            yield lambda s=s, par=par: self.cbar[s].passes(par)
            yield from self.fin_barrier(0)
            g = self.si[s]
            if g == END:
                return
            assert v < len(self.groups), "finishers passed the conv barrier of a unit not yet issued"
            assert g == self.groups[v], "finishers took another unit's stage"
            valid = L.valid[g]
            if valid:
                assert self.conv[s] == v, "conv inputs of another unit"
                # the q/k share of this CTA to buffer q of every CTA of the cluster (the other
                # finisher warps send their part here too, before the barrier below)
                for peer in self.peers():
                    def deliver(peer=peer, q=q, v=v, r=self.r):
                        assert not peer.qk_readers[q], "q/k share written while consumers read the buffer"
                        assert peer.qk[q][r] is None or peer.qk[q][r] < v
                        peer.qk[q][r] = v
                        peer.qkbar[q].complete_tx(1)
                    L.post("share", deliver)
                self.vsb[s] = v
            yield from self.fin_barrier(0)
            if valid:
                self.qkbar[q].arrive(expect_tx=L.G)
            else:
                self.qkbar[q].arrive()
            if L.mistake != "no_qk_wait":
                par_q = (v // qb) & 1
                yield lambda q=q, par_q=par_q: self.qkbar[q].passes(par_q)
            self.full[s].arrive()
            if valid:
                assert all(u == v for u in self.qk[q]), "norms from a q/k buffer without every share"
            self.pub[s].arrive()
            v += 1

    # ---------------------------------------------------------------- consumers
    def consumer(self, team):
        L, ns, qb = self.L, self.L.NSTAGE, self.L.QB
        u = team
        while True:
            s, q = u % ns, u % qb
            par = (u // ns) & 1
            if u >= ns and L.mistake != "no_stage_release_wait":
                # the stage's previous unit, another team's when the teams do not divide the
                # stages, has been released: only then is the full barrier at most one phase
                # behind this unit (a parity wait two phases ahead would pass at once)
                par_e = ((u // ns) - 1) & 1
                yield lambda s=s, par_e=par_e: self.empty[s].passes(par_e)
            yield lambda s=s, par=par: self.full[s].passes(par)
            g = self.si[s]
            if g == END:
                return
            assert u < len(self.groups), "consumers passed the full barrier of a unit not yet issued"
            assert g == self.groups[u], "consumers took another unit's stage"
            if L.valid[g]:
                assert self.tile[s] == u, "state tile of another unit"
                assert all(x == u for x in self.qk[q]), "q/k buffer without every share of the unit"
                assert self.vsb[s] == u, "v of another unit"
                self.qk_readers[q].add(u)
                yield lambda: True  # the first pass over the tile (S^T k, S^T q)
                yield lambda s=s, par=par: self.pub[s].passes(par)
                assert self.tile[s] == u and all(x == u for x in self.qk[q]), "inputs changed under the update"
                yield lambda: True  # the update pass reads the tile and the k rows again
                assert self.tile[s] == u and all(x == u for x in self.qk[q]), "inputs changed under the update"
                self.qk_readers[q].discard(u)
            self.consumed.append(u)
            self.empty[s].arrive()
            u += L.NTEAMS


def launch(ngroups, ncl, G, nstage, bad=(), dyn=True, seed=0, policy="random", **kw):
    valid = [g not in bad for g in range(ngroups)]
    m = Launch(ngroups, ncl, G, nstage, valid, dyn=dyn, **kw)
    m.run(random.Random(seed), policy)
    m.check_end()
    return m


SCENARIOS = [
    # groups  clusters  G  stages  invalid groups  dynamic
    (1, 1, 1, 3, (), True),
    (7, 2, 2, 3, (), True),
    (12, 3, 2, 3, (4,), True),
    (20, 2, 4, 2, (0, 7, 8), True),
    (9, 4, 1, 3, (), True),      # more clusters than groups after the fixed units
    (9, 2, 2, 3, (3,), False),   # the static schedule
    (3, 3, 2, 3, (), True),      # as many clusters as groups
]
POLICIES = ["random", "agents_first", "async_first", "late_async", "newest_async"]


@pytest.mark.parametrize("scenario", SCENARIOS, ids=lambda s: f"g{s[0]}_cl{s[1]}_G{s[2]}_st{s[3]}_bad{len(s[4])}_{'dyn' if s[5] else 'static'}")
def test_persistent_protocol_under_random_schedules(scenario):
    ngroups, ncl, G, nstage, bad, dyn = scenario
    for policy in POLICIES:
        for seed in range(6 if policy == "random" else 2):
            launch(ngroups, ncl, G, nstage, bad, dyn, seed=seed, policy=policy)


@pytest.mark.parametrize("mistake,kw", [("qb_one_less", dict(qb_delta=-1)), ("small_ring", {}),
                                        ("empty_parity", {}), ("no_qk_wait", {}), ("one_end_marker", {}),
                                        ("no_stage_release_wait", {})])
def test_planted_protocol_mistakes_are_caught(mistake, kw):
    caught = 0
    for ngroups, ncl, G, nstage, bad, dyn in SCENARIOS:
        for policy in POLICIES:
            for seed in range(4):
                args = {}
                if "qb_delta" in kw:
                    args["qb"] = nstage + 2 + kw["qb_delta"]
                try:
                    launch(ngroups, ncl, G, nstage, bad, dyn, seed=seed, policy=policy,
                           mistake=None if "qb_delta" in kw else mistake, **args)
                except (AssertionError, Deadlock):
                    caught += 1
    assert caught > 0, mistake


def kernel_parameters():
    """(dk, dv) -> (NSTAGE, QB, NTEAMS) as the kernel's WS<DK, DV> computes them (restated; keep in
    step), and the namespace constants read from its source."""
    import pathlib
    import re
    src = (pathlib.Path(__file__).resolve().parents[1] / "gated_delta_rule_102_b200" / "csrc" /
           "gdn_decode_persistent.cu").read_text()
    const = {name: int(re.search(rf"constexpr int {name} = (\d+);", src).group(1))
             for name in ("kRing", "kFixedUnits", "kMaxConvWidthPersistent")}
    rup = lambda x, m: (x + m - 1) // m * m  # noqa: E731
    shapes = {}
    for dk in (16, 32, 64, 128):
        for dv in ((16,) if dk >= 32 else ()) + (32, 64, 128):
            team_warps = 4 if dv >= 128 else (2 if dv >= 64 else 1)
            maxnch = 2 * dk + dv
            cstage = rup(const["kMaxConvWidthPersistent"] * maxnch * 2, 16) + \
                rup(maxnch * const["kMaxConvWidthPersistent"] * 2, 16)
            per_stage = dk * dv * 4 + cstage + dv * 6 + 32 + 2 * dk * 4 + 24 + 32
            nstage = min(max((232448 - 3072 - 4 * dk * 4) // per_stage, 2), 8)
            shapes[(dk, dv)] = (nstage, nstage + 2, 8 // team_warps)
    return const, shapes


def test_protocol_at_every_instantiated_shape():
    const, shapes = kernel_parameters()
    assert const["kFixedUnits"] >= 1
    assert shapes[(128, 128)] == (3, 5, 2)  # the benchmark's shape: three stages, two teams
    for (dk, dv), (nstage, qb, nteams) in shapes.items():
        # the bounds the protocol rests on: at most NSTAGE + 1 relayed entries outstanding, and a
        # team's previous unit of a stage issued before its next one
        assert const["kRing"] >= nstage + 2, (dk, dv)
        assert nstage >= nteams, (dk, dv)
    for nstage, qb, nteams in sorted(set(shapes.values())):
        for ngroups, ncl, G in ((9, 2, 2), (14, 3, 1), (6, 1, 4)):
            for policy in POLICIES:
                for seed in range(2):
                    launch(ngroups, ncl, G, nstage, (ngroups // 2,), True, seed=seed, policy=policy,
                           nteams=nteams, fixed=const["kFixedUnits"], ring=const["kRing"], qb=qb)
