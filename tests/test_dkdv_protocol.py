"""A model of the dK/dV kernel's synchronisation, run under random interleavings.

``dkdv_union_kernel`` (``csrc/qsa_dkdv_union.cu``) is a persistent kernel: per
CTA a scheduler warp, gather warps (a fixed set per stage of a three-stage
ring: four each as built, each taking a quarter of a chunk's unions, or one),
one MMA thread and four epilogue warps hand chunks and accumulators to one
another through mbarriers, and across CTAs each (tile, group, tensor) passes
its FP32 partial from query phase to query phase through a counter in global
memory.  This test restates that protocol as coroutines (one per warp role and
CTA; the tensor core an in-order queue whose commits arrive when every earlier
MMA has completed) and runs it under many random schedules.  It checks what
the kernel's correctness rests on and what the GPU tests cannot force:

* no deadlock, for any schedule of co-resident CTAs;
* every mbarrier parity wait passes exactly at the phase it is meant for (the
  hardware passes a wait issued two phases early at once);
* no shared-memory stage (or a worker's share of one), ring slot or accumulator is
  overwritten before its reader is done;
* every (tile, group, tensor) adds its partials in phase order, each phase
  exactly once, and the last phase writes the result.

And on the abort path (every wait in the kernel is bounded: on expiry it sets
the CTA's abort flag, and every other wait gives up once it sees the flag):

* after any one wait expires, at any point, every role of every CTA still
  leaves its loop (no role is left in an unbounded named barrier), and the
  tensor memory is released only after the tensor-core queue has drained.

It models the protocol, not the kernel's code: a change to the kernel's
barriers needs the same change here.
"""

import random

import pytest

STAGES, RING, ACC_BUFS, UNIONS, PER_STAGE = 3, 16, 2, 8, 4


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phases = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phases += 1
            self.pending = self.count

    def ready(self, parity):
        # the hardware rule: a parity wait passes while the barrier's current
        # phase has the other parity
        return (self.phases & 1) != parity


class Wait:
    """A blocking point: `ready()` says whether it may pass, `check()` runs
    when it does.  `bounded` waits give up (the role receives False) once the
    CTA's abort flag is set, or when they expire."""

    def __init__(self, ready, check=lambda: None, bounded=True):
        self.ready, self.check, self.bounded = ready, check, bounded


def make_units(rng, n_tiles, P, G):
    """Per-phase work lists -> units in claim order (phase-major, dK before dV)."""
    lists = []
    ords = {}
    for p in range(P):
        items = []
        for tile in range(n_tiles):
            if rng.random() < 0.55:
                items.append([tile, rng.randint(1, 11)])
        lists.append(items)
    last_phase = {}
    for p, items in enumerate(lists):
        for tile, _ in items:
            last_phase[tile] = p
    units = []
    for p, items in enumerate(lists):
        for tensor in range(2):
            for tile, n_ent in items:
                for g in range(G):
                    key = (tile, g, tensor)
                    ords.setdefault(key, 0)
                    units.append(dict(tile=tile, g=g, tensor=tensor, phase=p, ord=ords[key],
                                      last=last_phase[tile] == p, n_ent=n_ent))
        for tile, _ in items:
            for tensor in range(2):
                for g in range(G):
                    ords[(tile, g, tensor)] += 1
    return units


class Model:
    """With `n_workers` = PER_STAGE x STAGES the warps of stage k % STAGES fill
    chunk k together (the kernel); otherwise `n_workers` warps take the chunks
    in turn, chunk k to warp k % n_workers;
    `collective_exit=False` restates an earlier epilogue in which each warp left
    on its own accumulator wait."""

    def __init__(self, units, n_ctas, seed, n_workers=STAGES * PER_STAGE, collective_exit=True, expire_at=None,
                 expire_roles=""):
        self.rng = random.Random(seed)
        self.n_workers = n_workers
        self.collective_exit = collective_exit
        # expire the expire_at-th bounded wait of the roles whose names start
        # with expire_roles (None: never)
        self.expire_at, self.expire_roles = expire_at, expire_roles
        self.n_bounded = 0
        self.units = units
        self.claim = 0
        self.done = {}            # (tile, g, tensor) -> published phases (the kernel's counter)
        self.partial = {}         # (tile, g, tensor) -> ords summed so far
        self.result = {}
        self.stored = {}          # (CTA, unit sequence number) -> epilogue warps done storing
        self.ctas = [self.cta_state() for _ in range(n_ctas)]
        self.roles = {}
        for i, c in enumerate(self.ctas):
            self.roles[(i, "sched")] = self.scheduler(c)
            for w in range(n_workers):
                self.roles[(i, f"w{w}")] = self.worker(c, w)
            self.roles[(i, "mma")] = self.mma(c)
            for e in range(4):
                self.roles[(i, f"epi{e}")] = self.epilogue(c, e)
        self.n_roles = {i: sum(1 for n in self.roles if n[0] == i) for i in range(n_ctas)}

    def cta_state(self):
        per_stage = PER_STAGE if self.n_workers == STAGES * PER_STAGE else 1
        return dict(full=[Bar(per_stage) for _ in range(STAGES)], empty=[Bar(1) for _ in range(STAGES)],
                    ring_full=[Bar(1) for _ in range(RING)], ring_empty=[Bar(per_stage) for _ in range(RING)],
                    acc_full=[Bar(2) for _ in range(ACC_BUFS)], acc_empty=[Bar(4) for _ in range(ACC_BUFS)],
                    drain=Bar(1), ring=[None] * RING, stage=[None] * STAGES,
                    half=[[None] * PER_STAGE for _ in range(STAGES)], acc=[None] * ACC_BUFS,
                    acc_desc=[None] * ACC_BUFS, acc_read={}, tc=[], abort=False, named={}, exited=0,
                    freed=False, per_stage=per_stage)

    def wait(self, bar, phase):
        def check():
            assert bar.phases == phase + 1, f"wait for phase {phase} passed with {bar.phases} completed"
        return Wait(lambda: bar.ready(phase & 1), check)

    def named_barrier(self, c, gen, flag):
        """The epilogue's `bar_or` over its four warps (not bounded)."""
        slot = c["named"].setdefault(gen, [0, False])
        slot[0] += 1
        slot[1] = slot[1] or flag
        return Wait(lambda: slot[0] == 4, bounded=False), slot

    # ------------------------------------------------------------------ roles
    def scheduler(self, c):
        k = 0
        ok = True
        while ok:
            U = self.claim
            self.claim += 1
            yield None                                   # claims interleave across CTAs
            if U >= len(self.units):
                break
            u = self.units[U]
            for p in range(0, u["n_ent"], UNIONS):
                n = min(UNIONS, u["n_ent"] - p)
                rs = k % RING
                if k >= RING and not (yield self.wait(c["ring_empty"][rs], k // RING - 1)):
                    ok = False
                    break
                c["ring"][rs] = dict(k=k, U=U, first=p == 0, last=p + n >= u["n_ent"])
                c["ring_full"][rs].arrive()
                k += 1
        markers = STAGES if c["per_stage"] == PER_STAGE else self.n_workers
        for j in range(markers if ok else 0):            # end markers; only the first reaches the MMA
            rs = k % RING
            if k >= RING and not (yield self.wait(c["ring_empty"][rs], k // RING - 1)):
                break
            c["ring"][rs] = dict(k=k, end=True, mma_end=j == 0)
            c["ring_full"][rs].arrive()
            k += 1

    def worker(self, c, w):
        pairs = c["per_stage"] == PER_STAGE
        step = STAGES if pairs else self.n_workers
        k = w % STAGES if pairs else w
        h = w // STAGES if pairs else 0
        while True:
            rs = k % RING
            if not (yield self.wait(c["ring_full"][rs], k // RING)):
                return
            d = c["ring"][rs]
            assert d["k"] == k, f"ring slot {rs} holds chunk {d['k']}, worker wants {k}"
            c["ring_empty"][rs].arrive()
            if d.get("end") and not d["mma_end"]:
                return
            s = k % STAGES
            if k >= STAGES and not (yield self.wait(c["empty"][s], k // STAGES - 1)):
                return
            if d.get("end"):
                if h == 0:
                    c["stage"][s] = dict(k=k, end=True)
                c["full"][s].arrive()
                return
            c["half"][s][h] = ("filling", k)
            yield None
            c["half"][s][h] = k
            if h == 0:
                c["stage"][s] = dict(d)
            c["full"][s].arrive()
            k += step

    def mma(self, c):
        useq = 0
        k = 0
        ok = True
        while True:
            s = k % STAGES
            if not (yield self.wait(c["full"][s], k // STAGES)):
                ok = False
                break
            d = c["stage"][s]
            assert d is not None and d["k"] == k, f"stage {s} descriptor {d}, MMA wants chunk {k}"
            if d.get("end"):
                break
            buf = useq % ACC_BUFS
            if d["first"] and useq >= ACC_BUFS and not (yield self.wait(c["acc_empty"][buf],
                                                                      useq // ACC_BUFS - 1)):
                ok = False
                break
            c["tc"].append(("mma", s, k, buf, d["U"], d["first"], useq))
            c["tc"].append(("commit", c["empty"][s]))
            if d["last"]:
                c["acc_desc"][buf] = d["U"]
                c["tc"].append(("commit", c["acc_full"][buf]))
                c["acc_full"][buf].arrive()              # the issuing thread's descriptor arrival
                useq += 1
            k += 1
        if ok:
            buf = useq % ACC_BUFS
            if useq < ACC_BUFS or (yield self.wait(c["acc_empty"][buf], useq // ACC_BUFS - 1)):
                c["acc_desc"][buf] = None                # end marker for the epilogue
                c["acc_full"][buf].arrive()
                c["acc_full"][buf].arrive()
        # every issued MMA completes before the tensor memory is released
        c["tc"].append(("commit", c["drain"]))
        yield Wait(lambda: c["drain"].phases >= 1, bounded=False)

    def epilogue(self, c, e):
        useq = 0
        gen = 0
        while True:
            buf = useq % ACC_BUFS
            got = yield self.wait(c["acc_full"][buf], useq // ACC_BUFS)
            if self.collective_exit:
                w, slot = self.named_barrier(c, gen, not got)
                gen += 1
                yield w
                if slot[1]:
                    return
            elif not got:
                return
            U = c["acc_desc"][buf]
            if U is None:
                return
            u = self.units[U]
            assert c["acc"][buf] == (U, "complete"), f"accumulator {buf} holds {c['acc'][buf]}, want unit {U}"
            key = (u["tile"], u["g"], u["tensor"])
            if u["ord"] > 0:
                fail = False
                if e == 0:                               # the leader polls the counter (bounded)
                    fail = not (yield Wait(lambda: self.done.get(key, 0) >= u["ord"]))
                w, slot = self.named_barrier(c, gen, fail)
                gen += 1
                yield w
                if slot[1]:
                    return
                assert self.partial[key] == list(range(u["ord"])), f"{key}: partial holds {self.partial[key]}"
            c["acc_read"][(buf, e)] = useq
            yield None
            c["acc_empty"][buf].arrive()
            if not u["last"]:
                w, slot = self.named_barrier(c, gen, False)   # every warp stored before the leader publishes
                gen += 1
                yield w
            self.stored.setdefault((id(c), useq), set()).add(e)
            if len(self.stored[(id(c), useq)]) == 4:
                summed = (self.partial.get(key, []) if u["ord"] > 0 else []) + [u["ord"]]
                if u["last"]:
                    assert key not in self.result, f"{key} written twice"
                    self.result[key] = summed
                else:
                    self.partial[key] = summed
                    assert self.done.get(key, 0) == u["ord"]
                    self.done[key] = u["ord"] + 1
            useq += 1

    # ------------------------------------------------------------------ tensor cores
    def tc_step(self, c):
        op = c["tc"].pop(0)
        if op[0] == "commit":
            op[1].arrive()
            return
        _, s, k, buf, U, first, useq = op
        halves = c["half"][s][:c["per_stage"]]
        assert all(x == k for x in halves) and c["stage"][s].get("k") == k, \
            f"stage {s} holds {halves} / {c['stage'][s]}, MMA of chunk {k} reads it"
        if first:
            if useq >= ACC_BUFS:   # every epilogue warp has read the unit two before
                assert all(c["acc_read"].get((buf, e), -1) >= useq - ACC_BUFS for e in range(4)), \
                    f"accumulator {buf} overwritten before its epilogue read it"
            c["acc"][buf] = (U, "partial")
        else:
            assert c["acc"][buf] == (U, "partial")
        if c["stage"][s]["last"]:
            c["acc"][buf] = (U, "complete")

    def _finish(self, name):
        i = name[0]
        del self.roles[name]
        c = self.ctas[i]
        c["exited"] += 1
        if c["exited"] == self.n_roles[i]:               # the CTA's final barrier: free the tensor memory
            assert not c["tc"], "tensor memory released with MMAs still queued"
            c["freed"] = True

    def run(self):
        blocked = {}
        expired = 0
        while self.roles or any(c["tc"] for c in self.ctas):
            def can_go(n):
                if n not in blocked:
                    return True
                w = blocked[n]
                return w.ready() or (w.bounded and self.ctas[n[0]]["abort"])
            choices = [n for n in self.roles if can_go(n)]
            choices += [i for i, c in enumerate(self.ctas) if c["tc"]]
            if not choices:
                stuck = [n for n, w in blocked.items() if w.bounded]
                if self.expire_at is None or not stuck:
                    raise AssertionError("deadlock: " + ", ".join(f"{n}" for n in self.roles))
                n = self.rng.choice(stuck)               # a bounded wait that nothing will satisfy expires
                self.ctas[n[0]]["abort"] = True
                expired += 1
                choices = [n]
            n = self.rng.choice(choices)
            if isinstance(n, int):
                self.tc_step(self.ctas[n])
                continue
            send = None
            if n in blocked:
                w = blocked.pop(n)
                if w.ready():
                    if w.bounded and n[1].startswith(self.expire_roles):
                        self.n_bounded += 1
                        if self.expire_at is not None and self.n_bounded == self.expire_at:
                            self.ctas[n[0]]["abort"] = True   # this wait expires although it could pass
                            send = False
                    if send is None:
                        w.check()
                        send = True
                else:
                    send = False                         # gave up: the CTA aborted
            try:
                y = self.roles[n].send(send)
            except StopIteration:
                self._finish(n)
                continue
            if y is not None:
                blocked[n] = y
        assert all(c["freed"] for c in self.ctas)
        return expired


def _structures():
    rng = random.Random(7)
    out = []
    for i in range(12):
        out.append((make_units(rng, rng.randint(1, 5), rng.randint(1, 5), rng.choice([1, 2])),
                    rng.randint(1, 4)))
    return out


@pytest.mark.parametrize("case", range(12))
@pytest.mark.parametrize("per_stage", [1, PER_STAGE])
def test_protocol_under_random_schedules(case, per_stage):
    units, n_ctas = _structures()[case]
    expected = {}
    for u in units:
        expected.setdefault((u["tile"], u["g"], u["tensor"]), []).append(u["ord"])
    for seed in range(25):
        m = Model(units, n_ctas, seed, n_workers=STAGES * per_stage)
        m.run()
        assert m.result == expected                      # each phase once, in phase order
        assert not any(c["abort"] for c in m.ctas)


@pytest.mark.parametrize("case", range(0, 12, 2))
def test_every_role_leaves_after_any_wait_expires(case):
    # One bounded wait expires (at a random point of a random schedule); the
    # other CTAs' waits on this CTA's partials then expire too.  Every role of
    # every CTA must still leave, the tensor memory being released only after
    # the CTA's tensor-core queue drained (both checked in run()).
    units, n_ctas = _structures()[case]
    base = Model(units, n_ctas, 0)
    base.run()
    rng = random.Random(case)
    for seed in range(20):
        m = Model(units, n_ctas, seed, expire_at=rng.randint(1, base.n_bounded))
        m.run()
    for seed in range(10):              # the same, aimed at the epilogue warps' waits
        epi = Model(units, n_ctas, seed, expire_at=10 ** 9, expire_roles="epi")
        epi.run()
        Model(units, n_ctas, seed, expire_at=rng.randint(1, epi.n_bounded), expire_roles="epi").run()


def test_the_model_catches_a_per_warp_epilogue_exit():
    # With each epilogue warp leaving on its own accumulator wait, a warp whose
    # wait expired leaves the other three in the epilogue's named barrier for
    # good; the model must find such a hang (on work lists with multi-phase
    # units, whose epilogues meet in those barriers).
    units, n_ctas = _structures()[0]
    rng = random.Random(11)
    hangs = 0
    for seed in range(30):
        count = Model(units, n_ctas, seed, expire_at=10 ** 9, expire_roles="epi")
        count.run()
        m = Model(units, n_ctas, seed, collective_exit=False, expire_at=rng.randint(1, count.n_bounded),
                  expire_roles="epi")
        try:
            m.run()
        except AssertionError as e:
            assert "deadlock" in str(e)
            hangs += 1
    assert hangs >= 10


def test_the_model_catches_workers_shared_between_stages():
    # An early version let 8 gather warps take chunks in turn over 6 stages
    # (here: 4 warps over 3), so chunks k and k + STAGES (one stage) could go to
    # different warps and a warp could wait for "stage free" while the stage's
    # barrier was still two phases behind; the hardware passes such a wait at
    # once.  The model must flag it (an early pass, a stage overwritten under its
    # MMA, or a stall).
    units = make_units(random.Random(3), 4, 4, 2)
    flagged = 0
    for seed in range(20):
        try:
            Model(units, 1, seed, n_workers=STAGES + 1).run()
        except AssertionError:
            flagged += 1
    assert flagged >= 15
    for seed in range(20):              # the kernel's design: a fixed set of warps per stage
        Model(units, 1, seed).run()
        Model(units, 1, seed, n_workers=STAGES).run()
