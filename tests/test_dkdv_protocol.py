"""A model of the dK/dV kernel's synchronisation, run under random interleavings.

``dkdv_union_kernel`` (``csrc/qsa_dkdv_union.cu``) is a persistent kernel: per
CTA a scheduler warp, six gather warps, one MMA thread and four epilogue warps
hand chunks and accumulators to one another through mbarriers, and across
CTAs each (tile, group, tensor) passes its FP32 partial from query phase to
query phase through a counter in global memory.  This test restates that
protocol as coroutines (one per warp role and CTA; the tensor core an in-order
queue whose commits arrive when every earlier MMA has completed) and runs it
under many random schedules.  It checks what the kernel's correctness rests
on and what the GPU tests cannot force:

* no deadlock, for any schedule of co-resident CTAs;
* every mbarrier parity wait passes exactly at the phase it is meant for (the
  hardware passes a wait issued two phases early at once);
* no shared-memory stage, ring slot or accumulator is overwritten before its
  reader is done;
* every (tile, group, tensor) adds its partials in phase order, each phase
  exactly once, and the last phase writes the result.

It models the protocol, not the kernel's code: a change to the kernel's
barriers needs the same change here.
"""

import random

import pytest

STAGES, RING, ACC_BUFS, UNIONS = 6, 16, 2, 4


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
    def __init__(self, units, n_ctas, seed, n_workers=STAGES):
        self.rng = random.Random(seed)
        self.n_workers = n_workers
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

    @staticmethod
    def cta_state():
        return dict(full=[Bar(1) for _ in range(STAGES)], empty=[Bar(1) for _ in range(STAGES)],
                    ring_full=[Bar(1) for _ in range(RING)], ring_empty=[Bar(1) for _ in range(RING)],
                    acc_full=[Bar(2) for _ in range(ACC_BUFS)], acc_empty=[Bar(4) for _ in range(ACC_BUFS)],
                    ring=[None] * RING, stage=[None] * STAGES, acc=[None] * ACC_BUFS,
                    acc_desc=[None] * ACC_BUFS, acc_read={}, tc=[])

    def wait(self, bar, phase):
        def ready():
            return bar.ready(phase & 1)

        def check():
            assert bar.phases == phase + 1, f"wait for phase {phase} passed with {bar.phases} completed"
        return ready, check

    # ------------------------------------------------------------------ roles
    def scheduler(self, c):
        k = 0
        while True:
            U = self.claim
            self.claim += 1
            yield None                                   # claims interleave across CTAs
            if U >= len(self.units):
                break
            u = self.units[U]
            for p in range(0, u["n_ent"], UNIONS):
                n = min(UNIONS, u["n_ent"] - p)
                rs = k % RING
                if k >= RING:
                    yield self.wait(c["ring_empty"][rs], k // RING - 1)
                c["ring"][rs] = dict(k=k, U=U, first=p == 0, last=p + n >= u["n_ent"])
                c["ring_full"][rs].arrive()
                k += 1
        for j in range(self.n_workers):                  # end markers; only the first reaches the MMA
            rs = k % RING
            if k >= RING:
                yield self.wait(c["ring_empty"][rs], k // RING - 1)
            c["ring"][rs] = dict(k=k, end=True, mma_end=j == 0)
            c["ring_full"][rs].arrive()
            k += 1

    def worker(self, c, w):
        k = w
        while True:
            rs = k % RING
            yield self.wait(c["ring_full"][rs], k // RING)
            d = c["ring"][rs]
            assert d["k"] == k, f"ring slot {rs} holds chunk {d['k']}, worker wants {k}"
            c["ring_empty"][rs].arrive()
            if d.get("end") and not d["mma_end"]:
                return
            s = k % STAGES
            if k >= STAGES:
                yield self.wait(c["empty"][s], k // STAGES - 1)
            if d.get("end"):
                c["stage"][s] = dict(k=k, end=True)
                c["full"][s].arrive()
                return
            c["stage"][s] = ("filling", k)
            yield None
            c["stage"][s] = dict(d)
            c["full"][s].arrive()
            k += self.n_workers

    def mma(self, c):
        useq = 0
        k = 0
        while True:
            s = k % STAGES
            yield self.wait(c["full"][s], k // STAGES)
            d = c["stage"][s]
            if d.get("end"):
                break
            buf = useq % ACC_BUFS
            if d["first"] and useq >= ACC_BUFS:
                yield self.wait(c["acc_empty"][buf], useq // ACC_BUFS - 1)
            c["tc"].append(("mma", s, k, buf, d["U"], d["first"], useq))
            c["tc"].append(("commit", c["empty"][s]))
            if d["last"]:
                c["acc_desc"][buf] = d["U"]
                c["tc"].append(("commit", c["acc_full"][buf]))
                c["acc_full"][buf].arrive()              # the issuing thread's descriptor arrival
                useq += 1
            k += 1
        buf = useq % ACC_BUFS
        if useq >= ACC_BUFS:
            yield self.wait(c["acc_empty"][buf], useq // ACC_BUFS - 1)
        c["acc_desc"][buf] = None                        # end marker for the epilogue
        c["acc_full"][buf].arrive()
        c["acc_full"][buf].arrive()

    def epilogue(self, c, e):
        useq = 0
        while True:
            buf = useq % ACC_BUFS
            yield self.wait(c["acc_full"][buf], useq // ACC_BUFS)
            U = c["acc_desc"][buf]
            if U is None:
                return
            u = self.units[U]
            assert c["acc"][buf] == (U, "complete"), f"accumulator {buf} holds {c['acc'][buf]}, want unit {U}"
            key = (u["tile"], u["g"], u["tensor"])
            if u["ord"] > 0:
                yield (lambda: self.done.get(key, 0) >= u["ord"], lambda: None)
                assert self.partial[key] == list(range(u["ord"])), f"{key}: partial holds {self.partial[key]}"
            c["acc_read"][(buf, e)] = useq
            yield None
            c["acc_empty"][buf].arrive()
            # the leader publishes once all four warps have stored (the kernel's
            # named barrier over the epilogue warps)
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
        assert isinstance(c["stage"][s], dict) and c["stage"][s].get("k") == k, \
            f"stage {s} holds {c['stage'][s]}, MMA of chunk {k} reads it"
        if first:
            if useq >= ACC_BUFS:   # every epilogue warp has read the unit two before
                assert all(c["acc_read"].get((buf, e), -1) >= useq - ACC_BUFS for e in range(4)), \
                    f"accumulator {buf} overwritten before its epilogue read it"
            c["acc"][buf] = (U, "partial")
        else:
            assert c["acc"][buf] == (U, "partial")
        if c["stage"][s]["last"]:
            c["acc"][buf] = (U, "complete")

    def run(self):
        blocked = {}
        while self.roles or any(c["tc"] for c in self.ctas):
            choices = [n for n in self.roles if n not in blocked or blocked[n][0]()]
            choices += [i for i, c in enumerate(self.ctas) if c["tc"]]
            if not choices:
                raise AssertionError("deadlock: " + ", ".join(f"{n}" for n in self.roles))
            n = self.rng.choice(choices)
            if isinstance(n, int):
                self.tc_step(self.ctas[n])
                continue
            if n in blocked:
                blocked.pop(n)[1]()
            try:
                w = next(self.roles[n])
            except StopIteration:
                del self.roles[n]
                continue
            if w is not None:
                blocked[n] = w


def _structures():
    rng = random.Random(7)
    out = []
    for i in range(12):
        out.append((make_units(rng, rng.randint(1, 5), rng.randint(1, 5), rng.choice([1, 2])),
                    rng.randint(1, 4)))
    return out


@pytest.mark.parametrize("case", range(12))
def test_protocol_under_random_schedules(case):
    units, n_ctas = _structures()[case]
    expected = {}
    for u in units:
        expected.setdefault((u["tile"], u["g"], u["tensor"]), []).append(u["ord"])
    for seed in range(25):
        m = Model(units, n_ctas, seed)
        m.run()
        assert m.result == expected                      # each phase once, in phase order


def test_the_model_catches_workers_shared_between_stages():
    # The first version let 8 gather warps take chunks in turn over 6 stages, so
    # chunks k and k + 6 (one stage) could go to different warps and a warp
    # could wait for "stage free" while the stage's barrier was still two phases
    # behind; the hardware passes such a wait at once.  The model must flag it
    # (an early pass, a stage overwritten under its MMA, or a stall).
    units = make_units(random.Random(3), 4, 4, 2)
    flagged = 0
    for seed in range(20):
        try:
            Model(units, 1, seed, n_workers=8).run()
        except AssertionError:
            flagged += 1
    assert flagged >= 15
    for seed in range(20):              # the kernel's design: one warp per stage
        Model(units, 1, seed).run()
