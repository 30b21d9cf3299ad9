"""Model check of the mbarrier protocols of the grouped-GEMM kernels (no GPU).

Each kernel hands buffers between roles through mbarriers waited on by phase
parity: a TMA ring of shared-memory stages (producer -> MMA), TMEM
accumulators or partial slots (MMA -> epilogue warps) and, in the NVFP4
kernel, a second hand between the TMA and the MMA (the scale threads, which
rearrange each stage's block scales before the MMA copies them to TMEM).  A parity
wait cannot tell a phase from the one two ahead, so a protocol is only right
if no waiter can ever be two phases behind.  Compute-sanitizer is not
available, so this test runs the protocols, as the kernels write them (the
same counters, parities and arrival counts), in a discrete-event model:

- an mbarrier completes a phase when its arrival count is reached;
  ``try_wait.parity(p)`` passes while the current phase's parity is not p;
- TMA copies land at any later moment, in any order; tcgen05 work completes
  in issue order (``tcgen05.commit`` arrives when all earlier MMAs are done);
- every buffer carries the tag of the data last written into it.

Under many random interleavings every consumer must read exactly the tag it
expects, no producer may overwrite data that has not been consumed, and every
role must finish.  Planted protocol mistakes must be caught, so the check is
not vacuous.
"""
import random
from collections import deque

import pytest


class Bar:
    """An mbarrier: a phase completes when its arrivals reach the count and its transaction
    count (bytes announced by expect_tx, less bytes landed; it may go below zero while the
    phase is open) is back to zero."""

    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._maybe_complete()

    def arrive_expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        self._maybe_complete()

    def passed(self, parity):
        return (self.phase & 1) != parity


class Violation(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Violation(msg)


class Sim:
    """Roles are generators that yield the predicate they wait on; async work is posted to
    queues (one FIFO per in-order engine, a fresh queue per out-of-order copy)."""

    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.roles = {}
        self.queues = {}
        self.n = 0

    def role(self, name, gen):
        self.roles[name] = [gen, lambda: True]

    def post(self, queue, fn):
        if queue is None:                       # out of order: its own queue
            self.n += 1
            queue = ("copy", self.n)
        self.queues.setdefault(queue, deque()).append(fn)

    def run(self, max_steps=2_000_000):
        for _ in range(max_steps):
            ready = [("role", k) for k, (g, pred) in self.roles.items() if pred()]
            ready += [("queue", k) for k, q in self.queues.items() if q]
            if not ready:
                if not self.roles:
                    return "done"
                return "deadlock: " + ", ".join(sorted(self.roles))
            kind, key = self.rng.choice(ready)
            if kind == "queue":
                self.queues[key].popleft()()
            else:
                g = self.roles[key][0]
                try:
                    self.roles[key][1] = next(g)
                except StopIteration:
                    del self.roles[key]
        return "no end"


# ----------------------------------------------------------------------------- bf16 / E4M3 grouped GEMM

def gemm(sim, units, k_stages, NS, n_epi=4, plant=None):
    """grouped_gemm_kernel: NS-stage TMA ring, two TMEM accumulators (tempty: 128 epilogue
    threads, modelled as 4 warps)."""
    full, empty = [Bar(1) for _ in range(NS)], [Bar(1) for _ in range(NS)]
    tfull, tempty = [Bar(1) for _ in range(2)], [Bar(n_epi) for _ in range(2)]
    smem, fresh = [None] * NS, [False] * NS       # fresh: landed and not yet consumed by the MMA
    tmem, readers = [None] * 2, [n_epi] * 2

    def producer():
        st, ph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: empty[s].passed(p ^ 1))

                def land(s=st, tag=(u, ks)):
                    check(not fresh[s], f"TMA overwrote stage {s} before the MMA consumed it")
                    smem[s], fresh[s] = tag, True
                    full[s].arrive()
                sim.post(None, land)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

    def mma():
        st, ph, acc, aph = 0, 0, 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tempty[a].passed(p ^ 1))
            check(readers[acc] == n_epi, f"MMA wrote accumulator {acc} while the epilogue was reading it")
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: full[s].passed(p))
                check(smem[st] == (u, ks), f"MMA read stage {st} holding {smem[st]}, expected {(u, ks)}")

                def mma_done(s=st, a=acc, first=ks == 0, u=u):
                    fresh[s] = False
                    if first:
                        tmem[a] = ("partial", u)
                    empty[s].arrive()
                sim.post("tc", mma_done)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

            def acc_done(a=acc, u=u):
                tmem[a], readers[a] = u, 0
                tfull[a].arrive()
            sim.post("tc", acc_done)
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    def epilogue(w):
        acc, aph = 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tfull[a].passed(p))
            if plant == "release_before_read":
                tempty[acc].arrive()
                yield (lambda: True)
                check(tmem[acc] == u, f"epilogue read accumulator {acc} holding {tmem[acc]}, expected {u}")
                readers[acc] += 1
            else:
                check(tmem[acc] == u, f"epilogue read accumulator {acc} holding {tmem[acc]}, expected {u}")
                readers[acc] += 1
                tempty[acc].arrive()
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    sim.role("producer", producer())
    sim.role("mma", mma())
    for w in range(n_epi):
        sim.role(f"epilogue{w}", epilogue(w))


# ----------------------------------------------------------------------------- FP8_B128 grouped GEMM

def gemm_b128(sim, units, k_stages, NS, NP=4, n_epi=4, plant=None):
    """grouped_gemm_b128_kernel: the TMA ring, and NP TMEM partial slots, one per K stage
    (pfull: the MMA's commit; pempty: 128 epilogue threads, modelled as 4 warps)."""
    full, empty = [Bar(1) for _ in range(NS)], [Bar(1) for _ in range(NS)]
    pfull, pempty = [Bar(1) for _ in range(NP)], [Bar(n_epi) for _ in range(NP)]
    smem, fresh = [None] * NS, [False] * NS
    part, readers = [None] * NP, [n_epi] * NP

    def producer():
        st, ph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: empty[s].passed(p ^ 1))

                def land(s=st, tag=(u, ks)):
                    check(not fresh[s], f"TMA overwrote stage {s} before the MMA consumed it")
                    smem[s], fresh[s] = tag, True
                    full[s].arrive()
                sim.post(None, land)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

    def mma():
        st, ph, ps, pph = 0, 0, 0, 0
        wait_parity = (lambda p: p) if plant == "wrong_parity" else (lambda p: p ^ 1)
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: full[s].passed(p))
                yield (lambda q=ps, p=pph: pempty[q].passed(wait_parity(p)))
                check(smem[st] == (u, ks), f"MMA read stage {st} holding {smem[st]}, expected {(u, ks)}")
                check(readers[ps] == n_epi, f"MMA wrote partial slot {ps} while the epilogue was reading it")
                readers[ps] = 0

                def mma_done(s=st, q=ps, tag=(u, ks)):
                    fresh[s] = False
                    part[q] = tag
                    empty[s].arrive()
                    pfull[q].arrive()
                sim.post("tc", mma_done)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1
                ps += 1
                if ps == NP:
                    ps, pph = 0, pph ^ 1

    def epilogue(w):
        ps, pph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda q=ps, p=pph: pfull[q].passed(p))
                check(part[ps] == (u, ks), f"epilogue read partial slot {ps} holding {part[ps]}, expected {(u, ks)}")
                readers[ps] += 1
                pempty[ps].arrive()
                ps += 1
                if ps == NP:
                    ps, pph = 0, pph ^ 1

    sim.role("producer", producer())
    sim.role("mma", mma())
    for w in range(n_epi):
        sim.role(f"epilogue{w}", epilogue(w))


# ----------------------------------------------------------------------------- NVFP4 grouped GEMM

def gemm_fp4(sim, units, k_stages, NS, n_sc=8, n_epi=4):
    """grouped_gemm_fp4_kernel: one TMA ring whose stages pass through two hands before the
    MMA frees them -- full (the TMA bytes), then sfready (every scale thread has written the
    stage's scale atoms), then empty (the MMA's commit) -- and two TMEM accumulators.  The
    128 scale threads are modelled as n_sc independent agents (any of them may run ahead)."""
    full, sfready, empty = [Bar(1) for _ in range(NS)], [Bar(n_sc) for _ in range(NS)], [Bar(1) for _ in range(NS)]
    tfull, tempty = [Bar(1) for _ in range(2)], [Bar(n_epi) for _ in range(2)]
    smem, fresh = [None] * NS, [False] * NS
    atoms = [[None] * n_sc for _ in range(NS)]
    tmem, readers = [None] * 2, [n_epi] * 2

    def producer():
        st, ph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: empty[s].passed(p ^ 1))

                def land(s=st, tag=(u, ks)):
                    check(not fresh[s], f"TMA overwrote stage {s} before the MMA consumed it")
                    smem[s], fresh[s] = tag, True
                    full[s].arrive()
                sim.post(None, land)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

    def scale_thread(i):
        st, ph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: full[s].passed(p))
                check(smem[st] == (u, ks), f"scale thread {i} read stage {st} holding {smem[st]}, expected {(u, ks)}")
                atoms[st][i] = (u, ks)
                sfready[st].arrive()
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

    def mma():
        st, ph, acc, aph = 0, 0, 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tempty[a].passed(p ^ 1))
            check(readers[acc] == n_epi, f"MMA wrote accumulator {acc} while the epilogue was reading it")
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: sfready[s].passed(p))
                check(smem[st] == (u, ks), f"MMA read stage {st} holding {smem[st]}, expected {(u, ks)}")
                check(all(t == (u, ks) for t in atoms[st]), f"MMA copied the atoms of stage {st}: {atoms[st]}")

                def mma_done(s=st):
                    fresh[s] = False
                    empty[s].arrive()
                sim.post("tc", mma_done)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

            def acc_done(a=acc, u=u):
                tmem[a], readers[a] = u, 0
                tfull[a].arrive()
            sim.post("tc", acc_done)
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    def epilogue(w):
        acc, aph = 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tfull[a].passed(p))
            check(tmem[acc] == u, f"epilogue read accumulator {acc} holding {tmem[acc]}, expected {u}")
            readers[acc] += 1
            tempty[acc].arrive()
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    sim.role("producer", producer())
    sim.role("mma", mma())
    for i in range(n_sc):
        sim.role(f"scale{i}", scale_thread(i))
    for w in range(n_epi):
        sim.role(f"epilogue{w}", epilogue(w))


# ----------------------------------------------------------------------------- CTA-pair grouped GEMM

def gemm_pair(sim, units, k_stages, NS, n_epi=4):
    """grouped_gemm_kernel_pair (cta_group::2): each CTA's producer waits its own `empty` and
    loads its half of the stage; the leader arms its `full` with both halves' bytes, and both
    halves complete transactions on the leader's `full` (the peer's may land before the
    leader arms it).  The leader's MMA commits to `empty` and `tfull` of both CTAs (multicast
    commit); the 4 epilogue warps of each CTA arrive on the leader's `tempty` (count 8)."""
    full = [Bar(1) for _ in range(NS)]                                   # leader only
    empty = [[Bar(1) for _ in range(NS)] for _ in range(2)]
    tfull = [[Bar(1) for _ in range(2)] for _ in range(2)]
    tempty = [Bar(2 * n_epi) for _ in range(2)]                          # leader only
    smem = [[None] * NS for _ in range(2)]
    fresh = [[False] * NS for _ in range(2)]
    tmem = [[None] * 2 for _ in range(2)]
    readers = [2 * n_epi] * 2

    def producer(rank):
        st, ph = 0, 0
        for u in range(units):
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: empty[rank][s].passed(p ^ 1))
                if rank == 0:
                    full[st].arrive_expect_tx(2)                         # both halves

                def land(s=st, tag=(u, ks)):
                    check(not fresh[rank][s], f"TMA overwrote stage {s} of CTA {rank} before the MMA consumed it")
                    smem[rank][s], fresh[rank][s] = tag, True
                    full[s].complete_tx(1)
                sim.post(None, land)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

    def mma():
        st, ph, acc, aph = 0, 0, 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tempty[a].passed(p ^ 1))
            check(readers[acc] == 2 * n_epi, f"MMA wrote accumulator {acc} while an epilogue was reading it")
            for ks in range(k_stages):
                yield (lambda s=st, p=ph: full[s].passed(p))
                for r in range(2):
                    check(smem[r][st] == (u, ks), f"MMA read stage {st} of CTA {r} holding {smem[r][st]}")

                def mma_done(s=st):
                    for r in range(2):
                        fresh[r][s] = False
                        empty[r][s].arrive()
                sim.post("tc", mma_done)
                st += 1
                if st == NS:
                    st, ph = 0, ph ^ 1

            def acc_done(a=acc, u=u):
                readers[a] = 0
                for r in range(2):
                    tmem[r][a] = u
                    tfull[r][a].arrive()
            sim.post("tc", acc_done)
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    def epilogue(rank, w):
        acc, aph = 0, 0
        for u in range(units):
            yield (lambda a=acc, p=aph: tfull[rank][a].passed(p))
            check(tmem[rank][acc] == u, f"epilogue of CTA {rank} read accumulator {acc} holding {tmem[rank][acc]}")
            readers[acc] += 1
            tempty[acc].arrive()
            acc += 1
            if acc == 2:
                acc, aph = 0, aph ^ 1

    for r in range(2):
        sim.role(f"producer{r}", producer(r))
        for w in range(n_epi):
            sim.role(f"epilogue{r}.{w}", epilogue(r, w))
    sim.role("mma", mma())


# ----------------------------------------------------------------------------- one-launch FFN (grouped_ffn.cu)

def ffn_fused(sim, n_ctas, entries, m_up, m_down, k_up, k_down, NS, n_epi=4, UQ=4, plant=None, form="bf16",
              n_sc=4, NP=4):
    """The one-launch FFNs on n_ctas CTAs (form "bf16": grouped_ffn_kernel; "fp4":
    grouped_ffn_fp4_kernel, whose stages also pass through the n_sc scale warps -- full, then
    sfready, then the MMA -- and whose scale warps read the unit queue too; "b128":
    grouped_ffn_b128_kernel, whose MMA writes one of NP TMEM partial slots per stage, read by
    every epilogue warp per stage instead of one accumulator per unit).  The units are the list [up units (entry, block)] +
    [down units]; each CTA's producer claims the next unit from a global counter (one atomic
    step, the next claim taken while the current unit loads) and publishes it in a UQ-slot
    queue in shared memory (uq_full: 1 arrival; uq_empty: the MMA thread and the n_epi epilogue
    warps), from which the MMA thread and every epilogue warp read the same sequence; then the
    per-CTA TMA ring and two accumulators of the grouped GEMM.  A down unit of entry s reads
    H[s]; its producer first waits until the global counter done[s] reaches n_epi * m_up (every
    epilogue warp of every up unit of s has stored its rows and reported).  Shared: the claim
    counter, done[] and, per entry, how many up epilogue warps have stored their rows of H."""
    n_up, n_down = entries * m_up, entries * m_down
    units = [("up", u // m_up) for u in range(n_up)] + [("down", u // m_down) for u in range(n_down)]
    n_units = len(units)
    claim = [0]
    done = [0] * entries
    stored = [0] * entries
    target = n_epi * m_up if plant != "early_read" else n_epi * (m_up - 1)   # planted: one up unit short
    uq_readers = 1 + n_epi if plant != "queue_short" else 1                 # planted: only the MMA frees a slot
    if form == "fp4" and plant not in ("queue_short", "queue_no_scale"):
        uq_readers += n_sc

    def cta(c):
        full, empty = [Bar(1) for _ in range(NS)], [Bar(1) for _ in range(NS)]
        tfull, tempty = [Bar(1) for _ in range(2)], [Bar(n_epi) for _ in range(2)]
        sfready, atoms = [Bar(n_sc) for _ in range(NS)], [[None] * n_sc for _ in range(NS)]
        pfull, pempty = [Bar(1) for _ in range(NP)], [Bar(n_epi) for _ in range(NP)]
        part, preaders = [None] * NP, [n_epi] * NP
        uq_full, uq_empty = [Bar(1) for _ in range(UQ)], [Bar(uq_readers) for _ in range(UQ)]
        uq = [None] * UQ
        published = []                      # the units this CTA claimed, in order
        smem, fresh = [None] * NS, [False] * NS
        tmem = [None] * 2

        def take(who, i, q, arrive=True):
            u = uq[q]
            check(u == (published[i] if i < len(published) else -1),
                  f"CTA {c}: {who} read unit {u} from queue slot {q}, expected entry {i} of {published}")
            if arrive:
                uq_empty[q].arrive()
            return u

        def producer():
            st, ph, q, qph = 0, 0, 0, 0
            nxt = claim[0]
            claim[0] += 1
            while True:
                u = nxt if nxt < n_units else -1
                yield (lambda q_=q, p=qph: uq_empty[q_].passed(p ^ 1))
                uq[q] = u
                if u >= 0:
                    published.append(u)
                uq_full[q].arrive()
                q += 1
                if q == UQ:
                    q, qph = 0, qph ^ 1
                if u < 0:
                    return
                yield (lambda: True)
                nxt = claim[0]
                claim[0] += 1
                kind, s = units[u]
                if kind == "down":
                    yield (lambda s=s: done[s] >= target)
                ks_n = k_up if kind == "up" else k_down
                for ks in range(ks_n):
                    yield (lambda s_=st, p=ph: empty[s_].passed(p ^ 1))

                    def land(s_=st, tag=(c, u, ks), kind=kind, s=s):
                        check(not fresh[s_], f"CTA {c}: TMA overwrote stage {s_} before the MMA consumed it")
                        if kind == "down":
                            check(stored[s] == n_epi * m_up, f"CTA {c}: read H of entry {s} with "
                                                             f"{stored[s]} of {n_epi * m_up} up warps stored")
                        smem[s_], fresh[s_] = tag, True
                        full[s_].arrive()
                    sim.post(None, land)
                    st += 1
                    if st == NS:
                        st, ph = 0, ph ^ 1

        def mma():
            st, ph, acc, aph, q, qph, i, ps, pph = 0, 0, 0, 0, 0, 0, 0, 0, 0
            while True:
                yield (lambda q_=q, p=qph: uq_full[q_].passed(p))
                u = take("MMA", i, q)
                i += 1
                q += 1
                if q == UQ:
                    q, qph = 0, qph ^ 1
                if u < 0:
                    return
                kind, s = units[u]
                if form != "b128":
                    yield (lambda a=acc, p=aph: tempty[a].passed(p ^ 1))
                for ks in range(k_up if kind == "up" else k_down):
                    if form == "fp4":
                        yield (lambda s_=st, p=ph: sfready[s_].passed(p))
                        check(all(t == (c, u, ks) for t in atoms[st]), f"CTA {c}: MMA copied atoms {atoms[st]}")
                    else:
                        yield (lambda s_=st, p=ph: full[s_].passed(p))
                    check(smem[st] == (c, u, ks), f"CTA {c}: MMA read stage {st} holding {smem[st]}")
                    if form == "b128":
                        yield (lambda q_=ps, p=pph: pempty[q_].passed(p ^ 1))
                        check(preaders[ps] == n_epi, f"CTA {c}: MMA wrote partial slot {ps} while it was read")
                        preaders[ps] = 0

                        def part_done(s_=st, q_=ps, tag=(u, ks)):
                            fresh[s_] = False
                            part[q_] = tag
                            empty[s_].arrive()
                            pfull[q_].arrive()
                        sim.post(("tc", c), part_done)
                        ps += 1
                        if ps == NP:
                            ps, pph = 0, pph ^ 1
                    else:
                        def mma_done(s_=st):
                            fresh[s_] = False
                            empty[s_].arrive()
                        sim.post(("tc", c), mma_done)
                    st += 1
                    if st == NS:
                        st, ph = 0, ph ^ 1
                if form == "b128":
                    continue

                def acc_done(a=acc, u=u):
                    tmem[a] = u
                    tfull[a].arrive()
                sim.post(("tc", c), acc_done)
                acc += 1
                if acc == 2:
                    acc, aph = 0, aph ^ 1

        def scale_warp(j):
            st, ph, q, qph, i = 0, 0, 0, 0, 0
            while True:
                yield (lambda q_=q, p=qph: uq_full[q_].passed(p))
                u = take(f"scale warp {j}", i, q)
                i += 1
                q += 1
                if q == UQ:
                    q, qph = 0, qph ^ 1
                if u < 0:
                    return
                kind, s = units[u]
                for ks in range(k_up if kind == "up" else k_down):
                    yield (lambda s_=st, p=ph: full[s_].passed(p))
                    check(smem[st] == (c, u, ks), f"CTA {c}: scale warp {j} read stage {st} holding {smem[st]}")
                    atoms[st][j] = (c, u, ks)
                    sfready[st].arrive()
                    st += 1
                    if st == NS:
                        st, ph = 0, ph ^ 1

        def epilogue(w):
            acc, aph, q, qph, i, ps, pph = 0, 0, 0, 0, 0, 0, 0
            while True:
                yield (lambda q_=q, p=qph: uq_full[q_].passed(p))
                u = take(f"epilogue warp {w}", i, q, arrive=plant != "queue_short")
                i += 1
                q += 1
                if q == UQ:
                    q, qph = 0, qph ^ 1
                if u < 0:
                    return
                kind, s = units[u]
                if form == "b128":
                    for ks in range(k_up if kind == "up" else k_down):
                        yield (lambda q_=ps, p=pph: pfull[q_].passed(p))
                        check(part[ps] == (u, ks), f"CTA {c}: epilogue read partial slot {ps} holding {part[ps]}")
                        preaders[ps] += 1
                        pempty[ps].arrive()
                        ps += 1
                        if ps == NP:
                            ps, pph = 0, pph ^ 1
                else:
                    yield (lambda a=acc, p=aph: tfull[a].passed(p))
                    check(tmem[acc] == u, f"CTA {c}: epilogue read accumulator {acc} holding {tmem[acc]}")
                    tempty[acc].arrive()
                if kind == "up":
                    stored[s] += 1           # this warp's rows of H are stored (and fenced)
                    yield (lambda: True)
                    done[s] += 1             # then reported with a release add
                acc += 1
                if acc == 2:
                    acc, aph = 0, aph ^ 1

        sim.role(f"producer{c}", producer())
        sim.role(f"mma{c}", mma())
        for w in range(n_epi):
            sim.role(f"epilogue{c}.{w}", epilogue(w))
        if form == "fp4":
            for j in range(n_sc):
                sim.role(f"scale{c}.{j}", scale_warp(j))

    for c in range(n_ctas):
        cta(c)

    def all_units_once():
        return claim[0] >= n_units
    return all_units_once


@pytest.mark.parametrize("n_ctas,entries,m_up,m_down,k_up,k_down,NS",
                         [(3, 4, 3, 4, 4, 3, 3), (2, 5, 2, 3, 3, 2, 2), (4, 3, 2, 2, 2, 2, 4), (5, 2, 3, 2, 2, 3, 2)])
def test_one_launch_ffn_protocol(n_ctas, entries, m_up, m_down, k_up, k_down, NS):
    for seed in range(25):
        sim = Sim(seed)
        claimed_all = ffn_fused(sim, n_ctas, entries, m_up, m_down, k_up, k_down, NS)
        assert sim.run() == "done" and claimed_all()


@pytest.mark.parametrize("form", ["fp4", "b128"])
@pytest.mark.parametrize("n_ctas,entries,m_up,m_down,k_up,k_down,NS",
                         [(3, 4, 3, 4, 4, 3, 3), (2, 5, 2, 3, 3, 2, 2), (4, 3, 2, 2, 2, 2, 4)])
def test_one_launch_ffn_protocol_nvfp4_and_b128(form, n_ctas, entries, m_up, m_down, k_up, k_down, NS):
    """The NVFP4 one-launch kernel (the scale warps read the unit queue and hand each stage on)
    and the FP8_B128 one (per-stage partial slots instead of per-unit accumulators)."""
    for seed in range(20):
        sim = Sim(seed)
        claimed_all = ffn_fused(sim, n_ctas, entries, m_up, m_down, k_up, k_down, NS, form=form)
        assert sim.run() == "done" and claimed_all()


def test_a_unit_queue_not_waiting_for_the_scale_warps_is_caught():
    """Planted: the NVFP4 queue slots count only the MMA thread and the epilogue warps, so the
    producer may overwrite a slot a scale warp has not read yet."""
    caught = 0
    for seed in range(40):
        sim = Sim(seed)
        ffn_fused(sim, 2, 6, 3, 3, 1, 1, 2, UQ=2, plant="queue_no_scale", form="fp4")
        try:
            sim.run()
        except Violation:
            caught += 1
    assert caught > 0


def test_a_unit_queue_freed_by_the_mma_alone_is_caught():
    """Planted: the queue slots count only the MMA thread's read, so the producer may overwrite a
    slot an epilogue warp has not read yet."""
    caught = 0
    for seed in range(40):
        sim = Sim(seed)
        ffn_fused(sim, 2, 6, 3, 3, 1, 1, 2, UQ=2, plant="queue_short")
        try:
            sim.run()
        except Violation:
            caught += 1
    assert caught > 0


def test_a_down_unit_waiting_for_too_few_reports_is_caught():
    caught = 0
    for seed in range(25):
        sim = Sim(seed)
        ffn_fused(sim, 4, 2, 3, 2, 3, 2, 2, plant="early_read")
        try:
            sim.run()
        except Violation:
            caught += 1
    assert caught > 0


SEEDS = range(40)


@pytest.mark.parametrize("units,k_stages,NS", [(5, 21, 8), (7, 3, 2), (4, 1, 3), (6, 42, 4)])
def test_grouped_gemm_protocol(units, k_stages, NS):
    for seed in SEEDS:
        sim = Sim(seed)
        gemm(sim, units, k_stages, NS)
        assert sim.run() == "done"


@pytest.mark.parametrize("units,k_stages,NS", [(5, 21, 6), (6, 3, 2), (4, 1, 3), (3, 42, 6)])
def test_cta_pair_gemm_protocol(units, k_stages, NS):
    for seed in SEEDS:
        sim = Sim(seed)
        gemm_pair(sim, units, k_stages, NS)
        assert sim.run() == "done"


@pytest.mark.parametrize("units,k_stages,NS", [(4, 21, 8), (6, 15, 8), (5, 3, 2), (3, 1, 4), (3, 9, 5)])
def test_fp8_b128_protocol(units, k_stages, NS):
    for seed in SEEDS:
        sim = Sim(seed)
        gemm_b128(sim, units, k_stages, NS)
        assert sim.run() == "done"


@pytest.mark.parametrize("units,k_stages,NS", [(3, 11, 4), (3, 8, 2), (4, 1, 3), (3, 2, 5), (2, 11, 8)])
def test_nvfp4_protocol(units, k_stages, NS):
    for seed in range(15):
        sim = Sim(seed)
        gemm_fp4(sim, units, k_stages, NS)
        assert sim.run() == "done"


def test_a_wait_on_the_wrong_parity_is_caught():
    sim = Sim(0)
    gemm_b128(sim, 3, 5, 4, plant="wrong_parity")
    assert sim.run().startswith("deadlock")


def test_releasing_an_accumulator_before_reading_it_is_caught():
    caught = 0
    for seed in SEEDS:
        sim = Sim(seed)
        gemm(sim, 6, 2, 2, plant="release_before_read")
        try:
            sim.run()
        except Violation:
            caught += 1
    assert caught > 0
