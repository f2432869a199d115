"""A model of the tensor-core forward kernel's mbarrier protocol, run under
random interleavings on the CPU.

Each role of the kernel's CTA is a generator that waits and arrives exactly
as the kernel does (a warpgroup's arrivals are one arrival here):

  * the TMA producer, loading a ring of stq Q/K slots and a ring of stv V
    slots in pair order;
  * three MMA issuers: one issues S = Q K^T of every chunk j = n * nch + c
    of the CTA's pairs in order, into S slot j % nslot once P.V of chunk
    j - nslot has finished with that slot; two issue P.V, issuer u taking
    the chunks of pairs u, u + 2, ... into O slot u, each once the softmax
    wrote its P and, for a pair's first chunk, once the epilogue read that
    O slot's previous pair (their "V loaded" and "P written" barriers are
    per issuer, with phase counts of their own);
  * ng softmax groups, group g taking pairs g, g + ng, ...: every chunk of
    its pair in order, each announced on the (slot, group) barrier, then the
    pair's row sums into shared memory (one slot per group and use parity,
    released by the epilogue); all groups meet to rebuild the CTA's bias
    table before every pair whose head differs from the previous pair's,
    and stay for the rebuilds after their own last pair;
  * the epilogue, taking every pair in order: row sums, then O.

The tensor core starts MMA groups in issue order but lets a group into one
accumulator overlap an earlier group into another (only MMAs into the same
accumulator are ordered); a commit arrives once every MMA that its thread
issued before it has finished.  TMA
loads land after random delays.  A
barrier holds a completed-phase count, and a parity wait succeeds when the
current phase's parity differs from the parity waited for, as
mbarrier.try_wait.parity does.  The model checks that:

  * every successful wait observes exactly the phase it was meant for (no
    parity aliasing);
  * no shared-memory slot is overwritten while an MMA still reads it, and
    every MMA reads the pair it was meant for;
  * no S slot is written by S = Q K^T while P.V still reads its P, no O slot
    is overwritten before the epilogue read it, no row-sum slot is
    overwritten before the epilogue read it, and the bias table is never
    rebuilt while a pair reads it;
  * every commit and load completion the CTA waits for has arrived by the
    time all roles are done, and nothing deadlocks.

It covers every shape the kernel builds: 1-3 stages per ring, 2-4 S slots,
1-5 chunks per pair, 1-3 softmax groups, and a head that is
constant or changes every pair or every third pair.  The last tests plant
five protocol mistakes -- S = Q K^T issued
into a slot without waiting for the P.V that reads it, a softmax group that
writes its row sums without waiting for the epilogue to free the slot, and
one "S ready" barrier per slot shared by the groups (met while building the
kernel: a group waiting on a slot's second phase saw the first phase's
parity), a group that skips the table rebuilds after its last pair, and
one "P written" barrier per slot shared by the two P.V issuers -- and check
that the model catches them.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.completed, self.pending = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completed += 1

    def try_wait(self, phase):
        """Wait for the completion of `phase` (parity phase & 1)."""
        ok = (self.completed & 1) != (phase & 1)
        if ok and self.completed != phase + 1:
            raise AssertionError(f"{self.name}: wait for phase {phase} passed with {self.completed} completed")
        return ok

    def fresh_ok(self, use):
        """A producer-side wait of the kernel: parity ((use) & 1) ^ 1, which a
        fresh barrier passes; use u waits for completion u - 1."""
        if use == 0:
            return True
        return self.try_wait(use - 1)


class ProtocolError(AssertionError):
    pass


def simulate(stq, stv, nslot, nch, ng, npairs, seed, head_period=0, skip_slot_wait=False,
             skip_l_empty=False, shared_s_full=False, skip_trailing_rebuilds=False, shared_p_full=False):
    """head_period > 0: the CTA's pairs change head every head_period pairs
    (0: one head throughout)."""
    rnd = random.Random(seed)
    kfull = [Barrier(f"kfull{s}") for s in range(stq)]
    kempty = [Barrier(f"kempty{s}") for s in range(stq)]
    # V "full" and P "ready" barriers per P.V issuer: the two issuers take
    # alternate pairs, and a waiter that runs ahead must not see the other
    # issuer's phase
    vfull = {(s, u): Barrier(f"vfull{s}{u}") for s in range(stv) for u in range(2)}
    vempty = [Barrier(f"vempty{s}") for s in range(stv)]
    head = [(n // head_period) % 3 if head_period else 0 for n in range(npairs)]
    tbl = Barrier("tbl", count=ng)
    table = {"head": None, "readers": set()}
    # one "S ready" barrier per (slot, softmax group): a slot's consecutive
    # chunks belong to different groups, and a group that reaches its wait
    # early must not see another group's phase
    s_full = {(s, g): Barrier(f"s_full{s}{g}") for s in range(nslot) for g in range(ng)}
    if shared_s_full:  # planted mistake: one barrier per slot for all groups
        for s in range(nslot):
            for g in range(1, ng):
                s_full[(s, g)] = s_full[(s, 0)]
    p_full = {(s, u): Barrier(f"p_full{s}{u}", count=1) for s in range(nslot) for u in range(2)}
    if shared_p_full:  # planted mistake: one barrier per slot for both P.V issuers
        for s in range(nslot):
            p_full[(s, 1)] = p_full[(s, 0)]
    slot_free = [Barrier(f"slot_free{s}") for s in range(nslot)]
    o_full = [Barrier(f"o_full{o}") for o in range(2)]   # one O slot per P.V issuer
    o_empty = [Barrier(f"o_empty{o}") for o in range(2)]
    l_full = {(g, par): Barrier(f"l_full{g}{par}") for g in range(ng) for par in (0, 1)}
    l_empty = {(g, par): Barrier(f"l_empty{g}{par}") for g in range(ng) for par in (0, 1)}
    lsum = {}

    kslot, vslot = [None] * stq, [None] * stv           # pair held by each shared-memory slot
    kreaders, vreaders = [set() for _ in range(stq)], [set() for _ in range(stv)]
    S = [None] * nslot                                   # chunk held by each S slot (S, then P)
    s_readers = [set() for _ in range(nslot)]            # P.V of a chunk reading the slot's P
    O = [None] * 2                                       # pair accumulated / held by each O slot
    events, clock, seq = [], [0], [0]
    pipe = {"last_start": 0}                             # the tensor core; per issuer, when its last MMA ends
    outstanding = [0]                                    # asynchronous completions not yet arrived

    def later(fn, delay):
        seq[0] += 1
        outstanding[0] += 1

        def fire():
            outstanding[0] -= 1
            fn()
        events.append((clock[0] + delay, seq[0], fire))

    def mma(start_fn, done_fn, who):
        """Issues one MMA group (one accumulator) from issuer `who`.  The tensor
        core starts groups in issue order and may overlap them: only MMAs into
        the same accumulator are ordered by the hardware, so a later group may
        write its accumulator while an earlier one still reads its
        operands."""
        start = max(clock[0] + 1, pipe["last_start"] + 1)
        end = start + rnd.randint(1, 12)
        pipe["last_start"] = start
        pipe[who] = max(pipe.get(who, 0), end)
        seq[0] += 1
        events.append((start, seq[0], start_fn))
        later(done_fn, end - clock[0])
        return end

    def commit(barrier, who):
        """tcgen05.commit: arrives once every MMA issued so far by this thread
        (issuer `who`) has finished."""
        later(barrier.arrive, max(1, pipe.get(who, 0) - clock[0]))

    def check(cond, what):
        if not cond:
            raise ProtocolError(what)

    def producer():
        # one thread loads both rings, in pair order: Q and K, then V
        for n in range(npairs):
            s = n % stq
            while not kempty[s].fresh_ok(n // stq):
                yield
            check(not kreaders[s], f"Q/K slot {s} reused while read")

            def land_k(n=n, s=s):
                check(not kreaders[s], f"Q/K slot {s} landed while read")
                kslot[s] = n
                kfull[s].arrive()
            later(land_k, rnd.randint(1, 20))
            s = n % stv
            while not vempty[s].fresh_ok(n // stv):
                yield
            check(not vreaders[s], f"V slot {s} reused while read")

            def land_v(n=n, s=s):
                check(not vreaders[s], f"V slot {s} landed while read")
                vslot[s] = n
                vfull[(s, n % 2)].arrive()
            later(land_v, rnd.randint(1, 20))
        yield "done"

    def qk_issuer():
        # S = Q K^T of every chunk in order, into slot j % nslot once P.V of
        # chunk j - nslot has finished with it
        total = npairs * nch
        for i in range(total):
            n, c, sl, s = i // nch, i % nch, i % nslot, (i // nch) % stq
            if c == 0:
                while not kfull[s].try_wait(n // stq):
                    yield
            if i >= nslot and not skip_slot_wait:
                while not slot_free[sl].try_wait(i // nslot - 1):
                    yield
            check(kslot[s] == n, f"QK({n},{c}) reads Q/K of pair {kslot[s]}")

            def qk_start(i=i, n=n, s=s, sl=sl):
                check(not s_readers[sl], f"QK chunk {i} writes slot {sl} while P.V reads it")
                check(kslot[s] == n, f"Q/K slot of pair {n} changed under QK")
                kreaders[s].add(i)
                S[sl] = ("S", i)

            def qk_done(i=i, s=s):
                kreaders[s].discard(i)
            mma(qk_start, qk_done, "qk")
            commit(s_full[(sl, n % ng)], "qk")
            if c == nch - 1:
                commit(kempty[s], "qk")
        yield "done"

    def pv_issuer(u):
        # P.V of every chunk of pairs u, u + 2, ... in order, into O slot u
        vuses, puses = [0] * stv, [0] * nslot  # this issuer's own phase counts (phase bits in the kernel)
        for n in range(u, npairs, 2):
            for c in range(nch):
                j = n * nch + c
                sl, s, o = j % nslot, n % stv, u
                phase = j // nslot if shared_p_full else puses[sl]
                while not p_full[(sl, u)].try_wait(phase):
                    yield
                puses[sl] += 1
                if c == 0:
                    while not vfull[(s, u)].try_wait(vuses[s]):
                        yield
                    vuses[s] += 1
                    while not o_empty[o].fresh_ok(n // 2):
                        yield
                check(S[sl] == ("P", j), f"PV chunk {j} finds slot {sl} holding {S[sl]}")

                def pv_start(j=j, n=n, c=c, s=s, sl=sl, o=o):
                    check(vslot[s] == n, f"PV({n},{c}) reads V of pair {vslot[s]}")
                    check(S[sl] == ("P", j), f"PV chunk {j} reads slot {sl} holding {S[sl]}")
                    if c == 0:
                        check(O[o] is None, f"PV({n}) overwrites O of pair {O[o]} before the epilogue read it")
                        O[o] = ("acc", n)
                    vreaders[s].add(j)
                    s_readers[sl].add(j)

                def pv_done(j=j, n=n, c=c, s=s, sl=sl, o=o):
                    vreaders[s].discard(j)
                    s_readers[sl].discard(j)
                    if c == nch - 1:
                        O[o] = ("done", n)
                mma(pv_start, pv_done, f"pv{u}")
                commit(slot_free[sl], f"pv{u}")
                if c == nch - 1:
                    commit(o_full[o], f"pv{u}")
                    commit(vempty[s], f"pv{u}")
        yield "done"

    def softmax_group(g):
        uses = [0] * nslot  # the group's own count of uses per slot (phase bits in the kernel)
        meetings = [0]
        state = {"next": 0, "prev": None}

        def meet():
            tbl.arrive()
            while not tbl.try_wait(meetings[0]):
                yield
            meetings[0] += 1

        def rebuild_until(last):
            # every group takes part in every table rebuild, in pair order
            while state["next"] <= last:
                m = state["next"]
                state["next"] += 1
                if head[m] == state["prev"]:
                    continue
                state["prev"] = head[m]
                yield from meet()  # every read of the previous table is done
                check(not table["readers"], f"table rebuilt for pair {m} while pairs {table['readers']} read it")
                table["head"] = ("building", head[m])
                for _ in range(rnd.randint(0, 3)):
                    yield
                yield from meet()  # the new table is complete
                table["head"] = head[m]

        for use, n in enumerate(range(g, npairs, ng)):
            yield from rebuild_until(n)
            check(table["head"] == head[n], f"pair {n} (head {head[n]}) finds the table of {table['head']}")
            table["readers"].add(n)
            for c in range(nch):
                j = n * nch + c
                sl = j % nslot
                phase = j // nslot if shared_s_full else uses[sl]
                while not s_full[(sl, g)].try_wait(phase):
                    yield
                uses[sl] += 1
                check(S[sl] == ("S", j), f"softmax of chunk {j} finds slot {sl} holding {S[sl]}")
                for _ in range(rnd.randint(0, 12)):
                    yield
                check(S[sl] == ("S", j), f"slot {sl} changed under the softmax of chunk {j}")
                check(table["head"] == head[n], f"table changed under pair {n}")
                S[sl] = ("P", j)
                p_full[(sl, n % 2)].arrive()
            table["readers"].discard(n)
            slot = (g, use & 1)
            if not skip_l_empty:
                while not l_empty[slot].fresh_ok(use >> 1):
                    yield
            check(lsum.get(slot, "read") == "read", f"row sums of pair {n} overwrite unread ones")
            lsum[slot] = n
            l_full[slot].arrive()
        if not skip_trailing_rebuilds:
            yield from rebuild_until(npairs - 1)
        yield "done"

    def epilogue():
        for n in range(npairs):
            g, use, o = n % ng, n // ng, n % 2
            slot = (g, use & 1)
            while not l_full[slot].try_wait(use >> 1):
                yield
            check(lsum[slot] == n, f"epilogue of pair {n} reads the row sums of pair {lsum[slot]}")
            for _ in range(rnd.randint(0, 3)):
                yield
            lsum[slot] = "read"
            l_empty[slot].arrive()
            while not o_full[o].try_wait(n // 2):
                yield
            check(O[o] == ("done", n), f"epilogue of pair {n} finds O slot {o} holding {O[o]}")
            for _ in range(rnd.randint(0, 5)):
                yield
            O[o] = None
            o_empty[o].arrive()
        yield "done"

    roles = [producer(), qk_issuer(), pv_issuer(0), pv_issuer(1)] + [softmax_group(g) for g in range(ng)] + [
        epilogue()]
    done = [False] * len(roles)
    for _ in range(10 ** 6):
        if all(done) and not events:
            check(outstanding[0] == 0, "completions still in flight at exit")
            return
        events.sort()
        while events and events[0][0] <= clock[0]:
            events.pop(0)[2]()
        i = rnd.randrange(len(roles))
        if not done[i] and next(roles[i]) == "done":
            done[i] = True
        clock[0] += 1
    raise ProtocolError("deadlock")


# (stq, stv, nslot, nch, ng): the shapes the kernel builds -- d = 32 with
# k <= 9 (3 + 3 stages, 3 S slots of 8 halo rows, 2 chunks), k = 11 and 13
# (2 + 2 or 2 + 1 stages, 4 slots of 4 rows, 5 chunks), d = 64 (2 slots,
# down to 1 + 1 stages) -- and some more.
COMBOS = [
    (3, 3, 3, 2, 2), (2, 2, 4, 5, 2), (2, 1, 4, 5, 2), (2, 2, 2, 2, 2), (2, 1, 2, 2, 2),
    (1, 1, 2, 5, 2), (1, 1, 2, 2, 2), (2, 3, 3, 1, 1), (1, 2, 4, 3, 3), (3, 1, 3, 5, 2),
]


@pytest.mark.parametrize("stq,stv,nslot,nch,ng", COMBOS)
@pytest.mark.parametrize("head_period", [0, 1, 3])
def test_protocol_under_random_interleavings(stq, stv, nslot, nch, ng, head_period):
    for seed in range(25):
        for npairs in (1, 2, 3, 5, 8, 13):
            simulate(stq, stv, nslot, nch, ng, npairs, seed * 100 + npairs, head_period)


def test_model_catches_a_slot_reused_before_its_pv_finished():
    # S = Q K^T issued into a slot without waiting for the P.V that reads
    # the slot's P: the two MMAs write and read different accumulators, so
    # nothing orders them and QK^T may overwrite P while P.V reads it
    with pytest.raises(AssertionError):
        for seed in range(200):
            for npairs in (3, 5, 8):
                simulate(2, 2, 2, 2, 2, npairs, seed, skip_slot_wait=True)


def test_model_catches_row_sums_written_before_the_epilogue_read_them():
    with pytest.raises(AssertionError):
        for seed in range(400):
            for npairs in (5, 8, 13):
                simulate(3, 3, 4, 1, 1, npairs, seed, skip_l_empty=True)


def test_model_catches_one_s_ready_barrier_per_slot_shared_by_the_groups():
    with pytest.raises(AssertionError):
        for seed in range(200):
            for npairs in (3, 5, 8):
                simulate(3, 3, 4, 5, 2, npairs, seed, shared_s_full=True)


def test_model_catches_a_group_that_skips_the_rebuilds_after_its_last_pair():
    # a group that leaves when its own pairs are done leaves the other group
    # waiting alone at the next table rebuild
    with pytest.raises(AssertionError):
        for seed in range(50):
            for npairs in (3, 4, 5):
                simulate(2, 2, 3, 2, 2, npairs, seed, head_period=1, skip_trailing_rebuilds=True)


def test_model_catches_one_p_ready_barrier_per_slot_shared_by_the_pv_issuers():
    with pytest.raises(AssertionError):
        for seed in range(200):
            for npairs in (3, 5, 8):
                simulate(3, 3, 3, 2, 2, npairs, seed, shared_p_full=True)
