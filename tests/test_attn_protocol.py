"""A model of attn_kernel's synchronisation protocol, run under random schedules on the CPU.

The kernel's roles are modelled one to one: the set-up thread (Q and the first dense K
tiles), the K and V producer threads with their joint drain, the S thread, the PV thread,
and the eight softmax warps (two warpgroups, each on one 64-key half of every tile).  The
model keeps the kernel's barrier counts and the parity each wait uses:

* mbarriers complete a phase when their arrivals (and, for a TMA fill, its bytes) are in;
  ``try_wait.parity(p)`` succeeds when the barrier's completed-phase count has the other
  parity.  Every wait also records which phase it meant, so a wait that passes for the
  wrong phase (its waiter two phases behind, or two phases ahead of the barrier, where the
  parity looks the same) is reported.
* a tcgen05.commit arrives when every MMA its thread issued before it has completed; MMAs
  of one thread run in issue order, MMAs of different threads in any order.
* named barriers (bar.sync) complete a generation when all participants have arrived.
* a bounded mbarrier wait can run out: the model lets one run out only when nothing else
  can move (or at random, to exercise the abort path), sets the CTA's abort flag, and from
  then on a wait whose phase is not complete returns at once, as the kernel's does.

Checked on every schedule: the run ends (no participant of a named barrier is missing;
without injected aborts no wait ever has to run out), every TMA load issued has landed
before the CTA ends, and, on runs without aborts, the data order: S_l is written before
the softmax reads it, P_l before its PV reads it, the PV has read P_l before S_{l+2}
overwrites that buffer, a warpgroup rescales O only between its PVs, a ring slot is
refilled only after its MMA has read it, and the epilogue reads O after every MMA.
"""
import random

import pytest

SLOTS = 5


def ring_tile(q):
    """The tile at ring position q (K0, K1, V0, K2, V1, K3, V2, ...): (is_k, l)."""
    if q < 2:
        return True, q
    if q % 2 == 0:
        return False, (q - 2) // 2
    return True, (q + 1) // 2


def pos_k(j):
    return j if j < 2 else 2 * j - 1


def pos_v(i):
    return 2 + 2 * i


class Deadlock(Exception):
    pass


class Sim:
    def __init__(self, n_iter, pre, seed, abort_p=0.0):
        self.rng = random.Random(seed)
        self.n = n_iter
        self.pre = pre
        self.abort_p = abort_p
        self.t = 0
        self.abort = False
        self.timeouts = 0
        self.bars = {}              # name -> [count, pending, phases, tx]
        self.nb = {}                # id -> [count, arrived, generation]
        self.events = []            # (time, seq, fn)
        self.seq = 0
        self.mma_q = {}             # thread -> list of [end_time or None, fn_on_done]
        self.log = {}               # (kind, ...) -> time
        self.issues = []            # protocol violations
        self.loads_in_flight = 0

    # ---------------------------------------------------------------- primitives
    def bar(self, name, count):
        self.bars[name] = [count, count, 0, 0]

    def arrive(self, name, tx=0):
        b = self.bars[name]
        b[1] -= 1
        b[3] += tx
        self._maybe_complete(name)

    def complete_tx(self, name, n):
        b = self.bars[name]
        b[3] -= n
        self._maybe_complete(name)

    def _maybe_complete(self, name):
        b = self.bars[name]
        if b[1] == 0 and b[3] == 0:
            b[2] += 1
            b[1] = b[0]

    def test(self, name, phase):
        """try_wait.parity for the phase index the caller means.  The parity answers right
        only while the barrier has completed phase - 1 or phase (or phase + 1 phases in
        all); a wait outside that window is reported."""
        done = self.bars[name][2]
        ok = (done & 1) != (phase & 1)
        if ok and done > phase + 1:
            self.issues.append(f"{name}: waiter of phase {phase} is {done - phase} phases behind")
        if ok and done < phase + 1:
            self.issues.append(f"{name}: wait for phase {phase} passed with {done} phases done")
        return ok

    def later(self, dt, fn):
        self.seq += 1
        self.events.append((self.t + dt, self.seq, fn))

    # MMAs: per issuing thread in order, random durations; commit arrives when the
    # thread's MMAs issued so far have completed
    def mma(self, thread, on_start, on_end):
        q = self.mma_q.setdefault(thread, [])
        q.append([None, on_start, on_end])
        if len(q) == 1:
            self._start_mma(thread)

    def _start_mma(self, thread):
        q = self.mma_q[thread]
        item = q[0]
        item[1](self.t)
        dur = self.rng.randint(1, 6)

        def done():
            item[2](self.t)
            q.pop(0)
            if q:
                self._start_mma(thread)
            for fn in list(self.commits.get(thread, [])):
                if fn[0] is item:
                    self.commits[thread].remove(fn)
                    fn[1]()
        self.later(dur, done)

    def commit(self, thread, name):
        q = self.mma_q.get(thread, [])
        if not q:
            self.arrive(name)
            return
        self.commits.setdefault(thread, []).append((q[-1], lambda: self.arrive(name)))

    def tma(self, name, nbytes, slot_key):
        self.arrive(name, tx=nbytes)
        self.loads_in_flight += 1
        t_issue = self.t

        def land():
            self.loads_in_flight -= 1
            self.log[("land",) + slot_key] = self.t
            self.log[("issue",) + slot_key] = t_issue
            self.complete_tx(name, nbytes)
        self.later(self.rng.randint(1, 25), land)

    # ---------------------------------------------------------------- the run
    def run(self, threads):
        self.commits = {}
        live = {name: gen for name, gen in threads.items()}
        waiting = {}                 # name -> condition (callable returning bool or None)
        for name in list(live):
            waiting[name] = None
        steps = 0
        while live:
            steps += 1
            if steps > 200000:
                raise Deadlock("no end")
            runnable = [n for n in live if waiting[n] is None or waiting[n][0]()]
            if runnable:
                name = self.rng.choice(runnable)
                w = waiting[name]
                value = w[1]() if w is not None else None
                waiting[name] = None
                try:
                    cond = live[name].send(value)
                except StopIteration:
                    del live[name]
                    del waiting[name]
                    continue
                waiting[name] = cond
                # advance time a little with every action
                self.t += 1
                self._fire()
                if self.abort_p and self.rng.random() < self.abort_p:
                    self._time_out_one(waiting)
                continue
            if self.events:
                self.t = max(self.t, min(e[0] for e in self.events))
                self._fire()
                continue
            # nothing can move: a bounded mbarrier wait runs out, else it is a deadlock
            if not self._time_out_one(waiting):
                raise Deadlock("blocked: " + ", ".join(f"{n}:{waiting[n][2]}" for n in live))
        if self.loads_in_flight:
            self.issues.append(f"{self.loads_in_flight} TMA loads in flight at the end")

    def _fire(self):
        due = sorted(e for e in self.events if e[0] <= self.t)
        self.events = [e for e in self.events if e[0] > self.t]
        for _, _, fn in due:
            fn()

    def _time_out_one(self, waiting):
        cands = [n for n, w in waiting.items() if w is not None and w[2].startswith("mbar ")
                 and not w[0]()]
        if not cands:
            return False
        name = self.rng.choice(cands)
        self.timeouts += 1
        self.abort = True
        waiting[name] = (lambda: True, lambda: False, "timed out")
        return True

    # conditions yielded by the threads: (ready, value, label)
    def mbar_wait(self, name, phase):
        """The kernel's bounded wait: True when the phase completed; False once aborted."""
        def ready():
            return self.test(name, phase) or self.abort
        return (ready, lambda: self.test(name, phase), f"mbar {name} phase {phase}")

    def drain_wait(self, name, phase):
        """The drain wait ignores the abort flag (it is bounded by time alone)."""
        return (lambda: self.test(name, phase), lambda: True, f"mbar-drain {name} phase {phase}")

    def nb_arrive(self, bid):
        """bar.arrive: counted in the current generation, no wait."""
        b = self.nb[bid]
        b[1] += 1
        if b[1] == b[0]:
            b[1] = 0
            b[2] += 1
        return (lambda: True, lambda: None, f"nbar-arrive {bid}")

    def nb_sync(self, bid):
        b = self.nb[bid]
        gen = b[2]
        b[1] += 1
        if b[1] == b[0]:
            b[1] = 0
            b[2] += 1
        return (lambda: self.nb[bid][2] > gen, lambda: None, f"nbar {bid} gen {gen}")


def run_model(n_iter, dense_first, seed, abort_p=0.0, rescale_p=0.2, softmax_arrive_only=False):
    n = n_iter
    pre = 0
    if dense_first:
        pre = min(2, n)
    sim = Sim(n, pre, seed, abort_p)
    for name in ("Q", "Done"):
        sim.bar(name, 1 if name == "Q" else 2)
    for s in range(2):
        sim.bar(f"SFull{s}", 1)
        sim.bar(f"PVDone{s}", 1)
    for x in range(SLOTS):
        sim.bar(f"full{x}", 1)
        sim.bar(f"empty{x}", 1)
    sim.nb = {"prod": [2, 0, 0], "P0": [5, 0, 0], "P1": [5, 0, 0], "epi": [8, 0, 0]}
    n_pos = 2 * n + 1
    stop = {}
    L = sim.log

    def load(q):
        is_k, l = ring_tile(q)
        sim.tma(f"full{q % SLOTS}", 1, (q,))

    # set-up thread: Q, then the first dense K tiles (positions below pre)
    sim.tma("Q", 1, ("Q",))
    for q in range(pre):
        load(q)

    def producer(kside):
        q = pre if kside else 2
        while q < n_pos:
            is_k, l = ring_tile(q)
            if is_k != kside or (is_k and l >= n):
                q += 1
                continue
            rnd = q // SLOTS
            if rnd > 0:
                ok = yield sim.mbar_wait(f"empty{q % SLOTS}", rnd - 1)
                if not ok:
                    break
                # the slot's previous load must have been read by its MMA
                prev = q - SLOTS
                if not sim.abort and ("read", prev) not in L:
                    sim.issues.append(f"slot of position {prev} refilled before its MMA read it")
            load(q)
            q += 1
        stop["K" if kside else "V"] = q
        yield sim.nb_sync("prod")
        if kside:
            qk, qv = stop["K"], stop["V"]

            def issued(x):
                if x >= n_pos:
                    return False
                is_k, lx = ring_tile(x)
                if is_k and lx >= n:
                    return False
                return x < (qk if is_k else qv)
            for x in range(max(0, min(qk, qv) - 2 * SLOTS), max(qk, qv)):
                if issued(x) and not issued(x + SLOTS):
                    yield sim.drain_wait(f"full{x % SLOTS}", x // SLOTS)

    def s_thread():
        ok = yield sim.mbar_wait("Q", 0)
        l = 0
        while ok and l < n:
            s = l & 1
            q = pos_k(l)
            ok = yield sim.mbar_wait(f"full{q % SLOTS}", q // SLOTS)
            if ok and l >= 2:
                ok = yield sim.mbar_wait(f"PVDone{s}", (l >> 1) - 1)
            if not ok:
                break
            ll = l

            def st(t, ll=ll, q=q):
                L[("S_start", ll)] = t
                L.setdefault(("read", q), t)
            sim.mma("S", st, lambda t, ll=ll: L.__setitem__(("S_end", ll), t))
            sim.commit("S", f"SFull{s}")
            sim.commit("S", f"empty{q % SLOTS}")
            l += 1
        sim.commit("S", "Done")

    def pv_thread():
        ok = True
        for l in range(n):
            s = l & 1
            qv = pos_v(l)
            if ok:
                ok = yield sim.mbar_wait(f"full{qv % SLOTS}", qv // SLOTS)
            for wg in range(2):
                yield sim.nb_sync(f"P{wg}")
                if ok:
                    def st(t, l=l, wg=wg, qv=qv):
                        L[("PV_start", l, wg)] = t
                        L.setdefault(("read", qv), t)
                    sim.mma("PV", st, lambda t, l=l, wg=wg: L.__setitem__(("PV_end", l, wg), t))
            if ok:
                sim.commit("PV", f"PVDone{s}")
                sim.commit("PV", f"empty{qv % SLOTS}")
        sim.commit("PV", "Done")

    def softmax(wg, warp):
        ok = True
        for l in range(n):
            sb = l & 1
            r = yield sim.mbar_wait(f"SFull{sb}", l >> 1)
            ok = r and ok
            L[("S_read", l, wg, warp)] = sim.t
            if l > 0 and sim.rng.random() < rescale_p:
                r = yield sim.mbar_wait(f"PVDone{sb ^ 1}", (l - 1) >> 1)
                ok = r and ok
                L[("rescale", l, wg, warp)] = sim.t
            L[("P_write", l, wg, warp)] = sim.t
            yield (sim.nb_arrive if softmax_arrive_only else sim.nb_sync)(f"P{wg}")
        r = yield sim.mbar_wait("Done", 0)
        L[("epilogue", wg, warp)] = sim.t
        yield sim.nb_sync("epi")

    threads = {"K": producer(True), "V": producer(False), "S": s_thread(), "PV": pv_thread()}
    for wg in range(2):
        for warp in range(4):
            threads[f"sm{wg}{warp}"] = softmax(wg, warp)
    sim.run(threads)
    return sim


def check_order(sim):
    L, n = sim.log, sim.n
    bad = list(sim.issues)
    inf = float("inf")

    def get(*k):
        return L.get(k)
    pv_ends = [get("PV_end", m, w) for m in range(n) for w in range(2)]
    for l in range(n):
        s_end, s_start = get("S_end", l), get("S_start", l)
        if s_end is None or s_start is None:
            bad.append(f"S_{l} never ran")
            continue
        for wg in range(2):
            pv_start, pv_end = get("PV_start", l, wg), get("PV_end", l, wg)
            if pv_start is None or pv_end is None:
                bad.append(f"PV_{l} of warpgroup {wg} never ran")
                continue
            for warp in range(4):
                if get("S_read", l, wg, warp) < s_end:
                    bad.append(f"S_{l} read before written")
                if get("P_write", l, wg, warp) > pv_start:
                    bad.append(f"PV_{l} of warpgroup {wg} started before P_{l} was written")
                t = get("rescale", l, wg, warp)
                if t is not None and (t < (get("PV_end", l - 1, wg) or inf) or t > pv_start):
                    bad.append(f"O_{wg} rescaled at tile {l} outside its PVs")
            if pv_start < get("land", pos_v(l)):
                bad.append(f"PV_{l} read V_{l} before it landed")
        if l + 2 < n and get("S_start", l + 2) is not None:
            for wg in range(2):
                if get("S_start", l + 2) < (get("PV_end", l, wg) or inf):
                    bad.append(f"S_{l + 2} overwrote P_{l} before its PV read it")
        if s_start < get("land", pos_k(l)):
            bad.append(f"S_{l} read K_{l} before it landed")
    last_pv = max((t for t in pv_ends if t is not None), default=0)
    for wg in range(2):
        for warp in range(4):
            if get("epilogue", wg, warp) < last_pv or None in pv_ends:
                bad.append("epilogue read O before the last PV")
    return bad


@pytest.mark.parametrize("n_iter", [1, 2, 3, 5, 8, 13])
def test_protocol_orders_and_ends(n_iter):
    for seed in range(40):
        sim = run_model(n_iter, dense_first=seed % 2 == 0, seed=1000 * n_iter + seed)
        assert sim.timeouts == 0, "a wait had to run out without an injected abort"
        assert check_order(sim) == []


@pytest.mark.parametrize("n_iter", [1, 2, 5, 9])
def test_protocol_ends_after_aborts(n_iter):
    """With waits running out at random, every named barrier still completes (both sides
    run all their iterations), the producers' drain still sees every load land, and the
    run ends."""
    aborted = 0
    for seed in range(60):
        sim = run_model(n_iter, dense_first=seed % 2 == 1, seed=7 + 31 * seed + n_iter,
                        abort_p=0.02)
        assert not any("in flight" in i for i in sim.issues), sim.issues
        aborted += sim.timeouts > 0
    assert aborted > 10          # the abort path was taken on many of the schedules


def test_model_finds_a_missing_wait(monkeypatch):
    """The model is not vacuous: an S thread that does not wait for the PV-done barrier
    (the barrier's test always passing) lets S_{l+2} overwrite P_l under a running PV."""
    orig = Sim.test

    def test(self, name, phase):
        return True if name.startswith("PVDone") else orig(self, name, phase)
    monkeypatch.setattr(Sim, "test", test)
    found = any(any("overwrote" in b for b in check_order(run_model(6, False, seed)))
                for seed in range(40))
    assert found


def test_model_finds_mixed_barrier_generations():
    """Why both sides wait on the P hand-off barrier: with the softmax warps only arriving
    (bar.arrive), an aborted run lets them run ahead, a generation completes with arrivals
    of two different tiles, and the PV thread's wait can be left without partners."""
    stuck = 0
    for seed in range(200):
        try:
            run_model(5, False, seed, abort_p=0.05, softmax_arrive_only=True)
        except Deadlock:
            stuck += 1
    assert stuck > 0
