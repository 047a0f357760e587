"""A model of the synchronisation of the gated-delta kernels (csrc/sfa_gdn.cu), run on the CPU.

Each kernel's warps coordinate through mbarriers and the completion order of the tensor
core and the TMA engine.  This model replays the waits the MMA warp, the TMA warp (the
recurrence kernel's copies) and the element-wise warps perform, in the same order, with the asynchronous engines (MMAs completing in issue
order, copies landing and stores reading shared memory at random later times), all
interleaved at random.  It checks, at the moment a buffer or TMEM column is overwritten,
that every reader of the old contents has finished; that no mbarrier wait can alias a
parity two phases old; and that no interleaving deadlocks.  It is a model: a change to a
kernel's waits has to be mirrored here.  Planted omissions of single waits must be caught
(the model's own check).  The element-wise warps are one actor here, so waits among them
(the staged barrier) are outside the model.
"""
import random

import pytest


class _Fail(AssertionError):
    pass


def _check(cond, msg):
    if not cond:
        raise _Fail(msg)


class _Engines:
    """Tensor core (in-order completion), copy engine (loads land in any order) and the
    store engine (stores finish reading shared memory in order), for one CTA."""

    def __init__(self, rng, done):
        self.rng, self.done = rng, done
        self.tc, self.copies, self.stores = [], [], []
        self.completed = set()      # MMA groups done: (kind, index)
        self.landed = {}            # buffer -> what landed there
        self.store_read = -1

    def mma(self, kind, idx, bar):
        self.tc.append((kind, idx, bar))

    def load(self, buf, what, bar):
        self.landed.pop(buf, None)
        self.copies.append((buf, what, bar))

    def actor(self):
        while True:
            if self.tc and self.rng.random() < 0.5:
                kind, idx, bar = self.tc.pop(0)
                self.completed.add((kind, idx))
                if bar:
                    self.done[bar] += 1
            if self.copies and self.rng.random() < 0.3:
                buf, what, bar = self.copies.pop(self.rng.randrange(len(self.copies)))
                self.landed[buf] = what
                self.done[bar] += 1
            if self.stores and self.rng.random() < 0.3:
                self.store_read = max(self.store_read, self.stores.pop(0))
            yield


def _wait(done, bar, k, name, drop):
    if name in drop:
        return
    while True:
        d = done[bar]
        _check(d in (k, k + 1), f"parity alias: {bar} phase {k}, {d} completed")
        if d == k + 1:
            return
        yield


def _run(rng, engine, finite):
    live, idle = list(finite), 0
    while live:
        gen = rng.choice(live + [engine])
        try:
            next(gen)
            idle += 1
        except StopIteration:
            live.remove(gen)
            idle = 0
        if idle > 200000:
            raise _Fail("deadlock")


def model_main(per, T, upd, rng, drop=frozenset(), NQ=4):
    """gdn_kernel, one CTA (its CTAs never wait for one another): T frames of `per` tiles each,
    or per[n] tiles in frame n (the kernel rotates the tiles of a frame over the CTAs, so a
    CTA's count changes from frame to frame when they do not divide evenly)."""
    pers = [per] * T if isinstance(per, int) else list(per)
    assert len(pers) == T
    done = {k: 0 for k in ("q0", "q1", "q2", "q3", "m0", "m1", "d_done", "s_free", "o_done0", "o_done1",
                           "s_ready")}
    done.update({f"o_staged{x}": 0 for x in range(NQ)})
    done.update({"m_free0": 0, "m_free1": 0})
    eng = _Engines(rng, done)
    st = {"s_frame": 0, "d_read": -1, "staged": set(), "stored": set()}
    total = sum(pers)

    def wait(bar, k, name):
        return _wait(done, bar, k, name, drop)

    def mma_warp():
        def issue(kind, idx, n, bar):
            _check(not upd or st["s_frame"] == n, f"MMA of frame {n} reads the state of frame {st['s_frame']}")
            eng.mma(kind, idx, bar)

        it = 0
        for n in range(T):
            if upd or n == 0:
                yield from wait("s_ready", n, "s_ready")
            if upd:
                yield from wait(f"m{n & 1}", n >> 1, "m_full")
                _check(eng.landed.get(f"m{n & 1}") == n, f"product of frame {n} issued before M landed")
                _check(st["d_read"] >= n - 1, "M S overwrites an unread product")
                issue("d", n, n, "d_done")
                eng.mma("m_free", n, f"m_free{n & 1}")
            for _ in range(pers[n]):
                s, u = it % NQ, it & 1
                yield from wait(f"q{s}", it // NQ, "q_full")
                _check(eng.landed.get(f"q{s}") == it, f"O MMA of tile {it} before its Q landed")
                if it >= 2:
                    yield from wait(f"o_staged{(it - 2) % NQ}", (it - 2) // NQ, "o_free")
                _check(it < 2 or (it - 2) in st["staged"], f"O of tile {it} overwrites an unread O")
                issue("qs", it, n, f"o_done{u}")
                it += 1
            eng.mma("s_free", n, "s_free")

    def tma_warp():
        last_store = [-1]

        def load_q(t):
            s = t % NQ
            if t >= NQ:
                p = t - NQ
                _check(("qs", p) in eng.completed and p in st["stored"] and eng.store_read >= p,
                       f"Q buffer {s} reloaded for tile {t} while tile {p} still uses it")
            eng.load(f"q{s}", t, f"q{s}")

        def load_m(n):
            if n >= 2:
                _check(("d", n - 2) in eng.completed, f"M slot {n & 1} reloaded while its product runs")
            eng.load(f"m{n & 1}", n, f"m{n & 1}")

        def store(t):
            _check(t in st["staged"], f"O of tile {t} stored before it was staged")
            st["stored"].add(t)
            eng.stores.append(t)
            last_store[0] = t

        for t in range(min(NQ, total)):
            load_q(t)
        if upd:
            for n in range(min(2, T)):
                load_m(n)
        t = 0
        for n in range(T):
            if upd and n + 2 < T:
                yield from wait(f"m_free{n & 1}", n >> 1, "m_slot")
                load_m(n + 2)
            # the frame's stores wait for the next frame's product (not when a Q buffer is
            # refilled within the frame)
            if upd and n + 1 < T and pers[n] <= NQ:
                yield from wait(f"m_free{(n + 1) & 1}", (n + 1) >> 1, "store_after_product")
            for _ in range(pers[n]):
                yield from wait(f"o_staged{t % NQ}", t // NQ, "o_staged")
                store(t)
                if t + NQ < total:
                    if "store_read" not in drop:
                        while eng.store_read < last_store[0]:
                            yield
                    load_q(t + NQ)
                t += 1

    def epilogue():
        done["s_ready"] += 1
        it = [0]

        def stage_o():
            t = it[0]
            u = t & 1
            yield from wait(f"o_done{u}", t >> 1, "o_done")
            _check(("qs", t) in eng.completed and eng.landed.get(f"q{t % NQ}") == t,
                   f"O of tile {t} staged too early or over a reloaded Q buffer")
            st["staged"].add(t)
            done[f"o_staged{t % NQ}"] += 1
            it[0] += 1

        for n in range(T):
            # the frame's O products past its second wait for the first ones' TMEM buffers,
            # and the frame's MMAs end before the state is rewritten: stage those first
            early = max(pers[n] - 2, 0) if upd else pers[n]
            if upd:
                yield from wait("d_done", n, "d_done")
                _check(("d", n) in eng.completed, f"product of frame {n} read before it was done")
                st["d_read"] = n
            for _ in range(early):
                yield from stage_o()
            if upd:
                yield from wait("s_free", n, "s_free")
                _check(not any(x[0] in ("d", "qs") for x in eng.tc), f"state of frame {n} rewritten while read")
                st["s_frame"] = n + 1
                done["s_ready"] += 1
            for _ in range(pers[n] - early):
                yield from stage_o()

    _run(rng, eng.actor(), [mma_warp(), tma_warp(), epilogue()])


def model_prep(nt, rng, drop=frozenset(), S=3):
    """gdn_prep_kernel, one CTA: nt tiles of one frame through S stages."""
    done = {k: 0 for k in ("kv0", "kv1", "kv2", "sc0", "sc1", "sc2", "md0", "md1", "md2", "fin")}
    eng = _Engines(rng, done)
    scaled = set()

    def wait(bar, k, name):
        return _wait(done, bar, k, name, drop)

    def mma_warp():
        def load(t):
            if t >= S:
                _check(("mm", t - S) in eng.completed, f"stage {t % S} reloaded while its MMAs run")
            eng.load(f"kv{t % S}", t, f"kv{t % S}")

        for t in range(min(S, nt)):
            load(t)
        for i in range(nt):
            s = i % S
            yield from wait(f"sc{s}", i // S, "scaled")
            _check(i in scaled, f"MMA of tile {i} before its operands were scaled")
            eng.mma("mm", i, f"md{s}")
            if i >= 1 and i + 2 < nt:
                p = i - 1
                yield from wait(f"md{p % S}", p // S, "mma_done")
                load(i + 2)
        eng.mma("fin", 0, "fin")

    def epilogue():
        for i in range(nt):
            s = i % S
            yield from wait(f"kv{s}", i // S, "kv_full")
            _check(eng.landed.get(f"kv{s}") == i, f"tile {i} scaled before it landed")
            scaled.add(i)
            done[f"sc{s}"] += 1
        yield from wait("fin", 0, "fin")
        _check(all(("mm", i) in eng.completed for i in range(nt)), "products staged while MMAs run")

    _run(rng, eng.actor(), [mma_warp(), epilogue()])


# per-frame tile counts that change from frame to frame, as the rotating assignment gives
# them (13 tiles over 12 CTAs: a CTA takes two tiles in one frame of every 12; 8 tiles over
# 3 CTAs: 3, 3, 2, 3, 3, 2, ...), in denser patterns than those
ROTATED = [[1, 2, 1, 1, 2], [2, 1, 1, 2, 1], [3, 2, 2, 3, 2], [1, 1, 2, 1, 1, 1], [1, 1, 1, 1, 1, 1, 1, 2, 1]]
MAIN_CASES = ([(per, T, upd) for per in (1, 2, 3, 5) for T in (1, 2, 3, 5) for upd in (True, False)] +
              [(pers, len(pers), upd) for pers in ROTATED for upd in (True, False)])
PREP_CASES = [(nt,) for nt in (1, 2, 3, 4, 7, 13)]


@pytest.mark.parametrize("seed", range(8))
def test_main_kernel_protocol_has_no_race_or_deadlock(seed):
    rng = random.Random(seed)
    for case in MAIN_CASES:
        model_main(*case, rng)


@pytest.mark.parametrize("seed", range(8))
def test_prep_kernel_protocol_has_no_race_or_deadlock(seed):
    rng = random.Random(seed)
    for case in PREP_CASES:
        model_prep(*case, rng)


def _caught(fn, cases, dropped):
    for seed in range(30):
        rng = random.Random(seed)
        try:
            for case in cases:
                fn(*case, rng, drop=frozenset({dropped}))
        except _Fail:
            return True
    return False


@pytest.mark.parametrize("dropped", ["s_ready", "m_full", "q_full", "o_free", "o_staged", "m_slot", "store_read",
                                     "d_done", "s_free", "o_done"])
def test_model_catches_a_missing_wait_in_the_main_kernel(dropped):
    assert _caught(model_main, [(2, 4, True), (1, 3, True), (3, 3, False), ([1, 2, 1, 2], 4, True)],
                   dropped), dropped


@pytest.mark.parametrize("dropped", ["scaled", "mma_done", "kv_full", "fin"])
def test_model_catches_a_missing_wait_in_the_prep_kernel(dropped):
    assert _caught(model_prep, [(7,), (13,)], dropped), dropped
