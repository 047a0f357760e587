"""A model of the synchronisation of the gated-delta kernel (csrc/sfa_gdn.cu), run on the CPU.

The kernel's warps coordinate through mbarriers, a global arrival counter and the
completion order of the tensor core and the TMA engine.  This model replays the waits the
kernel's MMA warp and epilogue warps perform, in the same order, with the asynchronous
engines (MMAs completing in issue order, copies landing and stores reading shared memory
at random later times) and the head's G CTAs as separate actors, all interleaved at random.
It checks, at the moment a buffer or TMEM column is overwritten, that every reader of the
old contents has finished; that no mbarrier wait can alias a parity two phases old; and
that no interleaving deadlocks.  It is a model: a change to the kernel's waits has to be
mirrored here.  Planted omissions of single waits must be caught (the model's own check);
the epilogue's threads are one actor here, so waits among them (the staged barrier) are
outside the model.
"""
import itertools
import random

import pytest

class _Fail(AssertionError):
    pass


def _check(cond, msg):
    if not cond:
        raise _Fail(msg)


def run_model(n_tiles, G, T, upd, rng, drop=frozenset()):
    """One kernel launch for one (batch, head): G CTAs, T frames, n_tiles tiles per frame."""
    spread = upd and G > 1
    count = [0]

    class CTA:
        pass

    ctas = []
    for g in range(G):
        c = CTA()
        c.g, c.per = g, (n_tiles - g + G - 1) // G
        c.done = {k: 0 for k in ("full0", "full1", "ks", "o", "u_full", "o_free", "sacc", "s_ready", "sum",
                                 "staged")}
        c.slot = [None, None]      # tile whose Q, K, V a slot holds
        c.stage = [None, None]     # frame whose sums occupy a slot's K and V buffers
        c.use = {}
        c.tc = []                  # MMA groups in issue order: (kind, tile, frame, barrier)
        c.copies = []              # in flight: (barrier, what lands)
        c.landed = [None, None]    # tile whose copies have landed in a slot
        c.sum_landed = -1          # frame whose sum has landed
        c.stores = []
        c.store_read = -1
        c.s_frame = 0              # frame whose state the bf16 S buffer holds
        c.sacc_frame_read = -1     # last frame whose S_acc the epilogue has read out
        ctas.append(c)

    def use(c, t):
        return c.use.setdefault(t, set())

    def wait(c, bar, k, name):
        if name in drop:
            return
        while True:
            d = c.done[bar]
            _check(d in (k, k + 1), f"parity alias: CTA {c.g} {bar} phase {k}, {d} completed")
            if d == k + 1:
                return
            yield

    def tensor_core(c):
        while True:
            if c.tc and rng.random() < 0.5:
                kind, t, _, bar = c.tc.pop(0)
                use(c, t).add(kind)
                c.done[bar] += 1
            yield

    def copy_engine(c):
        while True:
            if c.copies and rng.random() < 0.3:
                bar, what = c.copies.pop(rng.randrange(len(c.copies)))
                if bar == "sum":
                    c.sum_landed = what
                else:
                    c.landed[int(bar[-1])] = what
                c.done[bar] += 1
            if c.stores and rng.random() < 0.3:
                c.store_read = max(c.store_read, c.stores.pop(0))
            yield

    def mma_warp(c):
        total, per = c.per * T, c.per
        last_store = [-1]

        def load(t):
            s = t & 1
            prev = c.slot[s]
            if prev is not None:
                need = {"qs"} | ({"ks", "sacc", "u"} if upd else set())
                _check(need <= use(c, prev) and c.store_read >= prev,
                       f"slot {s} reloaded for tile {t} while tile {prev} still uses it")
            _check(c.stage[s] is None, f"slot {s} reloaded while it holds the sums of frame {c.stage[s]}")
            c.slot[s] = t
            c.landed[s] = None
            c.copies.append((f"full{s}", t))

        def store(t):
            _check("ostaged" in use(c, t) and c.slot[t & 1] == t, f"O of tile {t} stored before it was staged")
            c.stores.append(t)
            last_store[0] = t

        def issue(kind, t, n, bar):
            _check(not upd or c.s_frame == n, f"MMA of frame {n} reads the state of frame {c.s_frame}")
            c.tc.append((kind, t, n, bar))

        if total:
            load(0)
        for it in range(total):
            n, ii = divmod(it, per)
            s = it & 1
            if ii == 0 and (upd or n == 0):
                yield from wait(c, "s_ready", n, "s_ready")
            yield from wait(c, f"full{s}", it >> 1, "full")
            _check(c.slot[s] == it and c.landed[s] == it, f"MMA on tile {it} before its copies landed")
            if upd:
                _check(it == 0 or "u" in use(c, it - 1), f"KS of tile {it} overwrites an unread KS")
                issue("ks", it, n, "ks")
            if it > 0 and ii != 0:
                yield from wait(c, "o_free", it - 1, "o_free_prev")
                store(it - 1)
            _check(it == 0 or "oread" in use(c, it - 1), f"O of tile {it} overwrites an unread O")
            issue("qs", it, n, "o")
            if it + 1 < total:
                if upd and it > 0:
                    yield from wait(c, "sacc", it - 1, "sacc_prev")
                if "store_read" not in drop:
                    while c.store_read < last_store[0]:
                        yield
                load(it + 1)
            if upd:
                yield from wait(c, "u_full", it, "u_full")
                _check(ii > 0 or c.sacc_frame_read >= n - 1, f"S_acc of frame {n} restarted before it was read")
                issue("sacc", it, n, "sacc")
            if ii + 1 == per:
                yield from wait(c, "o_free", it, "o_free_last")
                store(it)

    def epilogue(c):
        c.done["s_ready"] += 1
        it = 0
        for n in range(T):
            for _ in range(c.per):
                s = it & 1
                if upd:
                    yield from wait(c, "ks", it, "ks_epi")
                    yield from wait(c, f"full{s}", it >> 1, "full")
                    _check("ks" in use(c, it) and c.landed[s] == it, f"U of tile {it} formed too early")
                    use(c, it).add("u")
                    c.done["u_full"] += 1
                yield from wait(c, "o", it, "o_epi")
                _check("qs" in use(c, it) and c.slot[s] == it, f"O of tile {it} staged over a busy Q buffer")
                use(c, it).update({"oread", "ostaged"})
                c.done["o_free"] += 1
                it += 1
            if not upd:
                continue
            yield from wait(c, "sacc", it - 1, "sacc_end")
            _check(all(x[2] > n for x in c.tc) and "sacc" in use(c, it - 1),
                   f"frame {n} ends with its MMAs in flight")
            s = (it - 1) & 1
            c.sacc_frame_read = n
            if spread:
                _check(c.slot[s] == it - 1, "sums staged over a reloaded slot")
                c.stage[s] = n
                c.done["staged"] += 1
                yield from wait(c, "staged", n, "staged")
                count[0] += 1
                while count[0] < G * (n + 1):
                    yield
                c.copies.append(("sum", n))
                yield from wait(c, "sum", n, "sum")
                _check(c.sum_landed == n, f"state of frame {n} updated before the head's sum landed")
                c.stage[s] = None
            c.s_frame = n + 1
            c.done["s_ready"] += 1

    finite, engines = [], []
    for c in ctas:
        finite += [mma_warp(c), epilogue(c)]
        engines += [tensor_core(c), copy_engine(c)]
    live, idle = list(finite), 0
    while live:
        gen = rng.choice(live + engines)
        try:
            next(gen)
            idle += 1
        except StopIteration:
            live.remove(gen)
            idle = 0
        if idle > 200000:
            raise _Fail("deadlock")


CASES = [(n, G, T, upd) for n, G, T, upd in itertools.product([1, 2, 3, 5, 13], [1, 2, 3, 7], [1, 2, 4], [True, False])
         if G <= n]


@pytest.mark.parametrize("seed", range(6))
def test_protocol_has_no_race_or_deadlock(seed):
    rng = random.Random(seed)
    for case in CASES:
        run_model(*case, rng)


@pytest.mark.parametrize("dropped", ["s_ready", "full", "sacc_prev", "store_read", "o_free_prev", "sum", "sacc_end",
                                     "u_full"])
def test_model_catches_a_missing_wait(dropped):
    caught = False
    for seed in range(20):
        rng = random.Random(seed)
        try:
            for case in [(13, 7, 3, True), (3, 1, 4, True), (5, 2, 3, True), (2, 1, 3, False)]:
                run_model(*case, rng, drop=frozenset({dropped}))
        except _Fail:
            caught = True
            break
    assert caught, f"dropping the {dropped} wait went unnoticed"
