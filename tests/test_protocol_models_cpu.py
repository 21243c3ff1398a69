"""Models of two kernels' mbarrier protocols, run as random schedules on the CPU.

An mbarrier wait names only the parity of the phase it wants, so a waiter
that is two or more completions behind (or ahead) reads the wrong phase.  Each
model below re-states one kernel's roles as Python generators with the same
barriers, counts and phase arithmetic, runs them under random interleavings
(TMA loads land in any order; tcgen05 MMAs and commits complete in issue
order), and asserts at every poll that the barrier is within one phase of the
one the waiter wants, and that the schedule always makes progress.

- attn_dense_kernel (csrc/attn_dense.cu): two 128-row tiles per work item, a
  K/V slot ring released by both tiles' MMA issuers, per-half score, P and
  P.V barriers, the rescale wait on the previous half's P.V.
- colmass_tc_kernel (csrc/attn_tc.cu): a q-tile ring, three TMEM score
  buffers (tile u in buffer u % 3), two reducer groups taking alternate tiles,
  and the keys barrier used only by work items that have row tiles.
- attn_pp_kernel (csrc/attn_tc.cu): K and V rings, two score issuers and a
  P.V issuer, per-half and per-parity score barriers, the P buffers' reuse
  wait, the rescale wait on the other group's P.V (four barriers by t mod 4),
  the named-barrier hand-off of the running reference between the two row
  groups, and the q barrier used only by work items that have column tiles.
- attn_tc_kernel (csrc/attn_tc.cu, the fixed-mass passes): one MMA thread
  alternating S(t) and P(t-1).V over two score buffers, and its q barrier
  used only by work items that have column tiles.
- tc_gemm_kernel (csrc/gemm_tc.cu): the A/B stage ring filled by the
  gathering warps and TMA, the MMA thread, and the two TMEM accumulators the
  epilogue drains while the next tile fills.

Each model also runs with a planted protocol mistake and must then fail:
that shows the checks can see the class of error they are there for.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Stuck(Exception):
    pass


def wait(bars, name, k):
    """Wait for the completion of phase k (k < 0: a fresh barrier's 'previous
    phase', always complete).  A poll checks k <= completed <= k + 1."""
    while True:
        b = bars[name]
        if k >= 0:
            assert k <= b.done <= k + 1, (name, k, b.done)
        if b.done > k:
            return
        yield None


def run_schedule(bars, threads, loads, pipe, rnd, idle_limit=20000):
    """Interleave the roles at random with the two asynchronous engines: TMA
    loads (complete in any order) and the MMA pipe (in issue order)."""
    alive, idle = list(threads), 0
    while alive:
        moved = False
        if loads and rnd.random() < 0.5:
            bars[loads.pop(rnd.randrange(len(loads)))].arrive()
            moved = True
        if pipe and rnd.random() < 0.5:
            kind, name = pipe.pop(0)
            if kind == "commit":
                bars[name].arrive()
            moved = True
        th = rnd.choice(alive)
        try:
            step = next(th)
            idle = 0 if (step is not None or moved) else idle + 1
        except StopIteration:
            alive.remove(th)
            idle = 0
        if idle > idle_limit and not loads and not pipe:
            raise Stuck()


# --------------------------------------------------------------- attn_dense_kernel
ROWS, COLS = 128, 128


def dn_tiles(S, p, x):
    first = p * 2 * ROWS + x * ROWS
    if first >= S:
        return 0
    return (min(S, first + ROWS) - 1 + COLS) // COLS


def dense_cta(S, H, grid, blk, stages, rnd, plant=None):
    pairs = (S + 2 * ROWS - 1) // (2 * ROWS)
    total = pairs * H
    items = list(range(blk, total, grid))
    item_p = lambda it: pairs - 1 - it % pairs
    B = {}
    for s in range(stages):
        B[("kv_full", s)] = Bar(1)
        B[("kv_empty", s)] = Bar(1 if plant == "kv_empty_count" else 2)
    for i in range(4):
        B[("s_full", i)] = Bar(1)
        B[("p_full", i)] = Bar(1)  # the 128 row threads move together in the model
    for x in range(2):
        for n in ("pv_done", "acc_full", "n_free", "q_full", "q_empty"):
            B[(n, x)] = Bar(1)
    B["fin"] = Bar(2)
    loads, pipe = [], []

    def tma():
        seq = 0
        for item in items:
            p = item_p(item)
            for _t in range(max(dn_tiles(S, p, 0), dn_tiles(S, p, 1))):
                for _kv in range(2):
                    yield from wait(B, ("kv_empty", seq % stages), seq // stages - 1)
                    loads.append(("kv_full", seq % stages))
                    seq += 1

    def issuer(x):
        seq = u = 0
        slot, phase = (lambda s: s % stages), (lambda s: s // stages)

        def skip(s):
            yield from wait(B, ("kv_full", slot(s)), phase(s))
            B[("kv_empty", slot(s))].arrive()

        for item_no, item in enumerate(items):
            p = item_p(item)
            my = dn_tiles(S, p, x)
            nt = max(dn_tiles(S, p, 0), dn_tiles(S, p, 1))
            yield from wait(B, ("q_full", x), item_no)
            if my == 0:
                pipe.append(("commit", ("q_empty", x)))
            base = seq
            if nt > 0:
                if my > 0:
                    yield from wait(B, ("kv_full", slot(base)), phase(base))
                    for hf in range(2):
                        pipe.extend([("mma", None), ("commit", ("s_full", 2 * x + hf))])
                    if my == 1:
                        pipe.append(("commit", ("q_empty", x)))
                    pipe.append(("commit", ("kv_empty", slot(base))))
                else:
                    yield from skip(base)
            for t in range(nt):
                vs, ks = base + 2 * t + 1, base + 2 * t + 2
                if t >= my:
                    yield from skip(vs)
                    if t + 1 < nt:
                        yield from skip(ks)
                    continue
                yield from wait(B, ("kv_full", slot(vs)), phase(vs))
                for hf in range(2):
                    if t == 0 and hf == 0 and item_no > 0:
                        yield from wait(B, ("n_free", x), item_no - 1)
                    yield from wait(B, ("p_full", 2 * x + hf), u >> 1)
                    pipe.extend([("mma", None), ("commit", ("pv_done", x))])
                    if t == my - 1 and hf == 1:
                        pipe.append(("commit", ("acc_full", x)))
                    if t + 1 < my:
                        if hf == 0:
                            yield from wait(B, ("kv_full", slot(ks)), phase(ks))
                        pipe.extend([("mma", None), ("commit", ("s_full", 2 * x + hf))])
                        if t + 1 == my - 1 and hf == 1:
                            pipe.append(("commit", ("q_empty", x)))
                    u += 1
                pipe.append(("commit", ("kv_empty", slot(vs))))
                if t + 1 < nt:
                    if t + 1 < my:
                        pipe.append(("commit", ("kv_empty", slot(ks))))
                    else:
                        yield from skip(ks)
            if my == 0:
                if item_no > 0:
                    yield from wait(B, ("n_free", x), item_no - 1)
                pipe.append(("commit", ("acc_full", x)))
            seq = base + 2 * nt
        pipe.append(("commit", "fin"))
        yield from wait(B, "fin", 0)

    def queries():
        if items:
            for x in range(2):
                B[("q_full", x)].arrive()
        for item_no in range(len(items) - 1):
            for x in range(2):
                yield from wait(B, ("q_empty", x), item_no)
                B[("q_full", x)].arrive()

    def rows(x):
        u = 0
        for item_no, item in enumerate(items):
            for t in range(dn_tiles(S, item_p(item), x)):
                for hf in range(2):
                    yield from wait(B, ("s_full", 2 * x + hf), u >> 1)
                    if (t > 0 or hf > 0) and rnd.random() < 0.3:  # the running maximum rose
                        k = u if plant == "pv_phase" else u - 1
                        yield from wait(B, ("pv_done", x), k)
                    for _ in range(rnd.randint(0, 3)):
                        yield None
                    B[("p_full", 2 * x + hf)].arrive()
                    u += 1
            yield from wait(B, ("acc_full", x), item_no)
            B[("n_free", x)].arrive()

    threads = [tma(), issuer(0), issuer(1), queries(), rows(0), rows(1)]
    run_schedule(B, threads, loads, pipe, rnd)


DENSE_SHAPES = [(256, 2, 4), (300, 2, 3), (40, 1, 1), (1000, 3, 5), (4096, 2, 7), (129, 2, 1), (513, 2, 148)]


@pytest.mark.parametrize("S,H,grid", DENSE_SHAPES)
def test_dense_protocol_phases_and_progress(S, H, grid):
    pairs = (S + 2 * ROWS - 1) // (2 * ROWS)
    for stages in (5, 10):
        for seed in range(3):
            rnd = random.Random(seed * 1000 + S)
            for blk in range(min(grid, pairs * H)):
                dense_cta(S, H, grid, blk, stages, rnd)


@pytest.mark.parametrize("plant", ["pv_phase", "kv_empty_count"])
def test_dense_protocol_model_catches_planted_mistakes(plant):
    caught = 0
    for seed in range(5):
        try:
            dense_cta(1000, 1, 1, 0, 5, random.Random(seed), plant=plant)
        except (AssertionError, Stuck):
            caught += 1
    assert caught > 0


# --------------------------------------------------------------- colmass_tc_kernel
def colmass_cta(nts, stages, nbuf, rnd, keys_every_item=False):
    """nts: row tiles of each of the CTA's work items (0: no row reaches the
    item's columns).  keys_every_item models a keys barrier completed by every
    item, with or without row tiles."""
    B = {}
    for s in range(stages):
        B[("full", s)] = Bar(1)
        B[("empty", s)] = Bar(2)  # the MMA commit + the tile's reducer group
    for b in range(nbuf):
        B[("s_full", b)] = Bar(1)
        B[("s_empty", b)] = Bar(1)
    B["a_ready"] = Bar(2)  # both reducer groups
    B["pair"] = Bar(2)  # the named barrier between the groups at an item's end
    loads, pipe = [], []

    def loader():
        fills = [0] * stages
        u = 0
        for nt in nts:
            for _t in range(nt):
                st = u % stages
                yield from wait(B, ("empty", st), fills[st] - 1)
                loads.append(("full", st))
                fills[st] += 1
                u += 1

    def mma():
        uses = [0] * stages
        u = ready_no = 0
        for item_no, nt in enumerate(nts):
            if keys_every_item:
                yield from wait(B, "a_ready", item_no)
            elif nt > 0:
                yield from wait(B, "a_ready", ready_no)
                ready_no += 1
            for _ in range(rnd.randint(0, 30)):  # a late MMA thread
                yield None
            for _t in range(nt):
                st = u % stages
                yield from wait(B, ("full", st), uses[st])
                uses[st] += 1
                if u >= nbuf:
                    yield from wait(B, ("s_empty", u % nbuf), u // nbuf - 1)
                pipe.extend([("mma", None), ("commit", ("s_full", u % nbuf)), ("commit", ("empty", st))])
                u += 1

    def reducers(grp):
        uses = [0] * stages
        u = gen = 0
        for nt in nts:
            if keys_every_item or nt > 0:
                B["a_ready"].arrive()
            for _t in range(nt):
                st = u % stages
                k = uses[st]
                uses[st] += 1
                if u % 2 == grp:
                    yield from wait(B, ("full", st), k)
                    yield from wait(B, ("s_full", u % nbuf), u // nbuf)
                    for _ in range(rnd.randint(0, 3)):
                        yield None
                    B[("s_empty", u % nbuf)].arrive()
                    for _ in range(rnd.randint(0, 3)):
                        yield None
                    B[("empty", st)].arrive()
                u += 1
            B["pair"].arrive()
            gen += 1
            yield from wait(B, "pair", gen - 1)

    run_schedule(B, [loader(), mma(), reducers(0), reducers(1)], loads, pipe, rnd, idle_limit=5000)


def _random_items(rnd):
    return [rnd.choice([0, 0, 1, 2, 3, 5]) for _ in range(rnd.randint(1, 8))]


def test_colmass_protocol_phases_and_progress():
    for seed in range(200):
        rnd = random.Random(seed)
        colmass_cta(_random_items(rnd), 4, 3, rnd)


def test_colmass_protocol_model_catches_a_keys_barrier_on_empty_items():
    caught = 0
    for seed in range(200):
        rnd = random.Random(seed)
        try:
            colmass_cta(_random_items(rnd), 4, 3, rnd, keys_every_item=True)
        except (AssertionError, Stuck):
            caught += 1
    assert caught > 0


# --------------------------------------------------------------- attn_pp_kernel
class NamedHandoff:
    """bar.arrive by the giving warp, bar.sync by the taking warp, one barrier
    id reused for every hand-off: a second give before the take would count
    towards the same barrier instance, so at most one may be outstanding."""

    def __init__(self):
        self.given = 0
        self.taken = 0

    def give(self):
        assert self.given == self.taken, "a second give before the take"
        self.given += 1

    def take(self):
        while self.given == self.taken:
            yield None
        self.taken += 1


def pp_cta(nts, stages, rnd, plant=None):
    """nts: column tiles of each of the CTA's work items (0: no selected column
    at or before the item's rows).  Row groups take alternate tiles by a
    block-wide counter u; both groups load the item's q and N halves, hand
    the running reference to each other per tile, and meet at the item's end."""
    B = {}
    for s in range(stages):
        B[("k_full", s)] = Bar(1)
        B[("k_empty", s)] = Bar(2)  # both score halves
        B[("v_full", s)] = Bar(1)
        B[("v_empty", s)] = Bar(1)
    for i in range(4):
        B[("s_full", i)] = Bar(1)
        B[("pv_done4", i)] = Bar(1)
    for i in range(2):
        B[("s_empty", i)] = Bar(1)  # the tile's group
        B[("p_full", i)] = Bar(1)
        B[("pv_done", i)] = Bar(1)
    B["q_ready"] = Bar(2)  # both groups
    B["end"] = Bar(2)
    hand = [NamedHandoff(), NamedHandoff()]  # hand[g]: group g gives to the other
    loads, pipe = [], []

    def loader():
        ks = vs = 0
        kfill = [0] * stages
        vfill = [0] * stages
        for nt in nts:
            for _t in range(nt):
                yield from wait(B, ("k_empty", ks), kfill[ks] - 1)
                loads.append(("k_full", ks))
                kfill[ks] += 1
                ks = (ks + 1) % stages
                yield from wait(B, ("v_empty", vs), vfill[vs] - 1)
                loads.append(("v_full", vs))
                vfill[vs] += 1
                vs = (vs + 1) % stages

    def s_half(half):
        u = item_no = 0
        for nt in nts:
            if nt == 0:
                continue
            yield from wait(B, "q_ready", item_no)
            item_no += 1
            for _t in range(nt):
                ks = u % stages
                yield from wait(B, ("k_full", ks), u // stages)
                if u > 0:
                    yield from wait(B, ("s_empty", half), u - 1)
                pipe.extend([("mma", None), ("commit", ("s_full", 2 * half + (u & 1))), ("commit", ("k_empty", ks))])
                u += 1

    def pv():
        u = 0
        for nt in nts:
            for _t in range(nt):
                yield from wait(B, ("p_full", u & 1), u >> 1)
                yield from wait(B, ("v_full", u % stages), u // stages)
                pipe.extend([("mma", None), ("commit", ("v_empty", u % stages)), ("commit", ("pv_done", u & 1)),
                             ("commit", ("pv_done4", u & 3))])
                u += 1

    def rows(grp):
        u = 0
        end_gen = 0
        for nt in nts:
            if nt > 0:
                B["q_ready"].arrive()
            for t in range(nt):
                b = u & 1
                if b != grp:
                    u += 1
                    continue
                yield from wait(B, ("s_full", b), u >> 1)
                B[("s_empty", 0)].arrive()
                if t > 0:
                    yield from hand[grp ^ 1].take()
                if t + 1 < nt:
                    hand[grp].give()
                if u >= 2:
                    yield from wait(B, ("pv_done", b), (u - 2) >> 1)
                if t > 0 and rnd.random() < 0.3:  # the reference rose: N waits for P(t-1).V
                    k = (u - 1) >> 2
                    if plant == "pv_done4_phase":
                        k += 1
                    yield from wait(B, ("pv_done4", (u - 1) & 3), k)
                for _ in range(rnd.randint(0, 3)):
                    yield None
                yield from wait(B, ("s_full", 2 + b), u >> 1)
                B[("s_empty", 1)].arrive()
                B[("p_full", b)].arrive()
                u += 1
            if nt > 0:
                yield from wait(B, ("pv_done4", (u - 1) & 3), (u - 1) >> 2)
            for _sync in range(2):
                B["end"].arrive()
                end_gen += 1
                yield from wait(B, "end", end_gen - 1)

    threads = [loader(), s_half(0), s_half(1), pv(), rows(0), rows(1)]
    run_schedule(B, threads, loads, pipe, rnd, idle_limit=5000)


def _pp_items(rnd):
    return [rnd.choice([0, 1, 1, 2, 3, 4, 5, 7]) for _ in range(rnd.randint(1, 7))]


def test_pp_protocol_phases_and_progress():
    for seed in range(300):
        rnd = random.Random(seed)
        pp_cta(_pp_items(rnd), 3, rnd)


def test_pp_protocol_model_catches_a_planted_phase():
    caught = 0
    for seed in range(100):
        rnd = random.Random(seed)
        try:
            pp_cta(_pp_items(rnd), 3, rnd, plant="pv_done4_phase")
        except (AssertionError, Stuck):
            caught += 1
    assert caught > 0


# --------------------------------------------------------------- tc_gemm_kernel
def gemm_cta(n_tiles, k_steps, stages, rnd, plant=None):
    """The persistent projection: per tile, k_steps stages of A rows (gathered
    by the producer warps, arriving when their copies land) and a B tile (TMA),
    an MMA thread consuming them in order into one of two TMEM accumulators,
    and the epilogue warps draining an accumulator while the next fills."""
    B = {}
    for s in range(stages):
        B[("full", s)] = Bar(2)  # the producers' arrival (cp.async landed) + the TMA's bytes
        B[("empty", s)] = Bar(1)
    for b in range(2):
        B[("acc_full", b)] = Bar(1)
        B[("acc_empty", b)] = Bar(1)  # the epilogue threads
    loads, pipe = [], []
    total = n_tiles * k_steps

    def producers():
        for i in range(total):
            st = i % stages
            yield from wait(B, ("empty", st), i // stages - 1)
            loads.append(("full", st))  # the gathered rows land

    def tma():
        for i in range(total):
            st = i % stages
            yield from wait(B, ("empty", st), i // stages - 1)
            loads.append(("full", st))

    def mma():
        i = 0
        for it in range(n_tiles):
            buf = it & 1
            k = it >> 1
            if plant == "acc_phase":
                k += 1
            yield from wait(B, ("acc_empty", buf), k - 1)
            for _k in range(k_steps):
                yield from wait(B, ("full", i % stages), i // stages)
                pipe.extend([("mma", None), ("commit", ("empty", i % stages))])
                i += 1
            pipe.append(("commit", ("acc_full", buf)))

    def epilogue():
        for it in range(n_tiles):
            buf = it & 1
            yield from wait(B, ("acc_full", buf), it >> 1)
            for _ in range(rnd.randint(0, 5)):
                yield None
            B[("acc_empty", buf)].arrive()

    run_schedule(B, [producers(), tma(), mma(), epilogue()], loads, pipe, rnd, idle_limit=5000)


def test_gemm_protocol_phases_and_progress():
    for seed in range(100):
        rnd = random.Random(seed)
        gemm_cta(rnd.randint(1, 7), rnd.randint(1, 9), 4, rnd)


def test_gemm_protocol_model_catches_a_planted_phase():
    caught = 0
    for seed in range(30):
        rnd = random.Random(seed)
        try:
            gemm_cta(5, 3, 4, rnd, plant="acc_phase")
        except (AssertionError, Stuck):
            caught += 1
    assert caught > 0


# --------------------------------------------------------------- attn_tc_kernel
def tc_cta(nts, stages, rnd, q_every_item=False):
    """The column-split update kernel of the fixed-mass passes: one MMA thread
    issues S(t) into score buffer t & 1, then P(t-1).V; all row threads take
    every tile.  q_every_item models a q barrier completed by every item,
    with or without column tiles."""
    B = {}
    for s in range(stages):
        B[("kv_full", s)] = Bar(1)
        B[("kv_empty", s)] = Bar(1)
    for i in range(2):
        B[("s_full", i)] = Bar(1)
        B[("p_full", i)] = Bar(1)  # the row threads move together in the model
        B[("pv_done", i)] = Bar(1)
    B["q_ready"] = Bar(1)
    loads, pipe = [], []

    def loader():
        fills = [0] * stages
        u = 0
        for nt in nts:
            for _t in range(nt):
                st = u % stages
                yield from wait(B, ("kv_empty", st), fills[st] - 1)
                loads.append(("kv_full", st))
                fills[st] += 1
                u += 1

    def mma():
        u = item_no = 0
        for nt in nts:
            if not q_every_item and nt == 0:
                continue
            yield from wait(B, "q_ready", item_no)
            item_no += 1
            for _ in range(rnd.randint(0, 30)):  # a late MMA thread
                yield None
            prev_stage = -1
            for t in range(nt + 1):
                if t < nt:
                    yield from wait(B, ("kv_full", u % stages), u // stages)
                    pipe.extend([("mma", None), ("commit", ("s_full", u & 1))])
                if t > 0:
                    up = u - 1
                    yield from wait(B, ("p_full", up & 1), up >> 1)
                    pipe.extend([("mma", None), ("commit", ("kv_empty", prev_stage)),
                                 ("commit", ("pv_done", up & 1))])
                if t < nt:
                    prev_stage = u % stages
                    u += 1

    def rows():
        u = 0
        for nt in nts:
            if q_every_item or nt > 0:
                B["q_ready"].arrive()
            for t in range(nt):
                yield from wait(B, ("s_full", u & 1), u >> 1)
                if t > 0 and rnd.random() < 0.3:  # the reference rose: N waits for P(t-1).V
                    yield from wait(B, ("pv_done", (u - 1) & 1), (u - 1) >> 1)
                for _ in range(rnd.randint(0, 3)):
                    yield None
                B[("p_full", u & 1)].arrive()
                u += 1
            if nt > 0:
                yield from wait(B, ("pv_done", (u - 1) & 1), (u - 1) >> 1)

    run_schedule(B, [loader(), mma(), rows()], loads, pipe, rnd, idle_limit=5000)


def test_tc_protocol_phases_and_progress():
    for seed in range(300):
        rnd = random.Random(seed)
        tc_cta(_pp_items(rnd), 3, rnd)


def test_tc_protocol_model_catches_a_q_barrier_on_empty_items():
    caught = 0
    for seed in range(300):
        rnd = random.Random(seed)
        items = [rnd.choice([0, 0, 1, 2, 3]) for _ in range(rnd.randint(2, 8))]
        try:
            tc_cta(items, 3, rnd, q_every_item=True)
        except (AssertionError, Stuck):
            caught += 1
    assert caught > 0
