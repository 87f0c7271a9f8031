"""A model of the chunked-prefill kernel's barrier protocol, checked on the CPU.

`prefill_tc_kernel` (csrc/prefill.cuh) runs four roles per CTA that meet only
at mbarriers: the TMA warp, the MMA thread (whose tensor-core operations and
commits complete in issue order), and two softmax warpgroups, one per
128-query tile. This test restates, role by role, the order of waits, copies,
MMAs, commits and arrivals the kernel uses. It then runs that model under
seeded random interleavings for every kind of tile range the kernel's
geometry produces: causal and windowed, a second query tile with or without
rows, one key tile or many.

A run fails on any of these:
- a deadlock;
- a wait satisfied by the wrong phase of its barrier (mbarrier parity waits
  only tell one phase from the next);
- a data hazard:
  - S written over a P that its P.V has not read;
  - O rescaled while a P.V on it is queued;
  - a K/V stage reloaded before the MMAs reading it completed;
  - a P.V reading V rows that still need zeroing;
  - the epilogue reading O before the last P.V.

The model has to change with the kernel: it encodes the protocol, not the
arithmetic."""
import random

import pytest

ROWS = KEYS = 128
STAGES = 2


def geometry(C, cached, row0, W, pair=False):
    """Tile ranges [jlo_x, jhi_x) of the two query tiles of a CTA (the
    kernel's formulas), the chunk's lowest needed key, and the context.
    pair: the two tiles are the same rows of two query heads."""
    row1 = row0 if pair else row0 + ROWS
    rows0 = min(ROWS, C - row0)
    rows1 = max(0, min(ROWS, C - row1))
    pf0 = cached + row0
    pf1 = cached + row1
    jlo0 = (max(0, pf0 - W + 1) if W > 0 else 0) // KEYS
    jlo1 = (max(0, pf1 - W + 1) if W > 0 else 0) // KEYS
    jhi0 = (pf0 + rows0 - 1) // KEYS + 1
    jhi1 = (pf1 + rows1 - 1) // KEYS + 1 if rows1 > 0 else jlo1
    chunk_lo = max(0, cached - W + 1) if W > 0 else 0
    return [(jlo0, jhi0), (jlo1, jhi1)], chunk_lo, cached + C


class Bar:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: arrival count underflow"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def ready(self, n):
        """try_wait.parity for completion number n (0-based): the hardware
        compares parities only, so a phase two ahead, or the previous one,
        must never be what the waiter sees."""
        assert self.done <= n + 1, f"{self.name}: waiting for phase {n}, {self.done} done"
        hw = (self.done & 1) != (n & 1)
        assert not hw or self.done == n + 1, f"{self.name}: phase {n} seen early"
        return hw


def run(C, cached, row0, W, seed, pair=False):
    """One seeded interleaving of the four roles for one CTA's geometry."""
    rnd = random.Random(seed)
    (r0, r1), chunk_lo, ctx = geometry(C, cached, row0, W, pair)
    ranges = [r0, r1]
    act = lambda x, j: ranges[x][0] <= j < ranges[x][1]
    jmin, jmax = r0[0], max(r0[1], r1[1])
    stage = lambda j: (j - jmin) % STAGES
    use = lambda j: (j - jmin) // STAGES
    # the query tile whose band reaches the last key tile zeroes its tail
    # rows (the first one in issue order when both do)
    zeroes_tail = [r0[1] == jmax, r1[1] == jmax and not r0[1] == jmax]

    B = {n: Bar(n) for n in ["q_full", "fin"] + [f"{k}{s}" for k in ("k_full", "k_free",
                                                                    "v_full", "v_free")
                                                for s in range(STAGES)]
         + [f"{k}{x}" for k in ("s_full", "o_full") for x in (0, 1)]}
    for x in (0, 1):
        B[f"p_full{x}"] = Bar(f"p_full{x}", 1)  # one arrival per softmax warp, modelled as one
    pipe, done, inflight = [], set(), []
    st = {"K": {}, "V": {}, "q": False, "S": {}, "O": {}, "zero_needed": set(), "zeroed": set()}
    for j in range(jmin, jmax):
        lo, hi = j * KEYS, (j + 1) * KEYS
        if hi > ctx or (W > 0 and j == jmin and lo < chunk_lo):
            st["zero_needed"].add(j)

    def tma():
        inflight.append(("q_full", "Q", None))
        yield
        for j in range(jmin, jmax):
            s, u = stage(j), use(j)
            if u > 0:
                while not B[f"k_free{s}"].ready(u - 1):
                    yield
                old = j - STAGES
                assert all(("S", x, old) in done for x in (0, 1) if act(x, old)), "K stage reloaded under S"
            inflight.append((f"k_full{s}", "K", j))
            yield
            if u > 0:
                while not B[f"v_free{s}"].ready(u - 1):
                    yield
                old = j - STAGES
                assert all(("PV", x, old) in done for x in (0, 1) if act(x, old)), "V stage reloaded under P.V"
            inflight.append((f"v_full{s}", "V", j))
            yield

    def mma():
        """The MMA thread: its operations and commits run in issue order."""
        while not B["q_full"].ready(0):
            yield

        def wait_k(j):
            while not B[f"k_full{stage(j)}"].ready(use(j)):
                yield

        def wait_v(j):
            while not B[f"v_full{stage(j)}"].ready(use(j)):
                yield

        def issue_s(x, j):  # K_j was waited for
            assert st["K"].get(stage(j)) == j, f"S of tile {j} over K stage {st['K']}"
            pipe.append(("S", x, j))
            pipe.append(("commit", f"s_full{x}"))
            yield

        def issue_pv(x, j):  # V_j was waited for; P is waited for here
            while not B[f"p_full{x}"].ready(j - ranges[x][0]):
                yield
            assert st["V"].get(stage(j)) == j, f"P.V of tile {j} over V stage {st['V']}"
            pipe.append(("PV", x, j))
            pipe.append(("commit", f"o_full{x}"))
            yield

        yield from wait_k(jmin)
        for x in (0, 1):
            if act(x, jmin):
                yield from issue_s(x, jmin)
        pipe.append(("commit", f"k_free{stage(jmin)}"))
        for j in range(jmin, jmax):
            # V_j and K_{j+1} first, then each query tile's P
            yield from wait_v(j)
            if act(0, j + 1) or act(1, j + 1):
                yield from wait_k(j + 1)
            for x in (0, 1):
                if act(x, j):
                    yield from issue_pv(x, j)
                if act(x, j + 1):
                    yield from issue_s(x, j + 1)
            if j + 1 < jmax:
                pipe.append(("commit", f"k_free{stage(j + 1)}"))
            pipe.append(("commit", f"v_free{stage(j)}"))
        pipe.append(("commit", "fin"))
        while not B["fin"].ready(0):
            yield

    def softmax(x):
        j0, j1 = ranges[x]
        for j in range(j0, j1):
            while not B[f"s_full{x}"].ready(j - j0):
                yield
            assert st["S"].get(x) == ("S", j), f"tile {j}: S of query tile {x} not there"
            yield
            if j > j0 and rnd.random() < 0.3:  # the row max grew: O rescaled in place
                assert ("PV", x, j - 1) in done, "rescale before the previous P.V completed"
                assert not any(op[0] == "PV" and op[1] == x for op in pipe), \
                    "rescale under a queued P.V"
            st["S"][x] = ("P", j)
            # the first consumer of a tile in issue order zeroes its rows
            # past the context or before the band
            if j in st["zero_needed"] and ((j == jmin and x == 0) or
                                           (j == j1 - 1 and zeroes_tail[x])):
                while not B[f"v_full{stage(j)}"].ready(use(j)):
                    yield
                st["zeroed"].add(j)
            B[f"p_full{x}"].arrive()
            yield
        if j1 > j0:
            while not B[f"o_full{x}"].ready(j1 - j0 - 1):
                yield
            assert all(("PV", x, j) in done for j in range(j0, j1)), "epilogue before the last P.V"

    def pipe_step():
        op = pipe.pop(0)
        if op[0] == "commit":
            B[op[1]].arrive()
            return
        kind, x, j = op
        assert st["q"], "MMA before Q landed"
        if kind == "S":
            cur = st["S"].get(x)
            assert cur is None or cur[0] == "P" and ("PV", x, cur[1]) in done, \
                f"S of tile {j} over an unread tile {cur}"
            st["S"][x] = ("S", j)
        else:
            assert st["S"].get(x) == ("P", j), f"P.V of tile {j} without its P"
            assert j not in st["zero_needed"] or j in st["zeroed"], \
                f"P.V of tile {j} reads unzeroed V rows"
        done.add((kind, x, j))

    roles = {"tma": tma(), "mma": mma(), "sm0": softmax(0), "sm1": softmax(1)}
    steps = 0
    while roles or pipe or inflight:
        choice = rnd.choice(list(roles) + ["pipe"] * bool(pipe) + ["copy"] * bool(inflight))
        if choice == "pipe":
            pipe_step()
        elif choice == "copy":
            bar, kind, j = inflight.pop(0)
            if kind == "Q":
                st["q"] = True
            else:
                st[kind][stage(j)] = j
            B[bar].arrive()
        else:
            try:
                next(roles[choice])
            except StopIteration:
                del roles[choice]
        steps += 1
        assert steps < 200000, f"deadlock: roles {list(roles)} waiting, queue {pipe}"
    assert B["fin"].done == 1


SHAPES = [(C, cached, row0, W)
          for C in (1, 100, 128, 129, 255, 256, 300, 512)
          for cached in (0, 5, 127, 128, 300, 1000)
          for row0 in (0, 256) if row0 < C
          for W in (0, 1, 64, 128, 200, 1024)]
# head-paired CTAs: both tiles cover the same 128 rows
PAIR_SHAPES = [(C, cached, row0, W)
               for C in (1, 100, 128, 129, 300, 512)
               for cached in (0, 5, 128, 1000)
               for row0 in (0, 128, 384) if row0 < C
               for W in (0, 1, 64, 200, 1024)]


def test_geometry_matches_the_causal_bound():
    # the last query of each tile sees exactly the keys up to its position
    for C, cached, row0, W in SHAPES:
        (r0, r1), _, ctx = geometry(C, cached, row0, W)
        last0 = cached + row0 + min(ROWS, C - row0) - 1
        assert r0[1] * KEYS > last0 >= (r0[1] - 1) * KEYS
        assert r0[1] * KEYS <= max(KEYS, ((ctx + KEYS - 1) // KEYS) * KEYS)
        if C - row0 > ROWS:
            last1 = cached + row0 + min(2 * ROWS, C - row0) - 1
            assert r1[1] * KEYS > last1 >= (r1[1] - 1) * KEYS
        else:
            assert r1[1] == r1[0]


@pytest.mark.parametrize("shape", SHAPES[::3])
def test_protocol_has_no_deadlock_alias_or_hazard(shape):
    for seed in range(6):
        run(*shape, seed)


@pytest.mark.parametrize("shape", PAIR_SHAPES[::3])
def test_head_paired_protocol_has_no_deadlock_alias_or_hazard(shape):
    for seed in range(6):
        run(*shape, seed, pair=True)


def test_head_pairs_share_one_key_range():
    # same rows: both query tiles stream exactly the same key tiles
    for C, cached, row0, W in PAIR_SHAPES:
        (r0, r1), _, _ = geometry(C, cached, row0, W, pair=True)
        assert r0 == r1


def test_model_catches_a_missing_wait():
    # the checker must notice a broken protocol: let the epilogue wait for
    # the first P.V instead of the last one
    old = Bar.ready

    def early(self, n):
        if self.name.startswith("o_full"):
            n = 0
        return old(self, n)

    Bar.ready = early
    try:
        with pytest.raises(AssertionError):
            for seed in range(20):
                run(512, 300, 0, 0, seed)
    finally:
        Bar.ready = old
