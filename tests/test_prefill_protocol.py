"""A model of the chunked-prefill kernel's barrier protocol, checked on the CPU.

`prefill_tc_kernel` (csrc/prefill.cuh) is persistent: one CTA per SM works
through a sequence of items, each two 128-query tiles and the key tiles they
need. Four roles meet only at mbarriers: the TMA warp, the MMA thread (whose
tensor-core operations and commits complete in issue order), and two softmax
warpgroups, one per query tile. Across items the K/V rings and the S/P phases
carry on; the next item's Q loads once the current item's last S has read Q
(q_free). An item's first P.V into O has no barrier of its own: it waits for
the item's first P, which the same softmax warps produce only after their
epilogue has read the previous item's O out.

This test restates, role by role, the order of waits, copies, MMAs, commits
and arrivals the kernel uses. It then runs that model under seeded random
interleavings, for single items of every kind of tile range the kernel's
geometry produces (causal and windowed, row-paired and head-paired tiles, a
second query tile with or without rows, one key tile or many) and for
sequences of such items through one CTA.

A run fails on any of these:
- a deadlock;
- a wait satisfied by the wrong phase of its barrier (mbarrier parity waits
  only tell one phase from the next);
- a data hazard:
  - S written over a P that its P.V has not read;
  - S computed from a Q tile of another item, or Q reloaded under a queued S;
  - O rescaled while a P.V on it is queued;
  - an item's first P.V overwriting an O the previous epilogue has not read;
  - a K/V stage reloaded before the MMAs reading it completed;
  - a P.V reading V rows that still need zeroing;
  - the epilogue reading O before the item's last P.V.

The model has to change with the kernel: it encodes the protocol, not the
arithmetic."""
import random

import pytest

ROWS = KEYS = 128
STAGES = 2


def geometry(C, cached, row0, W, pair=False):
    """Tile ranges [jlo_x, jhi_x) of the two query tiles of an item (the
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


class Item:
    """One work item's geometry and its first K/V tile in the CTA's count."""

    def __init__(self, n, shape, t0):
        C, cached, row0, W, pair = shape
        self.n, self.W = n, W
        self.ranges, self.chunk_lo, self.ctx = geometry(C, cached, row0, W, pair)
        (a0, b0), (a1, b1) = self.ranges
        self.jmin, self.jmax = a0, max(b0, b1)
        self.t0 = t0
        # the query tile whose band reaches the last key tile zeroes its
        # tail rows (the first one in issue order when both do)
        self.zeroes_tail = [b0 == self.jmax, b1 == self.jmax and not b0 == self.jmax]
        self.zero_needed = set()
        for j in range(self.jmin, self.jmax):
            lo, hi = j * KEYS, (j + 1) * KEYS
            if hi > self.ctx or (W > 0 and j == self.jmin and lo < self.chunk_lo):
                self.zero_needed.add(j)

    def act(self, x, j):
        return self.ranges[x][0] <= j < self.ranges[x][1]

    def t(self, j):  # the CTA-wide K/V tile count of key tile j
        return self.t0 + j - self.jmin


def run(shapes, seed):
    """One seeded interleaving of the four roles for a CTA that works
    through the items `shapes` (C, cached, row0, W, pair) in order."""
    rnd = random.Random(seed)
    items, t0 = [], 0
    for n, shape in enumerate(shapes):
        it = Item(n, shape, t0)
        items.append(it)
        t0 += it.jmax - it.jmin
    stage = lambda t: t % STAGES
    use = lambda t: t // STAGES

    names = (["q_full", "q_free", "fin"]
             + [f"{k}{s}" for k in ("k_full", "k_free", "v_full", "v_free") for s in range(STAGES)]
             + [f"{k}{x}" for k in ("s_full", "o_full") for x in (0, 1)])
    B = {n: Bar(n) for n in names}
    for x in (0, 1):  # one arrival per softmax warp, modelled as one
        B[f"p_full{x}"] = Bar(f"p_full{x}", 1)
    pipe, done, inflight = [], set(), []
    # K/V: stage -> tile count; Q: item whose tiles are loaded; S: per query
    # tile ("S"|"P", item, j); O: per query tile the item accumulating in it,
    # O_read: the last item whose O the epilogue read out
    st = {"K": {}, "V": {}, "Q": None, "S": {}, "O": {}, "O_read": {}, "zeroed": set()}

    def tma():
        t = 0
        for it in items:
            if it.n > 0:
                while not B["q_free"].ready(it.n - 1):
                    yield
                prev = items[it.n - 1]
                assert all(("S", x, prev.n, j) in done for x in (0, 1)
                           for j in range(prev.jmin, prev.jmax) if prev.act(x, j)), \
                    "Q reloaded before the previous item's S read it"
            inflight.append(("q_full", "Q", it.n))
            yield
            for j in range(it.jmin, it.jmax):
                s, u = stage(t), use(t)
                if u > 0:
                    while not B[f"k_free{s}"].ready(u - 1):
                        yield
                    assert not any(op[0] == "S" and op[4] == t - STAGES for op in pipe), \
                        "K stage reloaded under a queued S"
                inflight.append((f"k_full{s}", "K", t))
                yield
                if u > 0:
                    while not B[f"v_free{s}"].ready(u - 1):
                        yield
                    assert not any(op[0] == "PV" and op[4] == t - STAGES for op in pipe), \
                        "V stage reloaded under a queued P.V"
                inflight.append((f"v_full{s}", "V", t))
                yield
                t += 1

    def mma():
        """The MMA thread: its operations and commits run in issue order."""
        pc = [0, 0]

        def wait_k(t):
            while not B[f"k_full{stage(t)}"].ready(use(t)):
                yield

        def wait_v(t):
            while not B[f"v_full{stage(t)}"].ready(use(t)):
                yield

        def issue_s(it, x, j):  # K of tile j was waited for
            t = it.t(j)
            assert st["K"].get(stage(t)) == t, f"S of tile {j} over K stage {st['K']}"
            pipe.append(("S", x, it.n, j, t))
            pipe.append(("commit", f"s_full{x}"))

        for it in items:
            while not B["q_full"].ready(it.n):
                yield
            yield from wait_k(it.t(it.jmin))
            for x in (0, 1):
                if it.act(x, it.jmin):
                    issue_s(it, x, it.jmin)
            pipe.append(("commit", f"k_free{stage(it.t(it.jmin))}"))
            if it.jmax - it.jmin == 1:
                pipe.append(("commit", "q_free"))
            yield
            for j in range(it.jmin, it.jmax):
                t = it.t(j)
                # V_j and K_{j+1} first, then each query tile's P
                yield from wait_v(t)
                if it.act(0, j + 1) or it.act(1, j + 1):
                    yield from wait_k(t + 1)
                for x in (0, 1):
                    if it.act(x, j):
                        while not B[f"p_full{x}"].ready(pc[x]):
                            yield
                        pc[x] += 1
                        assert st["V"].get(stage(t)) == t, f"P.V of tile {j} over V {st['V']}"
                        pipe.append(("PV", x, it.n, j, t))
                        if j == it.ranges[x][1] - 1:  # the epilogue waits for the last P.V
                            pipe.append(("commit", f"o_full{x}"))
                    if it.act(x, j + 1):
                        issue_s(it, x, j + 1)
                    yield
                if j + 1 == it.jmax - 1:  # the item's last S reads Q
                    pipe.append(("commit", "q_free"))
                if j + 1 < it.jmax:
                    pipe.append(("commit", f"k_free{stage(t + 1)}"))
                pipe.append(("commit", f"v_free{stage(t)}"))
        pipe.append(("commit", "fin"))
        while not B["fin"].ready(0):
            yield

    def softmax(x):
        sc = oc = 0
        for it in items:
            j0, j1 = it.ranges[x]
            if j1 <= j0:
                continue
            for j in range(j0, j1):
                while not B[f"s_full{x}"].ready(sc):
                    yield
                sc += 1
                assert st["S"].get(x) == ("S", it.n, j), f"tile {j}: S of query tile {x} not there"
                yield
                if j > j0 and rnd.random() < 0.3:  # the row max grew: O rescaled in place
                    assert ("PV", x, it.n, j - 1) in done, "rescale before the previous P.V completed"
                    assert not any(op[0] == "PV" and op[1] == x for op in pipe), \
                        "rescale under a queued P.V"
                st["S"][x] = ("P", it.n, j)
                # the first consumer of a tile in issue order zeroes its rows
                # past the context or before the band
                if j in it.zero_needed and ((j == it.jmin and x == 0) or
                                            (j == j1 - 1 and it.zeroes_tail[x])):
                    while not B[f"v_full{stage(it.t(j))}"].ready(use(it.t(j))):
                        yield
                    st["zeroed"].add((it.n, j))
                B[f"p_full{x}"].arrive()
                yield
            while not B[f"o_full{x}"].ready(oc):
                yield
            oc += 1
            assert all(("PV", x, it.n, j) in done for j in range(j0, j1)), \
                "epilogue before the last P.V"
            assert st["O"].get(x) == it.n, "epilogue reads another item's O"
            yield
            st["O_read"][x] = it.n
            yield

    def pipe_step():
        op = pipe.pop(0)
        if op[0] == "commit":
            B[op[1]].arrive()
            return
        kind, x, n, j, t = op
        if kind == "S":
            assert st["Q"] == n, f"S of item {n} on the Q tiles of item {st['Q']}"
            cur = st["S"].get(x)
            assert cur is None or cur[0] == "P" and ("PV", x, cur[1], cur[2]) in done, \
                f"S of tile {j} over an unread tile {cur}"
            st["S"][x] = ("S", n, j)
        else:
            assert st["S"].get(x) == ("P", n, j), f"P.V of tile {j} without its P"
            it = items[n]
            assert j not in it.zero_needed or (n, j) in st["zeroed"], \
                f"P.V of tile {j} reads unzeroed V rows"
            if j == it.ranges[x][0]:  # the item's first P.V overwrites O
                prev = st["O"].get(x)
                assert prev is None or st["O_read"].get(x) == prev, \
                    f"P.V of item {n} over the unread O of item {prev}"
                st["O"][x] = n
        done.add((kind, x, n, j))

    roles = {"tma": tma(), "mma": mma(), "sm0": softmax(0), "sm1": softmax(1)}
    steps = 0
    while roles or pipe or inflight:
        choice = rnd.choice(list(roles) + ["pipe"] * bool(pipe) + ["copy"] * bool(inflight))
        if choice == "pipe":
            pipe_step()
        elif choice == "copy":
            bar, kind, t = inflight.pop(0)
            if kind == "Q":
                assert not any(op[0] == "S" for op in pipe), "Q reloaded under a queued S"
                st["Q"] = t
            else:
                st[kind][stage(t)] = t
            B[bar].arrive()
        else:
            try:
                next(roles[choice])
            except StopIteration:
                del roles[choice]
        steps += 1
        assert steps < 400000, f"deadlock: roles {list(roles)} waiting, queue {pipe}"
    assert B["fin"].done == 1


SHAPES = [(C, cached, row0, W, False)
          for C in (1, 100, 128, 129, 255, 256, 300, 512)
          for cached in (0, 5, 127, 128, 300, 1000)
          for row0 in (0, 256) if row0 < C
          for W in (0, 1, 64, 128, 200, 1024)]
# head-paired items: both tiles cover the same 128 rows
PAIR_SHAPES = [(C, cached, row0, W, True)
               for C in (1, 100, 128, 129, 300, 512)
               for cached in (0, 5, 128, 1000)
               for row0 in (0, 128, 384) if row0 < C
               for W in (0, 1, 64, 200, 1024)]


def test_geometry_matches_the_causal_bound():
    # the last query of each tile sees exactly the keys up to its position
    for C, cached, row0, W, _ in SHAPES:
        (r0, r1), _, ctx = geometry(C, cached, row0, W)
        last0 = cached + row0 + min(ROWS, C - row0) - 1
        assert r0[1] * KEYS > last0 >= (r0[1] - 1) * KEYS
        assert r0[1] * KEYS <= max(KEYS, ((ctx + KEYS - 1) // KEYS) * KEYS)
        if C - row0 > ROWS:
            last1 = cached + row0 + min(2 * ROWS, C - row0) - 1
            assert r1[1] * KEYS > last1 >= (r1[1] - 1) * KEYS
        else:
            assert r1[1] == r1[0]


def test_head_pairs_share_one_key_range():
    # same rows: both query tiles stream exactly the same key tiles
    for C, cached, row0, W, pair in PAIR_SHAPES:
        (r0, r1), _, _ = geometry(C, cached, row0, W, pair)
        assert r0 == r1


@pytest.mark.parametrize("shape", SHAPES[::3])
def test_single_item_has_no_deadlock_alias_or_hazard(shape):
    for seed in range(6):
        run([shape], seed)


@pytest.mark.parametrize("shape", PAIR_SHAPES[::3])
def test_single_head_paired_item_has_no_deadlock_alias_or_hazard(shape):
    for seed in range(6):
        run([shape], seed)


def _sequences():
    """Item sequences of one CTA: long and short items, one-tile items, a
    second tile without rows, windows, the modes mixed."""
    rnd = random.Random(1)
    pool = [s for s in SHAPES + PAIR_SHAPES if s[0] > s[2]]
    seqs = [[(512, 1000, 0, 0, True), (512, 1000, 128, 0, True), (1, 0, 0, 0, True)],
            [(100, 0, 0, 0, False), (300, 5, 256, 1, False), (129, 127, 0, 64, False)],
            [(1, 0, 0, 0, True)] * 4]
    for _ in range(24):
        seqs.append([rnd.choice(pool) for _ in range(rnd.randint(2, 4))])
    return seqs


@pytest.mark.parametrize("seq", _sequences(), ids=lambda s: "-".join(f"{x[0]}c{x[1]}r{x[2]}w{x[3]}{'p' if x[4] else ''}" for x in s))
def test_item_sequence_has_no_deadlock_alias_or_hazard(seq):
    for seed in range(4):
        run(seq, seed)


def test_model_catches_a_missing_wait():
    # the checker must notice a broken protocol: let the epilogue read O
    # without waiting for the last P.V
    old = Bar.ready

    def early(self, n):
        if self.name.startswith("o_full"):
            return True
        return old(self, n)

    Bar.ready = early
    try:
        with pytest.raises(AssertionError):
            for seed in range(20):
                run([(512, 300, 0, 0, False)], seed)
    finally:
        Bar.ready = old


def test_model_catches_an_early_q_reload():
    # and a Q reload that does not wait for the previous item's last S
    old = Bar.ready

    def early(self, n):
        if self.name == "q_free":
            return True
        return old(self, n)

    Bar.ready = early
    try:
        with pytest.raises(AssertionError):
            for seed in range(20):
                run([(512, 1000, 0, 0, True), (512, 1000, 128, 0, True)], seed)
    finally:
        Bar.ready = old


def item_of(r, b, G):
    """CTA b's r-th item in the persistent kernel's dealing: rounds of one item
    per CTA, every other round reversed."""
    return r * G + ((G - 1 - b) if r & 1 else b)


@pytest.mark.parametrize("n_items,G", [(1, 148), (147, 148), (148, 148), (149, 148), (512, 148),
                                       (1152, 148), (5, 3), (7, 1), (4096, 132)])
def test_dealing_gives_every_item_to_one_cta(n_items, G):
    G = min(G, n_items)  # the host launches min(items, SMs) CTAs
    seen = []
    for b in range(G):
        r = 0
        while item_of(r, b, G) < n_items:
            seen.append(item_of(r, b, G))
            r += 1
    assert sorted(seen) == list(range(n_items))


def test_dealing_balances_the_mixed_launch():
    """The mixed launch's 512 items dealt over 148 CTAs (cost of an item: its
    key tiles plus 0.3 of a tile for its start and epilogue): the busiest CTA
    within 4 % of the mean, no worse than a greedy longest-first assignment."""
    import heapq
    cached = [round(i * 4096 / 7) for i in range(8)]
    work = []  # in item order: chunks from the last, row tiles from the last, heads fastest
    for c in reversed(cached):
        for rt in reversed(range(4)):
            pf = c + rt * ROWS
            work += [(pf + ROWS - 1) // KEYS + 1 + 0.3] * 16
    G = 148
    load = [0.0] * G
    for b in range(G):
        r = 0
        while item_of(r, b, G) < len(work):
            load[b] += work[item_of(r, b, G)]
            r += 1
    heap = [(0.0, b) for b in range(G)]
    for w in sorted(work, reverse=True):
        l, b = heapq.heappop(heap)
        heapq.heappush(heap, (l + w, b))
    greedy = max(l for l, _ in heap)
    assert max(load) <= 1.04 * sum(load) / G
    assert max(load) <= greedy * 1.001
