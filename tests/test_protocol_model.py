"""A CPU model of the dense prefill kernel's barrier protocol.

The roles of prefill_fwd_kernel (TMA producer, MMA issuer, the two softmax
warpgroups, the epilogue) are generators that take the same barrier steps in
the same order as the kernel's dense path: per-tile Q buffers released after
each query tile's last S, 2-stage K/V rings, S/P per query tile, O handed to
the epilogue and freed again, a 2-slot ring of row statistics, and the next
item's first S0 issued early when a non-blocking test finds its Q0 and first
K tile already landed.  TMA copies land in any order; tcgen05 commits and the
MMAs before them complete in issue order; both at random times.

Besides phases, the model tracks what every shared buffer holds:
- no TMA copy may start into a Q tile or K/V stage that a pending MMA still
  reads, and every MMA must find its own item's (or KV tile's) data there;
- the first P V of an item into O_t may start only after the epilogue has
  read O_t of the previous item, and the epilogue may read O_t only after all
  of its item's P V products have landed.
For many random interleavings over the work-item schedules of causal,
non-causal, windowed and ragged problems, every run must finish and no wait or
test may see its barrier two phases ahead of the phase it names (a parity wait
would read the wrong phase).  Three planted slips of the protocol must be
caught.  The block-sparse path (a lister warp writing each item's tile list
one item ahead into two buffers, per-tile sets, empty sets skipped) is
modelled below the dense one, with its own planted slip.  A change to the
kernel's protocol has to be made here too.
"""

import random

import pytest

NS = 2  # K/V ring stages


class ProtocolError(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise ProtocolError(msg)


class Bar:
    def __init__(self, count=1):
        self.count = count
        self.pending = count
        self.done = 0  # completed phases

    def arrive(self):
        self.pending -= 1
        check(self.pending >= 0, "barrier over-arrived")
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def dense_items(B, H, N, causal, window_left, G, c):
    """The work items CTA c of G is dealt, as the kernel's prefill_item
    computes them: (lo0, hi0, lo1, hi1, has1)."""
    num_m = (N + 255) // 256
    out = []
    r = 0
    while True:
        idx = r * G + ((G - 1 - c) if (r & 1) else c)
        if idx >= num_m * B * H:
            return out
        rank = idx // (B * H)
        m = (num_m - 1 - rank) if causal else rank
        tiles = []
        for t in range(2):
            r0 = m * 256 + 128 * t
            if t == 1 and r0 >= N:
                tiles.append((0, 0))
                continue
            first = max(0, r0 - window_left) if window_left >= 0 else 0
            last = min(r0 + 127, N - 1) if causal else N - 1
            tiles.append((first // 128, last // 128 + 1))
        (lo0, hi0), (lo1, hi1) = tiles
        out.append((lo0, hi0, lo1, hi1, m * 256 + 128 < N))
        r += 1


def run_model(items, early_s0, seed, slip=None):
    rnd = random.Random(seed)
    bars = {}
    for t in range(2):
        for n in ("QF", "QE", "SF", "PF", "OF", "OR"):
            bars[f"{n}{t}"] = Bar()
        for s in range(2):
            bars[f"STF{t}{s}"] = Bar()
            bars[f"STE{t}{s}"] = Bar()
    for s in range(NS):
        for n in ("KF", "KE", "VF", "VE"):
            bars[f"{n}{s}"] = Bar()

    holder = {}       # buffer -> what it holds (set when a TMA copy lands)
    tma = []          # copies in flight: (buffer, value, barrier)
    pipe = []         # tcgen05 work in issue order: ("read", buf, value) / ("pv", t, item, first) / ("arrive", bar)
    o_item = [None, None]      # item whose P V products O_t holds
    o_read = [None, None]      # last item whose O_t the epilogue has read

    def active(it, t, j):
        lo, hi = (it[0], it[1]) if t == 0 else (it[2], it[3])
        return lo <= j < hi

    def wait(name, k):
        while True:
            b = bars[name]
            check(b.done <= k + 1, f"{name}: phase {k} waited for with {b.done} completed (parity alias)")
            if b.done > k:
                return
            yield

    def test(name, k):
        b = bars[name]
        check(b.done <= k + 1, f"{name}: phase {k} tested with {b.done} completed (parity alias)")
        return b.done > k

    def copy(buf, value, full):
        check(not any(e[0] == "read" and e[1] == buf for e in pipe), f"TMA into {buf} while an MMA still reads it")
        check(not any(x[0] == buf for x in tma), f"two copies into {buf}")
        tma.append((buf, value, full))

    def mma_s(t, item, stage, g):
        pipe.append(("read", f"Q{t}", item))
        pipe.append(("read", f"K{stage}", g))

    def mma_pv(t, item, stage, g, first):
        pipe.append(("read", f"V{stage}", g))
        pipe.append(("pv", t, item, first))

    def commit(name):
        pipe.append(("arrive", name))

    def retire(e):
        if e[0] == "arrive":
            bars[e[1]].arrive()
        elif e[0] == "read":
            check(holder.get(e[1]) == e[2], f"MMA read {e[1]} holding {holder.get(e[1])}, needs {e[2]}")
        else:
            _, t, item, first = e
            if first:
                check(o_item[t] is None or o_read[t] == o_item[t], f"O{t} of item {o_item[t]} overwritten unread")
                o_item[t] = item
            check(o_item[t] == item, f"P V of item {item} into O{t} of item {o_item[t]}")

    def producer():
        kv = 0
        q_issued = [0, 0]
        for r, it in enumerate(items):
            lo0, hi0, lo1, hi1, has1 = it
            jb, je = lo0, max(hi0, hi1 if has1 else 0)

            def load(kind, g):
                st, rd = g % NS, g // NS
                if rd > 0:
                    yield from wait(f"{kind}E{st}", rd - 1)
                copy(f"{kind}{st}", g, f"{kind}F{st}")

            yield from load("K", kv)
            for t in range(2):
                if t == 1 and not has1:
                    break
                if q_issued[t] > 0:
                    yield from wait(f"QE{t}", q_issued[t] - 1)
                copy(f"Q{t}", r, f"QF{t}")
                q_issued[t] += 1
            yield from load("V", kv)
            kv += 1
            for _ in range(jb + 1, je):
                yield from load("K", kv)
                yield from load("V", kv)
                kv += 1

    def mma():
        kv_it = 0
        p_cnt = [0, 0]
        o_cnt = [0, 0]
        q_cnt = [0, 0]
        s0_early = False
        for r, it in enumerate(items):
            lo0, hi0, lo1, hi1, has1 = it
            jb, je = lo0, max(hi0, hi1 if has1 else 0)
            have_nx = early_s0 and r + 1 < len(items)
            nkv = je - jb
            st = kv_it % NS
            if not s0_early:
                yield from wait("QF0", q_cnt[0])
                q_cnt[0] += 1
                yield from wait(f"KF{st}", kv_it // NS)
                if active(it, 0, jb):
                    mma_s(0, r, st, kv_it)
                    commit("SF0")
            s0_early = False
            if has1:
                yield from wait("QF1", q_cnt[1])
                q_cnt[1] += 1
                if active(it, 1, jb):
                    mma_s(1, r, st, kv_it)
                    commit("SF1")
            commit(f"KE{st}")
            if hi0 - 1 == jb or slip == "q0_released_early":
                commit("QE0")
            if has1 and hi1 - 1 == jb:
                commit("QE1")
            for j in range(jb, je):
                g = kv_it + (j - jb)
                st, st1 = g % NS, (g + 1) % NS
                v_ready = k_ready = False
                if active(it, 0, j):
                    yield from wait("PF0", p_cnt[0])
                    p_cnt[0] += 1
                    if j == lo0 and o_cnt[0] > 0 and slip != "no_o_free_wait":
                        yield from wait("OR0", o_cnt[0] - 1)
                    yield from wait(f"VF{st}", g // NS)
                    v_ready = True
                    mma_pv(0, r, st, g, j == lo0)
                    if j + 1 == hi0:
                        commit("OF0")
                        o_cnt[0] += 1
                    if active(it, 0, j + 1):
                        yield from wait(f"KF{st1}", (g + 1) // NS)
                        k_ready = True
                        mma_s(0, r, st1, g + 1)
                        commit("SF0")
                        if j + 2 == hi0 and slip != "q0_released_early":
                            commit("QE0")
                if active(it, 1, j):
                    yield from wait("PF1", p_cnt[1])
                    p_cnt[1] += 1
                    if j == lo1 and o_cnt[1] > 0:
                        yield from wait("OR1", o_cnt[1] - 1)
                    if not v_ready:
                        yield from wait(f"VF{st}", g // NS)
                    mma_pv(1, r, st, g, j == lo1)
                    if j + 1 == hi1:
                        commit("OF1")
                        o_cnt[1] += 1
                if active(it, 1, j + 1):
                    if not k_ready:
                        yield from wait(f"KF{st1}", (g + 1) // NS)
                    mma_s(1, r, st1, g + 1)
                    commit("SF1")
                    if j + 2 == hi1:
                        commit("QE1")
                commit(f"VE{st}")
                if j + 1 < je:
                    commit(f"KE{st1}")
                if early_s0 and j + 1 == hi0 and have_nx:
                    gn = kv_it + nkv
                    landed = test("QF0", q_cnt[0]) and test(f"KF{gn % NS}", gn // NS)
                    if landed or slip == "early_s0_untested":
                        q_cnt[0] += 1
                        mma_s(0, r + 1, gn % NS, gn)
                        commit("SF0")
                        s0_early = True
                yield
            kv_it += nkv

    def softmax(t):
        s_cnt = 0
        st_cnt = 0
        for it in items:
            if t == 1 and not it[4]:
                continue
            lo, hi = (it[0], it[1]) if t == 0 else (it[2], it[3])
            for _ in range(lo, hi):
                yield from wait(f"SF{t}", s_cnt)
                s_cnt += 1
                yield  # exponentials
                bars[f"PF{t}"].arrive()
            slot = st_cnt & 1
            if st_cnt >= 2:
                yield from wait(f"STE{t}{slot}", (st_cnt >> 1) - 1)
            bars[f"STF{t}{slot}"].arrive()
            st_cnt += 1

    def epilogue():
        st_cnt = [0, 0]
        for r, it in enumerate(items):
            for t in range(2):
                if t == 1 and not it[4]:
                    continue
                n = st_cnt[t]
                yield from wait(f"OF{t}", n)
                yield from wait(f"STF{t}{n & 1}", n >> 1)
                bars[f"STE{t}{n & 1}"].arrive()
                st_cnt[t] += 1
                check(o_item[t] == r and not any(e[0] == "pv" and e[1] == t for e in pipe),
                      f"O{t} of item {r} read before its P V products landed")
                yield  # O out of tensor memory
                o_read[t] = r
                bars[f"OR{t}"].arrive()

    live = {"producer": producer(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1),
            "epilogue": epilogue()}
    spins = 0
    while live or tma or pipe:
        choices = list(live) + (["tma"] if tma else []) + (["pipe"] if pipe else [])
        pick = rnd.choice(choices)
        if pick == "tma":
            buf, value, full = tma.pop(rnd.randrange(len(tma)))
            holder[buf] = value
            bars[full].arrive()
            spins = 0
        elif pick == "pipe":
            retire(pipe.pop(0))
            spins = 0
        else:
            try:
                next(live[pick])
            except StopIteration:
                del live[pick]
            spins += 1
            check(spins < 20_000, f"deadlock: {sorted(live)} all waiting")


CASES = [
    # B, H, N, causal, window_left, G (CTAs)
    (1, 2, 300, True, -1, 2),
    (1, 2, 300, False, -1, 2),
    (2, 3, 1000, True, -1, 3),
    (1, 2, 2048, True, -1, 1),
    (1, 1, 1200, True, 300, 1),     # a window: query tile 1 may start a tile after query tile 0
    (1, 2, 777, False, 200, 2),     # a window without causality
    (1, 4, 129, True, -1, 2),       # ragged: items without a second query tile
    (1, 1, 128, False, -1, 1),
]


@pytest.mark.parametrize("B,H,N,causal,window,G", CASES)
def test_protocol_finishes_without_hazards(B, H, N, causal, window, G):
    early = window < 0  # the kernel issues the early S0 in every dense kernel but the windowed one
    for c in range(G):
        items = dense_items(B, H, N, causal, window, G, c)
        for seed in range(20):
            run_model(items, early, seed)
            run_model(items, False, seed)


@pytest.mark.parametrize("slip", ["q0_released_early", "early_s0_untested", "no_o_free_wait"])
def test_planted_slips_are_caught(slip):
    # Non-causal items: there Q0's last S comes a tile after the K ring lets the
    # producer move on (in causal items the ring's back-pressure masks an early
    # Q0 release).
    items = dense_items(1, 2, 2048, False, -1, 1, 0)
    caught = 0
    for seed in range(40):
        try:
            run_model(items, True, seed, slip=slip)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"the model missed the planted slip {slip}"


# -- the block-sparse path ---------------------------------------------------------
#
# Each query tile visits an arbitrary set of KV tiles (a subset of its visible
# range); the producer walks their union; the lister warp writes each item's
# tile list one item ahead into one of two buffers (ListFull / ListEmpty); the
# MMA thread walks the list with the dense issue order; a query tile with an
# empty set is skipped by its softmax warpgroup and written as zeros by the
# epilogue without any wait.

def sparse_items(B, H, N, causal, G, c, density, rnd):
    out = []
    for lo0, hi0, lo1, hi1, has1 in dense_items(B, H, N, causal, -1, G, c):
        s0 = [j for j in range(lo0, hi0) if rnd.random() < density]
        s1 = [j for j in range(lo1, hi1) if rnd.random() < density] if has1 else []
        out.append((s0, s1, has1))
    return out


def run_sparse_model(items, seed, slip=None):
    rnd = random.Random(seed)
    bars = {}
    for t in range(2):
        for n in ("QF", "QE", "SF", "PF", "OF", "OR", "LF", "LE"):
            bars[f"{n}{t}"] = Bar()
        for s in range(2):
            bars[f"STF{t}{s}"] = Bar()
            bars[f"STE{t}{s}"] = Bar()
    for s in range(NS):
        for n in ("KF", "KE", "VF", "VE"):
            bars[f"{n}{s}"] = Bar()
    holder = {}
    tma = []
    pipe = []
    o_item = [None, None]
    o_read = [None, None]
    lists = [None, None]          # item whose list each buffer holds
    walking = [None, None]        # item whose list the MMA thread is walking, per buffer

    def wait(name, k):
        while True:
            b = bars[name]
            check(b.done <= k + 1, f"{name}: phase {k} waited for with {b.done} completed (parity alias)")
            if b.done > k:
                return
            yield

    def copy(buf, value, full):
        check(not any(e[0] == "read" and e[1] == buf for e in pipe), f"TMA into {buf} while an MMA still reads it")
        tma.append((buf, value, full))

    def retire(e):
        if e[0] == "arrive":
            bars[e[1]].arrive()
        elif e[0] == "read":
            check(holder.get(e[1]) == e[2], f"MMA read {e[1]} holding {holder.get(e[1])}, needs {e[2]}")
        else:
            _, t, item, first = e
            if first:
                check(o_item[t] is None or o_read[t] == o_item[t], f"O{t} of item {o_item[t]} overwritten unread")
                o_item[t] = item
            check(o_item[t] == item, f"P V of item {item} into O{t} of item {o_item[t]}")

    def union(it):
        return sorted(set(it[0]) | set(it[1]))

    def lister():
        for r in range(len(items) + 1):
            buf = r & 1
            if r >= 2:
                yield from wait(f"LE{buf}", (r >> 1) - 1)
            check(walking[buf] is None, f"list buffer {buf} rewritten while item {walking[buf]} is walked")
            lists[buf] = r if r < len(items) else -1
            yield
            bars[f"LF{buf}"].arrive()

    def producer():
        kv = 0
        q_issued = [0, 0]
        for r, it in enumerate(items):
            tiles = union(it)
            if not tiles:
                continue

            def load(kind, g):
                st, rd = g % NS, g // NS
                if rd > 0:
                    yield from wait(f"{kind}E{st}", rd - 1)
                copy(f"{kind}{st}", g, f"{kind}F{st}")

            yield from load("K", kv)
            for t in range(2):
                if t == 1 and not it[2]:
                    break
                if q_issued[t] > 0:
                    yield from wait(f"QE{t}", q_issued[t] - 1)
                copy(f"Q{t}", r, f"QF{t}")
                q_issued[t] += 1
            yield from load("V", kv)
            kv += 1
            for _ in tiles[1:]:
                yield from load("K", kv)
                yield from load("V", kv)
                kv += 1

    def mma():
        kv_it = 0
        p_cnt = [0, 0]
        o_cnt = [0, 0]
        q_cnt = [0, 0]
        r = 0
        while True:
            buf = r & 1
            yield from wait(f"LF{buf}", r >> 1)
            check(lists[buf] == (r if r < len(items) else -1), "MMA thread reads another item's list")
            if lists[buf] == -1:
                return
            it = items[r]
            tiles = union(it)
            n = len(tiles)
            if n == 0:
                bars[f"LE{buf}"].arrive()
                r += 1
                continue
            walking[buf] = r
            if slip == "list_released_early":
                walking[buf] = None
                bars[f"LE{buf}"].arrive()
            on = [set(it[0]), set(it[1])]
            has1 = it[2]
            yield from wait("QF0", q_cnt[0])
            q_cnt[0] += 1
            if has1:
                yield from wait("QF1", q_cnt[1])
                q_cnt[1] += 1
            st = kv_it % NS
            yield from wait(f"KF{st}", kv_it // NS)
            for t in range(2):
                if tiles[0] in on[t]:
                    pipe.extend([("read", f"Q{t}", r), ("read", f"K{st}", kv_it), ("arrive", f"SF{t}")])
            pipe.append(("arrive", f"KE{st}"))
            if n == 1:
                pipe.append(("arrive", "QE0"))
                if has1:
                    pipe.append(("arrive", "QE1"))
            for u in range(n):
                check(lists[buf] == r, "list rewritten under the MMA thread")
                j = tiles[u]
                more = u + 1 < n
                jn = tiles[u + 1] if more else None
                g = kv_it + u
                st, st1 = g % NS, (g + 1) % NS
                v_ready = k_ready = False
                for t in range(2):
                    if j in on[t]:
                        yield from wait(f"PF{t}", p_cnt[t])
                        p_cnt[t] += 1
                        first = j == min(on[t])
                        if first and o_cnt[t] > 0:
                            yield from wait(f"OR{t}", o_cnt[t] - 1)
                        if not v_ready:
                            yield from wait(f"VF{st}", g // NS)
                            v_ready = True
                        pipe.extend([("read", f"V{st}", g), ("pv", t, r, first)])
                        if j == max(on[t]):
                            pipe.append(("arrive", f"OF{t}"))
                            o_cnt[t] += 1
                    if more and jn in on[t]:
                        if not k_ready:
                            yield from wait(f"KF{st1}", (g + 1) // NS)
                            k_ready = True
                        pipe.extend([("read", f"Q{t}", r), ("read", f"K{st1}", g + 1), ("arrive", f"SF{t}")])
                pipe.append(("arrive", f"VE{st}"))
                if more:
                    pipe.append(("arrive", f"KE{st1}"))
                if u + 2 == n:
                    pipe.append(("arrive", "QE0"))
                    if has1:
                        pipe.append(("arrive", "QE1"))
                yield
            kv_it += n
            if slip != "list_released_early":
                walking[buf] = None
                bars[f"LE{buf}"].arrive()
            r += 1

    def softmax(t):
        s_cnt = 0
        st_cnt = 0
        for it in items:
            for _ in it[t]:
                yield from wait(f"SF{t}", s_cnt)
                s_cnt += 1
                yield
                bars[f"PF{t}"].arrive()
            if not it[t]:
                continue
            slot = st_cnt & 1
            if st_cnt >= 2:
                yield from wait(f"STE{t}{slot}", (st_cnt >> 1) - 1)
            bars[f"STF{t}{slot}"].arrive()
            st_cnt += 1

    def epilogue():
        st_cnt = [0, 0]
        for r, it in enumerate(items):
            for t in range(2):
                if not it[t]:
                    continue  # no key visible: zeros, nothing to wait for
                n = st_cnt[t]
                yield from wait(f"OF{t}", n)
                yield from wait(f"STF{t}{n & 1}", n >> 1)
                bars[f"STE{t}{n & 1}"].arrive()
                st_cnt[t] += 1
                check(o_item[t] == r and not any(e[0] == "pv" and e[1] == t for e in pipe),
                      f"O{t} of item {r} read before its P V products landed")
                yield
                o_read[t] = r
                bars[f"OR{t}"].arrive()

    live = {"lister": lister(), "producer": producer(), "mma": mma(), "softmax0": softmax(0),
            "softmax1": softmax(1), "epilogue": epilogue()}
    spins = 0
    while live or tma or pipe:
        choices = list(live) + (["tma"] if tma else []) + (["pipe"] if pipe else [])
        pick = rnd.choice(choices)
        if pick == "tma":
            buf, value, full = tma.pop(rnd.randrange(len(tma)))
            holder[buf] = value
            bars[full].arrive()
            spins = 0
        elif pick == "pipe":
            retire(pipe.pop(0))
            spins = 0
        else:
            try:
                next(live[pick])
            except StopIteration:
                del live[pick]
            spins += 1
            check(spins < 20_000, f"deadlock: {sorted(live)} all waiting")


@pytest.mark.parametrize("N,causal,density", [(700, True, 0.5), (700, False, 0.3), (1300, True, 0.15),
                                              (300, True, 1.0), (129, False, 0.5), (900, True, 0.0)])
def test_block_sparse_protocol_finishes_without_hazards(N, causal, density):
    rnd = random.Random(N)
    for c in range(2):
        items = sparse_items(1, 3, N, causal, 2, c, density, rnd)
        for seed in range(15):
            run_sparse_model(items, seed)


def test_block_sparse_planted_slip_is_caught():
    """The MMA thread handing its list buffer back before walking it lets the
    lister rewrite the list under it."""
    rnd = random.Random(3)
    items = sparse_items(1, 2, 1300, False, 1, 0, 0.6, rnd)
    caught = 0
    for seed in range(40):
        try:
            run_sparse_model(items, seed, slip="list_released_early")
        except ProtocolError:
            caught += 1
    assert caught > 0
