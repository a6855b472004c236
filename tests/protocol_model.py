"""CPU model of attn_kernel's mbarrier protocol (csrc/kernels_tc.cuh).

The model runs the kernel's roles -- TMA producer, one MMA issuer per row
tile, the softmax warpgroups (CS column shares of each row tile, which swap
their half-row maxima every job and their row sums at the end of an item
through an exchange barrier) -- as coroutines that wait on mbarriers with the
kernel's arrival counts and phase parities, in random interleavings, with TMA
and MMA completions arriving after random delays.  It mirrors the kernel's
item decoding, stage rings (shared ring, or one ring per warpgroup in
interleaved mode), query slots, the score-ahead/value MMA order and the
epilogue placement (deferred into the next item in the decode, at the item's
end in the split passes).

It checks: no deadlock; no mbarrier phase receives more arrivals than its
count; every score MMA reads the key/value stage and query slot holding the
tile and item it expects; the score buffer is never overwritten before every
share of the softmax read it; both shares of a row take the same exchanged
values; every output (the (m, l) pair of a partial row, each share's columns
of its O row, each token row) is written exactly once.
"""
import random
import sys

TOK = 128


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completions = name, count, 0, 0
        self.tx = 0

    def arrive(self, n=1):
        self.pending += n
        self._check()

    def expect_tx(self, b):
        self.tx += b
        self.arrive()

    def complete_tx(self, b):
        self.tx -= b
        self._check()

    def _check(self):
        if self.pending >= self.count and self.tx == 0:
            assert self.pending == self.count, (self.name, self.pending)
            self.pending = 0
            self.completions += 1

    def passed(self, parity):
        return (self.completions & 1) != parity


def decode_item(p, item):
    it = {}
    NW = p["NW"]
    if p["mode"] == "split":
        G = p["row_groups"]
        g = item % G
        rest = item // G
        c = rest % p["chunks"]
        it["bh"] = rest // p["chunks"]
        it["qrow0"] = g * (128 if p["interleave"] else NW * 128)
        it["t_begin"] = c * p["chunk_tiles"]
        it["t_end"] = min(p["kv_tiles"], it["t_begin"] + p["chunk_tiles"])
        it["part"] = NW * c if p["interleave"] else c
    else:
        pi = item % p["q_groups"]
        it["bh"] = item // p["q_groups"]
        it["qrow0"] = pi * NW * 128
        it["t_begin"], it["t_end"], it["part"] = 0, p["kv_tiles"], 0
    return it


def simulate(p, grid, NST, QS, seed):
    rng = random.Random(seed)
    events = []  # (time, fn)
    now = [0]

    def later(fn):
        events.append((now[0] + rng.randint(1, 30), fn))

    bars = {}
    for i in range(NST):
        bars[f"kv_full{i}"] = Bar(f"kv_full{i}", 1); bars[f"kv_empty{i}"] = Bar(f"kv_empty{i}", 1 if p["interleave"] else p["NW"])
    for i in range(QS):
        bars[f"q_full{i}"] = Bar(f"q_full{i}", 1); bars[f"q_empty{i}"] = Bar(f"q_empty{i}", p["NW"])
    CS = p.get("CS", 1)
    for w in range(p["NW"]):
        # plant "sfree_one_share": the score buffer released by one share only
        sfree_count = 4 if p.get("plant") == "sfree_one_share" else 4 * CS
        bars[f"sfull{w}"] = Bar(f"sfull{w}", 1); bars[f"sfree{w}"] = Bar(f"sfree{w}", sfree_count)
        bars[f"pfull{w}"] = Bar(f"pfull{w}", 4 * CS); bars[f"pfree{w}"] = Bar(f"pfree{w}", 1)
        bars[f"xbar{w}"] = Bar(f"xbar{w}", CS)       # one arrival per share (all its lanes)
    xvals = {}                                        # (row tile, exchange index) -> {share: value}
    writes = p["writes"]
    # buffer state for hazards
    S_state = ["free"] * p["NW"]
    S_reads = [0] * p["NW"]                           # shares that have read the current scores
    kv_contents = [None] * NST
    q_contents = [None] * QS
    outstanding_mma = []            # list of (bars_to_commit...) - commits complete when all prior done

    blk = p["blk"]

    R = NST // p["NW"]

    def producer():
        kv_load = q_load = 0
        wg_load = [0] * p["NW"]
        for item in range(blk, p["items"], grid):
            it = decode_item(p, item)
            slot = q_load % QS
            yield ("wait", f"q_empty{slot}", ((q_load // QS) & 1) ^ 1)
            nbytes = 1 if p["interleave"] else p["NW"]
            q_contents[slot] = item
            bars[f"q_full{slot}"].expect_tx(nbytes)
            for _ in range(nbytes):
                later(lambda s=slot: bars[f"q_full{s}"].complete_tx(1))
            qz_planes = p["q_planes"]
            qz = (it["bh"] % p["H"]) if p["q_shared"] else it["bh"]
            assert 0 <= qz < qz_planes
            q_load += 1
            for t in range(it["t_begin"], it["t_end"]):
                if p["interleave"] and not p.get("shared_ring"):
                    ow = (t - it["t_begin"]) % p["NW"]
                    st = ow * R + wg_load[ow] % R
                    fill = wg_load[ow] // R
                    wg_load[ow] += 1
                else:
                    st = kv_load % NST
                    fill = kv_load // NST
                yield ("wait", f"kv_empty{st}", (fill & 1) ^ 1)
                kv_contents[st] = (it["bh"], t)
                n = 1 if p["kv_same"] else 2
                bars[f"kv_full{st}"].expect_tx(n)
                for _ in range(n):
                    later(lambda s=st: bars[f"kv_full{s}"].complete_tx(1))
                assert 0 <= t * p["KT"] < p["kv_rows"] + p["KT"]
                kv_load += 1

    def mma(w):
        chain = {"t": 0}

        def commit(name):
            chain["t"] = max(chain["t"], now[0]) + rng.randint(1, 20)
            events.append((chain["t"], lambda: bars[name].arrive()))

        class Cur:
            pass

        state = {"ok": True}

        def settle(c, score):
            while c.item < p["items"]:
                c.info = decode_item(p, c.item)
                c.t = c.info["t_begin"] + (w if p["interleave"] else 0)
                assert w < p["NW"]
                c.nj = 0
                if c.t < c.info["t_end"]:
                    c.valid = True
                    return
                if score:
                    slot = c.item_count % QS
                    yield ("wait", f"q_full{slot}", (c.item_count // QS) & 1)
                    commit(f"q_empty{slot}")
                c.tiles_before += c.info["t_end"] - c.info["t_begin"]
                c.item_count += 1
                c.item += grid
            c.valid = False

        def first(c, score):
            c.item = blk; c.tiles_before = 0; c.item_count = 0
            yield from settle(c, score)

        def nxt(c, score):
            c.nj += 1
            c.t += p["NW"] if p["interleave"] else 1
            if c.t < c.info["t_end"]:
                return
            c.tiles_before += c.info["t_end"] - c.info["t_begin"]
            c.item_count += 1
            c.item += grid
            yield from settle(c, score)

        s_iss = [0]; pv_iss = [0]

        def stage_of(c, j):
            if p["interleave"] and not p.get("shared_ring"):
                return w * R + j % R, j // R
            g = c.tiles_before + (c.t - c.info["t_begin"])
            return g % NST, g // NST

        def issue_s(c):
            slot = c.item_count % QS
            if c.nj == 0:
                yield ("wait", f"q_full{slot}", (c.item_count // QS) & 1)
            st, fill = stage_of(c, s_iss[0])
            yield ("wait", f"kv_full{st}", fill & 1)
            assert kv_contents[st] == (c.info["bh"], c.t), ("kv stage holds wrong tile", kv_contents[st], c.t)
            assert q_contents[slot] == c.item, ("q slot holds wrong item", q_contents[slot], c.item)
            yield ("wait", f"sfree{w}", (s_iss[0] & 1) ^ 1)
            assert S_state[w] == "free" or (S_state[w] == "read" and S_reads[w] == CS), \
                ("S overwritten before read", w, S_state[w], S_reads[w])
            S_reads[w] = 0
            S_state[w] = "computing"
            commit(f"sfull{w}")
            s_iss[0] += 1
            if c.t + (p["NW"] if p["interleave"] else 1) >= c.info["t_end"]:
                commit(f"q_empty{slot}")

        def issue_pv(c):
            yield ("wait", f"pfull{w}", pv_iss[0] & 1)
            st, _ = stage_of(c, pv_iss[0])
            assert kv_contents[st] == (c.info["bh"], c.t), ("V stage holds wrong tile", kv_contents[st], c.t)
            commit(f"pfree{w}")
            pv_iss[0] += 1
            commit(f"kv_empty{st}")

        sc, pc = Cur(), Cur()
        yield from first(sc, True)
        yield from first(pc, False)
        if sc.valid:
            yield from issue_s(sc); yield from nxt(sc, True)
        while pc.valid:
            if sc.valid:
                yield from issue_s(sc); yield from nxt(sc, True)
            yield from issue_pv(pc); yield from nxt(pc, False)

    def softmax(wg, half):
        sfull_waits = pfree_waits = jobs_done = 0
        xph = [0]
        defer = p["mode"] == "decode"

        def exchange(value):
            # the kernel's exchange(): publish, arrive, wait for the other share
            if CS == 1:
                return value
            key = (wg, xph[0])
            xvals.setdefault(key, {})[half] = value
            bars[f"xbar{wg}"].arrive()
            yield ("wait", f"xbar{wg}", xph[0] & 1)
            other = xvals[key][half ^ 1]
            xph[0] += 1
            return other

        def outputs(it, njobs):
            for row in range(128):
                if p["mode"] == "split":
                    r = it["qrow0"] + (0 if p["interleave"] else wg * 128) + row
                    part = it["part"] + wg if p["interleave"] else it["part"]
                    if r < p["M"]:
                        assert part < p["parts"]
                        keys = [("O", part, it["bh"], r, half)]          # each share its D / CS columns
                        if half == 0:
                            keys.append(("ml", part, it["bh"], r))
                        for key in keys:
                            writes[key] = writes.get(key, 0) + 1
                else:
                    n = it["qrow0"] + wg * 128 + row
                    if n < p["N"] and njobs > 0:
                        key = ("y", it["bh"], n, half)
                        writes[key] = writes.get(key, 0) + 1

        pend = None
        for item in range(blk, p["items"], grid):
            it = decode_item(p, item)
            njobs = 0
            step = p["NW"] if p["interleave"] else 1
            for t in range(it["t_begin"] + (wg if p["interleave"] else 0), it["t_end"], step):
                yield ("wait", f"sfull{wg}", sfull_waits & 1)
                sfull_waits += 1
                assert S_state[wg] in ("computing", "read") or True
                S_state[wg] = "read"
                S_reads[wg] += 1
                if p.get("plant") != "sfree_one_share" or half == 0:
                    for _ in range(4):
                        bars[f"sfree{wg}"].arrive()
                mine = (item, t, half)
                other = yield from exchange(mine)
                if CS > 1:
                    assert other == (item, t, half ^ 1), ("exchange pairs different jobs", mine, other)

                while pfree_waits < jobs_done:
                    yield ("wait", f"pfree{wg}", pfree_waits & 1)
                    pfree_waits += 1
                if defer and pend is not None:
                    outputs(*pend)
                    pend = None
                for _ in range(4):
                    bars[f"pfull{wg}"].arrive()
                jobs_done += 1; njobs += 1
            if njobs == 0:
                outputs(it, 0)
            elif defer:
                other = yield from exchange(("l", item, half))
                if CS > 1:
                    assert other == ("l", item, half ^ 1), ("row-sum exchange pairs different items", other)
                pend = (it, njobs)
            else:
                other = yield from exchange(("l", item, half))
                if CS > 1:
                    assert other == ("l", item, half ^ 1), ("row-sum exchange pairs different items", other)
                while pfree_waits < jobs_done:
                    yield ("wait", f"pfree{wg}", pfree_waits & 1)
                    pfree_waits += 1
                outputs(it, njobs)
        if pend is not None:
            while pfree_waits < jobs_done:
                yield ("wait", f"pfree{wg}", pfree_waits & 1)
                pfree_waits += 1
            outputs(*pend)

    NWc = p["NW"]
    roles = [producer()] + [mma(w) for w in range(NWc)] + [softmax(w, h) for w in range(NWc) for h in range(CS)]
    state = [None] * len(roles)
    done = [False] * len(roles)
    steps = 0
    while not all(done):
        progressed = False
        order = list(range(len(roles))); rng.shuffle(order)
        for i in order:
            if done[i]:
                continue
            if state[i] is not None:
                _, b, par = state[i]
                if not bars[b].passed(par):
                    continue
            try:
                state[i] = next(roles[i])
            except StopIteration:
                done[i] = True
                state[i] = None
            progressed = True
        # fire events
        events.sort(key=lambda e: e[0])
        if events and (not progressed or rng.random() < 0.5):
            now[0] = max(now[0], events[0][0])
            events.pop(0)[1]()
            progressed = True
        if not progressed:
            raise RuntimeError(f"deadlock: states={state}")
        steps += 1
    while events:
        events.sort(key=lambda e: e[0]); events.pop(0)[1]()


def choose_chunks(units, tiles, sms=148, jobs_div=1):
    # Same cost model as the host planner: waves * (2 + jobs per item).
    best_c, best = 1, float("inf")
    for c in range(1, tiles + 1):
        per = -(-tiles // c)
        if c > 1 and -(-tiles // per) < c:
            continue
        cost = -(-units * c // sms) * (2 + -(-per // jobs_div))
        if cost <= best:
            best, best_c = cost, c
    return best_c


def check(B, H, N, M, D, grid=148, mode="both", seed=0, force_chunks=0, NW=3, shared_ring=False, CS=None,
          plant=None):
    BH = B * H
    KT = 64 if NW == 3 else 128
    kv_tiles = (N + KT - 1) // KT
    inter = NW == 3 or M <= 128
    rg = (M + 127) // 128 if inter else (M + NW * 128 - 1) // (NW * 128)
    chunks = force_chunks or choose_chunks(BH * rg, kv_tiles, jobs_div=NW if inter else 1)
    chunks = min(chunks, kv_tiles)
    tpc = -(-kv_tiles // chunks)
    chunks = -(-kv_tiles // tpc)
    NST = (6 if D == 64 else 9) if NW == 3 else (4 if D == 64 else 6)
    res = []
    for md in (["split", "decode"] if mode == "both" else [mode]):
        for kv_same in ([1, 0] if md == "split" else [0]):
            if md == "split":
                p = dict(mode="split", NW=NW, H=H, M=M, N=N, kv_rows=N, kv_tiles=kv_tiles, interleave=inter,
                         row_groups=rg, chunks=chunks, chunk_tiles=tpc, items=BH * chunks * rg,
                         q_shared=1, q_planes=H, kv_same=kv_same, parts=chunks * (NW if inter else 1))
            else:
                qg = -(-N // (NW * 128))
                p = dict(mode="decode", NW=NW, H=H, M=M, N=N, kv_rows=M, kv_tiles=-(-M // KT), interleave=False,
                         q_groups=qg, items=BH * qg, q_shared=0, q_planes=BH, kv_same=0, parts=1)
            p["KT"] = KT
            p["D"] = D
            # the kernel splits the score columns between two warps per row in
            # the split passes on 128-column jobs at D = 64
            p["CS"] = CS if CS is not None else (2 if md == "split" and KT == 128 and D == 64 else 1)
            p["shared_ring"] = shared_ring
            p["plant"] = plant
            g = min(grid, p["items"])
            writes = {}
            p["writes"] = writes
            for blk in range(g):
                p["blk"] = blk
                simulate(p, g, NST, 2, seed=blk + 7919 * seed)
            shares = list(range(p["CS"]))
            if md == "split":
                exp = {("ml", pt, bh, r) for bh in range(BH) for r in range(M) for pt in range(p["parts"])}
                exp |= {("O", pt, bh, r, h) for bh in range(BH) for r in range(M) for pt in range(p["parts"])
                        for h in shares}
            else:
                exp = {("y", bh, n, h) for bh in range(BH) for n in range(N) for h in shares}
            assert set(writes) == exp, (md, len(set(writes) ^ exp))
            assert all(v == 1 for v in writes.values()), md
            res.append((md, kv_same, p["items"], g, chunks))
    return res


