"""CPU model of the backward kernel's mbarrier protocol (bwd_tc::bwd_kernel,
csrc/kernels_bwd_tc.cuh).

The kernel's roles -- the TMA producer (row tiles in QS slots, a ring of NST
column stages, column statistics on the same barrier), one MMA issuer per
softmax warpgroup (score and dP MMAs one job ahead of the accumulating MMAs),
the softmax warpgroups (4 warps arriving on sfree and pfull, column
statistics read from the stage after an acquire on its full barrier, the
epilogue after the last accumulating MMA of the item) -- run as coroutines
that wait on mbarriers with the kernel's arrival counts and phase parities,
in random interleavings, with TMA and MMA completions arriving after random
delays.  Item decoding and chunking mirror the kernel.

Checked: no deadlock; no mbarrier phase gets more arrivals than its count;
every score MMA reads the row slot holding its item and the column stage
holding its tile; every accumulating MMA reads the stage holding its tile and
the P/dS buffer holding its job; the softmax reads column statistics from the
stage holding its tile; S/dP is never overwritten before the softmax read it,
nor P/dS while an accumulating MMA still reads it; the accumulators are never
reset for an item before the previous item's epilogue read them; every
output row is written exactly once.
"""
import random

from protocol_model import Bar

QT = 128      # rows per warpgroup tile
KT = 32       # columns per job
KT_WIDE = 64  # columns per job of a latent pass with one accumulator and row statistics


def decode_item(p, item):
    g = item % p["row_groups"]
    rest = item // p["row_groups"]
    chunk = rest % p["chunks"]
    bh = rest // p["chunks"]
    t0 = chunk * p["chunk_tiles"]
    return dict(bh=bh, row0=g * p["NW"] * QT, t_begin=t0, t_end=min(p["col_tiles"], t0 + p["chunk_tiles"]),
                chunk=chunk)


def simulate(p, blk, grid, seed, writes):
    rng = random.Random(seed)
    NW, NST, QS = p["NW"], p["NST"], p["QS"]
    events = []
    now = [0]

    def later(fn, lo=1, hi=30):
        events.append((now[0] + rng.randint(lo, hi), fn))

    bars = {}
    for i in range(QS):
        bars[f"row_full{i}"] = Bar(f"row_full{i}", 1)
        bars[f"row_empty{i}"] = Bar(f"row_empty{i}", NW)
    for i in range(NST):
        bars[f"col_full{i}"] = Bar(f"col_full{i}", 1)
        bars[f"col_empty{i}"] = Bar(f"col_empty{i}", NW)
    for w in range(NW):
        bars[f"sfull{w}"] = Bar(f"sfull{w}", 1)
        bars[f"sfree{w}"] = Bar(f"sfree{w}", 4)
        bars[f"pfull{w}"] = Bar(f"pfull{w}", 4)
        bars[f"pfree{w}"] = Bar(f"pfree{w}", 1)

    row_contents = [None] * QS          # item whose row tiles the slot holds
    col_contents = [None] * NST         # (bh, t) whose column tiles and statistics the stage holds
    S_state = ["free"] * NW             # free / computing / ready / read
    P_job = [None] * NW                 # job whose P, dS the warpgroup's TMEM buffer holds
    P_readers = [0] * NW                # accumulating MMAs still reading P/dS
    acc_item = [None] * NW              # item the accumulators belong to
    acc_done = [{} for _ in range(NW)]  # item -> its accumulating MMAs completed
    epilogue_done = [set() for _ in range(NW)]

    def producer():
        ic = g = 0
        for item in range(blk, p["items"], grid):
            it = decode_item(p, item)
            slot = ic % QS
            yield ("wait", f"row_empty{slot}", ((ic // QS) & 1) ^ 1)
            row_contents[slot] = item
            n = NW * p["row_tiles"]
            bars[f"row_full{slot}"].expect_tx(n)
            for _ in range(n):
                later(lambda s=slot: bars[f"row_full{s}"].complete_tx(1))
            ic += 1
            for t in range(it["t_begin"], it["t_end"]):
                st = g % NST
                yield ("wait", f"col_empty{st}", ((g // NST) & 1) ^ 1)
                col_contents[st] = (it["bh"], t)
                n = p["col_tiles_per_stage"] + (1 if p["col_stats"] else 0)
                bars[f"col_full{st}"].expect_tx(n)
                for _ in range(n):
                    later(lambda s=st: bars[f"col_full{s}"].complete_tx(1))
                g += 1

    def jobs():
        """The CTA's job stream: (item, info, t, ic, g, first, last)."""
        ic = g = 0
        for item in range(blk, p["items"], grid):
            it = decode_item(p, item)
            for t in range(it["t_begin"], it["t_end"]):
                yield item, it, t, ic, g, t == it["t_begin"], t + 1 >= it["t_end"]
                g += 1
            ic += 1

    def mma(w):
        chain = {"t": 0}

        def commit(fn):
            # MMA completions of one issuer land in issue order
            chain["t"] = max(chain["t"], now[0]) + rng.randint(1, 20)
            events.append((chain["t"], fn))

        s_issued = [0]
        a_issued = [0]

        def issue_s(j):
            item, it, t, ic, g, first, last = j
            slot = ic % QS
            if first:
                yield ("wait", f"row_full{slot}", (ic // QS) & 1)
            st = g % NST
            yield ("wait", f"col_full{st}", (g // NST) & 1)
            yield ("wait", f"sfree{w}", (s_issued[0] & 1) ^ 1)
            assert row_contents[slot] == item, ("row slot holds wrong item", row_contents[slot], item)
            assert col_contents[st] == (it["bh"], t), ("column stage holds wrong tile", col_contents[st], t)
            assert S_state[w] in ("free", "read"), ("S/dP overwritten before read", w, S_state[w])
            S_state[w] = "computing"

            def done(w=w):
                S_state[w] = "ready"
                bars[f"sfull{w}"].arrive()
            commit(done)
            s_issued[0] += 1
            if last:
                commit(lambda s=slot: bars[f"row_empty{s}"].arrive())

        def issue_acc(j):
            item, it, t, ic, g, first, last = j
            yield ("wait", f"pfull{w}", a_issued[0] & 1)
            st = g % NST
            assert col_contents[st] == (it["bh"], t), ("accumulating MMA: stage holds wrong tile", t)
            assert P_job[w] == (item, t), ("accumulating MMA reads the wrong P/dS", P_job[w], (item, t))
            if first:
                assert acc_item[w] is None or acc_item[w] in epilogue_done[w], \
                    ("accumulators reset before the previous item's epilogue", acc_item[w])
                acc_item[w] = item
            P_readers[w] += 1

            def done(w=w, st=st, item=item):
                P_readers[w] -= 1
                acc_done[w][item] = acc_done[w].get(item, 0) + 1
                bars[f"pfree{w}"].arrive()
                bars[f"col_empty{st}"].arrive()
            commit(done)
            a_issued[0] += 1

        s_stream, a_stream = jobs(), jobs()
        sj = next(s_stream, None)
        aj = next(a_stream, None)
        if sj is not None:
            yield from issue_s(sj)
            sj = next(s_stream, None)
        while aj is not None:
            if sj is not None:
                yield from issue_s(sj)
                sj = next(s_stream, None)
            yield from issue_acc(aj)
            aj = next(a_stream, None)

    def softmax(wg):
        sfull_waits = pfree_waits = jobs_done = 0
        pend = None                      # the finished item whose epilogue is deferred

        def epilogue(item, it):
            assert acc_item[wg] == item, ("epilogue reads another item's accumulators", acc_item[wg], item)
            assert P_readers[wg] == 0, ("epilogue while an accumulating MMA still runs", wg)
            assert acc_done[wg].get(item, 0) == it["t_end"] - it["t_begin"], \
                ("epilogue before the item's last accumulation", acc_done[wg].get(item, 0))
            epilogue_done[wg].add(item)
            for row in range(QT):
                r = it["row0"] + wg * QT + row
                if r < p["row_count"]:
                    key = (it["chunk"], it["bh"], r)
                    writes[key] = writes.get(key, 0) + 1

        for item, it, t, ic, g, first, last in jobs():
            yield ("wait", f"sfull{wg}", sfull_waits & 1)
            sfull_waits += 1
            assert S_state[wg] == "ready", ("S/dP read before computed", S_state[wg])
            S_state[wg] = "read"
            for _ in range(4):
                bars[f"sfree{wg}"].arrive()
            st = g % NST
            if p["col_stats"]:
                yield ("wait", f"col_full{st}", (g // NST) & 1)
                assert col_contents[st] == (it["bh"], t), ("statistics of the wrong tile", col_contents[st], t)
            while pfree_waits < jobs_done and not p.get("skip_pfree_wait"):
                yield ("wait", f"pfree{wg}", pfree_waits & 1)
                pfree_waits += 1
            assert P_readers[wg] == 0, ("P/dS overwritten while an accumulating MMA reads it", wg)
            P_job[wg] = (item, t)
            if pend is not None and not p.get("no_deferred_wait"):
                # the previous item's accumulators, read before this job's
                # accumulating MMA (released by pfull) overwrites them
                epilogue(*pend)
                pend = None
            for _ in range(4):
                bars[f"pfull{wg}"].arrive()
            jobs_done += 1
            if last:
                if p.get("no_deferred_wait"):
                    # planted: the epilogue without waiting for the item's last accumulating MMA
                    epilogue(item, it)
                elif p["deferred"]:
                    pend = (item, it)
                else:
                    while pfree_waits < jobs_done:
                        yield ("wait", f"pfree{wg}", pfree_waits & 1)
                        pfree_waits += 1
                    epilogue(item, it)
        if pend is not None:
            while pfree_waits < jobs_done:
                yield ("wait", f"pfree{wg}", pfree_waits & 1)
                pfree_waits += 1
            epilogue(*pend)

    roles = [producer()] + [mma(w) for w in range(NW)] + [softmax(w) for w in range(NW)]
    state = [None] * len(roles)
    done = [False] * len(roles)
    while not all(done):
        progressed = False
        order = list(range(len(roles)))
        rng.shuffle(order)
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
        events.sort(key=lambda e: e[0])
        if events and (not progressed or rng.random() < 0.5):
            now[0] = max(now[0], events[0][0])
            events.pop(0)[1]()
            progressed = True
        if not progressed:
            raise RuntimeError(f"deadlock: states={state}")
    while events:
        events.sort(key=lambda e: e[0])
        events.pop(0)[1]()


def choose_chunks(units, tiles, sms=148):
    # the forward split pass's cost model, as the backward's host planner uses it
    best_c, best = 1, float("inf")
    for c in range(1, tiles + 1):
        per = -(-tiles // c)
        if c > 1 and -(-tiles // per) < c:
            continue
        cost = -(-units * c // sms) * (2 + per)
        if cost <= best:
            best, best_c = cost, c
    return best_c


def check(B, H, N, M, D, side, col_stats, grid=148, seed=0, force_chunks=0, dual=False, skip_pfree_wait=False,
          no_deferred_wait=False):
    """side: "latent" (rows = M latents, columns = a chunk of the N tokens) or
    "token" (rows = N tokens, columns = all M latents); col_stats: the
    statistics come with the column tiles (else they belong to the rows)."""
    BH = B * H
    NW = 1 if D == 128 else 2
    rows, cols = (M, N) if side == "latent" else (N, M)
    rg = -(-rows // (NW * QT))
    if side == "latent":
        # tokens per chunk: a multiple of the wide tile, planned over wide tiles;
        # a latent pass with row statistics and two warpgroups takes wide jobs
        wide = -(-cols // KT_WIDE)
        c = min(force_chunks or choose_chunks(BH * rg, wide), wide)
        chunk_len = -(-wide // c) * KT_WIDE
        kt = KT_WIDE if (NW == 2 and not col_stats and not dual) else KT
        col_tiles = -(-cols // kt)
        tpc = chunk_len // kt
        chunks = -(-col_tiles // tpc)
        assert chunks == -(-cols // chunk_len)          # the partial slots the reduction reads
    else:
        # the synthesis token side (one accumulator after merging) takes wide jobs
        kt = KT_WIDE if (NW == 2 and not dual) else KT
        col_tiles = -(-cols // kt)
        tpc = col_tiles
        chunks = 1
    p = dict(NW=NW, NST=4, QS=1 if dual else 2, row_groups=rg, chunks=chunks, chunk_tiles=tpc,
             col_tiles=col_tiles, items=BH * chunks * rg, row_count=rows,
             row_tiles=3 if dual else 2, col_tiles_per_stage=3 if dual else 2,
             col_stats=dual or col_stats, skip_pfree_wait=skip_pfree_wait, no_deferred_wait=no_deferred_wait,
             deferred=dual)
    g = min(grid, p["items"])
    writes = {}
    for blk in range(g):
        simulate(p, blk, g, seed=blk + 7919 * seed, writes=writes)
    exp = {(c, bh, r) for bh in range(BH) for r in range(rows) for c in range(chunks)}
    assert set(writes) == exp, (side, len(set(writes) ^ exp))
    assert all(v == 1 for v in writes.values())
    return p["items"], g, chunks
