"""Randomized model checks of the mbarrier protocols of the pipelined kernels (the
forward's fused attention kernel, its state kernel and state chain, the backward's
dq and dk/dv kernels and reverse chain, the projection GEMMs on one CTA and on a CTA
pair): every role of a CTA is
written as a step function that waits on barriers by completion index, TMA copies
and tensor-core commits complete at random later times (commits in issue order,
each after every product issued before it), and a random scheduler interleaves
everything. Each run must finish (no deadlock) and no barrier may ever be more than
one phase ahead of a waiter that still has to observe an earlier phase (a parity
wait would then miss it). This checks the protocol as written in the kernels' loop
structure, for every tile count they meet; it runs no GPU code."""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self, n=1, tag=None):
        # a tagged arrival belongs to phase `tag` (counted from 0): it must not land
        # while the barrier is still in an earlier phase or already in a later one
        assert tag is None or tag == self.done, \
            f"{self.name}: arrival for phase {tag} while in phase {self.done}"
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than the count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class Sim:
    """Roles are generators yielding ('wait', bar, k) (wait for completion k, counted
    from 0), ('arrive', bar, n[, tag]), ('tma', bar[, tag]) (a copy that completes bar
    later), ('mma',) (a product), ('commit', bar or [bars]) (arrives on the bar, or on
    each bar of a multicast list, once every earlier product is done) or ('named', id,
    members) (a named barrier of the CTA, or of a cluster). An optional tag names the
    phase an arrival belongs to (checked by Bar.arrive)."""

    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.bars = {}
        self.tma = []          # pending copies (bar)
        self.mma_queue = []    # issued products and commits, in order

    def bar(self, name, count=1):
        self.bars[name] = Bar(name, count)
        return self.bars[name]

    def run(self, roles, max_steps=2_000_000):
        state = {r: None for r in roles}   # the pending request of each role
        for step in range(max_steps):
            ready = []
            for r, req in list(state.items()):
                if req is None:
                    try:
                        req = next(roles[r])
                    except StopIteration:
                        del state[r]
                        continue
                    state[r] = req
                if req[0] == 'wait':
                    b, k = req[1], req[2]
                    # a waiter for completion k must not find the barrier past k + 1 (its
                    # parity would then match a later phase) nor before k (it would match
                    # an older one)
                    assert b.done <= k + 1, f"{b.name}: phase skipped (waiter for {k}, done {b.done})"
                    assert b.done >= k, f"{b.name}: stale phase (waiter for {k}, done {b.done})"
                    if b.done >= k + 1:
                        ready.append(r)
                elif req[0] == 'named':
                    nid, members = req[1], req[2]
                    arrived = [x for x in members if x in state and state[x] is not None
                               and state[x][0] == 'named' and state[x][1] == nid]
                    if len(arrived) == len(members):
                        ready.append(r)
                else:
                    ready.append(r)
            events = []  # asynchronous completions (named apart from the roles)
            if self.tma:
                events.append('<copy done>')
            if self.mma_queue:
                events.append('<product done>')
            if not state and not self.tma and not self.mma_queue:
                return step
            if not ready and not events:
                raise AssertionError("deadlock: " + ", ".join(
                    f"{r} waits {req[1].name if hasattr(req[1], 'name') else req[1]}"
                    f"#{req[2] if len(req) > 2 else ''}" for r, req in state.items()))
            choice = self.rng.choice(ready + events)
            if choice == '<copy done>':
                b, tag = self.tma.pop(self.rng.randrange(len(self.tma)))
                b.arrive(1, tag)
            elif choice == '<product done>':
                item = self.mma_queue.pop(0)   # in issue order
                for b in (item if isinstance(item, list) else [item] if item else []):
                    b.arrive()
            else:
                req = state[choice]
                kind = req[0]
                if kind == 'arrive':
                    req[1].arrive(req[2], req[3] if len(req) > 3 else None)
                elif kind == 'tma':
                    self.tma.append((req[1], req[2] if len(req) > 2 else None))
                elif kind == 'mma':
                    self.mma_queue.append(None)
                elif kind == 'commit':
                    self.mma_queue.append(req[1])
                elif kind == 'named':
                    nid, members = req[1], req[2]
                    for m in members:
                        state[m] = None
                    continue
                state[choice] = None
        raise AssertionError("did not finish")


# ------------------------------------------------------------------------------
# dq kernel: loads n = 0 .. 2 nk - 1 (two sweeps over nk key tiles), halves h = 2n + a
# ------------------------------------------------------------------------------
def dq_roles(sim, nk):
    nl, nh = 2 * nk, 4 * nk
    ONCE, X, DONE, M1, M2 = (sim.bar(n) for n in ("once", "x", "done", "m1", "m2"))
    FULL = [sim.bar(f"full{i}") for i in range(2)]
    FREE = [sim.bar(f"free{i}") for i in range(2)]
    SFULL = [sim.bar(f"sfull{i}") for i in range(2)]
    PFULL = [sim.bar(f"pfull{i}", 4) for i in range(2)]
    SK, SK2 = sim.bar("sk", 8), sim.bar("sk2", 8)

    def producer():
        yield ('tma', ONCE)
        for n in range(nl):
            st = n & 1
            if n >= 2:
                yield ('wait', FREE[st], (n >> 1) - 1)
            yield ('tma', FULL[st])
        yield ('wait', FREE[0], (nl - 2) >> 1)
        yield ('tma', X)

    def mma():
        def issue_sdp(h):
            n, a = h >> 1, h & 1
            st = n & 1
            if a == 0:
                yield ('wait', FULL[st], n >> 1)
            yield ('mma',)
            yield ('commit', SFULL[a])
            if n < nk and a == 1:
                yield ('commit', FREE[st])
        yield ('wait', ONCE, 0)
        yield from issue_sdp(0)
        yield from issue_sdp(1)
        for h in range(nh):
            n, a = h >> 1, h & 1
            yield ('wait', PFULL[a], n)
            if n >= nk:
                yield ('mma',)
                if a == 1:
                    yield ('commit', FREE[n & 1])
            if h + 2 < nh:
                yield from issue_sdp(h + 2)
        yield ('commit', DONE)
        yield ('wait', X, 0)
        yield ('wait', SK, 0)
        yield ('mma',)
        yield ('commit', M1)
        yield ('wait', SK2, 0)
        yield ('mma',)
        yield ('commit', M2)

    wgs = ("wg0", "wg1")

    def wg(w):
        for n in range(nk):
            yield ('wait', SFULL[w], n)
            yield ('arrive', PFULL[w], 4)
        yield ('named', 'merge', wgs)
        for n in range(nk, nl):
            yield ('wait', SFULL[w], n)
            yield ('arrive', PFULL[w], 4)
        yield ('wait', DONE, 0)
        yield ('wait', X, 0)
        yield ('named', 'den', wgs)
        yield ('arrive', SK, 4)
        yield ('wait', M1, 0)
        yield ('named', 'dd', wgs)
        yield ('arrive', SK2, 4)
        yield ('wait', M2, 0)
        yield ('named', 'sums', wgs)

    return {"producer": producer(), "mma": mma(), "wg0": wg(0), "wg1": wg(1)}


# ------------------------------------------------------------------------------
# dk/dv kernel: loads n = 0 .. nl - 1 (query tiles at or after the key tile)
# ------------------------------------------------------------------------------
def dkdv_roles(sim, nl, delta):
    nh = 2 * nl
    sx = nl & 1
    ONCE, X, DONE, M1, M2 = (sim.bar(n) for n in ("once", "x", "done", "m1", "m2"))
    FULL = [sim.bar(f"full{i}") for i in range(2)]
    FREE = [sim.bar(f"free{i}") for i in range(2)]
    SFULL = [sim.bar(f"sfull{i}") for i in range(2)]
    PFULL = [sim.bar(f"pfull{i}", 4) for i in range(2)]
    SK, SK2 = sim.bar("sk", 8), sim.bar("sk2", 8)

    def producer():
        yield ('tma', ONCE)
        for n in range(nl):
            st = n & 1
            if n >= 2:
                yield ('wait', FREE[st], (n >> 1) - 1)
            yield ('tma', FULL[st])
        if nl >= 2:
            yield ('wait', FREE[sx], (nl - 2) >> 1)
        yield ('tma', X)

    def mma():
        def issue_sdp(h):
            n, a = h >> 1, h & 1
            if a == 0:
                yield ('wait', FULL[n & 1], n >> 1)
            yield ('mma',)
            yield ('commit', SFULL[a])
        yield ('wait', ONCE, 0)
        yield from issue_sdp(0)
        yield from issue_sdp(1)
        for h in range(nh):
            n, a = h >> 1, h & 1
            yield ('wait', PFULL[a], n)
            yield ('mma',)
            if a == 1:
                yield ('commit', FREE[n & 1])
            if h + 2 < nh:
                yield from issue_sdp(h + 2)
        yield ('commit', DONE)
        yield ('wait', X, 0)
        yield ('wait', SK, 0)
        yield ('mma',)
        yield ('commit', M1)
        if delta:
            yield ('wait', SK2, 0)
            yield ('mma',)
            yield ('commit', M2)

    wgs = ("wg0", "wg1")

    def wg(w):
        for n in range(nl):
            yield ('wait', FULL[n & 1], n >> 1)
            yield ('wait', SFULL[w], n)
            yield ('arrive', PFULL[w], 4)
        yield ('wait', DONE, 0)
        if delta:
            yield ('wait', X, 0)
        yield ('named', 'den', wgs)
        yield ('arrive', SK, 4)
        if delta:
            yield ('wait', M1, 0)
            yield ('named', 'dd', wgs)
            yield ('arrive', SK2, 4)
            yield ('named', 'sdd', wgs)
            yield ('named', 'gz', wgs)
            yield ('wait', M2, 0)
        else:
            yield ('wait', M1, 0)

    return {"producer": producer(), "mma": mma(), "wg0": wg(0), "wg1": wg(1)}


# ------------------------------------------------------------------------------
# projection GEMM: a CTA's output tiles, k-steps through a ring, two accumulators
# ------------------------------------------------------------------------------
def gemm_roles(sim, tiles, ksteps, stages):
    FULL = [sim.bar(f"full{i}") for i in range(stages)]
    EMPTY = [sim.bar(f"empty{i}") for i in range(stages)]
    AFULL = [sim.bar(f"afull{i}") for i in range(2)]
    AEMPTY = [sim.bar(f"aempty{i}", 4) for i in range(2)]

    def producer():
        it = 0
        for _ in range(tiles):
            for _ in range(ksteps):
                st, use = it % stages, it // stages
                if use > 0:
                    yield ('wait', EMPTY[st], use - 1)
                yield ('tma', FULL[st])
                it += 1

    def mma():
        it = 0
        for lt in range(tiles):
            acc, use = lt & 1, lt >> 1
            if use > 0:
                yield ('wait', AEMPTY[acc], use - 1)
            for ks in range(ksteps):
                st = it % stages
                yield ('wait', FULL[st], it // stages)
                yield ('mma',)
                yield ('commit', EMPTY[st])
                if ks == ksteps - 1:
                    yield ('commit', AFULL[acc])
                it += 1

    def epilogue():
        for lt in range(tiles):
            yield ('wait', AFULL[lt & 1], lt >> 1)
            yield ('arrive', AEMPTY[lt & 1], 4)

    return {"producer": producer(), "mma": mma(), "epilogue": epilogue()}


# ------------------------------------------------------------------------------
# projection GEMM on a CTA pair (cluster of two, cta_group::2 MMAs from the even CTA):
# each CTA's copies complete on the even CTA's FULL barrier, whose producer expects the
# pair's bytes (count: its arrival + one completion per CTA's copies); the MMA commits
# are multicast to both CTAs' EMPTY / AFULL / DRAIN barriers; both CTAs' epilogues
# release an accumulator on the even CTA's AEMPTY (4 warps each); before the cluster
# barrier every producer waits for its stages' last release and the even CTA's MMA
# warp for the last accumulator releases.
# ------------------------------------------------------------------------------
def pair_gemm_roles(sim, tiles, ksteps, stages, full_count=3, empty_mask=(0, 1)):
    FULL = [sim.bar(f"full{i}", full_count) for i in range(stages)]        # CTA 0's
    EMPTY = [[sim.bar(f"empty{c}.{i}") for i in range(stages)] for c in range(2)]
    AFULL = [[sim.bar(f"afull{c}.{i}") for i in range(2)] for c in range(2)]
    AEMPTY = [sim.bar(f"aempty{i}", 8) for i in range(2)]                  # CTA 0's
    DRAIN = [sim.bar(f"drain{c}") for c in range(2)]
    members = [f"{r}{c}" for c in range(2) for r in ("producer", "mma", "epilogue")]

    def producer(c):
        it, last = 0, {}
        for _ in range(tiles):
            for _ in range(ksteps):
                st, use = it % stages, it // stages
                if use > 0:
                    yield ('wait', EMPTY[c][st], use - 1)
                if c == 0:
                    yield ('arrive', FULL[st], 1, use)   # arrive.expect_tx (the pair's bytes)
                yield ('tma', FULL[st], use)            # this CTA's A half and B half
                last[st] = use
                it += 1
        for st, use in last.items():                     # tail: no copy still landing
            yield ('wait', EMPTY[c][st], use)
        yield ('named', 'cluster', members)

    def mma(c):
        if c == 0:
            it = 0
            for lt in range(tiles):
                acc, use = lt & 1, lt >> 1
                if use > 0:
                    yield ('wait', AEMPTY[acc], use - 1)
                for ks in range(ksteps):
                    st = it % stages
                    yield ('wait', FULL[st], it // stages)
                    yield ('mma',)
                    yield ('commit', [EMPTY[x][st] for x in empty_mask])
                    if ks == ksteps - 1:
                        yield ('commit', [AFULL[0][acc], AFULL[1][acc]])
                    it += 1
            yield ('commit', [DRAIN[0], DRAIN[1]])
            for acc in range(2):                          # tail: the last releases landed
                uses = (tiles + 1 - acc) // 2
                if uses > 0:
                    yield ('wait', AEMPTY[acc], uses - 1)
        yield ('wait', DRAIN[c], 0)
        yield ('named', 'cluster', members)

    def epilogue(c):
        for lt in range(tiles):
            yield ('wait', AFULL[c][lt & 1], lt >> 1)
            yield ('arrive', AEMPTY[lt & 1], 4)
        yield ('named', 'cluster', members)

    roles = {}
    for c in range(2):
        roles[f"producer{c}"] = producer(c)
        roles[f"mma{c}"] = mma(c)
        roles[f"epilogue{c}"] = epilogue(c)
    return roles


@pytest.mark.parametrize("tiles,ksteps,stages", [(1, 1, 5), (3, 16, 5), (4, 4, 5), (7, 2, 5),
                                                 (2, 9, 3), (5, 16, 6)])
def test_pair_gemm_pipeline_protocol(tiles, ksteps, stages):
    for seed in range(40):
        sim = Sim(seed * 1000 + tiles * 10 + ksteps + stages)
        sim.run(pair_gemm_roles(sim, tiles, ksteps, stages))


def test_pair_gemm_model_detects_a_barrier_expecting_one_cta():
    """A FULL barrier that counts only the even CTA's copies completes early, and the
    odd CTA's copy then lands in the next phase."""
    with pytest.raises(AssertionError, match="arrival for phase|phase skipped|stale"):
        for seed in range(40):
            sim = Sim(seed)
            sim.run(pair_gemm_roles(sim, 4, 8, 5, full_count=2))


def test_pair_gemm_model_detects_a_commit_to_one_cta():
    """Ring stages released only in the even CTA: the odd CTA's producer never sees
    its stages free."""
    with pytest.raises(AssertionError, match="deadlock"):
        sim = Sim(1)
        sim.run(pair_gemm_roles(sim, 3, 8, 5, empty_mask=(0,)))


@pytest.mark.parametrize("nk", [1, 2, 3, 4, 7, 16])
def test_dq_pipeline_protocol(nk):
    for seed in range(40):
        sim = Sim(seed * 1000 + nk)
        sim.run(dq_roles(sim, nk))


@pytest.mark.parametrize("delta", [False, True])
@pytest.mark.parametrize("nl", [1, 2, 3, 4, 7, 16])
def test_dkdv_pipeline_protocol(nl, delta):
    for seed in range(40):
        sim = Sim(seed * 1000 + nl + 100 * delta)
        sim.run(dkdv_roles(sim, nl, delta))


@pytest.mark.parametrize("tiles,ksteps,stages", [(1, 1, 3), (3, 8, 3), (5, 16, 4), (2, 2, 4),
                                                 (7, 1, 3)])
def test_gemm_pipeline_protocol(tiles, ksteps, stages):
    for seed in range(40):
        sim = Sim(seed * 1000 + tiles * 10 + ksteps)
        sim.run(gemm_roles(sim, tiles, ksteps, stages))


def test_model_detects_a_phase_skip():
    """Planted mistake: the dq producer no longer waits for the ring stage to be freed
    before refilling it (FULL then completes twice before the MMA warp has seen the
    first completion)."""
    def broken(sim, nk):
        roles = dq_roles(sim, nk)
        FULL = [sim.bars["full0"], sim.bars["full1"]]
        ONCE = sim.bars["once"]

        def producer():
            yield ('tma', ONCE)
            for n in range(2 * nk):
                yield ('tma', FULL[n & 1])
        roles["producer"] = producer()
        return roles
    failures = 0
    for seed in range(40):
        sim = Sim(seed)
        try:
            sim.run(broken(sim, 4))
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_detects_a_deadlock():
    """Planted mistake: the dk/dv MMA warp frees a ring stage only after the next
    tile's scores, which wait for that stage to be refilled."""
    def broken(sim, nl):
        roles = dkdv_roles(sim, nl, False)
        FULL = [sim.bars["full0"], sim.bars["full1"]]
        FREE = [sim.bars["free0"], sim.bars["free1"]]
        SFULL = [sim.bars["sfull0"], sim.bars["sfull1"]]
        PFULL = [sim.bars["pfull0"], sim.bars["pfull1"]]
        ONCE, DONE = sim.bars["once"], sim.bars["done"]

        def mma():
            yield ('wait', ONCE, 0)
            for n in range(nl):
                yield ('wait', FULL[n & 1], n >> 1)
                for a in range(2):
                    yield ('mma',)
                    yield ('commit', SFULL[a])
                for a in range(2):
                    yield ('wait', PFULL[a], n)
                    yield ('mma',)
                if n + 2 < nl:
                    yield ('wait', FULL[n & 1], (n + 2) >> 1)  # waits for its own refill
                yield ('commit', FREE[n & 1])
            yield ('commit', DONE)
        roles["mma"] = mma()
        return roles
    with pytest.raises(AssertionError):
        sim = Sim(1)
        sim.run(broken(sim, 4))


# ------------------------------------------------------------------------------
# the forward attention kernel (one persistent CTA walking its list of query tiles)
# ------------------------------------------------------------------------------
def attn_roles(sim, tiles):
    """tiles: list of (nkv, tma_out[, piece, merges]) per query tile of the CTA's list;
    piece: the tile is one piece of a split key range (its record is written and
    counted: the split barriers), merges: this piece finished last and writes the
    merged output (otherwise it writes none)."""
    QFULL, QEMPTY = sim.bar("qfull"), sim.bar("qempty", 9)   # QK commit + 8 softmax warps
    KFULL = [sim.bar(f"kfull{i}") for i in range(2)]
    SFREE = [sim.bar(f"sfree{i}") for i in range(2)]
    VFULL = [sim.bar(f"vfull{i}") for i in range(2)]
    VEMPTY = [sim.bar(f"vempty{i}") for i in range(2)]
    SFULL = [sim.bar(f"sfull{i}") for i in range(2)]
    PFULL = [sim.bar(f"pfull{i}", 8) for i in range(2)]   # one per S buffer
    RDONE = sim.bar("rdone")
    SQFULL = sim.bar("sqfull", 8)
    DRAIN = sim.bar("drain", 2)
    PAIR = [sim.bar(f"pair{i}", 2) for i in range(4)]
    OFULL = [sim.bar(f"ofull{i}", 4) for i in range(2)]
    OFREE = [sim.bar(f"ofree{i}") for i in range(2)]
    STORE = [sim.bar(f"storeread{i}") for i in range(2)]  # a TMA store has read its tile
    SPLW, SPLF = sim.bar("split_written", 8), sim.bar("split_flag")
    ntiles = len(tiles)

    def producer():
        k_use, v_use = [0, 0], [0, 0]
        kst, vst = [0], [0]

        def issue_k():
            st = kst[0]
            if k_use[st] > 0:
                yield ('wait', SFULL[st], k_use[st] - 1)
            yield ('tma', KFULL[st])
            k_use[st] += 1
            kst[0] ^= 1

        def issue_v():
            st = vst[0]
            if v_use[st] > 0:
                yield ('wait', VEMPTY[st], v_use[st] - 1)
            yield ('tma', VFULL[st])
            v_use[st] += 1
            vst[0] ^= 1
        for tc, tile in enumerate(tiles):
            nkv = tile[0]
            if tc > 0:
                yield ('wait', QEMPTY, tc - 1)
            yield ('tma', QFULL)                   # Q (and z), after the descriptor slot
            yield from issue_k()
            if nkv >= 2:
                yield from issue_k()
            yield from issue_v()                   # item 0: M_hi
            for j in range(nkv):
                if j + 2 < nkv:
                    yield from issue_k()
                yield from issue_v()               # V_j
        if ntiles > 0:
            yield ('wait', QEMPTY, ntiles - 1)
        yield ('arrive', QFULL, 1)                 # the end marker

    def qk():
        n = 0
        for tc in range(ntiles + 1):
            yield ('wait', QFULL, tc)
            if tc == ntiles:
                break
            nkv = tiles[tc][0]
            for j in range(nkv):
                st = n & 1
                if n >= 2:
                    yield ('wait', SFREE[st], (n >> 1) - 1)
                yield ('wait', KFULL[st], n >> 1)
                yield ('mma', 'qk')
                yield ('commit', SFULL[st], 'qk')
                if j == nkv - 1:
                    yield ('commit', QEMPTY, 'qk')
                n += 1
        yield ('commit', DRAIN, 'qk')
        yield ('wait', DRAIN, 0)

    def pv():
        n, vit = 0, 0
        for tc in range(ntiles + 1):
            yield ('wait', SQFULL, tc)
            if tc == ntiles:
                break
            nkv = tiles[tc][0]
            st = vit & 1
            yield ('wait', VFULL[st], vit >> 1)
            yield ('mma', 'pv')                       # R = sigma(Q) M_hi
            yield ('commit', VEMPTY[st], 'pv')
            yield ('commit', RDONE, 'pv')
            vit += 1
            for j in range(nkv):
                st = vit & 1
                yield ('wait', PFULL[n & 1], n >> 1)
                yield ('wait', VFULL[st], vit >> 1)
                yield ('mma', 'pv')
                yield ('commit', VEMPTY[st], 'pv')
                yield ('commit', SFREE[n & 1], 'pv')       # P V done: S free, O readable
                vit += 1
                n += 1
        yield ('commit', DRAIN, 'pv')
        yield ('wait', DRAIN, 0)

    rescale_rng = random.Random(len(tiles) * 7919 + sum(t[0] for t in tiles))

    def softmax(w):
        half, wq = w // 4, w % 4
        rng = random.Random(rescale_rng.random() + w)   # each warp decides its own rescales
        issuer = wq == 0
        kc, pph, oc, stores, sc = 0, 0, 0, 0, 0
        yield ('wait', QFULL, 0)
        if ntiles == 0:
            yield ('arrive', SQFULL, 1)
            return
        yield ('arrive', QEMPTY, 1)                   # sigma(Q) of tile 0
        yield ('arrive', SQFULL, 1)
        for tc, tile in enumerate(tiles):
            nkv, tma_out = tile[0], tile[1]
            piece = len(tile) > 2 and tile[2]
            emit = not piece or tile[3]
            for j in range(nkv):
                yield ('wait', SFULL[kc & 1], kc >> 1)
                kc += 1
                yield ('arrive', PAIR[wq], 1)
                yield ('wait', PAIR[wq], pph)
                pph += 1
                if j > 0 and rng.random() < 0.3:           # a rescale of O: P V of the
                    yield ('wait', SFREE[(kc - 2) & 1], (kc - 2) >> 1)   # previous step
                yield ('arrive', PFULL[(kc - 1) & 1], 1)
            yield ('arrive', PAIR[wq], 1)              # epilogue: row sums exchanged
            yield ('wait', PAIR[wq], pph)
            pph += 1
            yield ('wait', SFREE[(kc - 1) & 1], (kc - 1) >> 1)    # the tile's last P V
            yield ('wait', RDONE, tc)
            if piece:                                  # record written, then counted
                yield ('arrive', SPLW, 1)
                if w == 0:
                    yield ('wait', SPLW, sc)
                    yield ('arrive', SPLF, 1)           # the merge decision, broadcast
                yield ('wait', SPLF, sc)
                sc += 1
            if tma_out and emit:
                if oc > 0:
                    if issuer:
                        yield ('wait', STORE[half], stores - 1)   # its last store has read
                        yield ('arrive', OFREE[half], 1)
                    yield ('wait', OFREE[half], oc - 1)
                yield ('arrive', OFULL[half], 1)
                if issuer:
                    yield ('wait', OFULL[half], oc)
                    yield ('tma', STORE[half])                     # TMA store reads the tile
                    stores += 1
                oc += 1
            yield ('wait', QFULL, tc + 1)
            if tc + 1 == ntiles:
                yield ('arrive', SQFULL, 1)            # the end marker reaches the P V warp
            else:
                yield ('arrive', QEMPTY, 1)            # sigma(Q) of the next tile
                yield ('arrive', SQFULL, 1)

    roles = {"producer": producer(), "qk": qk(), "pv": pv()}
    for w in range(8):
        roles[f"softmax{w}"] = softmax(w)
    return roles


class SimPerWarp(Sim):
    """Products and commits complete in issue order per issuing warp (the two MMA
    warps issue independently)."""

    def run(self, roles, max_steps=4_000_000):
        queues = {}

        # route ('mma', who) and ('commit', bar, who) into per-warp queues
        def gen_wrap(g):
            for req in g:
                if req[0] == 'mma':
                    yield ('mma_w', req[1])
                elif req[0] == 'commit' and len(req) == 3:
                    yield ('commit_w', req[1], req[2])
                else:
                    yield req
        roles = {k: gen_wrap(v) for k, v in roles.items()}
        state = {r: None for r in roles}
        for step in range(max_steps):
            ready = []
            for r, req in list(state.items()):
                if req is None:
                    try:
                        req = next(roles[r])
                    except StopIteration:
                        del state[r]
                        continue
                    state[r] = req
                if req[0] == 'wait':
                    b, k = req[1], req[2]
                    assert b.done <= k + 1, f"{b.name}: phase skipped (waiter for {k}, done {b.done})"
                    assert b.done >= k, f"{b.name}: stale phase (waiter for {k}, done {b.done})"
                    if b.done >= k + 1:
                        ready.append(r)
                else:
                    ready.append(r)
            events = ['<copy done>'] if self.tma else []
            events += [f'<product done {w}>' for w, q in queues.items() if q]
            if not state and not self.tma and not any(queues.values()):
                return step
            if not ready and not events:
                raise AssertionError("deadlock: " + ", ".join(
                    f"{r} waits {req[1].name}#{req[2]}" for r, req in state.items()
                    if req[0] == 'wait'))
            choice = self.rng.choice(ready + events)
            if choice == '<copy done>':
                self.tma.pop(self.rng.randrange(len(self.tma))).arrive()
            elif choice.startswith('<product done'):
                w = choice[len('<product done '):-1]
                item = queues[w].pop(0)
                if item is not None:
                    item.arrive()
            else:
                req = state[choice]
                if req[0] == 'arrive':
                    req[1].arrive(req[2])
                elif req[0] == 'tma':
                    self.tma.append(req[1])
                elif req[0] == 'mma_w':
                    queues.setdefault(req[1], []).append(None)
                elif req[0] == 'commit_w':
                    queues.setdefault(req[2], []).append(req[1])
                state[choice] = None
        raise AssertionError("did not finish")


@pytest.mark.parametrize("seed", range(30))
def test_attention_kernel_protocol(seed):
    """Random tile lists of a persistent CTA: 0 to 6 tiles of 1 to 6 key tiles each,
    whole tiles (TMA-stored through shared memory) and ragged ones (stored directly)."""
    rng = random.Random(seed)
    tiles = [(rng.randint(1, 6), rng.random() < 0.8) for _ in range(rng.randint(0, 6))]
    sim = SimPerWarp(seed)
    sim.run(attn_roles(sim, tiles))


@pytest.mark.parametrize("seed", range(30))
def test_attention_kernel_protocol_split_pieces(seed):
    """Split mode: lists that mix whole tiles with pieces of split key ranges (1 to 4
    key tiles), some of which merge and store the tile and some of which only leave
    their record."""
    rng = random.Random(1000 + seed)
    tiles = []
    for _ in range(rng.randint(1, 7)):
        piece = rng.random() < 0.7
        tiles.append((rng.randint(1, 4), rng.random() < 0.8, piece, rng.random() < 0.5))
    sim = SimPerWarp(seed)
    sim.run(attn_roles(sim, tiles))


def test_attention_model_detects_a_wrong_split_count():
    """Planted mistake: the records barrier counts one arrival per warp of one
    warpgroup (4) instead of all eight softmax warps, so it completes twice per piece
    and the counting warp's parity wait would see a later phase."""
    def broken(sim, tiles):
        roles = attn_roles(sim, tiles)
        sim.bars["split_written"].count = sim.bars["split_written"].pending = 4
        return roles
    failures = 0
    for seed in range(30):
        sim = SimPerWarp(seed)
        try:
            sim.run(broken(sim, [(2, True, True, False), (1, True, True, True),
                                 (3, False, True, False), (2, True, True, True)]))
        except AssertionError:
            failures += 1
    assert failures > 0


def test_attention_model_detects_a_conditional_wait_on_a_shared_pv_barrier():
    """Planted mistake: one P-V-done barrier committed after every P V and waited only
    when a rescale needs O. Skipped phases leave it behind the waiter's count, where a
    parity wait would pass on an older phase (the kernel waits on the S buffer's S-free
    barrier instead, which the Q K^T warp keeps in step)."""
    def broken(sim, tiles):
        roles = attn_roles(sim, tiles)
        PV = sim.bar("pvdone_shared")
        SFREE = [sim.bars["sfree0"], sim.bars["sfree1"]]
        old_pv, softs = roles["pv"], {w: roles[f"softmax{w}"] for w in range(8)}

        def pv():
            for req in old_pv:
                yield req
                if req[0] == 'commit' and req[1] in SFREE:
                    yield ('commit', PV, 'pv')

        def soft(g):
            count = 0
            for req in g:
                if req[0] == 'wait' and req[1] in SFREE:
                    yield ('wait', PV, req[2] * 2 + SFREE.index(req[1]))
                    continue
                yield req
        roles["pv"] = pv()
        for w in range(8):
            roles[f"softmax{w}"] = soft(softs[w])
        return roles
    failures = 0
    for seed in range(30):
        sim = SimPerWarp(seed)
        try:
            sim.run(broken(sim, [(6, True), (5, True), (6, False), (4, True)]))
        except AssertionError:
            failures += 1
    assert failures > 0


def test_attention_model_detects_a_missing_sfree_wait():
    """Planted mistake: Q K^T no longer waits for the P V that last read its S buffer."""
    def broken(sim, tiles):
        roles = attn_roles(sim, tiles)
        QFULL, KFULL = sim.bars["qfull"], [sim.bars["kfull0"], sim.bars["kfull1"]]
        SFULL = [sim.bars["sfull0"], sim.bars["sfull1"]]
        QEMPTY, DRAIN = sim.bars["qempty"], sim.bars["drain"]

        def qk():
            n = 0
            for tc in range(len(tiles) + 1):
                yield ('wait', QFULL, tc)
                if tc == len(tiles):
                    break
                for j in range(tiles[tc][0]):
                    yield ('wait', KFULL[n & 1], n >> 1)
                    yield ('mma', 'qk')
                    yield ('commit', SFULL[n & 1], 'qk')
                    if j == tiles[tc][0] - 1:
                        yield ('commit', QEMPTY, 'qk')
                    n += 1
            yield ('commit', DRAIN, 'qk')
            yield ('wait', DRAIN, 0)
        roles["qk"] = qk()
        return roles
    failures = 0
    for seed in range(30):
        sim = SimPerWarp(seed)
        try:
            sim.run(broken(sim, [(6, True), (5, True), (6, False)]))
        except AssertionError:
            failures += 1
    assert failures > 0


# ------------------------------------------------------------------------------
# the forward's state kernel (one chunk of one segment) and the state chains
# ------------------------------------------------------------------------------
def state_roles(sim, units, stages=3, conv_warps=16, zsum=True):
    """The persistent state kernel: a CTA walks units (head, segment, chunk) of
    units[i] slabs each; the ring and its barrier phases run on across units; the MMA
    warp commits DONE once per unit with tokens and DRAIN at the end; the converters
    wait for such a unit's DONE before draining its accumulator (a unit without
    tokens writes zeros and waits for nothing), and (zsum) meet at a named barrier
    twice per unit around the shared sum area."""
    FULL = [sim.bar(f"full{i}") for i in range(stages)]
    CONV = [sim.bar(f"conv{i}", conv_warps) for i in range(stages)]
    MMA = [sim.bar(f"mma{i}") for i in range(stages)]
    DONE = sim.bar("done")
    DRAIN = sim.bar("drain")
    convs = [f"conv{w}" for w in range(conv_warps)]

    def producer():
        g = 0
        for nslab in units:
            for _ in range(nslab):
                stg = g % stages
                if g >= stages:
                    yield ('wait', MMA[stg], g // stages - 1)
                yield ('tma', FULL[stg], g // stages)
                g += 1

    def mma():
        g = 0
        for nslab in units:
            for _ in range(nslab):
                stg = g % stages
                yield ('wait', CONV[stg], g // stages)
                yield ('mma',)
                yield ('commit', MMA[stg])
                g += 1
            if nslab > 0:
                yield ('commit', DONE)
        yield ('commit', DRAIN)
        yield ('wait', DRAIN, 0)

    def converter():
        g, dn = 0, 0
        for un, nslab in enumerate(units):
            for _ in range(nslab):
                stg = g % stages
                yield ('wait', FULL[stg], g // stages)
                yield ('arrive', CONV[stg], 1)  # operands converted in place
                g += 1
            if nslab > 0:
                yield ('wait', DONE, dn)        # then the accumulator is drained
                dn += 1
            if zsum:
                yield ('named', f"zred{un}a", convs)
                yield ('named', f"zred{un}b", convs)

    roles = {"producer": producer(), "mma": mma()}
    for w in convs:
        roles[w] = converter()
    return roles


def chain_roles(sim, S, CH, delta=True):
    """The forward chain and the backward's reverse chain share this protocol: per
    segment the four row warps write their block of M (or dM) transposed and arrive;
    the MMA warp multiplies by the segment's G chunks (double-buffered TMA, the next
    chunk's load issued before waiting for the current one) and signals the segment."""
    G = [sim.bar(f"g{i}") for i in range(2)]
    MT, MMA, SEG = sim.bar("mt", 4), sim.bar("mma"), sim.bar("seg")

    def mma():
        if not delta:
            return
        total, n = S * CH, 0
        yield ('tma', G[0])
        for q in range(S):
            yield ('wait', MT, q)
            for c in range(CH):
                buf = n & 1
                if n + 1 < total:
                    yield ('tma', G[buf ^ 1])   # the other buffer's last MMA is done
                yield ('wait', G[buf], n >> 1)
                yield ('mma',)
                yield ('commit', MMA)
                if c == CH - 1:
                    yield ('commit', SEG)
                yield ('wait', MMA, n)
                n += 1

    def rows():
        for q in range(S):
            if delta:
                yield ('arrive', MT, 1)         # the M block transposed, for G M
                yield ('wait', SEG, q)

    roles = {"mma": mma()}
    for w in range(4):
        roles[f"rows{w}"] = rows()
    return roles


@pytest.mark.parametrize("units", [[1], [8], [32], [8, 8, 8], [0, 3, 5], [2, 0], [5, 1, 7, 2],
                                   [32, 32, 1]])
def test_state_kernel_protocol(units):
    for seed in range(30):
        sim = Sim(seed * 1000 + sum(units) + len(units))
        sim.run(state_roles(sim, units))


def test_state_model_detects_a_commit_for_a_unit_without_tokens():
    """DONE committed for a unit without tokens as well: the two commits of units
    [2, 0] complete the barrier twice before the converters' first wait."""
    def broken(sim, units):
        roles = state_roles(sim, units, zsum=False)
        stages = 3
        CONV = [sim.bars[f"conv{i}"] for i in range(stages)]
        MMA = [sim.bars[f"mma{i}"] for i in range(stages)]

        def mma():
            g = 0
            for nslab in units:
                for _ in range(nslab):
                    stg = g % stages
                    yield ('wait', CONV[stg], g // stages)
                    yield ('mma',)
                    yield ('commit', MMA[stg])
                    g += 1
                yield ('commit', sim.bars["done"])
            yield ('commit', sim.bars["drain"])
            yield ('wait', sim.bars["drain"], 0)
        roles["mma"] = mma()
        return roles
    with pytest.raises(AssertionError, match="phase skipped"):
        for seed in range(40):
            sim = Sim(seed)
            sim.run(broken(sim, [2, 0]))


def test_state_model_detects_a_done_barrier_committed_once():
    """DONE committed once for the whole CTA instead of once per unit: the converters'
    wait for the second unit's sums never completes."""
    def broken(sim, units):
        roles = state_roles(sim, units, zsum=False)
        stages = 3
        FULL = [sim.bars[f"full{i}"] for i in range(stages)]
        CONV = [sim.bars[f"conv{i}"] for i in range(stages)]
        MMA = [sim.bars[f"mma{i}"] for i in range(stages)]

        def mma():
            g = 0
            for nslab in units:
                for _ in range(nslab):
                    stg = g % stages
                    yield ('wait', CONV[stg], g // stages)
                    yield ('mma',)
                    yield ('commit', MMA[stg])
                    g += 1
            yield ('commit', sim.bars["done"])
            yield ('commit', sim.bars["drain"])
            yield ('wait', sim.bars["drain"], 0)
        roles["mma"] = mma()
        return roles
    with pytest.raises(AssertionError, match="deadlock"):
        sim = Sim(5)
        sim.run(broken(sim, [4, 4]))


@pytest.mark.parametrize("S,CH", [(1, 1), (1, 8), (3, 2), (16, 1), (5, 4)])
def test_chain_protocol(S, CH):
    for seed in range(20):
        sim = Sim(seed * 100 + S * 10 + CH)
        sim.run(chain_roles(sim, S, CH))


# ------------------------------------------------------------------------------
# one-segment update (step_state_kernel): slabs n through two stages; converter group
# g (eight warps, one arrival each) takes the slabs of stage g; Linear+Delta issues
# R of slab n, then the update product of slab n - 1
# ------------------------------------------------------------------------------
def step_state_roles(sim, nslab, delta):
    FULL = [sim.bar(f"full{i}", 2) for i in range(2)]     # expect_tx arrival + the copies
    CONV1 = [sim.bar(f"conv1_{i}", 8) for i in range(2)]
    RDONE = [sim.bar(f"rdone{i}") for i in range(2)]
    CONV2 = [sim.bar(f"conv2_{i}", 8) for i in range(2)]
    FREE = [sim.bar(f"free{i}") for i in range(2)]
    MFULL = sim.bar("mfull", 2)
    DONE = sim.bar("done")

    def producer():
        if delta:
            yield ('arrive', MFULL, 1, 0)
            yield ('tma', MFULL, 0)
        for n in range(nslab):
            st = n & 1
            if n >= 2:
                yield ('wait', FREE[st], (n >> 1) - 1)
            yield ('arrive', FULL[st], 1, n >> 1)
            yield ('tma', FULL[st], n >> 1)

    def mma():
        if delta and nslab > 0:
            yield ('wait', MFULL, 0)
        for n in range(nslab):
            st = n & 1
            yield ('wait', CONV1[st], n >> 1)
            if not delta:
                yield ('mma',)
                yield ('commit', FREE[st])
                continue
            yield ('mma',)                      # R of slab n
            yield ('commit', RDONE[st])
            if n > 0:
                yield ('wait', CONV2[(n - 1) & 1], (n - 1) >> 1)
                yield ('mma',)                  # update of slab n - 1
                yield ('commit', FREE[(n - 1) & 1])
        if delta and nslab > 0:
            yield ('wait', CONV2[(nslab - 1) & 1], (nslab - 1) >> 1)
            yield ('mma',)
            yield ('commit', FREE[(nslab - 1) & 1])
        yield ('commit', DONE)

    def converters(g):
        for n in range(g, nslab, 2):
            st = n & 1
            yield ('wait', FULL[st], n >> 1)
            yield ('arrive', CONV1[st], 8)      # sigma(K) hi/lo and 1/den written
            if not delta:
                continue
            yield ('wait', CONV1[st], n >> 1)   # every warp's 1/den of the slab
            yield ('wait', RDONE[st], n >> 1)
            yield ('arrive', CONV2[st], 8)      # U = V - R / den written
        yield ('wait', DONE, 0)

    return {"producer": producer(), "mma": mma(), "conv0": converters(0), "conv1": converters(1)}


@pytest.mark.parametrize("delta", [False, True])
@pytest.mark.parametrize("nslab", [0, 1, 2, 3, 4, 7, 16])
def test_step_state_kernel_protocol(nslab, delta):
    for seed in range(40):
        sim = Sim(seed * 1000 + nslab + 100 * delta)
        sim.run(step_state_roles(sim, nslab, delta))


def test_step_state_model_detects_a_wait_for_the_wrong_slab():
    """The update of slab n - 1 waiting for the U of slab n's completion index: the U
    it waits for needs an R that is issued only after that update."""
    def broken(sim, nslab):
        roles = step_state_roles(sim, nslab, True)
        CONV1 = [sim.bars["conv1_0"], sim.bars["conv1_1"]]
        CONV2 = [sim.bars["conv2_0"], sim.bars["conv2_1"]]
        RDONE = [sim.bars["rdone0"], sim.bars["rdone1"]]
        FREE = [sim.bars["free0"], sim.bars["free1"]]

        def mma():
            yield ('wait', sim.bars["mfull"], 0)
            for n in range(nslab):
                st = n & 1
                yield ('wait', CONV1[st], n >> 1)
                yield ('mma',)
                yield ('commit', RDONE[st])
                if n > 0:
                    yield ('wait', CONV2[(n - 1) & 1], n >> 1)   # should be (n - 1) >> 1
                    yield ('mma',)
                    yield ('commit', FREE[(n - 1) & 1])
            yield ('commit', sim.bars["done"])
        roles["mma"] = mma()
        return roles
    with pytest.raises(AssertionError, match="deadlock|phase"):
        sim = Sim(3)
        sim.run(broken(sim, 8))
