"""Race detection for the tcgen05 kernels' barrier protocols (CPU only).

Each kernel's roles (TMA thread, MMA-issuing thread, softmax or epilogue
warps) are restated as generators of the same waits, arrivals and commits
the CUDA source performs, and run under random schedules in which copies
finish in any order and tensor-core operations finish in issue order.  At
every wait the model asserts what a parity wait needs to be exact: when the
wait begins its barrier is at most one phase behind, and while it waits the
barrier never gets two phases ahead.  It also asserts the data hazards the
barriers exist for (TMEM columns and shared-memory stages are reused only
after their readers finished) and that no schedule deadlocks.

These are models of the protocols, kept next to the sources they restate
(qkv_tc.cu, its K split across a cluster included, prefill_pair.cu,
prefill_fa.cu, decode_tc.cu, decode_hn.cu); a change to a kernel's waits
belongs in both.  The decode's former final waits, and a K-split leader that
reads its partner's partial sums before the cluster barrier, are kept as
planted mistakes that the model flags.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.done = 0


def run(roles, bars, seed, max_steps=200000):
    """Random schedule of `roles` (name -> generator); returns the event log."""
    rng = random.Random(seed)
    nxt = {}
    queue = []          # issued asynchronous operations: (name, barriers to arrive on)
    log = []

    def arrive(b):
        bar = bars[b]
        bar.pending -= 1
        assert bar.pending >= 0, f"more arrivals than expected on {b}"
        if bar.pending == 0:
            bar.done += 1
            bar.pending = bar.count

    def fetch(n, g):
        a = next(g, None)
        if a is not None and a[0] == "wait":
            assert bars[a[1]].done >= a[2], f"{n} waits phase {a[2]} of {a[1]} with only {bars[a[1]].done} done"
        nxt[n] = a

    gens = dict(roles)
    for n, g in gens.items():
        fetch(n, g)
    for _ in range(max_steps):
        ready = []
        for n, a in nxt.items():
            if a is None:
                continue
            if a[0] == "wait":
                bar = bars[a[1]]
                assert bar.done <= a[2] + 1, f"{n}: {a[1]} two phases past the awaited phase {a[2]}"
                if bar.done >= a[2] + 1:
                    ready.append(n)
            else:
                ready.append(n)
        copies = [i for i, (name, _) in enumerate(queue) if name.startswith("load")]
        tensor = [i for i, (name, _) in enumerate(queue) if not name.startswith("load")]
        choices = ready + [("op", i) for i in copies] + ([("op", tensor[0])] if tensor else [])
        if not choices:
            stuck = {n: a for n, a in nxt.items() if a is not None}
            assert not stuck, f"deadlock: {stuck}"
            return log
        pick = rng.choice(choices)
        if isinstance(pick, tuple):
            name, comps = queue.pop(pick[1])
            log.append(("done", name))
            for b in comps:
                arrive(b)
            continue
        a = nxt[pick]
        if a[0] == "arrive":
            arrive(a[1])
        elif a[0] == "issue":
            queue.append((a[1], a[2]))
            log.append(("issue", a[1]))
        elif a[0] == "event":
            log.append(("event", a[1]))
        fetch(pick, gens[pick])
    raise AssertionError("schedule did not finish")


def first(log):
    pos = {}
    for i, e in enumerate(log):
        pos.setdefault(e, i)
    return pos


def ring_load(kind, t, S, full):
    """One TMA copy into stage t % S of a ring, after the stage was freed."""
    s = t % S
    if t >= S:
        yield ("wait", f"{kind}_empty{s}", t // S - 1)
    yield ("issue", f"load_{kind}{t}", [full or f"{kind}_full{s}"])


# ---------------------------------------------------------------- qkv_tc.cu
def qkv_tc(n_tiles, n_kb, STAGES=4, warps=4):
    bars = {"drain": Bar(1)}
    for s in range(STAGES):
        bars[f"ab_full{s}"] = Bar(1)
        bars[f"ab_empty{s}"] = Bar(1)
    for b in range(2):
        bars[f"acc_full{b}"] = Bar(1)
        bars[f"acc_empty{b}"] = Bar(warps)

    def producer():
        for j in range(n_tiles * n_kb):
            yield from ring_load("ab", j, STAGES, None)

    def mma():
        j = 0
        for it in range(n_tiles):
            buf = it & 1
            if it >= 2:
                yield ("wait", f"acc_empty{buf}", (it >> 1) - 1)
            yield ("event", f"acc_write{it}")
            for kb in range(n_kb):
                yield ("wait", f"ab_full{j % STAGES}", j // STAGES)
                yield ("issue", f"mma{j}", [f"ab_empty{j % STAGES}"])
                j += 1
            yield ("issue", f"acc{it}", [f"acc_full{buf}"])
        yield ("issue", "drain", ["drain"])
        yield ("wait", "drain", 0)

    def epilogue(w):
        for it in range(n_tiles):
            yield ("wait", f"acc_full{it & 1}", it >> 1)
            yield ("event", f"acc_read{it}_{w}")
            yield ("arrive", f"acc_empty{it & 1}")

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"epi{w}": epilogue(w) for w in range(warps)})
    return roles, bars


@pytest.mark.parametrize("n_tiles,n_kb", [(1, 1), (2, 3), (3, 5), (5, 2)])
def test_qkv_gemm_protocol(n_tiles, n_kb):
    for seed in range(60):
        roles, bars = qkv_tc(n_tiles, n_kb)
        pos = first(run(roles, bars, seed))
        for it in range(n_tiles):
            for w in range(4):
                assert pos[("done", f"acc{it}")] < pos[("event", f"acc_read{it}_{w}")]
                if it + 2 < n_tiles:
                    assert pos[("event", f"acc_read{it}_{w}")] < pos[("event", f"acc_write{it + 2}")]
        for j in range(4, n_tiles * n_kb):
            assert pos[("done", f"mma{j - 4}")] < pos[("issue", f"load_ab{j}")]


def qkv_tc_ksplit(n_kb, STAGES=4, warps=4, ks=2, leader_waits=True):
    """The K split of qkv_tc.cu: the ks CTAs of a cluster each take one
    tile's k-blocks [r n_kb / ks, (r + 1) n_kb / ks); ranks above 0 write
    their accumulator rows to their own shared memory, every thread of every
    rank meets at a cluster barrier, the leader's epilogue warps read those
    rows, and a second cluster barrier keeps the other ranks alive until then.
    ``leader_waits=False`` plants the mistake of reading before the first
    cluster barrier."""
    n_roles = ks * (2 + warps)
    bars = {"cluster1": Bar(n_roles), "cluster2": Bar(n_roles)}
    roles = {}
    for r in range(ks):
        kb0, kb1 = r * n_kb // ks, (r + 1) * n_kb // ks
        bars[f"drain_{r}"] = Bar(1)
        bars[f"acc_full_{r}"] = Bar(1)
        for s in range(STAGES):
            bars[f"ab{r}_full{s}"] = Bar(1)
            bars[f"ab{r}_empty{s}"] = Bar(1)

        def producer(r=r, kb0=kb0, kb1=kb1):
            for j in range(kb1 - kb0):
                yield from ring_load(f"ab{r}", j, STAGES, None)
            yield ("arrive", "cluster1")
            yield ("wait", "cluster1", 0)
            yield ("arrive", "cluster2")
            yield ("wait", "cluster2", 0)

        def mma(r=r, kb0=kb0, kb1=kb1):
            for j in range(kb1 - kb0):
                yield ("wait", f"ab{r}_full{j % STAGES}", j // STAGES)
                yield ("issue", f"mma{r}_{j}", [f"ab{r}_empty{j % STAGES}"])
            yield ("issue", f"acc{r}", [f"acc_full_{r}"])
            yield ("issue", f"drain{r}", [f"drain_{r}"])
            yield ("wait", f"drain_{r}", 0)
            yield ("arrive", "cluster1")
            yield ("wait", "cluster1", 0)
            yield ("arrive", "cluster2")
            yield ("wait", "cluster2", 0)

        def epilogue(w, r=r):
            yield ("wait", f"acc_full_{r}", 0)
            if r > 0:
                yield ("event", f"partial_write{r}_{w}")
            if r == 0 and not leader_waits:
                for q in range(1, ks):
                    yield ("event", f"partial_read{q}_{w}")
            yield ("arrive", "cluster1")
            yield ("wait", "cluster1", 0)
            if r == 0:
                if leader_waits:
                    for q in range(1, ks):
                        yield ("event", f"partial_read{q}_{w}")
                yield ("event", f"tile_epilogue_{w}")
            yield ("arrive", "cluster2")
            yield ("wait", "cluster2", 0)
            yield ("event", f"exit{r}_{w}")

        roles[f"tma{r}"] = producer()
        roles[f"mma{r}"] = mma()
        roles.update({f"epi{r}_{w}": epilogue(w) for w in range(warps)})
    return roles, bars


def check_ksplit(pos, ks, warps=4):
    for q in range(1, ks):
        for w in range(warps):
            assert pos[("done", f"acc{q}")] < pos[("event", f"partial_write{q}_{w}")]
            for w2 in range(warps):
                # every row of rank q is written before the leader reads any, and read before rank q leaves
                assert pos[("event", f"partial_write{q}_{w}")] < pos[("event", f"partial_read{q}_{w2}")]
                assert pos[("event", f"partial_read{q}_{w2}")] < pos[("event", f"exit{q}_{w}")]
    for w in range(warps):
        assert pos[("done", "acc0")] < pos[("event", f"tile_epilogue_{w}")]


@pytest.mark.parametrize("n_kb,ks", [(8, 2), (9, 2), (12, 3), (16, 4)])
def test_qkv_gemm_ksplit_protocol(n_kb, ks):
    for seed in range(60):
        roles, bars = qkv_tc_ksplit(n_kb, ks=ks)
        check_ksplit(first(run(roles, bars, seed)), ks)


def test_planted_ksplit_read_before_the_cluster_barrier_is_flagged():
    flagged = False
    for seed in range(60):
        roles, bars = qkv_tc_ksplit(8, leader_waits=False)
        try:
            check_ksplit(first(run(roles, bars, seed)), 2)
        except AssertionError:
            flagged = True
            break
    assert flagged


# ---------------------------------------------------------------- prefill_pair.cu
def prefill_pair(n, KS=3, VS=2, warps=4, rescale_at=(), p_before_pv_wait=True):
    """S | P | O in TMEM: the softmax frees S once it holds it in registers
    (s_free), the MMA lane issues the next S at once, and the softmax writes
    P(t) only after P(t-1).V has read the P columns.  ``p_before_pv_wait``
    False plants the mistake of storing P without that wait."""
    bars = {"q_full": Bar(1), "s_full": Bar(1), "s_free": Bar(warps), "p_full": Bar(warps), "o_done": Bar(1),
            "drain": Bar(1)}
    for i in range(KS):
        bars[f"k_full{i}"], bars[f"k_empty{i}"] = Bar(1), Bar(1)
    for i in range(VS):
        bars[f"v_full{i}"], bars[f"v_empty{i}"] = Bar(1), Bar(1)

    def tma():
        yield ("issue", "load_q", ["q_full"])
        yield from ring_load("k", 0, KS, None)
        if n > 1:
            yield from ring_load("k", 1, KS, None)
        for t in range(n):
            if t + 2 < n:
                yield from ring_load("k", t + 2, KS, None)
            yield from ring_load("v", t, VS, None)

    def issue_s(t):
        yield ("wait", f"k_full{t % KS}", t // KS)
        yield ("event", f"S{t}_start")
        yield ("issue", f"S{t}", [f"k_empty{t % KS}", "s_full"])

    def mma():
        yield ("wait", "q_full", 0)
        yield from issue_s(0)
        for t in range(n):
            if t + 1 < n:                   # S columns free once every warp holds S(t)
                yield ("wait", "s_free", t)
                yield from issue_s(t + 1)
            yield ("wait", "p_full", t)
            yield ("wait", f"v_full{t % VS}", t // VS)
            yield ("event", f"PV{t}_start")
            yield ("issue", f"PV{t}", [f"v_empty{t % VS}", "o_done"])
        yield ("issue", "drain", ["drain"])
        yield ("wait", "drain", 0)

    def softmax(w):
        for t in range(n):
            yield ("wait", "s_full", t)
            yield ("event", f"readS{t}_{w}")
            yield ("arrive", "s_free")
            if t > 0 and (p_before_pv_wait or t in rescale_at):
                yield ("wait", "o_done", t - 1)
            if t in rescale_at:
                yield ("event", f"rescale{t}_{w}")
            yield ("event", f"writeP{t}_{w}")
            yield ("arrive", "p_full")
        if n > 0:
            yield ("wait", "o_done", n - 1)
        yield ("event", f"readO_{w}")

    roles = {"tma": tma(), "mma": mma()}
    roles.update({f"sm{w}": softmax(w) for w in range(warps)})
    return roles, bars


def check_pair(n, pos):
    for t in range(n):
        for w in range(4):
            assert pos[("done", f"S{t}")] < pos[("event", f"readS{t}_{w}")]
            assert pos[("event", f"writeP{t}_{w}")] < pos[("event", f"PV{t}_start")]
            if t + 1 < n:   # S(t+1) overwrites S only after every warp read S(t)
                assert pos[("event", f"readS{t}_{w}")] < pos[("event", f"S{t + 1}_start")]
            if t > 0:       # P(t) overwrites P(t-1) only after P(t-1).V has read it
                assert pos[("done", f"PV{t - 1}")] < pos[("event", f"writeP{t}_{w}")]
                if ("event", f"rescale{t}_{w}") in pos:
                    assert pos[("done", f"PV{t - 1}")] < pos[("event", f"rescale{t}_{w}")]
        if t >= 3:
            assert pos[("done", f"S{t - 3}")] < pos[("issue", f"load_k{t}")]
    assert all(pos[("done", f"PV{n - 1}")] < pos[("event", f"readO_{w}")] for w in range(4))


@pytest.mark.parametrize("n", [1, 2, 3, 6])
def test_prefill_pair_protocol(n):
    for seed in range(60):
        roles, bars = prefill_pair(n, rescale_at=tuple(range(1, n, 2)))
        check_pair(n, first(run(roles, bars, seed)))


def test_prefill_pair_protocol_flags_p_written_before_pv_read_it():
    """Planted mistake: P(t) stored without waiting for P(t-1).V."""
    failed = False
    for seed in range(200):
        roles, bars = prefill_pair(4, p_before_pv_wait=False)
        try:
            check_pair(4, first(run(roles, bars, seed)))
        except AssertionError:
            failed = True
            break
    assert failed


# ---------------------------------------------------------------- prefill_fa.cu
def prefill_fa(n0, n1, p_own, warps=4):
    KS = VS = 3 if p_own else 2
    nt = (n0, n1)
    n_kv = max(nt)
    bars = {"q_full": Bar(1), "drain": Bar(1)}
    for t in range(2):
        bars[f"s_full{t}"], bars[f"p_full{t}"], bars[f"o_done{t}"] = Bar(1), Bar(warps), Bar(1)
    for i in range(KS):
        bars[f"k_full{i}"], bars[f"k_empty{i}"] = Bar(1), Bar(1)
        bars[f"v_full{i}"], bars[f"v_empty{i}"] = Bar(1), Bar(1)

    def tma():
        yield ("issue", "load_q", ["q_full"])
        yield from ring_load("k", 0, KS, None)
        for i in range(n_kv):
            if i + 1 < n_kv:
                yield from ring_load("k", i + 1, KS, None)
            yield from ring_load("v", i, VS, None)

    def mma():
        yield ("wait", "q_full", 0)
        yield ("wait", "k_full0", 0)
        for t in range(2):
            if nt[t] > 0:
                yield ("event", f"S{t}_0_start")
                yield ("issue", f"S{t}_0", [f"s_full{t}"])
        yield ("issue", "kfree0", ["k_empty0"])
        for i in range(n_kv):
            vs, ks = i % VS, (i + 1) % KS
            yield ("wait", f"v_full{vs}", i // VS)
            for t in range(2):
                if i >= nt[t]:
                    continue
                yield ("wait", f"p_full{t}", i)
                yield ("event", f"PV{t}_{i}_start")
                yield ("issue", f"PV{t}_{i}", [f"o_done{t}"])
                if i + 1 < nt[t]:
                    yield ("wait", f"k_full{ks}", (i + 1) // KS)
                    if not p_own:             # aliased P: S_t's columns hold P_t until P_t.V is done
                        yield ("wait", f"o_done{t}", i)
                    yield ("event", f"S{t}_{i + 1}_start")
                    yield ("issue", f"S{t}_{i + 1}", [f"s_full{t}"])
            yield ("issue", f"vfree{i}", [f"v_empty{vs}"])
            if i + 1 < n_kv:
                yield ("issue", f"kfree{i + 1}", [f"k_empty{ks}"])
        yield ("issue", "drain", ["drain"])
        yield ("wait", "drain", 0)

    def softmax(t, w):
        for i in range(n_kv):
            if i >= nt[t]:
                continue
            yield ("wait", f"s_full{t}", i)
            yield ("event", f"readS{t}_{i}_{w}")
            if i % 2 == 1:                    # a row max that grew: O rescaled in TMEM
                yield ("wait", f"o_done{t}", i - 1)
                yield ("event", f"rescale{t}_{i}_{w}")
            if p_own and i > 0:               # own P columns: free once P_t.V_{i-1} has read them
                yield ("wait", f"o_done{t}", i - 1)
            yield ("event", f"writeP{t}_{i}_{w}")
            yield ("arrive", f"p_full{t}")
        if nt[t] > 0:
            yield ("wait", f"o_done{t}", nt[t] - 1)
        yield ("event", f"readO{t}_{w}")

    roles = {"tma": tma(), "mma": mma()}
    for t in range(2):
        roles.update({f"sm{t}{w}": softmax(t, w) for w in range(warps)})
    return roles, bars


@pytest.mark.parametrize("p_own", [True, False], ids=["hd64-own-P", "hd128-P-over-S"])
@pytest.mark.parametrize("n0,n1", [(1, 1), (1, 2), (2, 3), (4, 4), (3, 5)])
def test_prefill_two_tile_protocol(n0, n1, p_own):
    for seed in range(40):
        roles, bars = prefill_fa(n0, n1, p_own)
        pos = first(run(roles, bars, seed))
        for t, nt in ((0, n0), (1, n1)):
            for i in range(nt):
                for w in range(4):
                    assert pos[("done", f"S{t}_{i}")] < pos[("event", f"readS{t}_{i}_{w}")]
                    assert pos[("event", f"writeP{t}_{i}_{w}")] < pos[("event", f"PV{t}_{i}_start")]
                    if i > 0:          # P_t(i) written after P_t(i-1).V finished reading its columns
                        assert pos[("done", f"PV{t}_{i - 1}")] < pos[("event", f"writeP{t}_{i}_{w}")]
            assert all(pos[("done", f"PV{t}_{nt - 1}")] < pos[("event", f"readO{t}_{w}")] for w in range(4))


# ---------------------------------------------------------------- decode_tc.cu
def decode_tc(n, final="drain", KS=2, VS=2, warps=4):
    bars = {"q_full": Bar(1), "o_done": Bar(1), "drain": Bar(1)}
    for i in range(2):
        bars[f"s_full{i}"], bars[f"p_full{i}"] = Bar(1), Bar(warps)
    for i in range(KS):
        bars[f"k_full{i}"], bars[f"k_empty{i}"] = Bar(1), Bar(1)
    for i in range(VS):
        bars[f"v_full{i}"], bars[f"v_empty{i}"] = Bar(1), Bar(1)

    def tma():
        yield ("issue", "load_q", ["q_full"])
        yield from ring_load("k", 0, KS, None)
        for t in range(n):
            if t + 1 < n:
                yield from ring_load("k", t + 1, KS, None)
            yield from ring_load("v", t, VS, None)

    def mma():
        yield ("wait", "q_full", 0)

        def issue_s(t):     # S double-buffered: buffer t & 1 held P(t-2) until P(t-2).V completed
            yield ("wait", f"k_full{t % KS}", t // KS)
            if t >= 2:
                yield ("wait", "o_done", t - 2)
            yield ("event", f"S{t}_start")
            yield ("issue", f"S{t}", [f"k_empty{t % KS}", f"s_full{t & 1}"])
        yield from issue_s(0)
        for t in range(n):
            if t + 1 < n:
                yield from issue_s(t + 1)
            yield ("wait", f"p_full{t & 1}", t >> 1)
            yield ("wait", f"v_full{t % VS}", t // VS)
            yield ("event", f"PV{t}_start")
            yield ("issue", f"PV{t}", [f"v_empty{t % VS}", "o_done"])
        yield ("issue", "drain", ["drain"])
        yield ("wait", "drain", 0)

    def softmax(w):
        for t in range(n):
            yield ("wait", f"s_full{t & 1}", t >> 1)
            yield ("event", f"readS{t}_{w}")
            if t % 2 == 1:
                yield ("wait", "o_done", t - 1)
            yield ("event", f"writeP{t}_{w}")
            yield ("arrive", f"p_full{t & 1}")
        if final == "drain":
            if n > 0:
                yield ("wait", "drain", 0)
        else:
            if final == "last-two" and n > 1:
                yield ("wait", "o_done", n - 2)
            if n > 0:
                yield ("wait", "o_done", n - 1)
        yield ("event", f"readO_{w}")

    roles = {"tma": tma(), "mma": mma()}
    roles.update({f"sm{w}": softmax(w) for w in range(warps)})
    return roles, bars


@pytest.mark.parametrize("n", [1, 2, 3, 5])
def test_decode_tcgen05_protocol(n):
    for seed in range(60):
        roles, bars = decode_tc(n)
        pos = first(run(roles, bars, seed))
        for t in range(n):
            for w in range(4):
                assert pos[("done", f"S{t}")] < pos[("event", f"readS{t}_{w}")]
                assert pos[("event", f"writeP{t}_{w}")] < pos[("event", f"PV{t}_start")]
                if t >= 2:     # S(t) overwrites the buffer P(t-2) was read from
                    assert pos[("done", f"PV{t - 2}")] < pos[("event", f"S{t}_start")]
        assert all(pos[("done", f"PV{n - 1}")] < pos[("event", f"readO_{w}")] for w in range(4))


@pytest.mark.parametrize("final", ["last", "last-two"])
def test_planted_decode_final_waits_are_flagged(final):
    """Waiting on o_done for the last phase (or the last two) lets some
    schedules read O early or wait on a phase the barrier already passed."""
    flagged = 0
    for seed in range(100):
        roles, bars = decode_tc(3, final=final)
        try:
            run(roles, bars, seed)
        except AssertionError:
            flagged += 1
    assert flagged > 0


# ---------------------------------------------------------------- decode_hn.cu
def decode_hn(pieces, KS=3, VS=3, rescale=(), zero_v=(), warps=4, p_wait=True):
    """One CTA's range: `pieces` lists the tiles of each piece in order;
    tiles are numbered n = 0, 1, ... across pieces.  `rescale` holds the
    tiles whose softmax rescales O^T, `zero_v` the tiles whose V rows past
    kv_len the softmax zeroes.  `p_wait` False drops the single P buffer's
    wait (a planted mistake)."""
    bars = {"p_full": Bar(warps), "p_empty": Bar(1), "drain": Bar(1)}
    for i in range(2):
        bars[f"q_full{i}"], bars[f"q_empty{i}"] = Bar(1), Bar(1)
        bars[f"s_full{i}"], bars[f"s_free{i}"] = Bar(1), Bar(warps)
        bars[f"o_final{i}"], bars[f"o_empty{i}"] = Bar(1), Bar(warps)
        bars[f"ml_full{i}"], bars[f"ml_empty{i}"] = Bar(warps), Bar(warps)
    for i in range(KS):
        bars[f"k_full{i}"], bars[f"k_empty{i}"] = Bar(1), Bar(1)
    for i in range(VS):
        bars[f"v_full{i}"], bars[f"v_empty{i}"] = Bar(1), Bar(1)
    tiles = []            # (n, piece, first, last)
    for pi, cnt in enumerate(pieces):
        for t in range(cnt):
            tiles.append((len(tiles), pi, t == 0, t == cnt - 1))

    def tma():
        for pi in range(len(pieces)):
            q = pi & 1
            if pi >= 2:
                yield ("wait", f"q_empty{q}", (pi >> 1) - 1)
            yield ("issue", f"load_q{pi}", [f"q_full{q}"])
            for n, tp, _, _ in tiles:
                if tp != pi:
                    continue
                yield from ring_load("k", n, KS, None)
                if n >= 1:                      # V runs one tile behind K
                    yield from ring_load("v", n - 1, VS, None)
        if tiles:
            yield from ring_load("v", len(tiles) - 1, VS, None)

    def mma():
        def pv(m):
            _, pm, first, last = tiles[m]
            if first and pm >= 2:
                yield ("wait", f"o_empty{pm & 1}", (pm >> 1) - 1)
            yield ("wait", "p_full", m)
            yield ("wait", f"v_full{m % VS}", m // VS)
            yield ("event", f"PV{m}_start")
            yield ("issue", f"PV{m}", [f"v_empty{m % VS}", "p_empty"] + ([f"o_final{pm & 1}"] if last else []))
        for n, pi, first, last in tiles:
            if first:
                yield ("wait", f"q_full{pi & 1}", pi >> 1)
            yield ("wait", f"k_full{n % KS}", n // KS)
            if n >= 2:
                yield ("wait", f"s_free{n & 1}", (n - 2) >> 1)
            yield ("event", f"S{n}_start")
            yield ("issue", f"S{n}", [f"k_empty{n % KS}", f"s_full{n & 1}"] + ([f"q_empty{pi & 1}"] if last else []))
            if n >= 1:
                yield from pv(n - 1)
        if tiles:
            yield from pv(len(tiles) - 1)
        yield ("issue", "drain", ["drain"])
        yield ("wait", "drain", 0)

    def softmax(w):
        for n, pi, first, last in tiles:
            yield ("wait", f"s_full{n & 1}", n >> 1)
            yield ("event", f"readS{n}_{w}")
            yield ("arrive", f"s_free{n & 1}")
            if n >= 1 and p_wait:
                yield ("wait", "p_empty", n - 1)
            if n in rescale and not first:
                yield ("event", f"rescale{n}_{w}")
            yield ("event", f"writeP{n}_{w}")
            if n in zero_v:
                yield ("wait", f"v_full{n % VS}", n // VS)
                yield ("event", f"zeroV{n}_{w}")
            yield ("arrive", "p_full")
            if last:
                if pi >= 2:
                    yield ("wait", f"ml_empty{pi & 1}", (pi >> 1) - 1)
                yield ("event", f"writeM{pi}_{w}")
                yield ("arrive", f"ml_full{pi & 1}")

    def epilogue(w):
        for pi in range(len(pieces)):
            yield ("wait", f"o_final{pi & 1}", pi >> 1)
            yield ("wait", f"ml_full{pi & 1}", pi >> 1)
            yield ("event", f"readO{pi}_{w}")
            yield ("arrive", f"o_empty{pi & 1}")
            yield ("arrive", f"ml_empty{pi & 1}")

    roles = {"tma": tma(), "mma": mma()}
    roles.update({f"sm{w}": softmax(w) for w in range(warps)})
    roles.update({f"ep{w}": epilogue(w) for w in range(warps)})
    return roles, bars, tiles


def check_hn(tiles, pos, zero_v, KS, VS):
    W = range(4)
    piece_tiles = {}
    for n, pi, _, _ in tiles:
        piece_tiles.setdefault(pi, []).append(n)
    for n, pi, first, last in tiles:
        for w in W:
            assert pos[("done", f"S{n}")] < pos[("event", f"readS{n}_{w}")]
            assert pos[("event", f"writeP{n}_{w}")] < pos[("event", f"PV{n}_start")]
            if n >= 1:      # one P buffer: P(n) is written after P.V(n-1) read P(n-1)
                assert pos[("done", f"PV{n - 1}")] < pos[("event", f"writeP{n}_{w}")]
            if n >= 2:      # S(n) reuses the TMEM columns S(n-2) was read from
                assert pos[("event", f"readS{n - 2}_{w}")] < pos[("event", f"S{n}_start")]
            if ("event", f"rescale{n}_{w}") in pos:
                assert pos[("done", f"PV{n - 1}")] < pos[("event", f"rescale{n}_{w}")] < pos[("event", f"PV{n}_start")]
            if n in zero_v:
                assert pos[("done", f"load_v{n}")] < pos[("event", f"zeroV{n}_{w}")] < pos[("event", f"PV{n}_start")]
        if n >= KS:         # a K stage is reloaded only after the S that read it completed
            assert pos[("done", f"S{n - KS}")] < pos[("issue", f"load_k{n}")]
        if n >= VS:
            assert pos[("done", f"PV{n - VS}")] < pos[("issue", f"load_v{n}")]
    for pi, ns in piece_tiles.items():
        for w in W:         # O^T of a piece is read after its last P.V and before piece pi + 2 reuses it
            assert pos[("done", f"PV{ns[-1]}")] < pos[("event", f"readO{pi}_{w}")]
            assert pos[("event", f"writeM{pi}_{w}")] < pos[("event", f"readO{pi}_{w}")]
            if pi + 2 in piece_tiles:
                assert pos[("event", f"readO{pi}_{w}")] < pos[("event", f"PV{piece_tiles[pi + 2][0]}_start")]
                assert pos[("event", f"readO{pi}_{w}")] < pos[("event", f"writeM{pi + 2}_{w}")]
        if pi + 2 in piece_tiles:   # a Q buffer is reloaded after the piece's last S completed
            assert pos[("done", f"S{ns[-1]}")] < pos[("issue", f"load_q{pi + 2}")]


HN_CASES = [([1], (), (0,)), ([3], (0, 2), (2,)), ([2, 1], (0, 1), (1, 2)), ([1, 1, 1], (0, 1, 2), (0, 1, 2)),
            ([4, 2, 3], (0, 3, 5, 8), (3, 5)), ([5, 1, 1, 2], (0, 2, 5, 6, 7), (4, 6, 8))]


@pytest.mark.parametrize("pieces,rescale,zero_v", HN_CASES, ids=lambda c: str(c))
@pytest.mark.parametrize("KS,VS", [(3, 3), (2, 3), (3, 2)])
def test_decode_keys_as_rows_protocol(pieces, rescale, zero_v, KS, VS):
    for seed in range(40):
        roles, bars, tiles = decode_hn(pieces, KS, VS, rescale, zero_v)
        pos = first(run(roles, bars, seed))
        check_hn(tiles, pos, zero_v, KS, VS)


def test_planted_decode_keys_as_rows_missing_p_wait_is_flagged():
    """Without the wait for the previous P.V, the softmax can overwrite the
    single P buffer while the tensor cores still read it."""
    flagged = 0
    for seed in range(60):
        roles, bars, tiles = decode_hn([3, 2], 3, 3, (), (), p_wait=False)
        try:
            pos = first(run(roles, bars, seed))
            check_hn(tiles, pos, (), 3, 3)
        except AssertionError:
            flagged += 1
    assert flagged > 0
