"""Discrete-event models of the barrier protocols of the warp-specialised
kernels (csrc/prefill_sm100.cu prefill_kernel, csrc/prefill_bwd_sm100.cu
bt_dkv_kernel and bq_dq_kernel, and the CTA pair of
csrc/mla_decode_tc.cu mla_decode_tc_kernel, on mbarriers; csrc/mla_decode.cu
mla_decode_ws_kernel on named barriers), checked for deadlock, parity
aliasing, buffers refilled before they were read, and mismatched
named-barrier use under many random interleavings.

Each role of a kernel (TMA producers, MMA issuers, elementwise and epilogue
warps) is restated as the sequence of its waits, arrivals and MMA commits, in
the kernel's order.  The engine follows PTX semantics:
  * an mbarrier completes a phase when its expected arrival count is reached;
  * mbarrier.try_wait.parity(P) succeeds iff the number of completed phases
    has the other parity than P, so a waiter for phase p that is two phases
    behind the barrier succeeds wrongly (flagged as aliasing) and one that is
    two phases ahead hangs (a deadlock);
  * a TMA load arrives on its barrier some time after it is issued;
  * tcgen05.commit arrives once every MMA its thread issued before it has
    completed; each issuing thread's MMAs complete in issue order.
A mutation test checks that the engine catches a protocol bug of this kind.
"""
import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


def _simulate(bars, roles, seed, max_rounds=400000):
    """roles: name -> generator yielding ("wait", bar, phase), ("arrive", bar),
    ("load", bar[, key]) (a TMA load or bulk copy completing later on bar;
    with a key, its completion also marks a read of its source buffer),
    ("mma", issuer) / ("commit", issuer, bar), or ("mark", key) / ("expect",
    key, n) (a buffer read finished / a write that needs n reads done before
    it: a shortfall is reported with the aliasing events).  Returns (status,
    stuck waits, aliasing events)."""
    rng = random.Random(seed)
    B = {name: _Bar(count) for name, count in bars.items()}
    aliasing, loads, mma, marks = [], [], {}, {}
    cur = {k: None for k in roles}
    done = set()

    def wait_ok(name, p):
        d = B[name].done
        ok = (d & 1) != (p & 1)
        if ok and d < p + 1:
            aliasing.append((name, p, d))
        return ok

    for _ in range(max_rounds):
        if len(done) == len(roles):
            return "ok", None, aliasing
        progressed = False
        order = list(roles) + ["loads"] + ["mma:" + k for k in mma]
        rng.shuffle(order)
        for c in order:
            if c == "loads":
                if loads and rng.random() < 0.5:
                    name, key = loads.pop(0)
                    B[name].arrive()
                    if key is not None:
                        marks[key] = marks.get(key, 0) + 1
                    progressed = True
            elif c.startswith("mma:"):
                q = mma[c[4:]]
                if q and rng.random() < 0.5:
                    e = q.pop(0)
                    if e is not None:
                        B[e].arrive()
                    progressed = True
            elif c not in done:
                while True:
                    if cur[c] is None:
                        try:
                            cur[c] = next(roles[c])
                        except StopIteration:
                            done.add(c)
                            break
                    a = cur[c]
                    if a[0] == "wait":
                        if not wait_ok(a[1], a[2]):
                            break
                    elif a[0] == "arrive":
                        B[a[1]].arrive()
                    elif a[0] == "load":
                        loads.append((a[1], a[2] if len(a) > 2 else None))
                    elif a[0] == "mma":
                        mma.setdefault(a[1], []).append(None)
                    elif a[0] == "commit":
                        mma.setdefault(a[1], []).append(a[2])
                    elif a[0] == "mark":          # a read of a buffer finished
                        marks[a[1]] = marks.get(a[1], 0) + 1
                    elif a[0] == "expect":        # a write needs that many reads done first
                        if marks.get(a[1], 0) < a[2]:
                            aliasing.append(("overwrite", a[1], a[2], marks.get(a[1], 0)))
                    cur[c] = None
                    progressed = True
        if not progressed and not loads and not any(mma.values()):
            return "deadlock", {k: cur[k] for k in roles if k not in done}, aliasing
    return "timeout", None, aliasing


# ---------------------------------------------------------------- prefill_kernel
def _prefill_roles(tiles, rescale_rng):
    """tiles[n]: K/V tiles of work item n.  Two S buffers, two Q, K, V stages;
    softmax halves h = 0, 1; the epilogue warpgroup releases O (B_OFREE)."""
    NS = QS = KS = VS = 2
    bars = {"OFREE": 1, "UDONE": 2}
    for i in range(2):
        bars.update({f"QF{i}": 1, f"QE{i}": 1, f"KF{i}": 1, f"KE{i}": 1, f"VF{i}": 1, f"VE{i}": 1,
                     f"S{i}": 1, f"P0_{i}": 1, f"P1_{i}": 1, f"O{i}": 1})

    def tma_qk():
        gt = 0
        for n, T in enumerate(tiles):
            if n >= QS:
                yield ("wait", f"QE{n % QS}", n // QS - 1)
            yield ("load", f"QF{n % QS}")
            for _ in range(T):
                if gt >= KS:
                    yield ("wait", f"KE{gt % KS}", gt // KS - 1)
                yield ("load", f"KF{gt % KS}")
                gt += 1

    def tma_v():
        gt = 0
        for T in tiles:
            for _ in range(T):
                if gt >= VS:
                    yield ("wait", f"VE{gt % VS}", gt // VS - 1)
                yield ("load", f"VF{gt % VS}")
                gt += 1

    def qk():
        gt = 0
        for n, T in enumerate(tiles):
            yield ("wait", f"QF{n % QS}", n // QS)
            for _ in range(T):
                bf = gt % NS
                yield ("wait", f"KF{gt % KS}", gt // KS)
                if gt >= NS:
                    yield ("wait", f"O{bf}", (gt - NS) // NS)   # S buffer free: PV two tiles back done
                yield ("mma", "qk")
                yield ("commit", "qk", f"S{bf}")
                yield ("commit", "qk", f"KE{gt % KS}")
                gt += 1
            yield ("commit", "qk", f"QE{n % QS}")

    def pv():
        gt = 0
        for n, T in enumerate(tiles):
            for j in range(T):
                bf = gt % NS
                yield ("wait", f"VF{gt % VS}", gt // VS)
                if j == 0 and n > 0:
                    yield ("wait", "OFREE", n - 1)
                for h in range(2):
                    yield ("wait", f"P{h}_{bf}", gt // NS)
                    yield ("mma", "pv")
                yield ("commit", "pv", f"O{bf}")
                yield ("commit", "pv", f"VE{gt % VS}")
                gt += 1

    def softmax(h):
        gt = 0
        for n, T in enumerate(tiles):
            for j in range(T):
                yield ("wait", f"S{gt % NS}", gt // NS)
                if j > 0 and rescale_rng.random() < 0.3:   # the lazy rescale reads O after the last PV
                    yield ("wait", f"O{(gt - 1) % NS}", (gt - 1) // NS)
                yield ("arrive", f"P{h}_{gt % NS}")
                gt += 1
            if n > 0:
                yield ("wait", "OFREE", n - 1)   # exchange buffer read by the last epilogue
            yield ("arrive", "UDONE")

    def epilogue():
        gt = 0
        for n, T in enumerate(tiles):
            gt += T
            yield ("wait", "UDONE", n)
            yield ("wait", f"O{(gt - 1) % NS}", (gt - 1) // NS)
            yield ("arrive", "OFREE")

    roles = {"tma_qk": tma_qk(), "tma_v": tma_v(), "qk": qk(), "pv": pv(), "s0": softmax(0), "s1": softmax(1),
             "epi": epilogue()}
    return bars, roles


def _cases(seed, n_cases, max_items, max_len):
    rng = random.Random(seed)
    return [[1], [2], [1, 1], [3, 1, 2]] + [[rng.randint(1, max_len) for _ in range(rng.randint(1, max_items))]
                                            for _ in range(n_cases)]


def test_prefill_kernel_protocol():
    for items in _cases(3, 30, 6, 6):
        for seed in range(25):
            bars, roles = _prefill_roles(items, random.Random(seed + 1000))
            status, stuck, aliasing = _simulate(bars, roles, seed)
            assert status == "ok" and not aliasing, (items, seed, status, stuck, aliasing)


# ---------------------------------------------------------------- bt_dkv_kernel
def _dkv_roles(n, nbuf, qs):
    bars = {"KV": 1, "DV": 1, "DK": 1, "DRAIN": 2}
    for s in range(qs):
        bars.update({f"QT{s}": 1, f"QF{s}": 1, f"QE{s}": 2})
    for b in range(nbuf):
        bars.update({f"S{b}": 1, f"DP{b}": 1, f"P{b}": 1, f"DS{b}": 1})

    def tma():
        yield ("load", "KV")
        for s in range(n):
            if s >= qs:
                yield ("wait", f"QE{s % qs}", s // qs - 1)
            yield ("load", f"QT{s % qs}")

    def loader():
        for s in range(n):
            yield ("wait", f"QT{s % qs}", s // qs)
            yield ("arrive", f"QF{s % qs}")

    def issuer(side):
        prod, inp, acc = ("S", "P", "DV") if side == "p" else ("DP", "DS", "DK")
        yield ("wait", "KV", 0)
        for t in range(n + nbuf - 1):
            if t < n:
                yield ("wait", f"QF{t % qs}", t // qs)
                if t >= nbuf:
                    yield ("wait", acc, t - nbuf)   # buffer free: this side's accumulation nbuf steps back
                yield ("mma", side)
                yield ("commit", side, f"{prod}{t % nbuf}")
            s = t - (nbuf - 1)
            if s >= 0:
                yield ("wait", f"{inp}{s % nbuf}", s // nbuf)
                yield ("mma", side)
                yield ("commit", side, acc)
                yield ("commit", side, f"QE{s % qs}")
        yield ("commit", side, "DRAIN")

    def elementwise():
        for s in range(n):
            b = s % nbuf
            yield ("wait", f"QF{s % qs}", s // qs)
            yield ("wait", f"S{b}", s // nbuf)
            yield ("arrive", f"P{b}")
            yield ("wait", f"DP{b}", s // nbuf)
            yield ("arrive", f"DS{b}")
        yield ("wait", "DRAIN", 0)

    return bars, {"tma": tma(), "ld": loader(), "p": issuer("p"), "d": issuer("d"), "ew": elementwise()}


@pytest.mark.parametrize("nbuf,qs", [(2, 4), (1, 2)], ids=["64-query steps, two buffers", "128-query steps"])
def test_dkv_kernel_protocol(nbuf, qs):
    for n in range(1, 13):
        for seed in range(40):
            bars, roles = _dkv_roles(n, nbuf, qs)
            status, stuck, aliasing = _simulate(bars, roles, seed)
            assert status == "ok" and not aliasing, (n, seed, status, stuck, aliasing)


# ---------------------------------------------------------------- bq_dq_kernel
def _dq_roles(items, boundary_bug=False):
    """items[n]: key-tile steps of the n-th query tile a CTA walks (the kernel
    takes one; the persistent form, several, with Q/dO and dQ handed over
    between tiles)."""
    KST, VST = 3, 2
    bars = {"Q": 1, "QFREE": 2, "S": 1, "SC": 1, "DP": 1, "DS": 1, "DQ": 1, "DQDONE": 1, "DQFREE": 1, "DRAIN": 2}
    for s in range(KST):
        bars.update({f"KF{s}": 1, f"KE{s}": 1})
    for s in range(VST):
        bars.update({f"VF{s}": 1, f"VE{s}": 1})
    state = {"gj": 0}

    def tma():
        gj = 0

        def load_kv():
            nonlocal gj
            if gj >= KST:
                yield ("wait", f"KE{gj % KST}", gj // KST - 1)
            yield ("load", f"KF{gj % KST}")
            if gj >= VST:
                yield ("wait", f"VE{gj % VST}", gj // VST - 1)
            yield ("load", f"VF{gj % VST}")
            gj += 1
        for n, ns in enumerate(items):
            yield from load_kv()
            if n > 0:
                yield ("wait", "QFREE", n - 1)
            yield ("load", "Q")
            for _ in range(1, ns):
                yield from load_kv()

    def issuer_s():
        gj = 0
        for n, ns in enumerate(items):
            yield ("wait", "Q", n)
            for _ in range(ns):
                yield ("wait", f"KF{gj % KST}", gj // KST)
                if gj > 0:
                    yield ("wait", "SC", gj - 1)
                yield ("mma", "a")
                yield ("commit", "a", "S")
                gj += 1
            yield ("commit", "a", "QFREE")
        yield ("commit", "a", "DRAIN")

    def issuer_dp_dq():
        gj = 0

        def dq(x, first, n):
            if first and n > 0:
                yield ("wait", "DQFREE", n - 1)
            yield ("mma", "b")
            yield ("commit", "b", "DQ")
            yield ("commit", "b", f"KE{x % KST}")
        for n, ns in enumerate(items):
            yield ("wait", "Q", n)
            for j in range(ns):
                yield ("wait", f"VF{gj % VST}", gj // VST)
                if gj > 0:
                    yield ("wait", "DS", gj - 1)
                if j == 0 and gj > 0 and not boundary_bug:
                    yield ("wait", "DQ", gj - 1)
                elif gj > 1:
                    yield ("wait", "DQ", gj - 2)
                yield ("mma", "b")
                yield ("commit", "b", "DP")
                yield ("commit", "b", f"VE{gj % VST}")
                if j > 0:
                    yield from dq(gj - 1, j == 1, n)
                gj += 1
            yield ("commit", "b", "QFREE")
            yield ("wait", "DS", gj - 1)
            yield from dq(gj - 1, ns == 1, n)
            yield ("commit", "b", "DQDONE")
        yield ("commit", "b", "DRAIN")

    def elementwise():
        gj = 0
        for n, ns in enumerate(items):
            for _ in range(ns):
                yield ("wait", "S", gj)
                yield ("arrive", "SC")
                yield ("wait", "DP", gj)
                yield ("arrive", "DS")
                gj += 1
            yield ("wait", "DQDONE", n)
            yield ("arrive", "DQFREE")

    return bars, {"tma": tma(), "a": issuer_s(), "b": issuer_dp_dq(), "ew": elementwise()}


def test_dq_kernel_protocol():
    for items in [[n] for n in range(1, 12)] + _cases(7, 25, 5, 6):
        for seed in range(30):
            bars, roles = _dq_roles(items)
            status, stuck, aliasing = _simulate(bars, roles, seed)
            assert status == "ok" and not aliasing, (items, seed, status, stuck, aliasing)


def test_engine_catches_a_parity_aliasing_bug():
    """The dq protocol with several query tiles per CTA and the wait for
    dQ(gj-2) kept at a tile's first step (where the previous tile's last dQ,
    dQ(gj-1), may already have completed) deadlocks under some interleaving."""
    failures = 0
    for items in ([3, 3], [2, 1], [5, 4]):
        for seed in range(30):
            bars, roles = _dq_roles(items, boundary_bug=True)
            status, _, aliasing = _simulate(bars, roles, seed)
            failures += status != "ok" or bool(aliasing)
    assert failures > 0


# ---------------------------------------------------------------- mla_decode_tc_kernel
def _mla_tc_roles(nblk, rescale_rng, qk_runs_ahead=False, single_p_staging=False):
    """Both CTAs of a pair (ranks 0, 1), warps as roles; barrier names carry
    the rank.  Per CTA: TMA (three K/V stages), the MMA issuer (QK(j) into S
    buffer j % 2 once PV(j - 2) has completed, then PV(j - 1) once P(j - 1)
    is in), four owner warps (S, then the other CTA's partial scores, the
    softmax, a bulk copy of P to the other CTA, P in), four sender warps
    (S, then a push of the other CTA's rows to it) and four receiver warps
    (the other CTA's P, P in).  The receive buffers have no acknowledgement;
    "expect" checks that each is refilled only after its previous contents
    were read, that P is written over S only after S was read, and that an
    owner refills its P staging buffer only after the copy that last read
    it has completed (the copy completes on the other CTA's barrier; no
    bulk-group wait covers it, only the exchange's causal chain)."""
    ST = 3
    bars = {}
    for r in range(2):
        for i in range(ST):
            bars.update({f"{r}KF{i}": 1, f"{r}KE{i}": 1})
        for i in range(2):
            bars.update({f"{r}S{i}": 1, f"{r}PF{i}": 8, f"{r}O{i}": 1, f"{r}RS{i}": 4, f"{r}RP{i}": 1 + 4})

    def init(r):
        for i in range(2):
            yield ("arrive", f"{r}RP{i}")            # the receive buffers' first phases armed

    def tma(r):
        for j in range(nblk):
            if j >= ST:
                yield ("wait", f"{r}KE{j % ST}", j // ST - 1)
            yield ("load", f"{r}KF{j % ST}")

    def mma(r):
        for j in range(nblk + 1):
            if j < nblk:
                sb = j & 1
                yield ("wait", f"{r}KF{j % ST}", j // ST)
                if j >= 2:
                    yield ("wait", f"{r}O{sb}", (j - 2) >> 1)
                yield ("expect", f"{r}Sread{sb}", 8 * (j >> 1))   # S(j - 2) read by owners and senders
                yield ("mma", f"{r}")
                yield ("commit", f"{r}", f"{r}S{sb}")
            if j >= 1:
                i = j - 1
                yield ("wait", f"{r}PF{i & 1}", i >> 1)
                yield ("mma", f"{r}")
                yield ("commit", f"{r}", f"{r}O{i & 1}")
                yield ("commit", f"{r}", f"{r}KE{i % ST}")

    def owner(r, q):
        o = 1 - r
        for j in range(nblk):
            sb = j & 1
            yield ("wait", f"{r}S{sb}", j >> 1)
            yield ("mark", f"{r}Sread{sb}")
            yield ("wait", f"{r}RS{sb}", j >> 1)
            yield ("mark", f"{r}RSread{sb}")
            if j > 0 and rescale_rng.random() < 0.3:
                yield ("wait", f"{r}O{sb ^ 1}", (j - 1) >> 1)
            yield ("expect", f"{o}RPread{sb}", 4 * (j >> 1))   # the other CTA read P(j - 2) from buffer sb
            ps = 0 if single_p_staging else sb
            yield ("expect", f"{r}PSread{ps}{q}", j if single_p_staging else j >> 1)   # staging free
            yield ("load", f"{o}RP{sb}", f"{r}PSread{ps}{q}")     # bulk copy of P and the factors
            yield ("arrive", f"{r}PF{sb}")
        if nblk > 0:
            yield ("wait", f"{r}O{(nblk - 1) & 1}", (nblk - 1) >> 1)

    def sender(r, q):
        o = 1 - r
        for j in range(nblk):
            sb = j & 1
            yield ("wait", f"{r}S{sb}", j >> 1)
            yield ("mark", f"{r}Sread{sb}")
            yield ("mark", f"{r}Ssent{q}")
            yield ("expect", f"{o}RSread{sb}", 4 * (j >> 1))   # the other CTA read S(j - 2) from buffer sb
            yield ("arrive", f"{o}RS{sb}")

    def receiver(r, q):
        for j in range(nblk):
            sb = j & 1
            yield ("wait", f"{r}RP{sb}", j >> 1)
            if q == 0 and j + 2 < nblk:
                yield ("arrive", f"{r}RP{sb}")                 # one thread arms buffer sb's next phase
            yield ("mark", f"{r}RPread{sb}")
            if j > 0 and rescale_rng.random() < 0.3:
                yield ("wait", f"{r}O{sb ^ 1}", (j - 1) >> 1)
            yield ("expect", f"{r}Ssent{q}", j + 1)            # P over S(j) only after the sender read it
            yield ("arrive", f"{r}PF{sb}")
        if nblk > 0:
            yield ("wait", f"{r}O{(nblk - 1) & 1}", (nblk - 1) >> 1)

    def qk_only(r):   # the mutation: QK issued as soon as its rows land
        for j in range(nblk):
            yield ("wait", f"{r}KF{j % ST}", j // ST)
            yield ("expect", f"{r}Sread{j & 1}", 8 * (j >> 1))
            yield ("mma", f"{r}q")
            yield ("commit", f"{r}q", f"{r}S{j & 1}")

    def pv_only(r):
        for i in range(nblk):
            yield ("wait", f"{r}PF{i & 1}", i >> 1)
            yield ("mma", f"{r}p")
            yield ("commit", f"{r}p", f"{r}O{i & 1}")
            yield ("commit", f"{r}p", f"{r}KE{i % ST}")

    roles = {}
    for r in range(2):
        roles[f"init{r}"] = init(r)
        roles[f"tma{r}"] = tma(r)
        if qk_runs_ahead:
            roles[f"qk{r}"] = qk_only(r)
            roles[f"pv{r}"] = pv_only(r)
        else:
            roles[f"mma{r}"] = mma(r)
        for q in range(4):
            roles[f"own{r}{q}"] = owner(r, q)
            roles[f"snd{r}{q}"] = sender(r, q)
            roles[f"rcv{r}{q}"] = receiver(r, q)
    return bars, roles


def test_mla_tc_kernel_pair_protocol():
    for nblk in list(range(0, 9)) + [13, 20]:
        for seed in range(30):
            bars, roles = _mla_tc_roles(nblk, random.Random(seed + 77))
            status, stuck, aliasing = _simulate(bars, roles, seed)
            assert status == "ok" and not aliasing, (nblk, seed, status, stuck, aliasing)


def test_mla_tc_model_catches_a_single_p_staging_buffer():
    """With one P staging buffer per owner warp instead of two, block j's
    stores could overwrite P(j - 1) while its copy to the other CTA still
    reads it: nothing in the exchange orders the two."""
    flagged = 0
    for seed in range(30):
        bars, roles = _mla_tc_roles(8, random.Random(seed), single_p_staging=True)
        status, _, aliasing = _simulate(bars, roles, seed)
        flagged += status != "ok" or bool(aliasing)
    assert flagged > 0


def test_mla_tc_model_catches_a_missing_buffer_wait():
    """If QK ran ahead of the PV products (issued as soon as its rows land,
    without the wait for PV(j - 2)), S(j - 2) could be overwritten before it
    is read and the phases of its barrier alias."""
    flagged = 0
    for seed in range(30):
        bars, roles = _mla_tc_roles(8, random.Random(seed), qk_runs_ahead=True)
        status, _, aliasing = _simulate(bars, roles, seed)
        flagged += status != "ok" or bool(aliasing)
    assert flagged > 0


# ---------------------------------------------------------------- mla_decode_ws_kernel
def _simulate_named(nblk, seed, skip_p_read_sync=False):
    """Named barriers (bar.sync / bar.arrive with 384 threads: the QK
    warpgroup, 128, and the eight PV warps, 256).  A barrier completes a
    generation when both groups have arrived; bar.sync also waits for that
    generation.  A group arriving twice in one generation (its next use
    counted toward the current one) is flagged."""
    rng = random.Random(seed)
    gen = {i: 0 for i in range(1, 7)}
    arrived = {i: set() for i in range(1, 7)}
    misuse = []

    def arrive(i, who):
        if who in arrived[i]:
            misuse.append((i, who, gen[i]))
        arrived[i].add(who)
        if arrived[i] == {"qk", "pv"}:
            arrived[i] = set()
            gen[i] += 1
            return gen[i] - 1
        return gen[i]

    def qk():
        for kb in range(nblk):
            bb = kb & 1
            yield ("sync", 1 + bb)          # block kb landed
            if kb >= 2 and not skip_p_read_sync:
                yield ("sync", 5 + bb)      # P buffer bb read by the PV warps (block kb - 2)
            yield ("arrive", 3 + bb)        # P of block kb ready

    def pv():
        if nblk > 0:
            yield ("arrive", 1)             # block 0 landed
        for kb in range(nblk):
            bb = kb & 1
            if kb + 1 < nblk:
                yield ("arrive", 1 + (bb ^ 1))   # block kb + 1 landed
            yield ("sync", 3 + bb)          # P of block kb ready
            if kb + 2 < nblk:
                yield ("arrive", 5 + bb)    # P buffer bb read

    roles = {"qk": qk(), "pv": pv()}
    cur = {"qk": None, "pv": None}
    waiting = {}   # role -> (barrier, generation it waits to complete)
    done = set()
    for _ in range(100000):
        if len(done) == 2:
            return "ok", misuse
        progressed = False
        for who in rng.sample(list(roles), 2):
            if who in done:
                continue
            if who in waiting:
                i, g = waiting[who]
                if gen[i] > g:
                    del waiting[who]
                    progressed = True
                continue
            try:
                a = next(roles[who])
            except StopIteration:
                done.add(who)
                progressed = True
                continue
            g = arrive(a[1], who)
            if a[0] == "sync" and gen[a[1]] <= g:
                waiting[who] = (a[1], g)
            progressed = True
        if not progressed:
            return "deadlock", misuse
    return "timeout", misuse


def test_mla_ws_kernel_named_barrier_protocol():
    for nblk in range(0, 12):
        for seed in range(40):
            status, misuse = _simulate_named(nblk, seed)
            assert status == "ok" and not misuse, (nblk, seed, status, misuse)


def test_named_barrier_engine_catches_a_missing_sync():
    """Without the QK warps' wait for "P buffer read", the PV warps' arrivals
    pile up on that barrier (two arrivals of one group in a generation)."""
    flagged = 0
    for seed in range(20):
        status, misuse = _simulate_named(6, seed, skip_p_read_sync=True)
        flagged += status != "ok" or bool(misuse)
    assert flagged > 0
