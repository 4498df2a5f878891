"""The mbarrier hand-off protocols of the GEMM kernels, model-checked
on the CPU under random interleavings.

A GPU run only samples the interleavings its warps happen to take.  Here
each role of a kernel (producer, compute or decoder warps, MMA issuer,
epilogue) is a Python generator that issues the same barrier operations as
the kernel in the same order.  The barriers follow the mbarrier rules: a
phase completes when its pending arrivals and its transaction bytes both
reach zero; a parity wait succeeds once the phase of that parity has
completed.  Bulk copies and MMAs complete asynchronously, at random later
points.  Each shared buffer holds a tag of what was last written to it; every
read checks that the tag is the one the reader expects, so a refill that
overtakes a reader, or a reader that runs ahead of its data, fails.  Runs
that stop with roles still waiting are deadlocks.

The schedules are those of the kernels: stream-K ranges of (tile, k-block)
units over the CTAs, walked as runs of one tile (first and last flags); the
split of one CTA's range is what matters, so one CTA is modelled.  Planted
protocol mistakes (an empty barrier that counts one consumer too few, a
hand-off without its wait) must be caught, which shows that the checks can
fail.
"""
import random

import pytest


class Barrier:
    def __init__(self, count, name):
        self.count, self.pending, self.tx, self.phase, self.name = count, count, 0, 0, name

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        if self.pending < 0:
            raise Stale(f"{self.name}: more arrivals than its count")
        self._settle()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._settle()

    def _settle(self):
        if self.pending == 0 and self.tx == 0:
            self.phase ^= 1
            self.pending = self.count

    def passed(self, parity):
        # the phase with this parity has completed (a fresh barrier has "completed" parity 1)
        return self.phase != parity


class Stale(AssertionError):
    pass


def run(roles, seed, max_steps=200000):
    """Interleave the generators at random; asynchronous completions are
    extra runnable events.  Raises Stale on a wrong read, RuntimeError on a
    deadlock."""
    rng = random.Random(seed)
    mem = {}
    events = []                                   # callables: bulk-copy completions, in any order
    commits = {}                                  # role -> its MMA commits, completing in issue order
    live = {i: (g, None) for i, g in enumerate(roles)}
    for i in list(live):
        live[i] = (live[i][0], next(live[i][0], None))
    for _ in range(max_steps):
        ready = [i for i, (g, op) in live.items() if op is not None and (op[0] != "wait" or op[1].passed(op[2]))]
        choices = ([("role", i) for i in ready] + [("event", j) for j in range(len(events))]
                   + [("commit", i) for i, q in commits.items() if q])
        if not choices:
            if all(op is None for _, op in live.values()):
                return
            waiting = [f"{op[1].name}@{op[2]}" for _, op in live.values() if op is not None]
            raise RuntimeError("deadlock: roles wait on " + ", ".join(waiting))
        kind, k = rng.choice(choices)
        if kind == "event":
            events.pop(k)(mem)
            continue
        if kind == "commit":
            commits[k].pop(0)(mem)
            continue
        g, op = live[k]
        res = None
        if op[0] == "arrive":                     # ("arrive", bar[, tx])
            op[1].arrive(op[2] if len(op) > 2 else 0)
        elif op[0] == "copy":                     # ("copy", bar, nbytes, key, tag): completes later
            _, bar, nbytes, key, tag = op
            events.append(lambda m, bar=bar, nbytes=nbytes, key=key, tag=tag: (m.__setitem__(key, tag),
                                                                               bar.complete_tx(nbytes)))
        elif op[0] == "commit":
            # ("commit", bar, [reads], [writes]): the MMAs issued since the last
            # commit read their operands and write their accumulators, then the
            # barrier gets an arrival.  A commit tracks every earlier MMA of the
            # issuing thread, so one role's commits complete in issue order.
            bar, reads = op[1], op[2]
            writes = op[3] if len(op) > 3 else []

            def done(m, bar=bar, reads=reads, writes=writes):
                for key, tag in reads:
                    if m.get(key) != tag:
                        raise Stale(f"MMA read {key}: {m.get(key)} instead of {tag}")
                for key, tag in writes:
                    m[key] = tag
                bar.arrive()
            commits.setdefault(k, []).append(done)
        elif op[0] == "write":
            mem[op[1]] = op[2]
        elif op[0] == "read":
            if mem.get(op[1]) != op[2]:
                raise Stale(f"read {op[1]}: {mem.get(op[1])} instead of {op[2]}")
        elif op[0] != "wait":
            raise ValueError(op)
        live[k] = (g, g.send(res) if res is not None else next(g, None))
    raise RuntimeError("step limit")


def units_of(total, ctas, c, KB):
    """CTA c's stream-K range as (tile, kb, first, last) steps."""
    u0, u1 = total * c // ctas, total * (c + 1) // ctas
    out, u = [], u0
    while u < u1:
        tile = u // KB
        end = min(u1, (tile + 1) * KB)
        for v in range(u, end):
            out.append((tile, v - tile * KB, v == u, v == end - 1))
        u = end
    return out


# ---------------------------------------------------------------- the CUDA-core product

def small_kernel_roles(steps, stages, groups, empty_short=0, skip_red_empty=False, early_refill=False):
    """Producer + compute warps (2 halves x `groups` column groups) of
    gemm_int4_small_kernel.  empty_short, skip_red_empty and early_refill
    plant mistakes."""
    full = [Barrier(1, f"full{s}") for s in range(stages)]
    empty = [Barrier(2 * groups - empty_short, f"empty{s}") for s in range(stages)]
    red_full, red_empty = Barrier(groups, "red_full"), Barrier(groups, "red_empty")

    def producer():
        for n, (tile, kb, _, _) in enumerate(steps):
            s, ph = n % stages, (n // stages) & 1
            if n >= stages and not (early_refill and n == stages):
                yield ("wait", empty[s], ph ^ 1)
            yield ("arrive", full[s], 2)          # arrive.expect_tx: codes+scales, then X
            yield ("copy", full[s], 1, ("w", s), n)
            yield ("copy", full[s], 1, ("x", s), n)

    def compute(h, grp):
        seg = 0
        for n, (tile, kb, first, last) in enumerate(steps):
            s, ph = n % stages, (n // stages) & 1
            yield ("wait", full[s], ph)
            yield ("read", ("w", s), n)
            yield ("read", ("x", s), n)
            yield ("arrive", empty[s])
            if last:
                rph = seg & 1
                if h == 1:
                    if not skip_red_empty:
                        yield ("wait", red_empty, rph ^ 1)
                    yield ("write", ("red", grp), seg)
                    yield ("arrive", red_full)
                else:
                    yield ("wait", red_full, rph)
                    yield ("read", ("red", grp), seg)
                    yield ("arrive", red_empty)
                seg += 1

    return [producer()] + [compute(h, g) for h in (0, 1) for g in range(groups)]


SCHEDULES = [
    # total units, CTAs, CTA modelled, k-blocks per tile, stages
    (12, 1, 0, 4, 2),       # three whole tiles
    (50, 7, 3, 6, 3),       # pieces of tiles at both ends
    (40, 3, 1, 40, 2),      # one tile over several CTAs
    (9, 9, 4, 1, 2),        # one unit: first and last at once
    (60, 4, 2, 3, 5),       # short tiles, deep ring
]


@pytest.mark.parametrize("total,ctas,c,KB,stages", SCHEDULES)
def test_small_kernel_protocol(total, ctas, c, KB, stages):
    steps = units_of(total, ctas, c, KB)
    for seed in range(150):
        run(small_kernel_roles(steps, stages, groups=2), seed)


CAUGHT = (Stale, RuntimeError)                    # a wrong read, or a deadlock


def test_small_kernel_protocol_catches_planted_mistakes():
    steps = units_of(60, 2, 0, 5)
    with pytest.raises(CAUGHT):                   # a refill that does not wait for every compute warp
        for seed in range(300):
            run(small_kernel_roles(steps, 2, groups=2, empty_short=1), seed)
    with pytest.raises(Stale):                    # the first reuse of a stage without its empty wait
        for seed in range(300):
            run(small_kernel_roles(steps, 2, groups=2, early_refill=True), seed)
    with pytest.raises(CAUGHT):                   # the second half overwriting sums not yet read
        for seed in range(300):
            run(small_kernel_roles(units_of(60, 1, 0, 1), 2, groups=2, skip_red_empty=True), seed)


# ---------------------------------------------------------------- the tensor-core product

def tensor_kernel_roles(steps, stages, na, decoders=2, issuers=2, sub=2, empty_short=0):
    """Producer, decoder warps, MMA issuers and epilogue warps of
    gemm_int4_decode_kernel: decoders fill a ring of `na` tensor-memory A
    buffers (`sub` per stage); each issuer's MMAs read A and X and commit to
    the A buffer's and the stage's empty barriers (asynchronously, when the
    MMAs complete), and to an accumulator's full barrier at a tile run's end;
    the epilogue drains the accumulator (two in turn)."""
    full = [Barrier(1, f"full{s}") for s in range(stages)]
    empty = [Barrier(decoders + issuers - empty_short, f"empty{s}") for s in range(stages)]
    a_full = [Barrier(decoders, f"a_full{b}") for b in range(na)]
    a_empty = [Barrier(issuers, f"a_empty{b}") for b in range(na)]
    t_full = [Barrier(issuers, f"tmem_full{d}") for d in range(2)]
    t_empty = [Barrier(1, f"tmem_empty{d}") for d in range(2)]

    def producer():
        for n, _ in enumerate(steps):
            s, ph = n % stages, (n // stages) & 1
            if n >= stages:
                yield ("wait", empty[s], ph ^ 1)
            yield ("arrive", full[s], 2)
            yield ("copy", full[s], 1, ("codes", s), n)
            yield ("copy", full[s], 1, ("x", s), n)

    def decoder(w):
        a, aph = 0, 0
        for n, _ in enumerate(steps):
            s, ph = n % stages, (n // stages) & 1
            yield ("wait", full[s], ph)
            yield ("read", ("codes", s), n)
            yield ("arrive", empty[s])
            for b in range(sub):
                yield ("wait", a_empty[a], aph ^ 1)
                yield ("write", ("A", a, w), (n, b))
                yield ("arrive", a_full[a])
                a += 1
                if a == na:
                    a, aph = 0, aph ^ 1

    def issuer(i):
        a, aph, seg, tph = 0, 0, 0, 0
        for n, (_, _, first, last) in enumerate(steps):
            s, ph = n % stages, (n // stages) & 1
            d = seg & 1
            if first:
                yield ("wait", t_empty[d], ((tph >> d) & 1) ^ 1)
            yield ("wait", full[s], ph)
            for b in range(sub):
                yield ("wait", a_full[a], aph)
                reads = [(("A", a, w), (n, b)) for w in range(decoders)] + [(("x", s), n)]
                yield ("commit", a_empty[a], reads)
                a += 1
                if a == na:
                    a, aph = 0, aph ^ 1
            yield ("commit", empty[s], [(("x", s), n)])
            if last:
                yield ("commit", t_full[d], [])
                tph ^= 1 << d
                seg += 1

    def epilogue():
        seg, tph = 0, 0
        for n, (_, _, _, last) in enumerate(steps):
            if not last:
                continue
            d = seg & 1
            yield ("wait", t_full[d], (tph >> d) & 1)
            yield ("arrive", t_empty[d])
            tph ^= 1 << d
            seg += 1

    return ([producer()] + [decoder(w) for w in range(decoders)] + [issuer(i) for i in range(issuers)]
            + [epilogue()])


@pytest.mark.parametrize("total,ctas,c,KB,stages", SCHEDULES)
@pytest.mark.parametrize("na", [2, 3])
def test_tensor_kernel_protocol(total, ctas, c, KB, stages, na):
    steps = units_of(total, ctas, c, KB)
    for seed in range(60):
        run(tensor_kernel_roles(steps, stages, na), seed)


def test_tensor_kernel_protocol_catches_a_premature_refill():
    steps = units_of(40, 1, 0, 4)
    with pytest.raises(CAUGHT):
        for seed in range(300):
            run(tensor_kernel_roles(steps, 2, 2, empty_short=1), seed)


# ---------------------------------------------------------------- the int8 decode GEMM

def decode_visits(total, ctas, c, KB, nob):
    """walk_stages of gemm_decode_kernel for CTA c: a run that starts a tile
    opens with the tile's nob outlier stages (kind 1, a segment of their own),
    then the run's weight stages (kind 0, one segment)."""
    out = []
    for tile, kb, first, last in units_of(total, ctas, c, KB):
        if kb == 0 and first:
            out += [(1, tile, b, b == 0, b == nob - 1) for b in range(nob)]
        out.append((0, tile, kb, first, last))
    return out


def decode_kernel_roles(visits, stages, nbuf, pre, two_producers=False):
    """Producer, MMA issuer and four epilogue warps of gemm_decode_kernel:
    one ring of stages for weight and outlier stages alike; the first `pre`
    weight stages are armed and requested before the programmatic wait, their
    X tiles after it; accumulator buffers seg % nbuf, each drained by the
    epilogue before the MMAs of a later segment reuse it.  two_producers
    plants the earlier design in which a second warp filled the outlier
    stages and skipped the weight slots."""
    full = [Barrier(1, f"full{s}") for s in range(stages)]
    empty = [Barrier(1, f"empty{s}") for s in range(stages)]
    t_full = [Barrier(1, f"tmem_full{b}") for b in range(nbuf)]
    t_empty = [Barrier(4, f"tmem_empty{b}") for b in range(nbuf)]

    # the first `pre` visits are weight stages in slots 0 .. pre-1 (the kernel
    # requests none early when its range may open with outlier stages)
    assert all(visits[i][0] == 0 for i in range(min(pre, len(visits))))

    def producer(kinds):
        if 0 in kinds:
            for i in range(pre):                       # before griddepcontrol.wait
                yield ("arrive", full[i], 2)
                yield ("copy", full[i], 1, ("w", i), i)
        stage, phase, n = 0, 0, 0
        for v, (kind, tile, j, _, _) in enumerate(visits):
            if kind in kinds:
                if kind == 0 and n < pre:
                    yield ("copy", full[stage], 1, ("x", stage), v)
                else:
                    yield ("wait", empty[stage], phase ^ 1)
                    yield ("arrive", full[stage], 2)
                    yield ("copy", full[stage], 1, ("w", stage), v)
                    yield ("copy", full[stage], 1, ("x", stage), v)
            if kind == 0:
                n += 1
            stage += 1
            if stage == stages:
                stage, phase = 0, phase ^ 1

    def issuer():
        stage, phase, seg, tph = 0, 0, 0, 0
        for v, (kind, tile, j, first, last) in enumerate(visits):
            buf = seg % nbuf
            if first:
                yield ("wait", t_empty[buf], ((tph >> buf) & 1) ^ 1)
            yield ("wait", full[stage], phase)
            yield ("commit", empty[stage], [(("w", stage), v), (("x", stage), v)], [(("D", buf), ("partial", seg))])
            if last:
                yield ("commit", t_full[buf], [], [(("D", buf), ("done", seg))])
                tph ^= 1 << buf
                seg += 1
            stage += 1
            if stage == stages:
                stage, phase = 0, phase ^ 1

    def epilogue():
        seg, tph = 0, 0
        for kind, tile, j, first, last in visits:
            if not last:
                continue
            buf = seg % nbuf
            yield ("wait", t_full[buf], (tph >> buf) & 1)
            yield ("read", ("D", buf), ("done", seg))
            yield ("arrive", t_empty[buf])
            tph ^= 1 << buf
            seg += 1

    producers = [producer({0}), producer({1})] if two_producers else [producer({0, 1})]
    return producers + [issuer()] + [epilogue() for _ in range(4)]


DECODE_SCHEDULES = [
    # total units, CTAs, CTA modelled, k-blocks per tile, outlier stages, ring stages, buffers
    (24, 2, 0, 6, 2, 3, 2),     # starts two tiles: outlier segments, no early requests
    (24, 5, 2, 6, 3, 2, 4),     # starts mid-tile, then a tile with outliers
    (40, 1, 0, 5, 1, 5, 3),     # ring wraps many times around segments of different kinds
    (30, 3, 1, 30, 4, 2, 2),    # one tile over several CTAs, this CTA's piece mid-tile
    (18, 1, 0, 3, 0, 4, 4),     # no outliers
]


def _pre(visits, stages, KB, total, ctas, c):
    u0 = total * c // ctas
    if visits and visits[0][0] == 1:
        return 0
    first_seg = min(total * (c + 1) // ctas, (u0 // KB + 1) * KB) - u0
    return min(stages, first_seg)


@pytest.mark.parametrize("total,ctas,c,KB,nob,stages,nbuf", DECODE_SCHEDULES)
def test_decode_kernel_protocol(total, ctas, c, KB, nob, stages, nbuf):
    visits = decode_visits(total, ctas, c, KB, nob)
    pre = _pre(visits, stages, KB, total, ctas, c)
    for seed in range(150):
        run(decode_kernel_roles(visits, stages, nbuf, pre), seed)


def test_decode_kernel_protocol_catches_the_two_producer_design():
    """The design that faulted on the GPU: weight and outlier stages of one ring
    filled by two warps, each skipping the other's slots.  A parity wait cannot
    tell a phase from the one two laps later, so the outlier producer can pass
    the consumer and overwrite a live stage."""
    visits = decode_visits(60, 1, 0, 4, 3)
    with pytest.raises(CAUGHT):
        for seed in range(400):
            run(decode_kernel_roles(visits, 2, 2, 0, two_producers=True), seed)


# ---------------------------------------------------------------- the int8 prefill GEMM (CTA pairs)

def prefill_visits(tiles, KB, nob, defer=4):
    """walk_schedule of gemm_prefill_pair_kernel for one cluster, `tiles`
    tiles in turn (it = 0, 1, ...): each tile's K-blocks, and a tile's
    outlier stages deferred into the next tile's after `defer` K-blocks (the
    last tile's at the end)."""
    defer = min(KB, defer)
    out, prev = [], -1
    for it in range(tiles):
        for kb in range(KB):
            out.append((0, it, kb))
            if kb + 1 == defer and prev >= 0:
                out += [(1, prev, ob) for ob in range(nob)]
                prev = -1
        prev = it
    if prev >= 0:
        out += [(1, prev, ob) for ob in range(nob)]
    return out


def prefill_kernel_roles(visits, tiles, KB, nob, stages, skip_conv_wait=False, skip_empty_wait=False):
    """The two CTAs' producers, the leader's MMA issuer and the 2 x 4 epilogue
    warps of gemm_prefill_pair_kernel.  Both producers' copies complete on the
    leader's full barrier (armed by the leader with both CTAs' bytes); the
    MMAs commit to both CTAs' empty, int_full and final_full barriers; the
    epilogue warps of both CTAs arrive on the leader's acc_conv and acc_empty
    (8 arrivals).  The accumulator of tile `it` is buffer it % 2; with
    outliers the epilogue rewrites it in place (int32 -> scaled fp32) before
    the deferred outlier MMAs accumulate onto it.  skip_conv_wait plants an
    outlier MMA that does not wait for the conversion, skip_empty_wait a tile
    that does not wait for its accumulator to be drained."""
    full = [Barrier(1, f"full{s}") for s in range(stages)]
    empty = [[Barrier(1, f"empty{r}.{s}") for s in range(stages)] for r in range(2)]
    int_full = [[Barrier(1, f"int_full{r}.{b}") for b in range(2)] for r in range(2)]
    fin_full = [[Barrier(1, f"final_full{r}.{b}") for b in range(2)] for r in range(2)]
    acc_conv = [Barrier(8, f"acc_conv{b}") for b in range(2)]
    acc_empty = [Barrier(8, f"acc_empty{b}") for b in range(2)]
    D = [(r, b, q) for r in range(2) for b in range(2) for q in range(4)]

    def producer(rank):
        for v, _ in enumerate(visits):
            s, ph = v % stages, (v // stages) & 1
            if v >= stages:
                yield ("wait", empty[rank][s], ph ^ 1)
            if rank == 0:
                yield ("arrive", full[s], 2)
            yield ("copy", full[s], 1, ("half", rank, s), v)

    def issuer():
        for v, (kind, it, blk) in enumerate(visits):
            s, ph = v % stages, (v // stages) & 1
            buf, use = it & 1, (it >> 1) & 1
            if kind == 0 and blk == 0 and not skip_empty_wait:
                yield ("wait", acc_empty[buf], use ^ 1)
            if kind == 1 and blk == 0 and not skip_conv_wait:
                yield ("wait", acc_conv[buf], use)
            yield ("wait", full[s], ph)
            reads = [(("half", r, s), v) for r in range(2)]
            if kind == 0:
                writes = [(("D",) + d, ("int", it)) for d in D if d[1] == buf]
            else:
                reads += [(("D",) + d, ("conv", it) if blk == 0 else ("outl", it)) for d in D if d[1] == buf]
                writes = [(("D",) + d, ("outl", it)) for d in D if d[1] == buf]
            for r in range(2):
                yield ("commit", empty[r][s], reads if r == 0 else [], writes if r == 0 else [])
            if kind == 0 and blk == KB - 1:
                for r in range(2):
                    yield ("commit", int_full[r][buf], [])
            if kind == 1 and blk == nob - 1:
                for r in range(2):
                    yield ("commit", fin_full[r][buf], [])

    def epilogue(rank, q):
        for it in range(tiles):
            buf, use = it & 1, (it >> 1) & 1
            key = ("D", rank, buf, q)
            yield ("wait", int_full[rank][buf], use)
            yield ("read", key, ("int", it))
            if nob:
                yield ("write", key, ("conv", it))
                yield ("arrive", acc_conv[buf])
                yield ("wait", fin_full[rank][buf], use)
                yield ("read", key, ("outl", it))
            yield ("arrive", acc_empty[buf])

    return ([producer(0), producer(1), issuer()]
            + [epilogue(r, q) for r in range(2) for q in range(4)])


PREFILL_SCHEDULES = [
    # tiles of this cluster, K-blocks per tile, outlier stages, ring stages (3 in the kernel)
    (5, 6, 2, 3),
    (4, 2, 3, 3),      # fewer K-blocks than the deferral: outlier stages after the next tile's last
    (6, 5, 0, 3),      # no outliers
    (1, 4, 1, 3),      # one tile: its outlier stages at the end
    (7, 8, 4, 2),
]


@pytest.mark.parametrize("tiles,KB,nob,stages", PREFILL_SCHEDULES)
def test_prefill_kernel_protocol(tiles, KB, nob, stages):
    visits = prefill_visits(tiles, KB, nob)
    for seed in range(100):
        run(prefill_kernel_roles(visits, tiles, KB, nob, stages), seed)


def test_prefill_kernel_protocol_catches_planted_mistakes():
    visits = prefill_visits(4, 3, 2)
    with pytest.raises(Stale):                    # outlier MMAs onto an unconverted accumulator
        for seed in range(300):
            run(prefill_kernel_roles(visits, 4, 3, 2, 3, skip_conv_wait=True), seed)
    visits = prefill_visits(5, 2, 0)
    with pytest.raises(Stale):                    # a tile's MMAs over an accumulator not yet drained
        for seed in range(300):
            run(prefill_kernel_roles(visits, 5, 2, 0, 3, skip_empty_wait=True), seed)


# ---------------------------------------------------------------- the cooperative activation kernel

def grid_barrier_run(blocks, failing, seed, fail_after_arrive=False):
    """The grid barrier of activation_fused_kernel, one step per memory
    operation.  Block b ORs its rows' bit into the mask if its row copies
    arrived (all but `failing`); a block whose copies never arrived sets the
    fail word; every block then adds itself to the counter and waits (bounded)
    for all.  A block that goes on (counter complete, fail word clear) reads
    the mask, which must hold the bits of every block.  Returns the blocks
    that went on and the blocks whose wait gave up."""
    rng = random.Random(seed)
    mem = {"mask": 0, "ctr": 0, "fail": 0}

    def block(b):
        ok = b not in failing
        if ok:
            mem["mask"] |= 1 << b
            yield
        if not ok and not fail_after_arrive:
            mem["fail"] = 1
            yield
        mem["ctr"] += 1
        yield
        if not ok and fail_after_arrive:
            mem["fail"] = 1
            yield
        for _ in range(50):                           # the bounded wait
            if mem["ctr"] >= blocks:
                break
            yield
        else:
            return ("gave_up", b)
        yield
        if ok and mem["fail"] == 0:
            if mem["mask"] != (1 << blocks) - 1:
                raise Stale(f"block {b} went on with mask {mem['mask']:b}")
            return ("went_on", b)
        return ("stopped", b)

    gens = {b: block(b) for b in range(blocks)}
    result = {}
    while gens:
        b = rng.choice(list(gens))
        try:
            next(gens[b])
        except StopIteration as e:
            result[b] = e.value
            del gens[b]
    return result


@pytest.mark.parametrize("blocks,failing", [(6, set()), (6, {2}), (5, {0, 4}), (8, {7})])
def test_grid_barrier_never_goes_on_with_an_incomplete_mask(blocks, failing):
    for seed in range(400):
        out = grid_barrier_run(blocks, failing, seed)
        went = [b for b, (what, _) in out.items() if what == "went_on"]
        if failing:
            assert not went                            # the fail word stops every block
        else:
            assert all(what in ("went_on", "gave_up") for what, _ in out.values())


def test_grid_barrier_model_catches_a_late_fail_word():
    """Setting the fail word after arriving (the earlier ordering) lets a fast
    block pass the barrier with a mask that lacks the failed block's rows."""
    with pytest.raises(Stale):
        for seed in range(400):
            grid_barrier_run(6, {3}, seed, fail_after_arrive=True)
