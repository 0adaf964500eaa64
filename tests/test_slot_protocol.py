"""A discrete model of one CTA's expert-slot and accumulator-buffer protocol
in msk_kernel.cu, checked on the CPU.

The kernel's producer warp fills the expert slots (full barrier xfull[s],
one phase per fill), the two issuing warps and the consumer warps consume
them, and the slots are released by the tensor-core commits (xempty[s], two
arrivals) or by the consumer warps (xempty_cc[s]).  The block-scaled items
hand their fp32 accumulators over through dfull2 / dempty2.  Every waiter
tracks the barriers by parity only, so a wait is correct only if the waiter
is never two phases ahead of the barrier.  The parts of one layer come in
this order: block-scaled gate/up, CUDA-core gate/up, block-scaled down,
CUDA-core down; each agent skips over the parts it does not consume by
flipping its parities (fill_parity / fill_parity_run in the kernel).

The model runs the three agents as coroutines under a random scheduler with
random item counts per part and asserts that every wait passes on exactly
the fill (or the item's commits) it means.  It transcribes the kernel's
bookkeeping: prod_xslot / prod_xdrain, the issuer's gate/up and down loops
(the down items alternate between the issuing warps), expert_gu_tc,
expert_mma and expert_dt_tc.  The issuing warps' wait for the gate/up phase
to end before the block-scaled down fills is what keeps their first down
wait from matching a CUDA-core gate/up fill two phases earlier; the second
test shows the model finds that mistake when the wait is left out.

The tensor-core products complete asynchronously, after their issue, and
the commits that follow them arrive only then.  A scale-factor copy into
TMEM is not ordered after earlier products that read the same columns, so
the model also checks that every such copy comes after those products have
completed, as seen through the slot chain; the third test shows that this
needs down items of at most two K chunks.
"""
import random


class Barrier:
    """mbarrier: `count` arrivals complete a phase; try_wait.parity(p) is
    true when the phase with parity p has completed (current parity != p)."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, (self.name, "more arrivals than the phase takes")
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1

    def ready(self, parity):
        return (self.done & 1) != parity


def fill_parity(n_items, nkc, ns):
    n, m = n_items * nkc, 0
    for s in range(ns):
        if ((n // ns) + (1 if s < n % ns else 0)) & 1:
            m |= 1 << s
    return m


def fill_parity_run(nkc, ns, i):
    m = 0
    for j in range(i * nkc, (i + 1) * nkc):
        m ^= 1 << (j % ns)
    return m


def simulate(seed, layers=4, issuer_waits_for_gate_up=True, dt_chunks=(1, 2)):
    """Returns None when every wait matched its fill and every scale buffer
    was reused only after the products that read it completed, else a
    description.  dt_chunks: the K chunks per block-scaled down item to draw
    from (512-wide chunks: f / 512)."""
    rnd = random.Random(seed)
    xfull = [Barrier(f"xfull{i}", 1) for i in range(4)]
    xempty = [Barrier(f"xempty{i}", 2) for i in range(4)]
    xempty_cc = [Barrier(f"xempty_cc{i}", 1) for i in range(4)]  # the 8 consumer warps as one arrival
    dfull = [Barrier(f"dfull2_{i}", 2) for i in range(2)]
    dempty = [Barrier(f"dempty2_{i}", 1) for i in range(2)]
    fills = {s: [] for s in range(4)}
    state = {"route": 0, "gu_done": 0, "ring_free": 0}
    # per layer: (items, chunks per item, slots) of each part
    geo = []
    for _ in range(layers):
        g = {"tc": (rnd.randint(0, 3), 8, 4), "cc": (rnd.randint(0, 3), 4, 2),
             "dt": (rnd.randint(0, 4), rnd.choice(dt_chunks), 3), "dn": (rnd.randint(0, 3), 1, 3)}
        # whether the layer has block-scaled units / CUDA-core units at all
        # (the same on every CTA; a CTA's share of a part may still be empty)
        g["tc_on"], g["cc_on"] = rnd.random() < 0.9, rnd.random() < 0.7
        g["dt_on"] = g["tc_on"]
        for name, on in (("tc", g["tc_on"]), ("dt", g["dt_on"]), ("cc", g["cc_on"]), ("dn", g["cc_on"])):
            if not on:
                g[name] = (0,) + g[name][1:]
        geo.append(g)
    errors = []
    # the tensor pipe: per issuing warp, its issued chunks' products in issue
    # order, completing later; the commits after them arrive on completion
    pipe = {0: [], 1: []}
    # scale-factor TMEM columns in units of (buffer 0-3, half 0-1) of 16
    # columns: gate/up chunk j uses buffer j mod 4, half = the warp's role;
    # a down chunk uses both halves of buffer 2 (its warp's chunk count mod 2)
    # + role.  scale_user: the products that read a unit last
    scale_user = {}

    def issue(role, key, units, arrivals):
        op = {"key": key, "done": False, "arrivals": arrivals}
        for u in units:
            prev = scale_user.get(u)
            if prev is not None and not prev["done"]:
                errors.append(f"issuer {role}: scale columns {u} copied for {key} while the products of "
                              f"{prev['key']} may still read them")
            scale_user[u] = op
        pipe[role].append(op)

    def tensor_pipe():
        while True:
            busy = [r for r in (0, 1) if pipe[r]]
            if busy:
                op = pipe[rnd.choice(busy)].pop(0)
                op["done"] = True
                for bar, n in op["arrivals"]:
                    bar.arrive(n)
            yield

    def check_fill(s, key, who):
        idx = fills[s].index(key) if key in fills[s] else None
        if idx is None or xfull[s].done != idx + 1:
            errors.append(f"{who}: slot {s} wait for {key} passed with {xfull[s].done} fills landed")

    def producer():
        used = last_tc = par_tc = par_cc = 0

        def slot(s, tc):
            nonlocal used, last_tc, par_tc, par_cc
            if (used >> s) & 1:
                ltc = (last_tc >> s) & 1
                bar = xempty[s] if ltc else xempty_cc[s]
                par = (((par_tc if ltc else par_cc) >> s) & 1) ^ 1
                while not bar.ready(par):
                    yield
            used |= 1 << s
            if tc:
                par_tc ^= 1 << s
                last_tc |= 1 << s
            else:
                par_cc ^= 1 << s
                last_tc &= ~(1 << s)

        def drain():
            for s in range(4):
                if (used >> s) & 1:
                    ltc = (last_tc >> s) & 1
                    bar = xempty[s] if ltc else xempty_cc[s]
                    par = (((par_tc if ltc else par_cc) >> s) & 1) ^ 1
                    while not bar.ready(par):
                        yield

        def part(l, name, tc):
            n_items, nkc, ns = geo[l][name]
            for j in range(n_items * nkc):
                s = j % ns
                yield from slot(s, tc)
                fills[s].append((l, name, j // nkc, j % nkc))
                xfull[s].arrive()
                yield

        for l in range(layers):
            while state["route"] <= l:
                yield
            g = geo[l]
            if g["tc_on"]:
                yield from part(l, "tc", True)
            if g["tc_on"] and g["cc_on"]:
                yield from drain()
            if g["cc_on"]:
                yield from part(l, "cc", False)
            while state["gu_done"] <= l:
                yield
            if g["dt_on"]:
                yield from drain()
                yield from part(l, "dt", True)
            if g["cc_on"]:
                if g["dt_on"]:
                    yield from drain()
                yield from part(l, "dn", False)
            while state["ring_free"] <= l:
                yield

    def issuer(role):
        bits = 0  # 0-3 slot parities, 4-5 dempty2 parities, 6-7 buffer used
        for l in range(layers):
            g = geo[l]
            while state["route"] <= l:
                yield
            n_items, nkc, ns = g["tc"]
            for j in range(n_items * nkc):
                it, kc, s = j // nkc, j % nkc, j % ns
                db = it & 1
                while not xfull[s].ready((bits >> s) & 1):
                    yield
                check_fill(s, (l, "tc", it, kc), f"issuer {role} gate/up")
                bits ^= 1 << s
                if kc == 0 and (bits >> (6 + db)) & 1:
                    while not dempty[db].ready((bits >> (4 + db)) & 1):
                        yield
                    bits ^= 1 << (4 + db)
                issue(role, (l, "tc", it, kc), [(j & 3, role)],
                      [(xempty[s], 1)] + ([(dfull[db], 1)] if kc == nkc - 1 else []))
                if kc == nkc - 1:
                    bits |= 1 << (6 + db)
                yield
            bits ^= fill_parity(*g["cc"])
            if g["dt_on"] and issuer_waits_for_gate_up:
                while state["gu_done"] <= l:
                    yield
            n_items, nkc, ns = g["dt"]
            jr = 0  # chunks this warp issued
            for j in range(n_items * nkc):
                it, kc, s = j // nkc, j % nkc, j % ns
                db = it & 1
                mine = db == role
                if mine:
                    while not xfull[s].ready((bits >> s) & 1):
                        yield
                    check_fill(s, (l, "dt", it, kc), f"issuer {role} down")
                bits ^= 1 << s
                if kc == 0 and (bits >> (6 + db)) & 1:
                    if mine:
                        while not dempty[db].ready((bits >> (4 + db)) & 1):
                            yield
                    bits ^= 1 << (4 + db)
                if mine:
                    b = 2 * (jr & 1) + role
                    issue(role, (l, "dt", it, kc), [(b, 0), (b, 1)],
                          [(xempty[s], 2)] + ([(dfull[db], 2)] if kc == nkc - 1 else []))
                    jr += 1
                if kc == nkc - 1:
                    bits |= 1 << (6 + db)
                yield
            bits ^= fill_parity(*g["dn"])

    def consumers():
        xpar = 0  # 0-3 slot parities, 12-13 dfull2 parities
        items_seen = [0, 0]
        for l in range(layers):
            g = geo[l]
            state["route"] = l + 1

            def epilogues(name):
                nonlocal xpar
                n_items, nkc, ns = g[name]
                for it in range(n_items):
                    db = it & 1
                    xpar ^= fill_parity_run(nkc, ns, it)
                    dp = (xpar >> (12 + db)) & 1
                    xpar ^= 1 << (12 + db)
                    while not dfull[db].ready(dp):
                        yield
                    items_seen[db] += 1
                    if dfull[db].done != items_seen[db]:
                        errors.append(f"consumers: buffer {db} read for {(l, name, it)} after "
                                      f"{dfull[db].done} completions")
                    dempty[db].arrive()
                    yield

            def cuda_core(name):
                nonlocal xpar
                n_items, nkc, ns = g[name]
                for j in range(n_items * nkc):
                    s = j % ns
                    while not xfull[s].ready((xpar >> s) & 1):
                        yield
                    check_fill(s, (l, name, j // nkc, j % nkc), f"consumers {name}")
                    xpar ^= 1 << s
                    xempty_cc[s].arrive()
                    yield

            yield from epilogues("tc")
            yield from cuda_core("cc")
            state["gu_done"] = l + 1  # the grid barrier after gate/up
            if g["dt_on"]:
                yield from epilogues("dt")
            yield from cuda_core("dn")
            state["ring_free"] = l + 1
            yield

    agents = [producer(), issuer(0), issuer(1), consumers()]
    tp = tensor_pipe()
    steps = 0
    while agents and not errors:
        a = rnd.choice(agents + [tp])
        if a is tp:
            next(tp)
        else:
            try:
                next(a)
            except StopIteration:
                agents.remove(a)
        steps += 1
        if steps > 400_000:
            return "no progress"
    return errors[0] if errors else None


def test_every_wait_matches_its_fill():
    for seed in range(400):
        assert simulate(seed) is None, (seed, simulate(seed))


def test_model_finds_the_early_wait_without_the_gate_up_wait():
    found = [seed for seed in range(400) if simulate(seed, issuer_waits_for_gate_up=False) is not None]
    assert found, "the model should find a down wait matching a gate/up fill"


def test_scale_buffers_need_items_of_at_most_two_chunks():
    # four 512-wide chunks per down item (f = 2048): a warp reuses a scale
    # buffer two chunks later within one item, before the slot chain has
    # seen those products complete (why msk_create keeps such shapes on the
    # CUDA-core down path)
    found = [seed for seed in range(400) if simulate(seed, dt_chunks=(4,)) is not None]
    assert found and all("scale columns" in simulate(s, dt_chunks=(4,)) for s in found[:5])
