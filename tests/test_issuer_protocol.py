"""A model of the mbarrier protocol of the two tensor-core GEMMs (k_qgemm, k_wgemm).

Roles, as the kernels run them: a producer fills a ring of stages in order, the unpack warps
mark each stage ready (afull), two MMA issuers take alternate stages (all of a unit's adapter
atoms go to one issuer), TMEM accumulator buffers are handed to the epilogue (accf) and back
(acce). Waits are mbarrier parity waits: a wait for phase n of a barrier is only sound while
the barrier has completed n or n+1 phases. With n-1 it passes before the phase happened (an
issuer would read a stage that is not loaded, or overwrite a buffer still being drained); with
n+2 it never passes.

The model runs random interleavings of the roles and asserts every wait is sound. It checks the
rules the kernels use: issuer q owns TMEM buffers q, q+2, ...; after skipping an adapter block,
an issuer waits on adone, and the owner of the next block first waits on aack (phase 0 of aack
is completed at set-up); the epilogue follows the stage parity of each K block. A control runs
the earlier rules (a shared round-robin buffer index, no handshake) and must find an unsound
wait.
"""
import random

import pytest


class Unsound(Exception):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def parity_passes(self, n):
        # try_wait.parity(n & 1): true while the current (open) phase has the other parity
        return (self.done & 1) != (n & 1)


def _wait(bar, n, who):
    while not bar.parity_passes(n):
        if bar.done >= n + 2:
            raise Unsound(f"{who}: lapped on {bar.name}, waits for phase {n}, {bar.done} completed")
        yield
    if bar.done < n + 1:
        raise Unsound(f"{who}: {bar.name} passed for phase {n} with only {bar.done} completed")


def run_model(NS, NB, units, n_ad, new_rules, rng, n_unpack=4, n_epi=8):
    """units: per unit, the number of groups of each K block (1, or 2 for g = 64)."""
    full = [Barrier(f"full{i}", 1) for i in range(NS)]
    afull = [Barrier(f"afull{i}", n_unpack) for i in range(NS)]
    empty = [Barrier(f"empty{i}", 1) for i in range(NS)]
    accf = [Barrier(f"accf{i}", 1) for i in range(NB)]
    acce = [Barrier(f"acce{i}", n_epi) for i in range(NB)]
    adone, aack = Barrier("adone", 1), Barrier("aack", 1)
    aack.arrive()
    pending = []  # asynchronous completions: [delay, callback]
    own_n = NB // 2

    def producer():
        it = 0
        for blocks in units:
            for _ in range(len(blocks) + n_ad):
                s, n = it % NS, it // NS
                if n > 0:
                    yield from _wait(empty[s], n - 1, "producer")
                pending.append([rng.randint(1, 6), full[s].arrive])
                it += 1
                yield

    def unpack(k):
        it = 0
        for blocks in units:
            for _ in range(len(blocks) + n_ad):
                s = it % NS
                yield from _wait(full[s], it // NS, f"unpack{k}")
                for _ in range(rng.randint(0, 3)):
                    yield
                afull[s].arrive()
                it += 1

    def issuer(q):
        it = gidx = own = blk = 0
        for blocks in units:
            nkb = len(blocks)
            ad_owner = (it + nkb) & 1
            for i in range(nkb + n_ad):
                s, n = it % NS, it // NS
                if i < nkb:
                    if (it & 1) != q:
                        gidx += blocks[i]
                        it += 1
                        continue
                    yield from _wait(afull[s], n, f"issuer{q}")
                    for _ in range(blocks[i]):
                        if new_rules:
                            b, use = q + 2 * (own % own_n), own // own_n
                            own += 1
                        else:
                            b, use = gidx % NB, gidx // NB
                        gidx += 1
                        if use > 0:
                            yield from _wait(acce[b], use - 1, f"issuer{q}")
                        yield
                        pending.append([rng.randint(1, 4), accf[b].arrive])
                else:
                    at = i - nkb
                    b, use = (q + 2 * (own % own_n), own // own_n) if new_rules else (gidx % NB, gidx // NB)
                    if ad_owner != q:
                        if at == n_ad - 1:
                            gidx += 1
                            if new_rules:
                                yield from _wait(adone, blk, f"issuer{q}")
                                aack.arrive()
                                blk += 1
                        it += 1
                        continue
                    yield from _wait(afull[s], n, f"issuer{q}")
                    if at == 0 and use > 0:
                        yield from _wait(acce[b], use - 1, f"issuer{q}")
                    yield
                    if at == n_ad - 1:
                        pending.append([rng.randint(1, 4), accf[b].arrive])
                        gidx += 1
                        own += 1
                pending.append([rng.randint(1, 4), empty[s].arrive])
                if new_rules and i >= nkb and i - nkb == n_ad - 1:
                    yield from _wait(aack, blk, f"issuer{q}")
                    adone.arrive()
                    blk += 1
                it += 1

    def epilogue(k):
        gidx, own, bit = 0, [0, 0], 0
        for blocks in units:
            n_groups = sum(blocks)
            two = max(blocks) == 2
            order = []
            for g in range(n_groups):
                order.append(bit)
                if not two or (g & 1) or g + 1 == n_groups:
                    bit ^= 1
            if n_ad:
                order.append(bit)
                bit ^= n_ad & 1
            for q in order:
                if new_rules:
                    b, use = q + 2 * (own[q] % own_n), own[q] // own_n
                    own[q] += 1
                else:
                    b, use = gidx % NB, gidx // NB
                gidx += 1
                yield from _wait(accf[b], use, f"epilogue{k}")
                for _ in range(rng.randint(0, 8)):
                    yield
                acce[b].arrive()

    roles = [producer(), issuer(0), issuer(1)] + [unpack(k) for k in range(n_unpack)]
    roles += [epilogue(k) for k in range(n_epi)]
    for step in range(400000):
        if not roles:
            return
        for p in list(pending):
            p[0] -= 1
            if p[0] <= 0:
                pending.remove(p)
                p[1]()
        r = rng.choice(roles)
        try:
            for _ in range(rng.randint(1, 3)):
                next(r)
        except StopIteration:
            roles.remove(r)
    raise Unsound("no progress (deadlock)")


# stage ring depth / TMEM buffers of each kernel instance: k_qgemm BN 16-32 / 64 / 128 / 192-256,
# k_wgemm BN 16-32 / 64 / 128 (operand slots as the ring)
SHAPES = [(6, 4), (5, 4), (4, 4), (3, 2), (4, 8), (3, 8), (2, 4)]
UNITS = {
    "g128": [[1] * 4] * 4,
    "g64": [[2] * 3] * 4,
    "ragged_g64": [[2, 2, 1]] * 4,
    "one_block": [[1]] * 5,
    "mixed": [[1] * (1 + u % 3) for u in range(5)],
}


@pytest.mark.parametrize("NS,NB", SHAPES)
@pytest.mark.parametrize("kind", sorted(UNITS))
@pytest.mark.parametrize("n_ad", [0, 1, 2, 5])
def test_every_wait_is_sound(NS, NB, kind, n_ad):
    for seed in range(4):
        run_model(NS, NB, UNITS[kind], n_ad, True, random.Random(seed))


@pytest.mark.parametrize("NS,NB,kind,n_ad", [
    (3, 2, "g128", 5),   # an adapter block longer than the stage ring
    (3, 2, "g64", 0),    # two groups per stage on two TMEM buffers
])
def test_earlier_rules_are_unsound(NS, NB, kind, n_ad):
    found = 0
    for seed in range(8):
        try:
            run_model(NS, NB, UNITS[kind], n_ad, False, random.Random(seed))
        except Unsound:
            found += 1
    assert found > 0
