"""Host-side models of the decode-batch product (k_qdec, T <= 16), run on CPU.

1. The schedule: CTA c of G takes blocks [c*NB/G, (c+1)*NB/G) of the tile-major (output tile, K
   block) order. The model checks that every block belongs to exactly one CTA (the closed form
   the kernel uses for "which CTA holds block f" agrees with the ranges), that no tile has more
   segments than the workspace holds (the partial slot index stays in bounds), and that the
   per-tile fix-up (the last of the tile's segments to arrive adds them in segment order) runs
   exactly once per tile, whatever order the CTAs finish in.
2. The mbarrier protocol: a producer fills the packed-block ring in order, two teams of four
   unpack warps take alternate blocks and put each into one of four TMEM A slots, two issuers take
   alternate blocks (issuer q owns accumulator slots q, q+2, ...), four epilogue warps drain the
   groups in block order. Three rings: packed blocks (freed by the unpack team once used),
   activation tiles (freed by the MMA commit) and scale slabs (freed by the epilogue). Random
   interleavings; every parity wait must be sound (the barrier has completed n or n+1 phases
   when a wait for phase n passes) and everything must finish.
"""
import random

import pytest

from test_issuer_protocol import Barrier, Unsound, _wait

KTILE, NTILE = 128, 128


def range_begin(c, NB, G):
    return c * NB // G


def cta_of(f, NB, G):
    return ((f + 1) * G - 1) // NB


def plan(N, K, n_sm=148):
    """The host plan of the decode product (plan_decode): tiles, blocks, grid, partial slots."""
    NT = -(-N // NTILE)
    KB = -(-K // KTILE)
    NB = NT * KB
    G = min(NB, n_sm)
    lmin = NB // G
    maxseg = (KB - 1) // lmin + 2
    return NT, KB, NB, G, maxseg


SHAPES = [(29568, 8192), (8192, 29568), (256, 256), (200, 384), (512, 1024), (136, 256), (640, 1024),
          (1536, 8960), (8960, 1536), (1024, 512), (128, 128), (384, 640), (14336, 4096), (4096, 14336),
          (1, 128), (129, 65 * 128), (100000, 128)]


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("n_sm", [148, 7, 1, 1000])
def test_schedule_covers_every_block_once_and_segments_fit(N, K, n_sm):
    NT, KB, NB, G, maxseg = plan(N, K, n_sm)
    owner = {}
    for c in range(G):
        b0, b1 = range_begin(c, NB, G), range_begin(c + 1, NB, G)
        assert b1 > b0                                   # every CTA streams at least one block
        for f in range(b0, b1):
            assert f not in owner
            owner[f] = c
            assert cta_of(f, NB, G) == c                 # the closed form the kernel uses
    assert len(owner) == NB
    lens = [range_begin(c + 1, NB, G) - range_begin(c, NB, G) for c in range(G)]
    assert max(lens) - min(lens) <= 1                    # equal shares
    for nt in range(NT):
        c_first = cta_of(nt * KB, NB, G)
        nseg = cta_of(nt * KB + KB - 1, NB, G) - c_first + 1
        assert 1 <= nseg <= maxseg
        segs = sorted({owner[nt * KB + kb] for kb in range(KB)})
        assert segs == list(range(c_first, c_first + nseg))   # segment index = c - c_first < maxseg


@pytest.mark.parametrize("N,K", [(29568, 8192), (8192, 29568), (640, 1024), (136, 256)])
def test_fixup_runs_once_per_tile_in_segment_order(N, K):
    NT, KB, NB, G, maxseg = plan(N, K)
    rng = random.Random(N + K)
    for trial in range(5):
        cnt = [0] * NT
        finalized = {}
        # each CTA finishes its segments in order; CTAs interleave at random
        queues = []
        for c in range(G):
            b0, b1 = range_begin(c, NB, G), range_begin(c + 1, NB, G)
            tiles = []
            for f in range(b0, b1):
                if not tiles or tiles[-1] != f // KB:
                    tiles.append(f // KB)
            queues.append([c, tiles])
        partial = {}
        while any(q[1] for q in queues):
            q = rng.choice([q for q in queues if q[1]])
            c, nt = q[0], q[1].pop(0)
            c_first = cta_of(nt * KB, NB, G)
            nseg = cta_of(nt * KB + KB - 1, NB, G) - c_first + 1
            seg = c - c_first
            if nseg == 1:
                finalized[nt] = [seg]
                continue
            partial[(nt, seg)] = c
            old = cnt[nt]
            cnt[nt] += 1
            if old == nseg - 1:
                assert nt not in finalized
                assert all((nt, s) in partial for s in range(nseg))  # every partial is there
                finalized[nt] = list(range(nseg))                   # summed in segment order
                cnt[nt] = 0
        assert sorted(finalized) == list(range(NT))
        assert all(v == 0 for v in cnt)                             # counters left at zero


def run_decode_model(nblk, gpb_of, NW, NX, NSS, NA, n_slots, rng, n_unpack=8, n_epi=4):
    """nblk blocks; gpb_of(i) = groups of block i (1, or 2 at g = 64)."""
    wfull = [Barrier(f"wfull{i}", 1) for i in range(NW)]
    wempty = [Barrier(f"wempty{i}", n_unpack // 2) for i in range(NW)]
    xfull = [Barrier(f"xfull{i}", 1) for i in range(NX)]
    xempty = [Barrier(f"xempty{i}", 1) for i in range(NX)]
    sfull = [Barrier(f"sfull{i}", 1) for i in range(NSS)]
    sempty = [Barrier(f"sempty{i}", n_epi) for i in range(NSS)]
    afull = [Barrier(f"afull{i}", n_unpack // 2) for i in range(NA)]
    aempty = [Barrier(f"aempty{i}", 1) for i in range(NA)]
    accf = [Barrier(f"accf{i}", 1) for i in range(n_slots)]
    acce = [Barrier(f"acce{i}", n_epi) for i in range(n_slots)]
    own_n = n_slots // 2
    pending = []

    def producer():
        for i in range(nblk):
            for full, empty, depth in ((wfull, wempty, NW), (xfull, xempty, NX), (sfull, sempty, NSS)):
                s, n = i % depth, i // depth
                if n > 0:
                    yield from _wait(empty[s], n - 1, "producer")
                pending.append([rng.randint(1, 8), full[s].arrive])
                yield

    def unpack(k):
        team = k // 4          # two teams of four warps take alternate blocks
        for i in range(team, nblk, 2):
            s, a = i % NW, i % NA
            yield from _wait(wfull[s], i // NW, f"unpack{k}")
            if i // NA > 0:
                yield from _wait(aempty[a], i // NA - 1, f"unpack{k}")
            for _ in range(rng.randint(0, 3)):
                yield
            wempty[s].arrive()     # the packed block has been used
            afull[a].arrive()

    def issuer(q):
        own = 0
        for i in range(q, nblk, 2):
            a, sx = i % NA, i % NX
            yield from _wait(afull[a], i // NA, f"issuer{q}")
            yield from _wait(xfull[sx], i // NX, f"issuer{q}")
            for _ in range(gpb_of(i)):
                slot, use = q + 2 * (own % own_n), own // own_n
                own += 1
                if use > 0:
                    yield from _wait(acce[slot], use - 1, f"issuer{q}")
                yield
                pending.append([rng.randint(1, 5), accf[slot].arrive])
            pending.append([rng.randint(1, 5), aempty[a].arrive])
            pending.append([rng.randint(1, 5), xempty[sx].arrive])

    def epilogue(k):
        n = [0, 0]
        for i in range(nblk):
            q, ss = i & 1, i % NSS
            yield from _wait(sfull[ss], i // NSS, f"epilogue{k}")   # the block's scale slabs
            for _ in range(gpb_of(i)):
                slot, use = q + 2 * (n[q] % own_n), n[q] // own_n
                n[q] += 1
                yield from _wait(accf[slot], use, f"epilogue{k}")
                for _ in range(rng.randint(0, 6)):
                    yield
                acce[slot].arrive()
            sempty[ss].arrive()    # scales read: the slot is free

    roles = [producer(), issuer(0), issuer(1)] + [unpack(k) for k in range(n_unpack)]
    roles += [epilogue(k) for k in range(n_epi)]
    for _ in range(2000000):
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


# rings (packed, tile, scales), A slots, accumulator slots of the three instances:
# int8 (16, 24, 24, 8, 16); W4 bf16 (12, 16, 16, 6, 8); W3 bf16 (16, 16, 16, 6, 8)
@pytest.mark.parametrize("NW,NX,NSS,NA,n_slots", [(16, 24, 24, 8, 16), (12, 16, 16, 6, 8), (16, 16, 16, 6, 8)])
@pytest.mark.parametrize("kind", ["g128", "g64", "ragged_g64", "one", "two"])
def test_decode_barrier_protocol_is_sound(NW, NX, NSS, NA, n_slots, kind):
    shapes = {
        "g128": (100, lambda i: 1),
        "g64": (60, lambda i: 2),
        "ragged_g64": (45, lambda i: 1 if i % 5 == 4 else 2),   # the last block of each tile holds one group
        "one": (1, lambda i: 1),
        "two": (2, lambda i: 2),
    }
    nblk, gpb_of = shapes[kind]
    for seed in range(3):
        run_decode_model(nblk, gpb_of, NW, NX, NSS, NA, n_slots, random.Random(seed))
