"""Host-side models of the decode-batch product (k_qdec, T <= 16), run on CPU.

1. The schedule: CTA c of G takes blocks [c*NB/G, (c+1)*NB/G) of the tile-major (output tile, K
   block) order. The model checks that every block belongs to exactly one CTA (the closed form
   the kernel uses for "which CTA holds block f" agrees with the ranges), that no tile has more
   segments than the workspace holds (the partial slot index stays in bounds), and that the
   per-tile fix-up (the last of the tile's segments to arrive adds them in segment order) runs
   exactly once per tile, whatever order the CTAs finish in.
2. The mbarrier protocol: one thread streams the packed blocks into a ring that the unpack team
   frees as soon as it has read a block; two teams of four unpack warps take alternate blocks;
   three issuers take every third block, each loading the activation tiles of its own blocks NA
   blocks ahead into a 2 NA ring (the tile of block j is requested after afull of block j - NA,
   which implies that block j - 2 NA's MMAs, the slot's previous user, are done), and commit once
   per block (freeing the A slot) and once per batch of groups (two batch buffers); four epilogue
   warps drain the batches in order. Random interleavings and random commit delays; every parity wait
   must be sound (the barrier has completed n or n+1 phases when a wait for phase n passes),
   every commit must land in the phase it is meant for, and everything must finish.
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


class TaggedBarrier(Barrier):
    """A barrier whose arrivals say which phase they belong to (a commit must never land in an
    earlier phase that is still open)."""

    def arrive_for(self, phase, who):
        if phase != self.done:
            raise Unsound(f"{who}: arrival for phase {phase} of {self.name} landed in phase {self.done}")
        self.arrive()


def run_decode_model(nblk, gpb_of, NW, NA, rng, NBUF=2, NBATCH=8, n_epi=4, n_iss=3, tiles_ahead=None):
    """nblk blocks; gpb_of(i) = groups of block i (1, or 2 at g = 64, 1 for the ragged last K block).
    tiles_ahead: how far ahead (in blocks) an issuer requests activation tiles; the kernel's NA."""
    ahead = NA if tiles_ahead is None else tiles_ahead
    wfull = [Barrier(f"wfull{i}", 1) for i in range(NW)]
    wempty = [Barrier(f"wempty{i}", 4) for i in range(NW)]
    NX = 2 * NA
    xfull = [TaggedBarrier(f"xfull{i}", 1) for i in range(NX)]
    x_reader_done = {}   # block -> its tile has been consumed by an issued MMA that completed
    afull = [Barrier(f"afull{i}", 4) for i in range(NA)]
    mdone = [TaggedBarrier(f"mdone{i}", 1) for i in range(NA)]
    accf = [TaggedBarrier(f"accf{i}", n_iss) for i in range(NBUF)]
    acce = [Barrier(f"acce{i}", n_epi) for i in range(NBUF)]
    ngroups = sum(gpb_of(i) for i in range(nblk))
    nbatch = -(-ngroups // NBATCH)
    pending = []

    def later(fn, *args):
        pending.append([rng.randint(1, 6), lambda: fn(*args)])

    def w_producer():
        for i in range(nblk):
            s, n = i % NW, i // NW
            if n > 0:
                yield from _wait(wempty[s], n - 1, "w_producer")
            later(wfull[s].arrive)
            yield

    def unpack(k):
        team = k // 4
        for i in range(team, nblk, 2):
            sw, s = i % NW, i % NA
            yield from _wait(wfull[sw], i // NW, f"unpack{k}")
            if i // NA > 0:
                yield from _wait(mdone[s], i // NA - 1, f"unpack{k}")
            for _ in range(rng.randint(0, 3)):
                yield
            wempty[sw].arrive()
            yield
            afull[s].arrive()

    def issuer(q):
        st = {"acq": 0, "com": 0}

        def acquire(b):
            while st["acq"] <= b:
                a = st["acq"]
                if a // NBUF > 0:
                    yield from _wait(acce[a % NBUF], a // NBUF - 1, f"issuer{q}")
                st["acq"] += 1

        def commit_before(b):
            while st["com"] < b:
                cb = st["com"]
                yield from acquire(cb)
                later(accf[cb % NBUF].arrive_for, cb // NBUF, f"issuer{q}")
                st["com"] += 1

        st["ix"] = q

        def request_tiles(upto):
            while st["ix"] < nblk and st["ix"] <= upto:
                j = st["ix"]
                if j >= NX and not x_reader_done.get(j - NX, False):
                    raise Unsound(f"issuer{q}: tile of block {j} requested while block {j - NX} may still read the slot")
                later(xfull[j % NX].arrive_for, j // NX, f"issuer{q}")
                st["ix"] += n_iss

        request_tiles(NA - 1)
        gidx = 0
        for i in range(nblk):
            ng = gpb_of(i)
            if i % n_iss != q:
                gidx += ng
                continue
            s = i % NA
            yield from _wait(afull[s], i // NA, f"issuer{q}")
            request_tiles(i + ahead)
            yield from _wait(xfull[i % NX], i // NX, f"issuer{q}")
            for _ in range(ng):
                bt = gidx // NBATCH
                yield from commit_before(bt)
                yield from acquire(bt)
                yield
                gidx += 1
            def mma_done(i=i, s=s):
                x_reader_done[i] = True
                mdone[s].arrive_for(i // NA, f"issuer{q}")
            later(mma_done)
        yield from commit_before(nbatch)

    def epilogue(k):
        for bt in range(nbatch):
            yield from _wait(accf[bt % NBUF], bt // NBUF, f"epilogue{k}")
            for _ in range(rng.randint(0, 4)):
                yield
            acce[bt % NBUF].arrive()

    roles = [w_producer()] + [issuer(q) for q in range(n_iss)] + [unpack(k) for k in range(8)]
    roles += [epilogue(k) for k in range(n_epi)]
    for _ in range(2000000):
        if not roles and not pending:
            assert all(b.done == -(-max(nblk - i, 0) // NA) for i, b in enumerate(mdone))
            return
        for p in list(pending):
            p[0] -= 1
            if p[0] <= 0:
                pending.remove(p)
                p[1]()
        if not roles:
            continue
        r = rng.choice(roles)
        try:
            for _ in range(rng.randint(1, 3)):
                next(r)
        except StopIteration:
            roles.remove(r)
    raise Unsound("no progress (deadlock)")


# packed-block ring, A slots, groups per batch of the three instances: int8 (20, 6, 8);
# W4 bf16 (20, 6, 4); W3 bf16 (24, 6, 4)
@pytest.mark.parametrize("NW,NA,NBATCH", [(20, 6, 8), (20, 6, 4), (24, 6, 4)])
@pytest.mark.parametrize("kind", ["g128", "g64", "ragged_g64", "one", "two", "three_g64", "seven"])
def test_decode_barrier_protocol_is_sound(NW, NA, NBATCH, kind):
    shapes = {
        "g128": (100, lambda i: 1),
        "g64": (60, lambda i: 2),
        "ragged_g64": (45, lambda i: 1 if i % 5 == 4 else 2),   # the last block of each tile holds one group
        "one": (1, lambda i: 1),
        "two": (2, lambda i: 2),
        "three_g64": (3, lambda i: 2),
        "seven": (7, lambda i: 1),
    }
    nblk, gpb_of = shapes[kind]
    for seed in range(3):
        run_decode_model(nblk, gpb_of, NW, NA, random.Random(seed), NBATCH=NBATCH)


@pytest.mark.parametrize("N,K,group", [(29568, 8192, 128), (8192, 29568, 128), (640, 1088, 64), (136, 320, 64)])
def test_group_count_closed_form(N, K, group):
    """The kernel counts a CTA's groups as nblk * gpb minus one per tile end in its range when the
    last K block of a tile holds one group (K = 64 mod 128 at g = 64)."""
    NT, KB, NB, G, _ = plan(N, K)
    gpb = 128 // group
    G_total = -(-K // group)
    for c in range(G):
        b0, b1 = range_begin(c, NB, G), range_begin(c + 1, NB, G)
        walk = sum(min(gpb, G_total - (f % KB) * gpb) for f in range(b0, b1))
        ragged = G_total < KB * gpb
        closed = (b1 - b0) * gpb - ((b1 // KB - b0 // KB) if ragged else 0)
        assert walk == closed


# (T, K, N, group, a_bits, w_bits, r_s, N_r, r_r): the 72B decode projections, the decode parity
# shapes' corners, and a rank that takes the adapters past the decode product's 384 columns
PLAN_SHAPES = [
    (16, 8192, 29568, 128, 8, 4, 32, 8, 4), (16, 29568, 8192, 128, 8, 4, 32, 8, 4), (1, 8192, 29568, 128, 16, 3, 32, 8, 4),
    (2, 320, 200, 64, 16, 3, 8, 4, 4), (7, 8192, 128, 128, 8, 4, 32, 8, 4), (16, 29568, 256, 128, 6, 4, 32, 8, 4),
    (16, 1024, 1000, 128, 8, 4, 0, 1, 0), (13, 1024, 640, 128, 6, 4, 32, 8, 32),
]


@pytest.mark.parametrize("T,K,N,group,a_bits,w_bits,rs,nr,rr", PLAN_SHAPES)
def test_library_decode_plan_matches_the_model(T, K, N, group, a_bits, w_bits, rs, nr, rr):
    """The schedule these models check is the one the library plans: qe_linear_plan reports the
    decode product's CTA count and segment bound, computed by the C code, host only."""
    import quantized_gemm_moe_b200 as qe
    try:
        qe.load()
    except Exception as e:  # pragma: no cover - the build step makes the library
        pytest.skip(f"libqe.so not built: {e}")
    p = qe.linear_plan(qe.make_desc(K, N, group, w_bits, a_bits, rs, nr, rr), T, qe.QE_BF16)
    assert p["decode_product"] == 1
    NT, KB, NB, G, maxseg = plan(N, K, p["decode_ctas"])
    assert p["decode_ctas"] == G
    assert p["decode_max_segments"] == maxseg
    assert p["product_tile_tokens"] == 16 and p["product_k_splits"] == 1


def test_library_decode_plan_limits():
    import quantized_gemm_moe_b200 as qe
    try:
        qe.load()
    except Exception as e:  # pragma: no cover
        pytest.skip(f"libqe.so not built: {e}")
    # 17 tokens, and adapters wider than 384 columns (R_pad = 448), run on the GEMM instead
    assert qe.linear_plan(qe.make_desc(8192, 4096, 128, 4, 8, 32, 8, 4), 17)["decode_product"] == 0
    wide = qe.linear_plan(qe.make_desc(8192, 4096, 128, 4, 8, 64, 8, 48), 16)
    assert wide["decode_product"] == 0 and wide["decode_ctas"] == 0 and wide["decode_max_segments"] == 0
    assert qe.linear_plan(qe.make_desc(8192, 4096, 128, 4, 8, 64, 8, 40), 16)["decode_product"] == 1  # R_pad 384


def test_decode_model_catches_early_tile_requests():
    """Control: requesting the activation tiles three blocks further ahead than the kernel does
    reuses a tile slot whose MMAs may still be reading it; the model must see that."""
    caught = 0
    for seed in range(10):
        try:
            run_decode_model(100, lambda i: 1, 20, 6, random.Random(seed), NBATCH=8, tiles_ahead=6 + 3)
        except Unsound:
            caught += 1
    assert caught >= 8


@pytest.mark.parametrize("nbatch", [1, 2, 3, 4, 5, 13, 40])
def test_scale_ring_reads_landed_slots_that_are_not_being_rewritten(nbatch):
    """The epilogue's group scales: each thread requests batch b's scales into slot b % R (R = 4)
    as one cp.async group, R - 1 batches ahead, and before reading batch b waits with
    cp.async.wait_group R - 1: every group except the R - 1 most recently committed has landed.
    Other groups land in any order."""
    R = 4
    rng = random.Random(nbatch)
    slot_owner = {}      # slot -> batch whose copy last went into it
    committed = []       # groups in commit order: batch, or None for an empty group
    landed = set()

    def request(b):
        if b < nbatch:
            slot_owner[b % R] = b
        committed.append(b if b < nbatch else None)   # an empty group is committed all the same

    for b in range(R - 1):
        request(b)
    for bt in range(nbatch):
        request(bt + R - 1)
        for g in committed:                  # some copies land early, in any order
            if g is not None and rng.random() < 0.3:
                landed.add(g)
        for g in committed[:-(R - 1)]:       # cp.async.wait_group R - 1
            if g is not None:
                landed.add(g)
        assert bt in landed                  # this batch's scales are there
        assert slot_owner[bt % R] == bt      # and no later batch has been requested into its slot


@pytest.mark.parametrize("R_pad", [64, 128, 192, 320, 384, 512])
@pytest.mark.parametrize("chunk", [1, 2, 3, 5, 8, 16, 100])
def test_route_quant_group_sum_layout_fits(R_pad, chunk):
    """k_route_quant with several warps per token: the token group's partial rows [g][R_pad] and
    its summed row fit in the group's wpt adapter rows, the logit partials in the static buffer,
    and the named barrier ids stay in 1..15."""
    kWarps, kThreads, kMaxRouted = 16, 512, 16
    wpt = 1
    while wpt * 2 * chunk <= kWarps:
        wpt *= 2
    nslot_w = kWarps // wpt
    if wpt == 1:
        return                                   # one warp per token: the per-warp path
    gthr = wpt * 32
    g = max(1, gthr // R_pad)
    assert (g + 1) * R_pad <= wpt * R_pad        # partials + summed row inside the group's rows
    for n_r in range(1, kMaxRouted + 1):
        lg = gthr // n_r
        assert lg >= 1 and lg * n_r <= gthr      # this group's share of the logit buffer
        assert (nslot_w - 1) * gthr + gthr <= kThreads
    assert 1 <= 1 + (nslot_w - 1) <= 15
