"""Host check of the balanced persistent decode schedule's integer arithmetic: the tile
partition among workers, the owner of a tile, and the merge pieces of units that workers
share.  The formulas are the ones decode_sk_kernel evaluates (restated here): worker W
owns flat tiles [W*T//NW, (W+1)*T//NW) with NW = min(workers, max(1, T // per)), per = 16
tiles of 16 tokens (8 of 32 tokens), or 4 when T // per workers would be under a quarter of
them, then rounded down to a multiple c of the unit count when 1 <= c < 8 (units that merge
in the launch) and that keeps three quarters of NW; the owner
of tile t is ((t+1)*NW + T-1)//T - 1;
a unit cut between workers leaves one piece per worker, side 1 for the worker where the
unit begins and side 0 for the others.  The last piece of a unit merges them in the same
launch, or, for launches whose units span many workers, a separate merge kernel reads the
same slots."""
import itertools
import random

import pytest


def n_workers(workers, T, tile_tokens=16, units=0):
    base = 16 * 16 // tile_tokens
    per = 4 if (T // base) * 4 < workers else base
    r = min(workers, max(1, T // per))
    c = r // units if units > 0 else 0
    if 1 <= c < 8 and 4 * c * units >= 3 * r:
        return c * units
    return r


def start(W, T, NW):
    return T if W >= NW else (W * T) // NW


def owner(t, T, NW):
    return ((t + 1) * NW + T - 1) // T - 1


def schedule(tiles_per_seq, U, workers):
    """Simulate every worker: returns (final writes, pieces) per unit, plus the slots."""
    pre = [0]
    for n in tiles_per_seq:
        pre.append(pre[-1] + n)
    T = U * pre[-1]
    NW = n_workers(workers, T, units=len(tiles_per_seq) * U)
    finals, pieces, slots = {}, {}, {}
    for W in range(workers):
        s, e = start(W, T, NW), start(W + 1, T, NW)
        for f in range(s, e):
            b = next(bb for bb in range(len(tiles_per_seq)) if U * pre[bb + 1] > f)
            nt = pre[b + 1] - pre[b]
            local = f - U * pre[b]
            y, tile = divmod(local, nt)
            if tile != nt - 1 and f != e - 1:
                continue
            us = U * pre[b] + y * nt
            ue = us + nt
            if us >= s and ue <= e:
                finals.setdefault((b, y), []).append(W)
            else:
                side = 0 if us < s else 1
                key = (W, side)
                assert key not in slots, "two units in one slot"
                slots[key] = (b, y)
                pieces.setdefault((b, y), []).append((W, side))
    return T, NW, finals, pieces


@pytest.mark.parametrize("workers,tile_tokens", [(1, 16), (3, 16), (4, 16), (7, 16), (16, 16),
                                                (64, 16), (4, 32), (16, 32), (64, 32)])
def test_partition_and_owner(workers, tile_tokens):
    base = 16 * 16 // tile_tokens
    for T in range(1, 300):
        NW = n_workers(workers, T, tile_tokens)
        cover = []
        for W in range(workers):
            cover += list(range(start(W, T, NW), start(W + 1, T, NW)))
        assert cover == list(range(T))
        sizes = [start(W + 1, T, NW) - start(W, T, NW) for W in range(NW)]
        per = 4 if (T // base) * 4 < workers else base
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= min(per, T)
        for t in range(T):
            W = owner(t, T, NW)
            assert start(W, T, NW) <= t < start(W + 1, T, NW)


def test_units_are_written_exactly_once():
    rng = random.Random(0)
    for trial in range(300):
        B = rng.randint(1, 7)
        tiles = [rng.choice([0, 1, 2, 3, 5, 8, 13, 40, 128]) for _ in range(B)]
        U = rng.choice([1, 2, 3, 8])
        workers = rng.choice([1, 2, 4, 12, 32])
        if sum(tiles) == 0:
            continue
        T, NW, finals, pieces = schedule(tiles, U, workers)
        for b, n in enumerate(tiles):
            for y in range(U):
                key = (b, y)
                if n == 0:
                    assert key not in finals and key not in pieces
                    continue
                assert (key in finals) != (key in pieces)
                if key in finals:
                    assert len(finals[key]) == 1
                    continue
                us = U * sum(tiles[:b]) + y * n
                ue = us + n
                w0, w1 = owner(us, T, NW), owner(ue - 1, T, NW)
                got = sorted(pieces[key])
                want = sorted([(w0, 1)] + [(W, 0) for W in range(w0 + 1, w1 + 1)])
                assert got == want, (tiles, U, workers, key)


@pytest.mark.parametrize("B,U,ntiles,workers", [(20, 8, 128, 1184), (32, 8, 128, 1184),
                                                (32, 8, 64, 1184), (64, 8, 128, 1184),
                                                (128, 8, 128, 1184), (3, 5, 17, 40)])
def test_unit_aligned_worker_count(B, U, ntiles, workers):
    """Units of equal length that merge in the launch: the worker count is a multiple c of
    the units, every unit is cut into exactly c pieces (or held whole when c = 1), and no
    worker holds parts of two units."""
    units = B * U
    T = units * ntiles
    NW = n_workers(workers, T, 16, units)
    r = n_workers(workers, T)
    c = NW // units
    assert NW % units == 0 and 1 <= c < 8 and 4 * NW >= 3 * r
    _, NW2, finals, pieces = schedule([ntiles] * B, U, workers)
    assert NW2 == NW
    if c == 1:
        assert not pieces and all(len(v) == 1 for v in finals.values()) and len(finals) == units
    else:
        assert not finals and all(len(v) == c for v in pieces.values()) and len(pieces) == units
        held = [W for v in pieces.values() for W, _ in v]
        assert len(held) == len(set(held)) == NW


def test_worker_count_unaligned_outside_the_in_launch_merge():
    # 11.84 workers per unit: the merge kernel's launch keeps the plain count
    assert n_workers(1184, 100 * 200, units=100) == n_workers(1184, 100 * 200) == 1184
    # B=16 at ctx 2048: 16 tiles per worker already give 8 per unit
    assert n_workers(1184, 128 * 128, units=128) == 1024
    # rounding would drop more than a quarter (640 units: c = 1 keeps 54%)
    assert n_workers(1184, 640 * 128, units=640) == 1184
    # a few long units (small launch, 32 per unit): unchanged
    assert n_workers(1184, 8 * 128, units=8) == n_workers(1184, 8 * 128) == 256


def test_slot_indices_stay_in_the_workspace():
    """Slots W*2+side < 2 * (SMs * CTAs per SM * 4 workers), the bound the workspace is
    sized for; counters b*U+y < B*Hq."""
    sms, per_sm, wpc = 160, 2, 4
    workers = sms * per_sm * wpc
    for B, Hq, Hk, hpc in itertools.product([1, 5, 64], [8, 32, 64], [1, 8], [1, 4, 16]):
        if Hq % Hk:
            continue
        g = Hq // Hk
        hpc = min(hpc, g)
        U = Hk * ((g + hpc - 1) // hpc)
        assert B * U <= B * Hq
        assert 2 * (workers - 1) + 1 < 2 * workers


def defers(B, Hq, Hk, pack, grid):
    """The host policy (decode_defers_merge): units averaging more than 8 workers each
    leave their pieces to the separate merge kernel."""
    g = Hq // Hk
    hpc = (min(g, 16 if g > 8 else 8)) if pack else 1
    if hpc > 8:
        return True  # the 16-head instance always leaves its pieces to the merge kernel
    units = B * Hk * ((g + hpc - 1) // hpc)
    return grid * 4 > 8 * units


def merge_kernel_reads(tiles_per_seq, U, workers):
    """The piece slots the merge kernel reads per unit: pieces of workers wfirst..wlast,
    slot W*2 + (1 if W == wfirst else 0), for units held by more than one worker."""
    pre = [0]
    for n in tiles_per_seq:
        pre.append(pre[-1] + n)
    T = U * pre[-1]
    NW = n_workers(workers, T, units=len(tiles_per_seq) * U)
    reads = {}
    for b, n in enumerate(tiles_per_seq):
        if n == 0:
            continue
        for y in range(U):
            us = U * pre[b] + y * n
            w0, w1 = owner(us, T, NW), owner(us + n - 1, T, NW)
            if w0 != w1:
                reads[(b, y)] = sorted([(w0, 1)] + [(W, 0) for W in range(w0 + 1, w1 + 1)])
    return reads


@pytest.mark.parametrize("workers", [4, 64, 1184])
def test_merge_kernel_reads_exactly_the_written_pieces(workers):
    """For every cut unit, the separate merge kernel reads exactly the slots the workers
    wrote, and no slot is written for two units."""
    rng = random.Random(workers)
    for trial in range(12):
        B = rng.randint(1, 6)
        tiles = [rng.choice([0, 1, 3, 64, 512]) for _ in range(B)]
        U = rng.choice([1, 8])
        _, _, _, pieces = schedule(tiles, U, workers)
        reads = merge_kernel_reads(tiles, U, workers)
        assert set(reads) == set(pieces), (tiles, U)
        seen = set()
        for key, slots in reads.items():
            assert slots == sorted(pieces[key]), (tiles, U, key)
            for s_ in slots:
                assert s_ not in seen
                seen.add(s_)


def test_defer_policy_on_the_named_shapes():
    grid = 148 * 2
    assert defers(4, 64, 8, True, grid)        # 70B long context: 32 units, 37 workers each
    assert defers(1, 32, 8, True, grid)        # one sequence
    assert not defers(64, 32, 8, True, grid)   # B=64 sweep: 2 workers per unit
    assert defers(16, 32, 8, True, grid)       # 7B-shaped batch: 9.25 grid workers per unit
    assert not defers(32, 32, 8, True, grid)   # 4.6 workers per unit
    assert not defers(8, 32, 8, False, grid)   # PackGQA off: one unit per head
    assert defers(64, 32, 2, True, grid)       # groups of 16: always the merge kernel
    assert not defers(64, 32, 2, False, grid)  # ... unless PackGQA is off
