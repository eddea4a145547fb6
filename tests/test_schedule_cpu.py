"""Host check of the balanced persistent decode schedule's integer arithmetic: the tile
partition among workers, the owner of a tile, and the merge pieces of units that workers
share.  The formulas are the ones decode_sk_kernel evaluates (restated here): worker W
owns flat tiles [W*T//NW, (W+1)*T//NW) with NW = min(workers, max(1, T // 16)); the owner
of tile t is ((t+1)*NW + T-1)//T - 1;
a unit cut between workers leaves one piece per worker, side 1 for the worker where the
unit begins and side 0 for the others; the pieces are merged up a binary tree whose
internal nodes are claimed by the second of their two children to arrive."""
import itertools
import random

import pytest


def n_workers(workers, T):
    return min(workers, max(1, T // 16))


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
    NW = n_workers(workers, T)
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


@pytest.mark.parametrize("workers", [1, 3, 4, 7, 16, 64])
def test_partition_and_owner(workers):
    for T in range(1, 300):
        NW = n_workers(workers, T)
        cover = []
        for W in range(workers):
            cover += list(range(start(W, T, NW), start(W + 1, T, NW)))
        assert cover == list(range(T))
        sizes = [start(W + 1, T, NW) - start(W, T, NW) for W in range(NW)]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= min(16, T)
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


def tree_merge(np_, order, levels_cap=12):
    """Replay the merge-tree protocol for np_ pieces whose leaf owners finish in `order`.
    Each owner climbs: no sibling -> move up; else arrive at the parent's counter; the
    first arrival stops, the second merges (left operand first) and climbs on.  Returns
    the root's operand tree and the counter ids used."""
    levels = 0
    while (1 << levels) < np_:
        levels += 1
    assert levels < levels_cap
    counters, results, roots, used = {}, {k: k for k in range(np_)}, [], set()
    pending = {}
    for k in order:
        node, lv, val = k, 0, k
        while lv < levels:
            sib = node ^ 1
            if (sib << lv) >= np_:
                node >>= 1
                lv += 1
                continue
            p0 = (node >> 1) << (lv + 1)
            cid = (p0, lv + 1)
            used.add(cid)
            counters[cid] = counters.get(cid, 0) + 1
            if counters[cid] == 1:
                pending[(lv, node)] = val
                break
            other = pending.pop((lv, sib))
            val = (val, other) if node < sib else (other, val)
            node >>= 1
            lv += 1
        else:
            roots.append(val)
    return roots, counters, used


def _tree_of(np_):
    levels = 0
    while (1 << levels) < np_:
        levels += 1
    def build(lv, node):
        lo = node << lv
        if lo >= np_:
            return None
        if lv == 0:
            return lo
        l, r = build(lv - 1, 2 * node), build(lv - 1, 2 * node + 1)
        return l if r is None else (l, r)
    return build(levels, 0)


@pytest.mark.parametrize("np_", [2, 3, 4, 5, 7, 8, 9, 16, 37, 100, 1280])
def test_merge_tree_has_one_root_and_a_fixed_shape(np_):
    rng = random.Random(np_)
    want = _tree_of(np_)
    for trial in range(20):
        order = list(range(np_))
        rng.shuffle(order)
        roots, counters, used = tree_merge(np_, order)
        assert len(roots) == 1, "exactly one worker writes the unit"
        assert roots[0] == want, "the result must not depend on the arrival order"
        assert all(c == 2 for c in counters.values()), "every counter is claimed by two children"
        # counter ids stay inside [2 * workers][12]: leaf slot < 2 * 1280, level < 12
        assert all(p0 < 1280 and 1 <= lv < 12 for p0, lv in used)
