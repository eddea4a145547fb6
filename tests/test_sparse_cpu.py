"""Pins of the page-level top-K sparse decode oracle (RocketKV's decode stage, as the page
"TensorRT-LLM 如何用 sparse_attention_config 配置 Sparse Attention 降低长上下文推理开销"
configures it: KT-cache page scores, the `topk` best pages plus a window of recent tokens
attended).  Each oracle step is checked against something other than itself: brute-force
minima and maxima of the keys, the maximum of q.k over the box's corners, the bound it
gives on every key, a sort of the scores, planted ties, window pages and a planted needle,
and dense attention over the chosen pages."""
import itertools

import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import inputs
from oracle import oracle
from tests._util import bits, oracle_decode


def _case(lens, Hq=8, Hk=2, D=64, P=16, seed=0, pt_stride=None):
    return inputs.make_decode_case(len(lens), Hq, Hk, D, P, lens, seed=seed, pt_stride=pt_stride,
                                   keep_dense=True)


def _kt(case):
    kv = case.kv
    return oracle.kt_build(bits(kv.k_pages), kv.page_table.numpy(), kv.seq_lens.numpy())


def _scores(case, kt=None):
    kv = case.kv
    kt = _kt(case) if kt is None else kt
    return oracle.page_scores(bits(case.q), kt, kv.page_table.numpy(), kv.seq_lens.numpy(),
                              kv.page_size)


def test_kt_entries_are_page_min_and_max():
    case = _case([37, 100, 16, 1], seed=1)
    kv = case.kv
    P = kv.page_size
    # finite garbage (not NaN, which min/max comparisons would skip) in the slots past
    # each sequence's end: an entry that took them in would show it
    for b, L in enumerate(kv.seq_lens.tolist()):
        if L % P:
            phys = int(kv.page_table[b, L // P])
            kv.k_pages[phys, :, L % P:, 0::2] = 100.0
            kv.k_pages[phys, :, L % P:, 1::2] = -100.0
    kt = _kt(case)
    cu = kv.cu_kv.tolist()
    for b, L in enumerate(kv.seq_lens.tolist()):
        kd = kv.k_dense[cu[b]:cu[b + 1]].double().numpy()          # [L][Hk][D]
        for p in range((L + P - 1) // P):
            blk = kd[p * P:min(L, (p + 1) * P)]
            phys = int(kv.page_table[b, p])
            np.testing.assert_array_equal(kt[phys, :, :, 0], blk.min(axis=0))
            np.testing.assert_array_equal(kt[phys, :, :, 1], blk.max(axis=0))


def test_page_score_is_the_box_maximum():
    """sum_d max(q_d min_d, q_d max_d) = max of q.k over the 2^D corners of the box, per
    query head; the kv head's score sums its heads'."""
    case = _case([53, 40], Hq=4, Hk=2, D=4, P=16, seed=2)
    kv = case.kv
    kt = _kt(case)
    sc = _scores(case, kt)
    q = case.q.double().numpy()
    g = 2
    for b, L in enumerate(kv.seq_lens.tolist()):
        for p in range((L + 15) // 16):
            phys = int(kv.page_table[b, p])
            for kvh in range(2):
                lo, hi = kt[phys, kvh, :, 0], kt[phys, kvh, :, 1]
                total = 0.0
                for j in range(g):
                    qh = q[b, kvh * g + j]
                    total += max(float(np.dot(qh, np.where(c, hi, lo)))
                                 for c in itertools.product([0, 1], repeat=4))
                assert sc[b, kvh, p] == pytest.approx(total, rel=1e-6, abs=1e-6)


def test_page_score_bounds_every_key():
    case = _case([200, 77], seed=3)
    kv = case.kv
    sc = _scores(case)
    q = case.q.double().numpy()
    cu = kv.cu_kv.tolist()
    g = 4
    for b, L in enumerate(kv.seq_lens.tolist()):
        kd = kv.k_dense[cu[b]:cu[b + 1]].double().numpy()
        for kvh in range(2):
            qs = q[b, kvh * g:(kvh + 1) * g]                         # [g][D]
            for t in range(L):
                dot = float((qs @ kd[t, kvh]).sum())
                assert sc[b, kvh, t // 16] >= dot - 1e-4
        assert np.all(np.isneginf(sc[b, :, (L + 15) // 16:]))


def _ref_select(scores, L, P, topk, window):
    np_ = (L + P - 1) // P
    win = sorted({t // P for t in range(max(L - window, 0), L)})
    wp = win[0] if win else np_
    cand = list(range(wp))
    if len(cand) > topk:
        cand = sorted(cand, key=lambda p: (-float(scores[p]), p))[:topk]
    return sorted(set(cand) | set(win))


@pytest.mark.parametrize("topk,window", [(0, 16), (1, 1), (3, 32), (4, 0), (5, 17), (100, 8),
                                         (2, 100000)])
def test_selection_matches_a_sort(topk, window):
    case = _case([300, 96, 129, 17, 0], seed=4)
    kv = case.kv
    sc = _scores(case)
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), 16, topk, window)
    for b, L in enumerate(kv.seq_lens.tolist()):
        for kvh in range(2):
            ref = _ref_select(sc[b, kvh], L, 16, topk, window)
            got = sel[b, kvh, :nsel[b, kvh]].tolist()
            assert got == ref, (b, kvh, topk, window)


def test_window_whose_start_is_a_page_boundary():
    """L - window a multiple of the page size: the window covers exactly its pages."""
    case = _case([96, 64 + 32], seed=5)
    kv = case.kv
    sc = _scores(case)
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), 16, 1, 32)
    for b in range(2):
        for kvh in range(2):
            got = sel[b, kvh, :nsel[b, kvh]].tolist()
            assert got[-2:] == [4, 5] and len(got) == 3 and got[0] < 4


def test_ties_go_to_the_lower_page():
    """One physical page repeated at several logical positions has identical scores there:
    the lower logical pages win."""
    case = _case([160], Hq=4, Hk=1, seed=6, pt_stride=10)
    kv = case.kv
    pt = kv.page_table.clone()
    dup = int(pt[0, 7])
    for p in (2, 5, 7):
        pt[0, p] = dup                                # pages 2, 5 and 7 are the same page
    kt = oracle.kt_build(bits(kv.k_pages), pt.numpy(), kv.seq_lens.numpy())
    sc = oracle.page_scores(bits(case.q), kt, pt.numpy(), kv.seq_lens.numpy(), 16)
    assert sc[0, 0, 2] == sc[0, 0, 5] == sc[0, 0, 7]
    # make the duplicated page the best one by a margin: choose topk = 2 among it
    order = sorted(range(9), key=lambda p: (-float(sc[0, 0, p]), p))
    rank_of_dup = order.index(2)
    topk = rank_of_dup + 2                            # takes pages 2 and 5, not 7
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), 16, topk, 16)
    got = set(sel[0, 0, :nsel[0, 0]].tolist())
    assert {2, 5} <= got and 7 not in got


def test_window_pages_are_chosen_whatever_their_score():
    case = _case([150], Hq=4, Hk=1, seed=7)
    kv = case.kv
    sc = _scores(case)
    sc[0, 0, 8:10] = -1e30                            # the window pages score lowest
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), 16, 2, 20)
    got = sel[0, 0, :nsel[0, 0]].tolist()
    assert got[-2:] == [8, 9] and len(got) == 4


def test_all_pages_chosen_equals_dense_decode():
    case = _case([300, 96, 129, 17, 0], seed=8)
    kv = case.kv
    sc = _scores(case)
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), 16, 1000, 32)
    out, lse = oracle.sparse_decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages),
                                    kv.page_table.numpy(), kv.seq_lens.numpy(), case.scale, sel,
                                    nsel)
    ro, rl = oracle_decode(case)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_sparse_equals_dense_attention_over_the_chosen_pages():
    """Per kv head: a dense decode of a cache holding only the chosen pages (a new page
    table listing them, the partial last page last) gives the sparse result."""
    case = _case([300, 96, 129], seed=9)
    kv = case.kv
    P, g = 16, 4
    sc = _scores(case)
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), P, 3, 20)
    out, lse = oracle.sparse_decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages),
                                    kv.page_table.numpy(), kv.seq_lens.numpy(), case.scale, sel,
                                    nsel)
    for b, L in enumerate(kv.seq_lens.tolist()):
        for kvh in range(2):
            pages = sel[b, kvh, :nsel[b, kvh]].tolist()
            pt = np.array([[int(kv.page_table[b, p]) for p in pages]], np.int32)
            n = sum(min(P, L - p * P) for p in pages)
            q = bits(case.q[b:b + 1, kvh * g:(kvh + 1) * g])
            kp = bits(kv.k_pages[:, kvh:kvh + 1].contiguous())
            vp = bits(kv.v_pages[:, kvh:kvh + 1].contiguous())
            ro, rl = oracle.decode(q, kp, vp, pt, np.array([n], np.int32), case.scale)
            np.testing.assert_allclose(out[b, kvh * g:(kvh + 1) * g], ro[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, kvh * g:(kvh + 1) * g], rl[0], rtol=0, atol=1e-12)


def test_needle_page_is_chosen():
    """Keys of one early page pointing where the group's queries point, with a large
    magnitude: its (point-like) box scores highest and it is chosen with topk = 1.  (The
    min/max bound of a page of random keys is loose, so the needle needs the magnitude.)"""
    case = _case([400], Hq=4, Hk=1, seed=10)
    kv = case.kv
    P, needle = 16, 6
    phys = int(kv.page_table[0, needle])
    qmean = case.q[0].float().mean(0)
    kv.k_pages[phys, 0] = (16.0 * torch.sign(qmean)).to(torch.bfloat16)
    sc = _scores(case)
    assert int(np.argmax(sc[0, 0, :20])) == needle
    sel, nsel = oracle.sparse_select(sc, kv.seq_lens.numpy(), P, 1, 16)
    assert sel[0, 0, :nsel[0, 0]].tolist() == [needle, 24]
