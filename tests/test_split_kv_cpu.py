"""Sequences spread over several GPUs (one process per GPU): the page-boundary partition,
each rank's local page-table rows and token counts, and the exchange of partial results,
on the CPU.  The per-rank attention and the merge are computed here by the fp64 oracle
(the GPU path runs gqa_paged_decode_partial and lse_combine; tests/test_split_kv_gpu.py
checks those).  Pins: a merge of decodes over any contiguous cut of every sequence's
tokens equals the uncut decode ("FasterTransformer source tour", section 6.1; the
log-sum-exp merge of the NumSplits section of "解锁GQA性能潜力…")."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gqa_attention_paged_b200 import inputs, split_kv
from oracle import oracle
from tests._util import bits, oracle_decode


def _rank_partials(case, world):
    """Oracle decode of every rank's share (the product's partition helpers)."""
    kv = case.kv
    P = kv.page_size
    max_pages = kv.page_table.shape[1]
    parts = []
    for r in range(world):
        p0, p1 = split_kv.rank_page_range(max_pages, world, r)
        pt = split_kv.local_page_table(kv.page_table, p0, p1)
        sl = split_kv.local_seq_lens(kv.seq_lens, P, p0, p1)
        o, l = oracle.decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages), pt.numpy(),
                             sl.numpy(), case.scale)
        parts.append((o, l, p0, p1, sl))
    return parts


def test_rank_page_ranges_cover_every_page_once():
    for max_pages in (0, 1, 7, 64, 129, 512):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for r in range(world):
                p0, p1 = split_kv.rank_page_range(max_pages, world, r)
                assert 0 <= p0 <= p1 <= max_pages
                seen += list(range(p0, p1))
            assert seen == list(range(max_pages))


def test_local_token_counts_sum_to_the_sequence():
    lens = torch.tensor([0, 1, 15, 16, 17, 100, 1000], dtype=torch.int32)
    P = 16
    max_pages = 63
    for world in (1, 2, 3, 5):
        tot = torch.zeros_like(lens)
        for r in range(world):
            p0, p1 = split_kv.rank_page_range(max_pages, world, r)
            sl = split_kv.local_seq_lens(lens, P, p0, p1)
            assert (sl >= 0).all() and (sl <= (p1 - p0) * P).all()
            tot += sl
        assert torch.equal(tot, lens)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_rank_partition_merge_equals_unsplit(world):
    """Per-rank oracle decodes over the product's partition, merged by the oracle's
    log-sum-exp merge, equal the uncut decode to fp64 rounding."""
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [300, 37, 129], seed=5, pt_stride=20)
    parts = _rank_partials(case, world)
    B, Hq, D = case.q.shape
    o_all = np.stack([p[0].reshape(B * Hq, D) for p in parts])
    l_all = np.stack([p[1].reshape(B * Hq) for p in parts])
    out, lse = oracle.lse_combine(o_all, l_all)
    ref_o, ref_l = oracle_decode(case)
    np.testing.assert_allclose(out, ref_o.reshape(B * Hq, D), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l.reshape(B * Hq), rtol=0, atol=1e-12)
    # a rank holding none of a sequence gives o = 0, lse = -inf for it
    for o, l, p0, p1, sl in parts:
        for b in range(B):
            if int(sl[b]) == 0:
                assert np.all(o[b] == 0) and np.all(np.isneginf(l[b]))


def test_any_contiguous_cut_merges_to_the_uncut_decode():
    """The merge identity the multi-GPU path rests on, for random cuts of each
    sequence's pages into contiguous ranges (empty ranges included)."""
    rng = np.random.default_rng(3)
    case = inputs.make_decode_case(2, 8, 2, 64, 16, [250, 91], seed=6, pt_stride=16)
    kv = case.kv
    B, Hq, D = case.q.shape
    L = kv.seq_lens.numpy()
    ref_o, ref_l = oracle_decode(case)
    for _ in range(5):
        R = int(rng.integers(2, 6))
        cuts = np.sort(rng.integers(0, 17, size=R - 1))
        bounds = [0] + list(cuts) + [16]
        os_, ls_ = [], []
        for r in range(R):
            p0, p1 = int(bounds[r]), int(bounds[r + 1])
            pt = kv.page_table[:, p0:max(p1, p0 + 1)].contiguous().numpy()
            sl = np.clip(L - p0 * 16, 0, (p1 - p0) * 16).astype(np.int32)
            o, l = oracle.decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages), pt, sl,
                                 case.scale)
            os_.append(o.reshape(B * Hq, D))
            ls_.append(l.reshape(B * Hq))
        out, lse = oracle.lse_combine(np.stack(os_), np.stack(ls_))
        np.testing.assert_allclose(out, ref_o.reshape(B * Hq, D), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l.reshape(B * Hq), rtol=0, atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        case = inputs.make_decode_case(3, 8, 2, 64, 16, [300, 37, 129], seed=5, pt_stride=20)
        kv = case.kv
        B, Hq, D = case.q.shape
        p0, p1 = split_kv.rank_page_range(kv.page_table.shape[1], world, rank)
        pt = split_kv.local_page_table(kv.page_table, p0, p1)
        sl = split_kv.local_seq_lens(kv.seq_lens, kv.page_size, p0, p1)
        o, l = oracle.decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages), pt.numpy(),
                             sl.numpy(), case.scale)
        o_t = torch.from_numpy(o.reshape(B * Hq, D)).float()
        l_t = torch.from_numpy(l.reshape(B * Hq)).float()
        o_all, l_all = split_kv.exchange_partials(o_t, l_t)
        out, lse = oracle.lse_combine(o_all.double().numpy(), l_all.double().numpy())
        q.put((rank, out, lse, o_all.numpy(), l_all.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gloo_ranks_exchange_and_merge(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [300, 37, 129], seed=5, pt_stride=20)
    ref_o, ref_l = oracle_decode(case)
    B, Hq, D = case.q.shape
    parts = _rank_partials(case, world)
    for r, out, lse, o_all, l_all in res:
        # every rank received every rank's partial, in rank order
        for k in range(world):
            np.testing.assert_array_equal(o_all[k], parts[k][0].reshape(B * Hq, D).astype(np.float32))
            np.testing.assert_array_equal(l_all[k], parts[k][1].reshape(B * Hq).astype(np.float32))
        # and the merge of the fp32 partials is the uncut decode to fp32 rounding
        np.testing.assert_allclose(out, ref_o.reshape(B * Hq, D), rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(lse, ref_l.reshape(B * Hq), rtol=1e-6, atol=1e-6)
    np.testing.assert_array_equal(res[0][1], res[1][1])  # both ranks hold the same result
