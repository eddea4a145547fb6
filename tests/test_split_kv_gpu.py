"""Decode of sequences spread over several GPUs, on one GPU: every rank's share is computed
in turn by gqa_paged_decode_partial (the kernels each rank runs), the partials are stacked
as the all-gather would deliver them, and lse_combine merges them.  Compared with the fp64
oracle: each rank's fp32 partial against the oracle's decode of the same tokens, and the
merge against the oracle's uncut decode (bf16 gate).  Ranks whose kernels would wait on
one another are never emulated: each rank's work is an ordinary, independent launch."""
import datetime
import socket

import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs, split_kv
from oracle import oracle
from tests._util import bf16_tol_ok, bits, err_report, np32, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dev(case):
    kv = case.kv
    d = dict(q=case.q.to(DEV), k=kv.k_pages.to(DEV), v=kv.v_pages.to(DEV))
    d["ks"] = None if kv.k_scale is None else kv.k_scale.to(DEV)
    d["vs"] = None if kv.v_scale is None else kv.v_scale.to(DEV)
    return d


def _partial_ok(got, ref, tag):
    """fp32 partials: |err| <= 1e-4 + 1e-3 |ref| (the kernels accumulate in fp32; only the
    final bf16 rounding of the full decode is missing here)."""
    got = np.asarray(got, np.float64)
    bad = ~(np.abs(got - ref) <= 1e-4 + 1e-3 * np.abs(ref))
    assert not bad.any(), f"{tag}: {err_report(got, ref)} bad={int(bad.sum())}"


def _simulate(case, world, S):
    kv = case.kv
    d = _dev(case)
    B, Hq, D = case.q.shape
    max_pages = kv.page_table.shape[1]
    os_, ls_ = [], []
    for r in range(world):
        p0, p1 = split_kv.rank_page_range(max_pages, world, r)
        pt = split_kv.local_page_table(kv.page_table, p0, p1)
        sl = split_kv.local_seq_lens(kv.seq_lens, kv.page_size, p0, p1)
        o, l = binding.gqa_paged_decode_partial(d["q"], d["k"], d["v"], pt.to(DEV), sl.to(DEV),
                                                case.scale, num_splits=S, k_scale=d["ks"],
                                                v_scale=d["vs"])
        torch.cuda.synchronize()
        ro, rl = oracle.decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages), pt.numpy(),
                               sl.numpy(), case.scale, np32(kv.k_scale), np32(kv.v_scale))
        _partial_ok(o.cpu().numpy(), ro, f"rank {r}/{world} o_part")
        lg = l.cpu().numpy().astype(np.float64)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isneginf(lg), np.isneginf(rl)), f"rank {r}: empty rows differ"
        np.testing.assert_allclose(lg[fin], rl[fin], rtol=1e-5, atol=1e-4)
        os_.append(o.view(B * Hq, D))
        ls_.append(l.view(B * Hq))
    out, lse = binding.lse_combine(torch.stack(os_), torch.stack(ls_))
    torch.cuda.synchronize()
    return out.view(B, Hq, D), lse.view(B, Hq)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("S", [0, binding.GQA_SPLITS_BALANCED, 3])
def test_split_ranks_llama7b(world, S):
    case = inputs.llama7b_decode(seed=31)
    out, lse = _simulate(case, world, S)
    ro, rl = oracle_decode(case)
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, f"world {world}: {err_report(o, ro)} bad={int(bad.sum())}"
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-5, atol=2e-4)


@pytest.mark.parametrize("world", [2, 4])
def test_split_ranks_long_sequences_bf16_and_fp8(world):
    """Few long sequences (each rank's share still spans many workers, so the balanced
    schedule's separate piece merge runs on every rank), bf16 and e4m3 KV."""
    for kvd in ("bf16", "fp8_e4m3"):
        case = inputs.make_decode_case(2, 32, 8, 128, 64, [6000, 2500], seed=32, kv_dtype=kvd,
                                       outlier_p=0.01)
        out, lse = _simulate(case, world, 0)
        ro, rl = oracle_decode(case)
        o = out.float().cpu().numpy()
        ok, bad = bf16_tol_ok(o, ro)
        assert ok, f"{kvd} world {world}: {err_report(o, ro)} bad={int(bad.sum())}"


def test_split_ranks_tiny_d64_with_empty_shares():
    """Head dim 64, and a rank count that leaves the short sequence with no tokens on the
    later ranks (o = 0, lse = -inf there, left out of the merge)."""
    case = inputs.tiny_decode(seed=3)
    out, lse = _simulate(case, 5, 1)
    ro, rl = oracle_decode(case)
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, err_report(o, ro)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_split_kv_decode_through_one_nccl_rank():
    """The whole multi-GPU call (partial decode, NCCL all-gathers, merge) in a one-rank
    process group: the collective path runs for real, with nothing to wait for."""
    import torch.distributed as dist
    case = inputs.llama7b_decode(seed=33)
    kv = case.kv
    d = _dev(case)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV))
    try:
        p0, p1 = split_kv.rank_page_range(kv.page_table.shape[1], 1, 0)
        out, lse = split_kv.split_kv_decode(
            d["q"], d["k"], d["v"], split_kv.local_page_table(kv.page_table, p0, p1).to(DEV),
            split_kv.local_seq_lens(kv.seq_lens, kv.page_size, p0, p1).to(DEV), case.scale)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ro, rl = oracle_decode(case)
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, err_report(o, ro)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-5, atol=2e-4)
