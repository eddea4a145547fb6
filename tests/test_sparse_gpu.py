"""Page-level top-K sparse decode on the GPU against the fp64 oracle: the KT entries and
the selection bit for bit (both sides take the selection's fp32 decisions the same way),
the attention over the chosen pages within the bf16 gate."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from oracle import oracle
from tests._util import bf16_tol_ok, bits, err_report, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dev(case):
    kv = case.kv
    return dict(q=case.q.to(DEV), k=kv.k_pages.to(DEV), v=kv.v_pages.to(DEV),
                pt=kv.page_table.to(DEV), sl=kv.seq_lens.to(DEV))


def _kt_bits_equal(kt_gpu, kt_ref, kv):
    """The GPU's bf16 entries equal the oracle's exact min / max on every referenced page."""
    g = kt_gpu.float().cpu().double().numpy()
    P = kv.page_size
    for b, L in enumerate(kv.seq_lens.tolist()):
        for p in range((L + P - 1) // P):
            phys = int(kv.page_table[b, p])
            np.testing.assert_array_equal(g[phys], kt_ref[phys], err_msg=f"b={b} p={p}")


CASES = {
    "llama7b": lambda: inputs.llama7b_decode(seed=41),
    "long_p64": lambda: inputs.make_decode_case(4, 64, 8, 128, 64, [3000, 9001, 1500, 700],
                                                seed=42, outlier_p=0.01),
    "tiny_d64": lambda: inputs.make_decode_case(3, 8, 2, 64, 16, [300, 37, 129], seed=43),
    "mqa_g16": lambda: inputs.make_decode_case(2, 16, 1, 128, 32, [1000, 400], seed=44),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_kt_build_is_bit_exact(name):
    case = CASES[name]()
    d = _dev(case)
    kt = binding.gqa_paged_kt_build(d["k"], d["pt"], d["sl"])
    torch.cuda.synchronize()
    kv = case.kv
    ref = oracle.kt_build(bits(kv.k_pages), kv.page_table.numpy(), kv.seq_lens.numpy())
    _kt_bits_equal(kt, ref, kv)


def test_kt_append_follows_the_appended_tokens():
    """Tokens appended one by one (crossing page boundaries): the appended entries equal a
    fresh build over the grown cache, and the oracle's."""
    # pages for the grown sequences are allocated up front (each sequence its own), the
    # appends overwrite them token by token
    L0 = torch.tensor([30, 47, 16], dtype=torch.int32)
    case = inputs.make_decode_case(3, 8, 2, 128, 16, (L0 + 40).tolist(), seed=45)
    kv = case.kv
    d = _dev(case)
    d["sl"] = L0.to(DEV)
    kt = binding.gqa_paged_kt_build(d["k"], d["pt"], d["sl"])
    gen = torch.Generator().manual_seed(46)
    sl = L0.clone()
    for step in range(40):
        sl = sl + 1
        sl_d = sl.to(DEV)
        k_new = torch.randn(3, 2, 128, generator=gen).to(torch.bfloat16).to(DEV)
        v_new = torch.randn(3, 2, 128, generator=gen).to(torch.bfloat16).to(DEV)
        binding.gqa_paged_append_kv(k_new, v_new, d["k"], d["v"], d["pt"], sl_d)
        binding.gqa_paged_kt_append(k_new, d["pt"], sl_d, kt, kv.page_size)
    torch.cuda.synchronize()
    fresh = binding.gqa_paged_kt_build(d["k"], d["pt"], sl.to(DEV))
    torch.cuda.synchronize()
    kv.seq_lens = sl
    ref = oracle.kt_build(bits(d["k"].cpu()), kv.page_table.numpy(), sl.numpy())
    kv.k_pages = d["k"].cpu()
    _kt_bits_equal(kt, ref, kv)
    _kt_bits_equal(fresh, ref, kv)


def _oracle_selection(case, topk, window, pt=None):
    kv = case.kv
    pt = kv.page_table if pt is None else pt
    kt = oracle.kt_build(bits(kv.k_pages), pt.numpy(), kv.seq_lens.numpy())
    sc = oracle.page_scores(bits(case.q), kt, pt.numpy(), kv.seq_lens.numpy(), kv.page_size)
    return oracle.sparse_select(sc, kv.seq_lens.numpy(), kv.page_size, topk, window)


def _check_selection(case, d, topk, window, pt=None):
    kv = case.kv
    pt_h = kv.page_table if pt is None else pt
    pt_d = pt_h.to(DEV)
    kt = binding.gqa_paged_kt_build(d["k"], pt_d, d["sl"])
    B, Hk = kv.page_table.shape[0], kv.k_pages.shape[1]
    ws = binding.new_workspace(binding.load().gqa_paged_sparse_select_workspace_size(
        B, Hk, pt_h.shape[1]), DEV)
    st, sl_, sp = binding.gqa_paged_sparse_select(d["q"], kt, d["k"], pt_d, d["sl"], topk, window,
                                                  workspace=ws)
    assert binding.gqa_get_error(ws) == 0
    sel, nsel = _oracle_selection(case, topk, window, pt_h)
    B, Hk = nsel.shape
    P = kv.page_size
    st, sl_, sp = st.cpu().numpy(), sl_.cpu().numpy(), sp.cpu().numpy()
    for b in range(B):
        L = int(kv.seq_lens[b])
        for j in range(Hk):
            r = b * Hk + j
            ref = sel[b, j, :nsel[b, j]].tolist()
            n = len(ref)
            assert sp[r, :n].tolist() == ref, (b, j)
            assert st[r, :n].tolist() == [int(pt_h[b, p]) * Hk + j for p in ref], (b, j)
            assert sl_[r] == sum(min(P, L - p * P) for p in ref), (b, j)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("topk,window", [(0, 32), (4, 32), (16, 1), (7, 0), (1000, 64)])
def test_selection_is_bit_exact(name, topk, window):
    case = CASES[name]()
    _check_selection(case, _dev(case), topk, window)


@pytest.mark.parametrize("topk,window", [(4, 32), (300, 16)])
def test_selection_is_bit_exact_on_a_table_of_more_than_1024_pages(topk, window):
    """A table of 1250 pages of 16 tokens: more pages than the pick's 512 threads, so each
    thread takes several pages in every radix pass, count and compaction."""
    case = inputs.make_decode_case(2, 16, 2, 128, 16, [20000, 5000], seed=48)
    assert case.kv.page_table.shape[1] > 1024
    _check_selection(case, _dev(case), topk, window)


def test_selection_ties_go_to_the_lower_page():
    case = inputs.make_decode_case(2, 32, 8, 128, 16, [320, 200], seed=47, pt_stride=20)
    pt = case.kv.page_table.clone()
    for b in range(2):
        dup = int(pt[b, 9])
        for p in (1, 4, 9):
            pt[b, p] = dup                      # the same full page at three positions
    _check_selection(case, _dev(case), 5, 16, pt)
    _check_selection(case, _dev(case), 1, 16, pt)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("topk,window,S", [(4, 32, 0), (16, 1, 0), (8, 64, 3)])
def test_sparse_decode_matches_the_oracle(name, topk, window, S):
    case = CASES[name]()
    kv = case.kv
    d = _dev(case)
    kt = binding.gqa_paged_kt_build(d["k"], d["pt"], d["sl"])
    out, lse = binding.gqa_paged_sparse_decode(d["q"], d["k"], d["v"], kt, d["pt"], d["sl"],
                                               case.scale, topk, window, num_splits=S)
    torch.cuda.synchronize()
    sel, nsel = _oracle_selection(case, topk, window)
    ro, rl = oracle.sparse_decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages),
                                  kv.page_table.numpy(), kv.seq_lens.numpy(), case.scale, sel, nsel)
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, f"{name}: {err_report(o, ro)} bad={int(bad.sum())}"
    lg = lse.cpu().numpy()
    fin = np.isfinite(rl)
    np.testing.assert_allclose(lg[fin], rl[fin], rtol=1e-5, atol=2e-4)


def test_sparse_with_every_page_is_the_dense_decode():
    case = CASES["llama7b"]()
    d = _dev(case)
    kt = binding.gqa_paged_kt_build(d["k"], d["pt"], d["sl"])
    out, lse = binding.gqa_paged_sparse_decode(d["q"], d["k"], d["v"], kt, d["pt"], d["sl"],
                                               case.scale, 10000, 32)
    torch.cuda.synchronize()
    ro, rl = oracle_decode(case)
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, err_report(o, ro)


def test_bad_page_entry_sets_the_error_word():
    case = CASES["tiny_d64"]()
    d = _dev(case)
    kt = binding.gqa_paged_kt_build(d["k"], d["pt"], d["sl"])
    pt = d["pt"].clone()
    pt[1, 1] = 10 ** 6
    ws = binding.new_workspace(
        binding.gqa_paged_sparse_decode_workspace_size(3, 8, 2, 64, 16, pt.shape[1], 1, 16), DEV)
    binding.gqa_paged_sparse_decode(d["q"], d["k"], d["v"], kt, pt, d["sl"], case.scale, 1, 16,
                                    workspace=ws)
    assert binding.gqa_get_error(ws) == -7
