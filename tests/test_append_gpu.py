"""GPU parity of the KV append (gqa_paged_append_kv) and of append + decode
(gqa_paged_append_decode) against the fp64 oracle, through the C ABI.  The append is
bit-exact: bf16 bits copied; e4m3 codes and per-(page, kv head) scales equal to the
oracle's (both divide in fp32 and round to nearest even).  The decode after it meets the
usual bf16 tolerance |gpu - ref| <= 2e-3 + 1e-2 |ref|."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from oracle import oracle
from tests._util import bf16_tol_ok, bits, err_report

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _new_tokens(B, Hk, D, seed):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Hk, D, generator=g) * 2).to(torch.bfloat16)
    v = (torch.randn(B, Hk, D, generator=g) * 2).to(torch.bfloat16)
    return k, v


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("P", [16, 64])
def test_append_is_bit_exact(kv_dtype, P):
    # lengths that open a page (slot 0), land mid-page and end a page, plus an empty one
    lens = [1, P + 1, 2 * P, 37, 0, 3 * P + 5]
    B, Hk, D = len(lens), 2, 128
    case = inputs.make_decode_case(B, 8, Hk, D, P, lens, seed=11, kv_dtype=kv_dtype)
    kv = case.kv
    kn, vn = _new_tokens(B, Hk, D, 7)
    want = oracle.append_kv(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                            kv.seq_lens.numpy(), bits(kn), bits(vn),
                            None if kv.k_scale is None else kv.k_scale.numpy(),
                            None if kv.v_scale is None else kv.v_scale.numpy())
    kp, vp = kv.k_pages.to(DEV), kv.v_pages.to(DEV)
    ks = None if kv.k_scale is None else kv.k_scale.to(DEV)
    vs = None if kv.v_scale is None else kv.v_scale.to(DEV)
    ws = binding.gqa_paged_append_kv(kn.to(DEV), vn.to(DEV), kp, vp, kv.page_table.to(DEV),
                                     kv.seq_lens.to(DEV), k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert binding.gqa_get_error(ws) == 0
    assert np.array_equal(bits(kp), want[0]) and np.array_equal(bits(vp), want[1])
    if ks is not None:
        assert np.array_equal(ks.cpu().numpy(), want[2]) and np.array_equal(vs.cpu().numpy(), want[3])


@pytest.mark.parametrize("S", [0, 3])
def test_append_decode_matches_the_oracle(S):
    case = inputs.llama7b_decode(seed=4)
    kv = case.kv
    B, Hq, D = case.q.shape
    kn, vn = _new_tokens(B, case.Hk, D, 8)
    kp_o, vp_o, _, _ = oracle.append_kv(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                                        kv.seq_lens.numpy(), bits(kn), bits(vn))
    ref_o, ref_l = oracle.decode(bits(case.q), kp_o, vp_o, kv.page_table.numpy(),
                                 kv.seq_lens.numpy(), case.scale)
    kp, vp = kv.k_pages.to(DEV), kv.v_pages.to(DEV)
    out, lse = binding.gqa_paged_append_decode(case.q.to(DEV), kn.to(DEV), vn.to(DEV), kp, vp,
                                               kv.page_table.to(DEV), kv.seq_lens.to(DEV),
                                               case.scale, num_splits=S)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ref_o)
    assert ok, f"{err_report(o, ref_o)} bad={int(bad.sum())}"
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(lse.cpu().numpy()[fin], ref_l[fin], rtol=1e-4, atol=2e-3)
    assert np.array_equal(bits(kp), kp_o)


def test_append_decode_fp8_matches_the_oracle():
    case = inputs.make_decode_case(8, 64, 8, 128, 64, [4096, 1, 65, 128, 2000, 64, 3000, 777],
                                   seed=9, kv_dtype="fp8_e4m3")
    kv = case.kv
    B, Hq, D = case.q.shape
    kn, vn = _new_tokens(B, case.Hk, D, 10)
    kp_o, vp_o, ks_o, vs_o = oracle.append_kv(bits(kv.k_pages), bits(kv.v_pages),
                                              kv.page_table.numpy(), kv.seq_lens.numpy(),
                                              bits(kn), bits(vn), kv.k_scale.numpy(),
                                              kv.v_scale.numpy())
    ref_o, ref_l = oracle.decode(bits(case.q), kp_o, vp_o, kv.page_table.numpy(),
                                 kv.seq_lens.numpy(), case.scale, ks_o, vs_o)
    kp, vp = kv.k_pages.to(DEV), kv.v_pages.to(DEV)
    ks, vs = kv.k_scale.to(DEV), kv.v_scale.to(DEV)
    out, lse = binding.gqa_paged_append_decode(case.q.to(DEV), kn.to(DEV), vn.to(DEV), kp, vp,
                                               kv.page_table.to(DEV), kv.seq_lens.to(DEV),
                                               case.scale, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ref_o)
    assert ok, f"{err_report(o, ref_o)} bad={int(bad.sum())}"
    assert np.array_equal(ks.cpu().numpy(), ks_o) and np.array_equal(vs.cpu().numpy(), vs_o)


def test_append_bad_page_entry_sets_the_error_word():
    case = inputs.make_decode_case(2, 8, 2, 64, 16, [20, 5], seed=12)
    kv = case.kv
    pt = kv.page_table.clone()
    pt[0, 1] = kv.k_pages.shape[0] + 5  # token 19 of sequence 0 lives in logical page 1
    kn, vn = _new_tokens(2, 2, 64, 13)
    kp, vp = kv.k_pages.to(DEV), kv.v_pages.to(DEV)
    before = bits(kp)
    ws = binding.gqa_paged_append_kv(kn.to(DEV), vn.to(DEV), kp, vp, pt.to(DEV),
                                     kv.seq_lens.to(DEV))
    assert binding.gqa_get_error(ws) == -7  # GQA_ERR_BAD_PAGE
    after = bits(kp)
    # sequence 1's token is written, nothing else changed
    phys1 = int(kv.page_table[1, 0])
    diff = before != after
    assert diff.any() and not diff[np.arange(diff.shape[0]) != phys1].any()
