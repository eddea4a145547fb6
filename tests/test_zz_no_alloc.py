"""gqa_paged_decode_static_scratch: decode for callers that cannot allocate device memory
(an engine plugin's enqueue, an allocation-free real-time loop, a host whose device memory
belongs to another allocator).  It keeps its split partials, merge pieces and merge
counters in a fixed array inside the library instead of a caller workspace.

Checked here through the C ABI against gqa_paged_decode (fresh workspace) and against the
fp64 oracle, within the bf16 tolerance of the other tests (|err| <= 2e-3 + 1e-2 |ref|),
on calls in a row on the one shared array: every call runs on the array as the previous
call left it.  The sequence covers the split schedule, then the balanced schedule (whose
merge counters sit where the previous call's split partials were), the balanced schedule
with its separate piece merge (a few long sequences), and a repeat of the first balanced
call, which must give the same bits.

This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from tests._util import bf16_tol_ok, err_report, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_call(d, case, S):
    """Raw C-ABI call of gqa_paged_decode_static_scratch; returns (status, out, lse)."""
    B, Hq, D = case.q.shape
    num_pages, Hk, P, _ = case.kv.k_pages.shape
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=DEV)
    kvd = 1 if case.kv.k_scale is not None else 0
    st = binding.load().gqa_paged_decode_static_scratch(
        _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d.get("ks")), _p(d.get("vs")), kvd, _p(d["pt"]),
        d["pt"].shape[1], _p(d["sl"]), B, Hq, Hk, D, P, num_pages, case.scale, S, 1, _p(out),
        _p(lse), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, out, lse


def _dev(case):
    kv = case.kv
    d = dict(q=case.q.to(DEV), k=kv.k_pages.to(DEV), v=kv.v_pages.to(DEV),
             pt=kv.page_table.to(DEV), sl=kv.seq_lens.to(DEV))
    if kv.k_scale is not None:
        d["ks"], d["vs"] = kv.k_scale.to(DEV), kv.v_scale.to(DEV)
    return d


def _check(case, d, S, tag):
    """One static-scratch call, compared with the workspace call and with the oracle."""
    ref_o, ref_l = binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"],
                                            case.scale, num_splits=S,
                                            k_scale=d.get("ks"), v_scale=d.get("vs"))
    st, out, lse = _static_call(d, case, S)
    assert st == 0, f"{tag}: {binding.status_string(st)}"
    o = out.float().cpu().numpy()
    ro = ref_o.float().cpu().numpy()
    ok, bad = bf16_tol_ok(o, ro)
    assert ok, f"{tag} vs workspace call: {err_report(o, ro)} bad={int(bad.sum())}"
    np.testing.assert_allclose(lse.cpu().numpy(), ref_l.cpu().numpy(), rtol=1e-4, atol=2e-3,
                               err_msg=f"{tag} lse vs workspace call")
    oo, ol = oracle_decode(case)
    ok, bad = bf16_tol_ok(o, oo)
    assert ok, f"{tag} vs oracle: {err_report(o, oo)} bad={int(bad.sum())}"
    np.testing.assert_allclose(lse.cpu().numpy(), ol, rtol=1e-4, atol=2e-3,
                               err_msg=f"{tag} lse vs oracle")
    return out, lse


def test_static_scratch_matches_workspace_decode_two_calls_in_a_row():
    calls = [(inputs.llama7b_decode(seed=11), 4),              # 4 splits of a ragged batch
             (inputs.make_decode_case(3, 16, 2, 64, 32, [300, 7, 129], seed=12), 3)]
    for i, (case, S) in enumerate(calls):
        _check(case, _dev(case), S, f"call {i}")


def test_static_scratch_balanced_after_split_calls():
    """split (S=4) -> balanced -> balanced with the separate piece merge -> balanced again.
    The first balanced call's merge counters occupy bytes the split call's partials
    overwrote, so they must be cleared by the call itself."""
    ragged = inputs.llama7b_decode(seed=21, B=48)
    few_long = inputs.make_decode_case(2, 32, 8, 128, 16, [4096, 3001], seed=22)
    d_r, d_f = _dev(ragged), _dev(few_long)
    # the second balanced shape really takes the separate piece merge
    assert binding.gqa_paged_decode_kernel_launches(2, 32, 8, 128, 16, 4096, 0, 0) == 2
    assert binding.gqa_paged_decode_kernel_launches(48, 32, 8, 128, 16, 2048, 0, 0) == 1
    _check(ragged, d_r, 4, "split S=4")
    o1, l1 = _check(ragged, d_r, 0, "balanced after split")
    _check(few_long, d_f, 0, "balanced, separate piece merge")
    o2, l2 = _check(ragged, d_r, 0, "balanced again")
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)), "repeated balanced calls differ"
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


def test_static_scratch_rejects_calls_that_do_not_fit():
    case = inputs.sweep_decode(64, seed=1, ctx=2048)
    need = binding.gqa_paged_decode_workspace_size(64, 32, 8, 128, 16,
                                                   case.kv.page_table.shape[1] * 16, 0, 64)
    assert need > 16 << 20
    d = _dev(case)
    st, out, _ = _static_call(d, case, 64)
    assert st == -5                       # GQA_ERR_WORKSPACE, nothing enqueued
    assert torch.isnan(out.float()).all()  # outputs untouched
