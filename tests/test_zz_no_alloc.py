"""gqa_paged_decode_static_scratch: decode for callers that cannot allocate device memory
(an engine plugin's enqueue, an allocation-free real-time loop, a host whose device memory
belongs to another allocator).  It keeps its split partials in a fixed array inside the
library instead of a caller workspace.  Checked here through the C ABI against
gqa_paged_decode on the same inputs, within the bf16 tolerance of the other tests
(|err| <= 2e-3 + 1e-2 |ref|), on two calls in a row with different shapes, so the second
call runs on the array as the first one left it.

This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from tests._util import bf16_tol_ok, err_report

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


def test_static_scratch_matches_workspace_decode_two_calls_in_a_row():
    calls = [(inputs.llama7b_decode(seed=11), 4),              # 4 splits of a ragged batch
             (inputs.make_decode_case(3, 16, 2, 64, 32, [300, 7, 129], seed=12), 3)]
    for i, (case, S) in enumerate(calls):
        d = _dev(case)
        ref_o, ref_l = binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"],
                                                case.scale, num_splits=S,
                                                k_scale=d.get("ks"), v_scale=d.get("vs"))
        st, out, lse = _static_call(d, case, S)
        assert st == 0, binding.status_string(st)
        ro, o = ref_o.float().cpu().numpy(), out.float().cpu().numpy()
        ok, bad = bf16_tol_ok(o, ro)
        assert ok, f"call {i}: {err_report(o, ro)} bad={int(bad.sum())}"
        rl, l = ref_l.cpu().numpy(), lse.cpu().numpy()
        np.testing.assert_allclose(l, rl, rtol=1e-4, atol=2e-3, err_msg=f"call {i}")


def test_static_scratch_rejects_calls_that_do_not_fit():
    case = inputs.sweep_decode(64, seed=1, ctx=2048)
    need = binding.gqa_paged_decode_workspace_size(64, 32, 8, 128, 16,
                                                   case.kv.page_table.shape[1] * 16, 0, 64)
    assert need > 16 << 20
    d = _dev(case)
    st, out, _ = _static_call(d, case, 64)
    assert st == -5                       # GQA_ERR_WORKSPACE, nothing enqueued
    assert torch.isnan(out.float()).all()  # outputs untouched
