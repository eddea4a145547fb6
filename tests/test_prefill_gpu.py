"""GPU parity of causal chunked prefill (tcgen05 kernel) against the fp64 oracle, through
the C ABI.  Tolerance: |gpu - ref| <= 2e-3 + 1e-2 |ref| per element."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from oracle import oracle
from tests._util import bf16_tol_ok, bits, err_report, oracle_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_prefill(case, causal=True, max_q_len=None, workspace=None):
    kv = case.kv
    out, lse = binding.gqa_paged_prefill(
        case.q.to(DEV), case.cu_q.to(DEV), kv.k_pages.to(DEV), kv.v_pages.to(DEV),
        kv.page_table.to(DEV), kv.seq_lens.to(DEV), case.scale,
        max_q_len=case.max_q_len if max_q_len is None else max_q_len, causal=causal,
        workspace=workspace)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check(out, lse, ref_o, ref_l, what=""):
    ok, bad = bf16_tol_ok(out, ref_o)
    assert ok, f"{what}: {err_report(out, ref_o)} bad={int(bad.sum())}"
    np.testing.assert_allclose(lse, ref_l, rtol=1e-4, atol=2e-3, err_msg=what)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_prefill(seed):
    case = inputs.make_prefill_case(3, 8, 2, 128, 16, [0, 20, 45], [17, 1, 40], seed=seed)
    ref_o, ref_l = oracle_prefill(case)
    out, lse = run_prefill(case)
    check(out, lse, ref_o, ref_l, f"tiny seed={seed}")


@pytest.mark.parametrize("Hq,Hk,P", [(32, 8, 16), (8, 8, 32), (8, 1, 64), (12, 4, 16),
                                     (64, 8, 64), (3, 1, 16)])
def test_prefill_group_sizes_and_pages(Hq, Hk, P):
    case = inputs.make_prefill_case(3, Hq, Hk, 128, P, [0, 130, 301], [77, 128, 200],
                                    seed=Hq + P)
    ref_o, ref_l = oracle_prefill(case)
    out, lse = run_prefill(case)
    check(out, lse, ref_o, ref_l, f"Hq={Hq} Hk={Hk} P={P}")


@pytest.mark.parametrize("Hq,Hk,P,causal", [(8, 2, 16, True), (32, 8, 16, True),
                                            (16, 16, 32, True), (8, 1, 64, False)])
def test_prefill_head_dim_64(Hq, Hk, P, causal):
    case = inputs.make_prefill_case(3, Hq, Hk, 64, P, [0, 70, 260], [33, 128, 150],
                                    seed=Hq + Hk + P)
    ref_o, ref_l = oracle_prefill(case, causal=causal)
    out, lse = run_prefill(case, causal=causal)
    check(out, lse, ref_o, ref_l, f"D=64 Hq={Hq} Hk={Hk} P={P} causal={causal}")


def test_prefill_non_causal():
    case = inputs.make_prefill_case(2, 8, 2, 128, 16, [50, 200], [60, 129], seed=4)
    ref_o, ref_l = oracle_prefill(case, causal=False)
    out, lse = run_prefill(case, causal=False)
    check(out, lse, ref_o, ref_l, "non-causal")


def test_prefill_last_row_matches_gpu_decode():
    case = inputs.make_prefill_case(4, 32, 8, 128, 16, [0, 100, 1000, 2047], [1, 64, 33, 200],
                                    seed=5)
    out, lse = run_prefill(case)
    kv = case.kv
    last = (case.cu_q[1:] - 1).long()
    dout, dlse = binding.gqa_paged_decode(case.q[last].contiguous().to(DEV), kv.k_pages.to(DEV),
                                          kv.v_pages.to(DEV), kv.page_table.to(DEV),
                                          kv.seq_lens.to(DEV), case.scale, num_splits=1)
    torch.cuda.synchronize()
    d = dout.float().cpu().numpy()
    ref_o, ref_l = oracle_prefill(case)
    check(out[last.numpy()], lse[last.numpy()], ref_o[last.numpy()], ref_l[last.numpy()], "last")
    ok, _ = bf16_tol_ok(d, ref_o[last.numpy()])
    assert ok
    # both paths agree with each other to bf16 rounding
    assert np.max(np.abs(out[last.numpy()] - d)) < 2e-2


def test_prefill_max_q_len_too_small_sets_error():
    case = inputs.make_prefill_case(2, 8, 2, 128, 16, [10, 10], [40, 100], seed=6)
    ws = binding.new_workspace(binding.gqa_paged_prefill_workspace_size(140, 8, 128), DEV)
    run_prefill(case, max_q_len=40, workspace=ws)
    assert binding.gqa_get_error(ws) == -2


def _sampled_prefill_oracle(case, k):
    """Oracle rows for the first k and the last k query tokens of every chunk: the first
    k form a chunk of their own ending at position L - Lq + k - 1, the last k one ending
    at L - 1; causal masking makes both exactly the full chunk's rows."""
    kv = case.kv
    cu = case.cu_q.numpy()
    L = kv.seq_lens.numpy()
    rows, refs_o, refs_l = [], [], []
    for part in ("first", "last"):
        qs, lens, cq = [], [], [0]
        for b in range(len(L)):
            Lq = cu[b + 1] - cu[b]
            kk = min(k, Lq)
            sel = np.arange(cu[b], cu[b] + kk) if part == "first" else np.arange(cu[b + 1] - kk, cu[b + 1])
            rows.append(sel)
            qs.append(sel)
            lens.append(L[b] - Lq + kk if part == "first" else L[b])
            cq.append(cq[-1] + kk)
        idx = np.concatenate(qs)
        o, l = oracle.prefill(bits(case.q[torch.from_numpy(idx)]), np.array(cq, np.int32),
                              bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                              np.array(lens, np.int32), case.scale)
        refs_o.append(o)
        refs_l.append(l)
    return np.concatenate(rows), np.concatenate(refs_o), np.concatenate(refs_l)


def test_chunked_prefill_full_config_sampled():
    case = inputs.chunked_prefill(seed=0)
    out, lse = run_prefill(case)
    rows, ref_o, ref_l = _sampled_prefill_oracle(case, 12)
    check(out[rows], lse[rows], ref_o, ref_l, "chunked prefill B=8 Lq=512")
    assert np.isfinite(out).all()


def test_chunked_prefill_full_config_every_row():
    """The whole chunked-prefill workload (B=8, 512-token chunks after priors ~ U[0, 4096],
    Hq=32, Hk=8, D=128, P=16), every output row against the oracle."""
    case = inputs.chunked_prefill(seed=3)
    out, lse = run_prefill(case)
    ref_o, ref_l = oracle_prefill(case)
    check(out, lse, ref_o, ref_l, "chunked prefill, every row")


def _scaled_v_case(scale_v, seed, D=128):
    """The same chunked-prefill inputs with V multiplied by a power of two (exact in bf16)."""
    case = inputs.make_prefill_case(3, 32, 8, D, 16, [0, 300, 900], [77, 256, 160], seed=seed)
    kv = case.kv
    v = (kv.v_pages.float() * scale_v).to(torch.bfloat16)
    kv2 = inputs.PagedKV(kv.k_pages, v, kv.page_table, kv.seq_lens, kv.page_size)
    return case, inputs.PrefillCase(case.q, case.cu_q, kv2, case.Hq, case.Hk, case.head_dim,
                                    case.scale, case.seed, case.max_q_len)


@pytest.mark.parametrize("log2s", [-12, 12, 14, 20])
def test_prefill_v_scale_covariance(log2s):
    """O is linear in V: out(V 2^s) / 2^s must match the oracle on V.  2^-12 pushes most
    values into the f16 subnormal range, 2^12 keeps them under 2^16, and 2^14 / 2^20 put
    some (or all) V tiles beyond the f16 range, where the kernel keeps those tiles bf16."""
    s = 2.0 ** log2s
    base, case = _scaled_v_case(s, seed=11 + log2s)
    ref_o, ref_l = oracle_prefill(base)
    out, lse = run_prefill(case)
    check(out / s, lse, ref_o, ref_l, f"V x 2^{log2s}")


@pytest.mark.parametrize("log2s", [-12, 20])
def test_prefill_v_scale_covariance_head_dim_64(log2s):
    s = 2.0 ** log2s
    base, case = _scaled_v_case(s, seed=31 + log2s, D=64)
    ref_o, ref_l = oracle_prefill(base)
    out, lse = run_prefill(case)
    check(out / s, lse, ref_o, ref_l, f"D=64 V x 2^{log2s}")
