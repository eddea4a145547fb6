"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these compare the oracle with itself: each checks it against a closed form, a
library routine, an exact invariant the pages state, or an independent dense numpy
brute force on contiguous (unpaged) data.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import inputs
from oracle import bruteforce, oracle
from tests._util import bits, np32, oracle_decode, oracle_prefill

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- decoders

def test_bf16_decoder_matches_torch_on_all_patterns():
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(pats)
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decoder_matches_torch_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decoder_golden_codes():
    for code, expr in _load("e4m3_codes.json")["codes"]:
        v = oracle.e4m3_to_f64(np.array([int(code, 16)], np.uint8))[0]
        if expr == "nan":
            assert math.isnan(v), code
        else:
            want = eval(expr, {"__builtins__": {}})
            assert v == want and math.copysign(1, v) == math.copysign(1, want), (code, v, want)


def test_e4m3_round_trip_and_saturation():
    """Representable values survive quantisation exactly; saturation at +-448."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_to_f64(codes)
    back = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    back = back.numpy()
    same = (back == codes) | ((vals == 0) & ((back & 0x7F) == 0))
    assert same.all()
    # the input generator clamps to +-448 before the cast: quantising 10 * absmax-block
    pool = torch.tensor([[[[1000.0, -1000.0, 3.0, 0.0]]]], dtype=torch.bfloat16)
    valid = torch.tensor([[True]])
    c, s = inputs.quantize_e4m3(pool, valid)
    deq = oracle.e4m3_to_f64(c.numpy()) * s.numpy()[:, :, None, None]
    assert deq[0, 0, 0, 0] == pytest.approx(1000.0) and deq[0, 0, 0, 1] == pytest.approx(-1000.0)


# --------------------------------------------------------------------------- closed forms

def _pool_from_dense(k, v, P=16):
    """Single-sequence page pool: k,v [L][Hk][D] floats -> bf16 pool with identity table."""
    L, Hk, D = k.shape
    npg = (L + P - 1) // P
    kp = torch.zeros(npg, Hk, P, D)
    vp = torch.zeros(npg, Hk, P, D)
    for t in range(L):
        kp[t // P, :, t % P] = torch.tensor(k[t])
        vp[t // P, :, t % P] = torch.tensor(v[t])
    table = np.arange(npg, dtype=np.int32)[None]
    return bits(kp.bfloat16()), bits(vp.bfloat16()), table, np.array([L], np.int32)


@pytest.mark.parametrize("case", _load("closed_form_attention.json")["cases"],
                         ids=lambda c: c["name"])
def test_closed_form_golden(case):
    q = torch.tensor(case["q"], dtype=torch.float32)[None].bfloat16()  # [1][Hq][D]
    k = np.array(case["k"], np.float64)
    v = np.array(case["v"], np.float64)
    kp, vp, table, lens = _pool_from_dense(k, v)
    out, lse = oracle.decode(bits(q), kp, vp, table, lens, case["scale"])
    env = {"e": math.e, "log": math.log, "__builtins__": {}}
    want_o = np.array([[eval(x, env) for x in row] for row in case["expect_o"]])
    want_l = np.array([eval(x, env) for x in case["expect_lse"]])
    np.testing.assert_allclose(out[0], want_o, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0], want_l, rtol=1e-14, atol=1e-15)


def test_equal_keys_give_mean_of_values():
    """All keys equal -> uniform weights -> o = mean_t V_t; scale 0 likewise."""
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [1, 29, 70], seed=3, keep_dense=True)
    kv = case.kv
    kp = kv.k_pages.clone()
    kp[:] = kv.k_pages[int(kv.page_table[0, 0]), 0, 0]  # one key vector in every slot
    out, lse = oracle.decode(bits(case.q), bits(kp), bits(kv.v_pages), kv.page_table.numpy(),
                             kv.seq_lens.numpy(), case.scale)
    out0, lse0 = oracle.decode(bits(case.q), bits(kv.k_pages), bits(kv.v_pages),
                               kv.page_table.numpy(), kv.seq_lens.numpy(), 0.0)
    g = case.Hq // case.Hk
    for b in range(3):
        lo, hi = int(kv.cu_kv[b]), int(kv.cu_kv[b + 1])
        mean = kv.v_dense[lo:hi].double().mean(0).numpy()  # [Hk][D]
        want = np.repeat(mean, g, axis=0)
        np.testing.assert_allclose(out[b], want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out0[b], want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse0[b], math.log(hi - lo), rtol=1e-14)


def test_one_hot_values_give_the_softmax_column():
    """V[t] = e_t (L <= D): o[t] is the weight of token t; weights sum to 1 and follow
    the scores' order, with ratio exp(s_t - s_u) between tokens t and u."""
    L, D = 23, 64
    gen = torch.Generator().manual_seed(11)
    q = torch.randn(1, 1, D, generator=gen).bfloat16()
    k = torch.randn(L, 1, D, generator=gen).bfloat16().double().numpy()
    v = np.zeros((L, 1, D))
    for t in range(L):
        v[t, 0, t] = 1.0
    kp, vp, table, lens = _pool_from_dense(k, v)
    out, lse = oracle.decode(bits(q), kp, vp, table, lens, 0.125)
    p = out[0, 0, :L]
    assert abs(p.sum() - 1.0) < 1e-14 and np.all(out[0, 0, L:] == 0)
    s = 0.125 * (k[:, 0, :] @ q.double().numpy()[0, 0])
    np.testing.assert_allclose(np.log(p[1:] / p[0]), s[1:] - s[0], rtol=1e-11, atol=1e-12)
    assert np.argmax(p) == np.argmax(s)
    np.testing.assert_allclose(lse[0, 0], s[0] - np.log(p[0]), rtol=1e-13)


def test_empty_sequence():
    case = inputs.make_decode_case(3, 4, 2, 64, 16, [0, 5, 0], seed=1)
    out, lse = oracle_decode(case)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    assert np.all(np.isfinite(out[1]))


# --------------------------------------------------------------------------- invariants

def _mha_from_gqa(case):
    """repeat_kv: a pool with Hq kv heads, kv head h holding the data of GQA kv head h/g."""
    g = case.Hq // case.Hk
    kv = case.kv
    kp = kv.k_pages.repeat_interleave(g, dim=1)
    vp = kv.v_pages.repeat_interleave(g, dim=1)
    return kp, vp


@pytest.mark.parametrize("Hq,Hk", [(8, 2), (32, 8), (12, 3), (4, 1)])
def test_gqa_equals_mha_after_repeat_kv(Hq, Hk):
    case = inputs.make_decode_case(3, Hq, Hk, 64, 16, [17, 64, 90], seed=Hq + Hk)
    out, lse = oracle_decode(case)
    kp, vp = _mha_from_gqa(case)
    out2, lse2 = oracle.decode(bits(case.q), bits(kp), bits(vp), case.kv.page_table.numpy(),
                               case.kv.seq_lens.numpy(), case.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_mha_and_mqa_special_cases_against_brute_force():
    for Hq, Hk in [(4, 4), (4, 1)]:
        case = inputs.make_decode_case(2, Hq, Hk, 64, 16, [33, 48], seed=5, keep_dense=True)
        out, lse = oracle_decode(case)
        _check_against_dense(case, out, lse)


@pytest.mark.parametrize("S", [1, 2, 3, 4, 7, 64])
def test_split_merge_equals_unsplit(S):
    case = inputs.make_decode_case(4, 8, 2, 64, 16, [1, 37, 100, 260], seed=S)
    out, lse = oracle_decode(case)
    op, lp = oracle_decode(case, num_splits=S)
    B, Hq, D = out.shape
    mo, ml = oracle.lse_combine(op.reshape(S, B * Hq, D), lp.reshape(S, B * Hq))
    np.testing.assert_allclose(mo.reshape(B, Hq, D), out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ml.reshape(B, Hq), lse, rtol=1e-13, atol=1e-13)
    # split s covers pages [s*c, (s+1)*c) with c = ceil(np/S): empty splits carry -inf
    for b, L in enumerate([1, 37, 100, 260]):
        npg = (L + 15) // 16
        c = (npg + S - 1) // S
        for s in range(S):
            assert np.isneginf(lp[s, b]).all() == (s * c >= npg)


def test_lse_combine_all_empty_rows():
    o = np.random.default_rng(0).normal(size=(3, 5, 8))
    l = np.full((3, 5), -np.inf)
    l[1, 2] = 0.5
    out, lse = oracle.lse_combine(o, l)
    assert np.all(out[[0, 1, 3, 4]] == 0) and np.all(np.isneginf(lse[[0, 1, 3, 4]]))
    np.testing.assert_allclose(out[2], o[1, 2], rtol=1e-15)
    assert lse[2] == 0.5


def test_lse_combine_leaves_out_empty_splits():
    """An empty split (lse = -inf) carries no tokens: whatever its partial holds (even
    NaN), the merge equals the merge of the other splits."""
    rng = np.random.default_rng(1)
    o = rng.normal(size=(3, 4, 8))
    l = rng.normal(size=(3, 4))
    ref, ref_l = oracle.lse_combine(o[[0, 2]], l[[0, 2]])
    o2 = o.copy()
    l2 = l.copy()
    l2[1] = -np.inf
    o2[1] = np.nan
    out, lse = oracle.lse_combine(o2, l2)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(lse, ref_l)


def test_physical_page_permutation_invariance():
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [40, 77, 128], seed=9)
    out, lse = oracle_decode(case)
    kv = case.kv
    perm = torch.randperm(kv.num_pages, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(perm)
    kp = kv.k_pages[perm]          # new page i holds old page perm[i]
    vp = kv.v_pages[perm]
    table = inv[kv.page_table.long()].to(torch.int32)  # old page j now lives at inv[j]
    out2, lse2 = oracle.decode(bits(case.q), bits(kp), bits(vp), table.numpy(),
                               kv.seq_lens.numpy(), case.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_shared_prefix_pages_equal_private_copies():
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [96, 70, 50], seed=4, alias_prefix=[0, 3, 2])
    kv = case.kv
    assert (kv.page_table[1, :3] == kv.page_table[0, :3]).all()
    out, lse = oracle_decode(case)
    # de-alias: give every referenced (b, p) its own copy of the page
    npg = [(int(L) + 15) // 16 for L in kv.seq_lens]
    n = sum(npg)
    kp = torch.empty(n, *kv.k_pages.shape[1:], dtype=kv.k_pages.dtype)
    vp = torch.empty_like(kp)
    table = torch.zeros_like(kv.page_table)
    i = 0
    for b in range(3):
        for p in range(npg[b]):
            kp[i] = kv.k_pages[int(kv.page_table[b, p])]
            vp[i] = kv.v_pages[int(kv.page_table[b, p])]
            table[b, p] = i
            i += 1
    out2, lse2 = oracle.decode(bits(case.q), bits(kp), bits(vp), table.numpy(),
                               kv.seq_lens.numpy(), case.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


# --------------------------------------------------------------------------- brute force

def _check_against_dense(case, out, lse, rtol=1e-11, atol=1e-12):
    kv = case.kv
    g = case.Hq // case.Hk
    for b in range(case.q.shape[0]):
        lo, hi = int(kv.cu_kv[b]), int(kv.cu_kv[b + 1])
        if hi == lo:
            continue
        q = case.q[b:b + 1].double().numpy()
        o, l = bruteforce.attention_dense(q, kv.k_dense[lo:hi].double().numpy(),
                                          kv.v_dense[lo:hi].double().numpy(), case.scale)
        np.testing.assert_allclose(out[b], o[0], rtol=rtol, atol=atol)
        np.testing.assert_allclose(lse[b], l[0], rtol=rtol, atol=atol)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_against_dense_brute_force(seed):
    case = inputs.tiny_decode(seed=seed, keep_dense=True)
    out, lse = oracle_decode(case)
    _check_against_dense(case, out, lse)


def test_ragged_decode_p32_p64_against_dense_brute_force():
    for P in (32, 64):
        case = inputs.make_decode_case(4, 12, 4, 128, P, [1, 63, 64, 200], seed=P,
                                       keep_dense=True)
        out, lse = oracle_decode(case)
        _check_against_dense(case, out, lse)


def test_fp8_decode_against_dense_dequantised_brute_force():
    case = inputs.make_decode_case(2, 8, 2, 128, 64, [100, 300], seed=2, kv_dtype="fp8_e4m3",
                                   outlier_p=0.01)
    kv = case.kv
    out, lse = oracle_decode(case)
    # dense dequantised copies, built from the codes by the library decoder (torch)
    deqk = kv.k_pages.view(torch.float8_e4m3fn).double() * kv.k_scale.double()[:, :, None, None]
    deqv = kv.v_pages.view(torch.float8_e4m3fn).double() * kv.v_scale.double()[:, :, None, None]
    for b in range(2):
        L = int(kv.seq_lens[b])
        t = torch.arange(L)
        phys = kv.page_table[b, t // 64].long()
        k = deqk[phys, :, t % 64, :].numpy()
        v = deqv[phys, :, t % 64, :].numpy()
        o, l = bruteforce.attention_dense(case.q[b:b + 1].double().numpy(), k, v, case.scale)
        np.testing.assert_allclose(out[b], o[0], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[b], l[0], rtol=1e-11, atol=1e-12)
    # and the quantised result stays near the unquantised bf16 one
    ref, _ = oracle_decode(case, use_bf16_pool=True)
    assert np.max(np.abs(out - ref)) < 0.1


def test_prefill_against_dense_causal_brute_force():
    case = inputs.make_prefill_case(3, 8, 2, 64, 16, [0, 20, 45], [17, 1, 40], seed=6,
                                    keep_dense=True)
    out, lse = oracle_prefill(case)
    kv = case.kv
    for b in range(3):
        lo, hi = int(kv.cu_kv[b]), int(kv.cu_kv[b + 1])
        q0, q1 = int(case.cu_q[b]), int(case.cu_q[b + 1])
        L, Lq = hi - lo, q1 - q0
        pos = np.arange(L - Lq, L)
        o, l = bruteforce.attention_dense(case.q[q0:q1].double().numpy(),
                                          kv.k_dense[lo:hi].double().numpy(),
                                          kv.v_dense[lo:hi].double().numpy(), case.scale, pos)
        np.testing.assert_allclose(out[q0:q1], o, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[q0:q1], l, rtol=1e-11, atol=1e-12)
    # non-causal: every row sees all L keys
    outn, _ = oracle_prefill(case, causal=False)
    b = 1
    lo, hi = int(kv.cu_kv[b]), int(kv.cu_kv[b + 1])
    q0, q1 = int(case.cu_q[b]), int(case.cu_q[b + 1])
    o, _ = bruteforce.attention_dense(case.q[q0:q1].double().numpy(),
                                      kv.k_dense[lo:hi].double().numpy(),
                                      kv.v_dense[lo:hi].double().numpy(), case.scale)
    np.testing.assert_allclose(outn[q0:q1], o, rtol=1e-11, atol=1e-12)


def test_prefill_last_row_equals_decode():
    """The chunk's last row sits at position L-1 and sees the whole sequence: exactly a
    decode step of that token."""
    case = inputs.make_prefill_case(3, 8, 2, 64, 16, [5, 33, 100], [4, 16, 9], seed=8)
    out, lse = oracle_prefill(case)
    last = (case.cu_q[1:] - 1).long()
    dcase = inputs.DecodeCase(case.q[last], case.kv, case.Hq, case.Hk, case.head_dim, case.scale,
                              case.seed)
    dout, dlse = oracle_decode(dcase)
    assert np.array_equal(out[last.numpy()], dout) and np.array_equal(lse[last.numpy()], dlse)


# --------------------------------------------------------------------------- gather

def test_gather_copies_tokens_in_logical_order():
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [37, 16, 90], seed=12, keep_dense=True)
    kv = case.kv
    ko, vo = oracle.gather(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                           kv.seq_lens.numpy())
    assert np.array_equal(ko, bits(kv.k_dense.bfloat16()))
    assert np.array_equal(vo, bits(kv.v_dense.bfloat16()))
    assert not np.isnan(kv.k_dense.numpy()).any()  # no poison slot was copied


def test_kv_bytes_model_matches_the_pages_figure():
    """32 query heads in 8 groups: KV bytes are 1/4 of MHA's (75% less)."""
    import bench
    fx = _load("kv_bytes_gqa.json")
    gqa = bench.decode_kv_bytes([2048] * 4, Hk=fx["Hk"], D=128, elem=2)
    mha = bench.decode_kv_bytes([2048] * 4, Hk=fx["Hq"], D=128, elem=2)
    assert gqa / mha == fx["kv_bytes_ratio_gqa_over_mha"]
    assert 1 - gqa / mha == fx["kv_reduction"]


def test_fp8_quantisation_error_sets_the_fp8_bound():
    """On the 70B-shaped long-context workload (1% outliers at 8 sigma), exact fp64
    attention over the dequantised e4m3 cache differs from attention over the unquantised
    values by ~2e-2: below the 5e-2 max-|err| bound adopted for the fp8 path, and above
    2e-3 + 5e-2|ref| in some elements, so that per-element form cannot be met by any
    implementation and is not the gate."""
    case = inputs.long70b_decode(seed=0, kv_dtype="fp8_e4m3")
    deq, _ = oracle_decode(case)
    ref, _ = oracle_decode(case, use_bf16_pool=True)
    d = np.abs(deq - ref)
    assert 5e-3 < d.max() <= 5e-2
    assert (d > 2e-3 + 5e-2 * np.abs(ref)).any()
