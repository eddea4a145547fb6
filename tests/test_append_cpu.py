"""Pins of the oracle's KV append (oracle.append_kv) and of its e4m3 encoder, against
what the format and the plain definition fix, on the CPU.

- The encoder round-trips every finite e4m3 code and agrees bit for bit with torch's
  float8_e4m3fn cast (round to nearest even) on values inside +-448, exact midpoints
  included; values beyond +-448 saturate.
- bf16 append writes exactly the new token's bits at position L - 1 and nothing else.
- e4m3 append: a token opening a page sets the scale so that its largest element encodes
  as +-448; every stored value is within half an e4m3 step of x.
- The attention read through the appended cache equals dense attention with the new
  token placed last (brute force)."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import inputs
from oracle import bruteforce, oracle
from tests._util import bits


def _codes_finite():
    return [c for c in range(256) if (c & 0x7f) != 0x7f]


def test_encoder_round_trips_every_finite_code():
    codes = np.array(_codes_finite(), np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    assert np.array_equal(oracle.f32_to_e4m3(vals), codes)


def test_encoder_matches_torch_cast_with_midpoints():
    pos = np.sort(oracle.e4m3_to_f64(np.arange(0, 0x7f, dtype=np.uint8)))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)  # exact in fp32: ties to even
    rng = np.random.default_rng(0)
    rnd = (np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 4000)) *
           rng.choice([-1.0, 1.0], 4000)).astype(np.float32)
    x = np.concatenate([mids, -mids, rnd, np.float32([0.0, 2.0 ** -9, 2.0 ** -10, 447.9, -448.0])])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3(x), want)


def test_encoder_saturates():
    assert list(oracle.f32_to_e4m3(np.float32([449.0, 1e30, -5e5, np.inf, -np.inf]))) == \
        [0x7e, 0x7e, 0xfe, 0x7e, 0xfe]
    assert oracle.f32_to_e4m3(np.float32([np.nan]))[0] == 0x7f


def _new_tokens(B, Hk, D, seed):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Hk, D, generator=g) * 2).to(torch.bfloat16)
    v = (torch.randn(B, Hk, D, generator=g) * 2).to(torch.bfloat16)
    return k, v


def test_bf16_append_writes_only_the_new_token():
    case = inputs.make_decode_case(3, 8, 2, 64, 16, [17, 32, 1], seed=4)
    kv = case.kv
    kn, vn = _new_tokens(3, 2, 64, 1)
    kp0, vp0 = bits(kv.k_pages), bits(kv.v_pages)
    kp, vp, _, _ = oracle.append_kv(kp0, vp0, kv.page_table.numpy(), kv.seq_lens.numpy(),
                                    bits(kn), bits(vn))
    changed = np.zeros(kp.shape, bool)
    for b, L in enumerate(kv.seq_lens.tolist()):
        t = L - 1
        phys = int(kv.page_table[b, t // 16])
        assert np.array_equal(kp[phys, :, t % 16, :], bits(kn)[b])
        assert np.array_equal(vp[phys, :, t % 16, :], bits(vn)[b])
        changed[phys, :, t % 16, :] = True
    assert np.array_equal(kp[~changed], kp0[~changed]) and np.array_equal(vp[~changed], vp0[~changed])


def test_fp8_append_scale_and_codes():
    # lengths 17 and 33 open a page (token 16, 32 at slot 0); 20 lands mid-page
    case = inputs.make_decode_case(3, 8, 2, 128, 16, [17, 20, 33], seed=5, kv_dtype="fp8_e4m3")
    kv = case.kv
    kn, vn = _new_tokens(3, 2, 128, 2)
    ks0 = kv.k_scale.numpy().copy()
    kp, vp, ks, vs = oracle.append_kv(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                                      kv.seq_lens.numpy(), bits(kn), bits(vn),
                                      kv.k_scale.numpy(), kv.v_scale.numpy())
    x = kn.float().numpy()
    for b, L in enumerate(kv.seq_lens.tolist()):
        t = L - 1
        phys = int(kv.page_table[b, t // 16])
        for j in range(2):
            codes = kp[phys, j, t % 16]
            if t % 16 == 0:
                assert ks[phys, j] == np.float32(np.abs(x[b, j]).max()) / np.float32(448.0)
                top = int(np.argmax(np.abs(x[b, j])))
                assert codes[top] & 0x7f == 0x7e  # the largest element encodes as +-448
            else:
                assert ks[phys, j] == ks0[phys, j]  # a later token keeps the page's scale
            dq = oracle.e4m3_to_f64(codes) * ks[phys, j]
            inside = np.abs(x[b, j]) <= 448.0 * ks[phys, j]
            # inside the page's range: within half an e4m3 step (3 mantissa bits) or the
            # subnormal spacing; beyond it (a later token larger than the page's first):
            # saturated at +-448 * scale
            tol = np.maximum(np.abs(x[b, j]) * 2.0 ** -4, 2.0 ** -10 * ks[phys, j])
            assert np.all(np.abs(dq - x[b, j])[inside] <= tol[inside] * 1.0000001), (b, j)
            assert np.all(np.abs(dq[~inside]) == 448.0 * float(ks[phys, j])), (b, j)
            assert np.all(np.sign(dq[~inside]) == np.sign(x[b, j][~inside])), (b, j)


def test_decode_after_append_equals_dense_attention():
    case = inputs.make_decode_case(2, 8, 2, 64, 16, [9, 40], seed=6, keep_dense=True)
    kv = case.kv
    kn, vn = _new_tokens(2, 2, 64, 3)
    kp, vp, _, _ = oracle.append_kv(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                                    kv.seq_lens.numpy(), bits(kn), bits(vn))
    out, lse = oracle.decode(bits(case.q), kp, vp, kv.page_table.numpy(), kv.seq_lens.numpy(),
                             case.scale)
    cu = kv.cu_kv.tolist()
    for b, L in enumerate(kv.seq_lens.tolist()):
        k = kv.k_dense[cu[b]:cu[b + 1]].double().clone()
        v = kv.v_dense[cu[b]:cu[b + 1]].double().clone()
        k[L - 1] = kn[b].double()
        v[L - 1] = vn[b].double()
        o, l = bruteforce.attention_dense(case.q[b:b + 1].double().numpy(), k.numpy(), v.numpy(),
                                          case.scale)
        np.testing.assert_allclose(out[b], o[0], rtol=1e-12, atol=1e-12)
