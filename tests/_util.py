"""Helpers shared by the tests: turn seeded input cases into the raw bit-pattern numpy
arrays the CPU oracle reads, and compare results."""
import numpy as np
import torch

from oracle import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a CPU tensor: bf16 -> uint16, e4m3/uint8 -> uint8."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return t.view(torch.uint8).numpy()
    raise TypeError(t.dtype)


def np32(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float32)


def oracle_decode(case, num_splits=0, use_bf16_pool=False):
    kv = case.kv
    if use_bf16_pool:
        kp, vp, ks, vs = kv.k_pages_bf16, kv.v_pages_bf16, None, None
    else:
        kp, vp, ks, vs = kv.k_pages, kv.v_pages, kv.k_scale, kv.v_scale
    return oracle.decode(bits(case.q), bits(kp), bits(vp), kv.page_table.numpy(),
                         kv.seq_lens.numpy(), case.scale, np32(ks), np32(vs), num_splits)


def oracle_prefill(case, causal=True):
    kv = case.kv
    return oracle.prefill(bits(case.q), case.cu_q.numpy(), bits(kv.k_pages), bits(kv.v_pages),
                          kv.page_table.numpy(), kv.seq_lens.numpy(), case.scale, causal)


def bf16_tol_ok(got, ref, atol=2e-3, rtol=1e-2):
    """Element-wise |got - ref| <= atol + rtol*|ref| (NaN anywhere fails)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bad = ~(np.abs(got - ref) <= atol + rtol * np.abs(ref))
    return not bad.any(), bad


def err_report(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(got - ref)
    return (f"max_abs={np.nanmax(d) if d.size else 0:.3e} "
            f"max_rel={np.nanmax(d / np.maximum(np.abs(ref), 1e-30)) if d.size else 0:.3e} "
            f"nan={int(np.isnan(got).sum())}")
