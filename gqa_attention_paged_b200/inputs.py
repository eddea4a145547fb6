"""Seeded synthetic inputs for paged GQA attention.

This module only MAKES inputs: random q/k/v, a shuffled page pool, page tables and
sequence lengths, and (for the fp8 KV variant) the e4m3 codes and per-(page, kv head)
scales a cache writer would have stored.  It holds none of the attention arithmetic, so
both the CUDA path and the CPU oracle can consume the same tensors.

Recipe (the workloads the pages describe, synthesised):
  - q, k, v ~ N(0, 1) drawn in fp32 from torch.Generator(seed) on the CPU, rounded to
    bf16.  Optional outliers: each k/v element is independently replaced, with
    probability `outlier_p`, by +-`outlier_mag` (random sign).
  - Physical pages: a random permutation of the pool; sequence b takes its logical pages
    in order from that permutation.  The pool holds ceil(used / (1 - unused_frac))
    pages, so about `unused_frac` of it is never referenced.
  - Poison: unused pool pages, the tail slots of each sequence's last page, and page
    table entries past the end of a sequence (which point at unused pages when there are
    any) are filled with NaN so that a kernel reading them shows it in its output.
  - fp8 e4m3 variant: per (page, kv head) block, scale = absmax / 448 over the block's
    valid tokens (1.0 if the block is all zero), code = round-to-nearest-even of
    x / scale (torch's float8_e4m3fn cast), clamped to +-448 first.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

E4M3_MAX = 448.0
BF16_NAN_BITS = 0x7FC0
E4M3_NAN_BITS = 0x7F


@dataclass
class PagedKV:
    """A page pool and page tables for B sequences."""
    k_pages: torch.Tensor            # [num_pages][Hk][P][D] bf16, or uint8 e4m3 codes
    v_pages: torch.Tensor
    page_table: torch.Tensor         # int32 [B][pt_stride]
    seq_lens: torch.Tensor           # int32 [B]
    page_size: int
    k_scale: Optional[torch.Tensor] = None   # fp32 [num_pages][Hk] (fp8 only)
    v_scale: Optional[torch.Tensor] = None
    # bf16 pools holding the unquantised values (fp8 variant only)
    k_pages_bf16: Optional[torch.Tensor] = None
    v_pages_bf16: Optional[torch.Tensor] = None
    # contiguous per-sequence copies [sum L][Hk][D] (fp32 holding exact bf16 values)
    k_dense: Optional[torch.Tensor] = None
    v_dense: Optional[torch.Tensor] = None
    cu_kv: Optional[torch.Tensor] = None     # int64 [B+1]

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def kv_dtype(self) -> str:
        return "fp8_e4m3" if self.k_scale is not None else "bf16"


@dataclass
class DecodeCase:
    q: torch.Tensor                  # bf16 [B][Hq][D]
    kv: PagedKV
    Hq: int
    Hk: int
    head_dim: int
    scale: float
    seed: int
    name: str = ""


@dataclass
class PrefillCase:
    q: torch.Tensor                  # bf16 [total_q][Hq][D]
    cu_q: torch.Tensor               # int32 [B+1]
    kv: PagedKV
    Hq: int
    Hk: int
    head_dim: int
    scale: float
    seed: int
    max_q_len: int = 0
    name: str = ""


def _randn(gen, shape, outlier_p=0.0, outlier_mag=8.0):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if outlier_p > 0:
        hit = torch.rand(shape, generator=gen) < outlier_p
        sign = torch.where(torch.rand(shape, generator=gen) < 0.5, -1.0, 1.0)
        x = torch.where(hit, sign * outlier_mag, x)
    return x.to(torch.bfloat16)


def make_paged_kv(seq_lens: Sequence[int], Hk: int, D: int, P: int, gen: torch.Generator,
                  unused_frac: float = 0.25, pool_pages: Optional[int] = None,
                  pt_stride: Optional[int] = None, kv_dtype: str = "bf16",
                  outlier_p: float = 0.0, keep_dense: bool = False, poison: bool = True,
                  alias_prefix: Optional[Sequence[int]] = None) -> PagedKV:
    """Build a shuffled page pool holding len(seq_lens) sequences.

    alias_prefix[b] (optional) = number of leading pages sequence b shares with
    sequence 0 (prefix sharing: the same physical pages, and so the same K/V).
    """
    B = len(seq_lens)
    L = [int(x) for x in seq_lens]
    npg = [(l + P - 1) // P for l in L]
    alias = [0] * B if alias_prefix is None else [int(a) for a in alias_prefix]
    for b in range(B):
        assert 0 <= alias[b] <= min(npg[b], npg[0]) and (b > 0 or alias[b] == 0)
        if alias[b]:
            assert L[0] >= alias[b] * P, "shared prefix pages must be full in sequence 0"
    own = [npg[b] - alias[b] for b in range(B)]
    used = sum(own)
    if pool_pages is None:
        pool_pages = max(1, math.ceil(used / (1.0 - unused_frac))) if used else 1
    assert pool_pages >= used
    if pt_stride is None:
        pt_stride = max(1, max(npg) if npg else 1)
    assert pt_stride >= max(npg + [0])

    perm = torch.randperm(pool_pages, generator=gen).to(torch.int32)
    unused = perm[used:]
    poison_page = int(unused[0]) if len(unused) else 0
    table = torch.full((B, pt_stride), poison_page, dtype=torch.int32)
    off = 0
    for b in range(B):
        if alias[b]:
            table[b, :alias[b]] = table[0, :alias[b]]
        table[b, alias[b]:npg[b]] = perm[off:off + own[b]]
        off += own[b]

    # K/V of the pages each sequence owns, drawn token by token: [own_pages*P][Hk][D]
    kpool = torch.full((pool_pages, Hk, P, D), float("nan"), dtype=torch.bfloat16)
    vpool = torch.full((pool_pages, Hk, P, D), float("nan"), dtype=torch.bfloat16)
    if not poison:
        kpool.zero_()
        vpool.zero_()
    if used:
        kt = _randn(gen, (used * P, Hk, D), outlier_p)
        vt = _randn(gen, (used * P, Hk, D), outlier_p)
        # tail slots past each sequence's end are poison
        tok_off = 0
        for b in range(B):
            start = alias[b] * P
            end_valid = L[b]
            n_own_tok = own[b] * P
            first_tail = end_valid - start  # index within this sequence's own tokens
            if poison and own[b] > 0 and first_tail < n_own_tok:
                kt[tok_off + first_tail: tok_off + n_own_tok] = float("nan")
                vt[tok_off + first_tail: tok_off + n_own_tok] = float("nan")
            tok_off += n_own_tok
        ids = perm[:used].long()
        kpool[ids] = kt.view(used, P, Hk, D).permute(0, 2, 1, 3)
        vpool[ids] = vt.view(used, P, Hk, D).permute(0, 2, 1, 3)

    kv = PagedKV(kpool, vpool, table, torch.tensor(L, dtype=torch.int32), P)
    if keep_dense:
        kv.k_dense, kv.v_dense, kv.cu_kv = dense_copy(kv)
    if kv_dtype == "fp8_e4m3":
        kv.k_pages_bf16, kv.v_pages_bf16 = kpool, vpool
        valid = valid_slot_mask(table, kv.seq_lens, pool_pages, P)
        kv.k_pages, kv.k_scale = quantize_e4m3(kpool, valid)
        kv.v_pages, kv.v_scale = quantize_e4m3(vpool, valid)
    elif kv_dtype != "bf16":
        raise ValueError(kv_dtype)
    return kv


def valid_slot_mask(table, seq_lens, pool_pages, P):
    """bool [pool_pages][P]: slot holds a token of some sequence."""
    m = torch.zeros(pool_pages, P, dtype=torch.bool)
    for b in range(table.shape[0]):
        Lb = int(seq_lens[b])
        for p in range((Lb + P - 1) // P):
            n = min(P, Lb - p * P)
            m[int(table[b, p]), :n] = True
    return m


def quantize_e4m3(pool_bf16: torch.Tensor, valid: torch.Tensor):
    """Per-(page, kv head) absmax e4m3 codes.  Invalid slots get the NaN code."""
    x = pool_bf16.float()
    vmask = valid[:, None, :, None].expand_as(x)
    absmax = torch.where(vmask, x.abs(), torch.zeros_like(x)).amax(dim=(2, 3))
    scale = torch.where(absmax > 0, absmax / E4M3_MAX, torch.ones_like(absmax))
    y = (x / scale[:, :, None, None]).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    codes = torch.where(vmask, codes, torch.full_like(codes, E4M3_NAN_BITS))
    return codes.contiguous(), scale.to(torch.float32).contiguous()


def dense_copy(kv: PagedKV):
    """Contiguous [sum L][Hk][D] fp32 copies of the pool's (bf16) contents, built by
    direct indexing of the generated pool (input bookkeeping for the brute-force check)."""
    P = kv.page_size
    pool_k = kv.k_pages_bf16 if kv.k_pages_bf16 is not None else kv.k_pages
    pool_v = kv.v_pages_bf16 if kv.v_pages_bf16 is not None else kv.v_pages
    ks, vs = [], []
    for b in range(kv.page_table.shape[0]):
        Lb = int(kv.seq_lens[b])
        t = torch.arange(Lb)
        phys = kv.page_table[b, (t // P)].long()
        ks.append(pool_k[phys, :, t % P, :].float())
        vs.append(pool_v[phys, :, t % P, :].float())
    cu = torch.zeros(len(ks) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(kv.seq_lens.to(torch.int64), 0)
    Hk, D = pool_k.shape[1], pool_k.shape[3]
    k = torch.cat(ks) if ks else torch.zeros(0, Hk, D)
    v = torch.cat(vs) if vs else torch.zeros(0, Hk, D)
    return k, v, cu


def make_decode_case(B: int, Hq: int, Hk: int, D: int, P: int, seq_lens: Sequence[int],
                     seed: int = 0, scale: Optional[float] = None, kv_dtype: str = "bf16",
                     outlier_p: float = 0.0, unused_frac: float = 0.25,
                     pool_pages: Optional[int] = None, pt_stride: Optional[int] = None,
                     keep_dense: bool = False, name: str = "",
                     alias_prefix: Optional[Sequence[int]] = None) -> DecodeCase:
    assert len(seq_lens) == B
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, Hq, D))
    kv = make_paged_kv(seq_lens, Hk, D, P, gen, unused_frac=unused_frac, pool_pages=pool_pages,
                       pt_stride=pt_stride, kv_dtype=kv_dtype, outlier_p=outlier_p,
                       keep_dense=keep_dense, alias_prefix=alias_prefix)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return DecodeCase(q, kv, Hq, Hk, D, float(scale), seed, name)


def make_prefill_case(B: int, Hq: int, Hk: int, D: int, P: int, prior_lens: Sequence[int],
                      q_lens: Sequence[int], seed: int = 0, scale: Optional[float] = None,
                      unused_frac: float = 0.25, keep_dense: bool = False,
                      name: str = "") -> PrefillCase:
    assert len(prior_lens) == B and len(q_lens) == B
    gen = torch.Generator().manual_seed(seed)
    total_q = int(sum(q_lens))
    q = _randn(gen, (total_q, Hq, D))
    seq_lens = [int(a) + int(b) for a, b in zip(prior_lens, q_lens)]
    kv = make_paged_kv(seq_lens, Hk, D, P, gen, unused_frac=unused_frac, keep_dense=keep_dense)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor([int(x) for x in q_lens], dtype=torch.int32), 0)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return PrefillCase(q, cu, kv, Hq, Hk, D, float(scale), seed,
                       max(int(x) for x in q_lens) if B else 0, name)


def uniform_lens(B: int, lo: int, hi: int, seed: int) -> List[int]:
    """B integers uniform in [lo, hi], drawn from their own generator."""
    g = torch.Generator().manual_seed(seed + 7919)
    return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g)]


# ---------------------------------------------------------------------------------
# Named workloads (the five configurations of the hot path).
# ---------------------------------------------------------------------------------

def tiny_decode(seed: int = 0, **kw) -> DecodeCase:
    """B=2, Hq=8, Hk=2, D=64, L={37,100}, P=16, pool of 16 pages (10 used)."""
    return make_decode_case(2, 8, 2, 64, 16, [37, 100], seed=seed, pool_pages=16,
                            scale=1.0 / 8.0, name="tiny_decode", **kw)


def llama7b_decode(seed: int = 0, B: int = 16, **kw) -> DecodeCase:
    """Llama-2-7B-GQA-shaped decode: Hq=32, Hk=8, D=128, L ~ U[512, 2048], P=16, 25% of
    the pool unused."""
    return make_decode_case(B, 32, 8, 128, 16, uniform_lens(B, 512, 2048, seed), seed=seed,
                            unused_frac=0.25, pt_stride=128, name="llama7b_decode", **kw)


def sweep_decode(B: int, seed: int = 0, ctx: int = 2048, **kw) -> DecodeCase:
    """Batch sweep point: Hq=32, Hk=8, D=128, every context 2048, P=16."""
    return make_decode_case(B, 32, 8, 128, 16, [ctx] * B, seed=seed,
                            name=f"sweep_decode_B{B}", **kw)


def long70b_decode(seed: int = 0, kv_dtype: str = "bf16", **kw) -> DecodeCase:
    """70B-shaped long-context decode: B=4, Hq=64, Hk=8, D=128, L={8K,16K,24K,32K},
    P=64, k/v with 1% outliers at 8 sigma."""
    return make_decode_case(4, 64, 8, 128, 64, [8192, 16384, 24576, 32768], seed=seed,
                            kv_dtype=kv_dtype, outlier_p=0.01, name=f"long70b_decode_{kv_dtype}",
                            **kw)


def chunked_prefill(seed: int = 0, B: int = 8, q_len: int = 512, **kw) -> PrefillCase:
    """Causal chunked prefill: B=8, Hq=32, Hk=8, D=128, 512 new tokens after a prior
    context ~ U[0, 4096], P=16."""
    prior = uniform_lens(B, 0, 4096, seed)
    return make_prefill_case(B, 32, 8, 128, 16, prior, [q_len] * B, seed=seed,
                             name="chunked_prefill", **kw)
