"""Decode of sequences whose KV pages are spread over several GPUs (one process per GPU).

A context too long for one device is cut across devices ("FasterTransformer source tour",
section 6.1); every rank holds a contiguous range of each sequence's logical pages, and a
decode step is:

  1. each rank: gqa_paged_decode_partial over the tokens it holds -> fp32 normalised
     o_part [B][Hq][D] and lse_part [B][Hq] (the kernels of the single-GPU decode);
  2. one exchange: every rank gathers every rank's (o_part, lse_part) -- (D + 1) * Hq * 4
     bytes per sequence per rank -- with torch.distributed all-gathers (NCCL over NVLink on
     GPUs) into local buffers;
  3. each rank: lse_combine over the R partials (the NumSplits log-sum-exp merge of
     "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", section
     "核心参数调优：PackGQA与NumSplits的协同舞蹈"), giving the full decode on every rank.

The partition is one page boundary for the whole batch: with C = ceil(max_pages / R) pages
per rank, rank r holds logical pages [r*C, (r+1)*C) of every sequence (a short sequence
simply has no tokens on the later ranks; its partials there are o = 0, lse = -inf, which
the merge leaves out).  The helpers below compute that partition and each rank's local
page-table rows and token counts on the host side of the tensors; every arithmetic step of
the attention runs in the library's kernels.  No peer memory is read directly: remote
partials arrive through the collective into this rank's buffers.
"""
from __future__ import annotations

import contextlib
from typing import Optional, Tuple

import torch

from . import binding


def rank_page_range(max_pages: int, world: int, rank: int) -> Tuple[int, int]:
    """Logical pages [p0, p1) rank `rank` of `world` holds: contiguous ranges of
    ceil(max_pages / world) pages (the last ranks may hold fewer, or none)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    per = -(-int(max_pages) // world) if max_pages > 0 else 0
    p0 = min(int(max_pages), rank * per)
    p1 = min(int(max_pages), (rank + 1) * per)
    return p0, p1


def local_seq_lens(seq_lens: torch.Tensor, page_size: int, p0: int, p1: int) -> torch.Tensor:
    """Tokens of each sequence that fall in logical pages [p0, p1):
    clamp(L - p0 * P, 0, (p1 - p0) * P)."""
    lo, cap = p0 * page_size, (p1 - p0) * page_size
    return (seq_lens.to(torch.int64) - lo).clamp(0, cap).to(torch.int32)


def local_page_table(page_table: torch.Tensor, p0: int, p1: int) -> torch.Tensor:
    """Columns [p0, p1) of a [B][pt_stride] page table, contiguous (at least one column,
    so the local table is never empty)."""
    if p1 <= p0:
        return page_table[:, :1].contiguous()
    return page_table[:, p0:p1].contiguous()


def exchange_partials(o_part: torch.Tensor, lse_part: torch.Tensor,
                      group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Gather every rank's partial result: returns (o_all [R][rows][D], lse_all [R][rows])
    in rank order, in buffers of this rank.  Two all-gathers into one contiguous
    allocation; every rank calls this with tensors of the same shape."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rows = lse_part.numel()
    D = o_part.numel() // max(rows, 1)
    buf = torch.empty(world * rows * (D + 1), dtype=torch.float32, device=o_part.device)
    o_all = buf[:world * rows * D]
    l_all = buf[world * rows * D:]
    dist.all_gather_into_tensor(o_all, o_part.reshape(-1).contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse_part.reshape(-1).contiguous(), group=group)
    return o_all.view(world, rows, D), l_all.view(world, rows)


def split_kv_decode(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                    page_table_local: torch.Tensor, seq_lens_local: torch.Tensor, scale: float,
                    group=None, k_scale: Optional[torch.Tensor] = None,
                    v_scale: Optional[torch.Tensor] = None, num_splits: int = 0,
                    workspace: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step of sequences spread over the ranks of `group`.  Every rank passes
    the same q [B][Hq][D] and its own pool, local page-table rows and local token counts
    (rank_page_range / local_page_table / local_seq_lens give them for the page-boundary
    partition).  Returns (out bf16 [B][Hq][D], lse fp32 [B][Hq]) on every rank.

    Everything is enqueued on `stream` (default: the current stream), which is made the
    current stream for the call so the collectives order themselves after the partial
    decode and before the merge."""
    B, Hq, D = q.shape
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        o_part, lse_part = binding.gqa_paged_decode_partial(
            q, k_pages, v_pages, page_table_local, seq_lens_local, scale,
            num_splits=num_splits, k_scale=k_scale, v_scale=v_scale, workspace=workspace)
        o_all, l_all = exchange_partials(o_part.view(B * Hq, D), lse_part.view(B * Hq), group)
        if out is None:
            out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
        binding.lse_combine(o_all, l_all, out=out.view(B * Hq, D), lse=lse.view(B * Hq))
    return out, lse
