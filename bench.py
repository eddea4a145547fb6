"""Benchmark of paged GQA decode on B200 (placeholder: byte model only)."""


def decode_kv_bytes(seq_lens, Hk, D, elem):
    """Algorithmic K+V bytes of one decode step: every valid token's K and V row of every
    kv head, read once."""
    return 2 * sum(int(L) for L in seq_lens) * Hk * D * elem
