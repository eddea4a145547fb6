"""Dense numpy fp64 brute force, used only to cross-check the C oracle on tiny shapes.

TEST INFRASTRUCTURE ONLY.  It works on CONTIGUOUS per-sequence K/V (never on pages),
materialises repeat_kv explicitly with np.repeat (the RepeatKVPlugin semantics of
"TensorRT对Grouped Query Attention的支持进展", section "图优化与算子融合"), and computes
softmax(q K^T * scale + mask) V as whole matrices, the decomposed MatMul -> Softmax ->
MatMul form of "TensorRT-LLM与TensorRT核心差异解析", section 4.1.
"""
import numpy as np


def repeat_kv(x, g):
    """[L][Hk][D] -> [L][Hk*g][D]: KV head j serves query heads j*g .. j*g+g-1."""
    return np.repeat(x, g, axis=1)


def attention_dense(q, k, v, scale, q_pos=None):
    """q [Lq][Hq][D], k/v [L][Hk][D] (fp64).  q_pos[i] = absolute position of query row i;
    when given, key t is visible to row i iff t <= q_pos[i].  Returns (o [Lq][Hq][D],
    lse [Lq][Hq])."""
    Lq, Hq, D = q.shape
    L, Hk, _ = k.shape
    kr = repeat_kv(k, Hq // Hk)  # [L][Hq][D]
    vr = repeat_kv(v, Hq // Hk)
    s = np.einsum("ihd,thd->hit", q, kr) * scale  # [Hq][Lq][L]
    if q_pos is not None:
        mask = np.arange(L)[None, :] > np.asarray(q_pos)[:, None]  # [Lq][L]
        s = np.where(mask[None], -np.inf, s)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    o = np.einsum("hit,thd->ihd", e / z, vr)
    lse = (m + np.log(z))[..., 0].T  # [Lq][Hq]
    return o, lse
