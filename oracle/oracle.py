"""ctypes front end of the fp64 CPU oracle (gqa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py.  It never imports the CUDA package and the CUDA package never
imports it.  Inputs are numpy arrays holding raw bit patterns (bf16 as uint16, e4m3 as
uint8), so the oracle decodes every number itself.

Each function restates one operation of grouped-query attention over a paged KV cache;
the C source names the page and section each follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_P = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_bf16_to_f64.restype = ctypes.c_double
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_e4m3_to_f64.restype = ctypes.c_double
        L.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_gather.restype = None
        L.oracle_gather.argtypes = [_P, _P, _P, ctypes.c_int, _P, _P, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]
        dec = [_P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, ctypes.c_int,
               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
               ctypes.c_double]
        L.oracle_decode.restype = None
        L.oracle_decode.argtypes = dec + [_P, _P]
        L.oracle_decode_split.restype = None
        L.oracle_decode_split.argtypes = dec + [ctypes.c_int, _P, _P]
        L.oracle_lse_combine.restype = None
        L.oracle_lse_combine.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]
        L.oracle_prefill.restype = None
        L.oracle_prefill.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                     _P, _P]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.oracle_append_kv.restype = None
        L.oracle_append_kv.argtypes = [_P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _P, _P]
        L.oracle_kt_build.restype = None
        L.oracle_kt_build.argtypes = [_P, _P, ctypes.c_int, _P, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, _P]
        L.oracle_page_scores.restype = None
        L.oracle_page_scores.argtypes = [_P, _P, _P, ctypes.c_int, _P, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, _P]
        L.oracle_sparse_select.restype = None
        L.oracle_sparse_select.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]
        L.oracle_sparse_decode.restype = None
        L.oracle_sparse_decode.argtypes = [_P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, _P, _P, _P, _P]
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(_P)


def _opt(a, dtype):
    if a is None:
        return None, None
    return _c(a, dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


def bf16_to_f64(bits):
    f = lib().oracle_bf16_to_f64
    return np.array([f(int(b)) for b in np.asarray(bits, np.uint16).ravel()]).reshape(np.shape(bits))


def e4m3_to_f64(codes):
    f = lib().oracle_e4m3_to_f64
    return np.array([f(int(b)) for b in np.asarray(codes, np.uint8).ravel()]).reshape(np.shape(codes))


def _kv(k_pages, v_pages):
    if k_pages.dtype == np.uint16:
        return 0, np.uint16
    if k_pages.dtype == np.uint8:
        return 1, np.uint8
    raise TypeError("k_pages must hold bf16 bits (uint16) or e4m3 codes (uint8)")


def gather(k_pages, v_pages, page_table, seq_lens):
    """Contiguous copy-out: returns (k, v) with shape [sum L][Hk][D], same bit patterns."""
    num_pages, Hk, P, D = k_pages.shape
    kd, dt = _kv(k_pages, v_pages)
    B = len(seq_lens)
    kp, kp_p = _c(k_pages, dt)
    vp, vp_p = _c(v_pages, dt)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    cu = np.zeros(B + 1, np.int64)
    cu[1:] = np.cumsum(sl)
    cu, cu_p = _c(cu, np.int64)
    ko = np.zeros((int(cu[-1]), Hk, D), dt)
    vo = np.zeros((int(cu[-1]), Hk, D), dt)
    lib().oracle_gather(kp_p, vp_p, pt_p, pt.shape[1], sl_p, cu_p, B, Hk, D, P,
                        np.dtype(dt).itemsize, ko.ctypes.data_as(_P), vo.ctypes.data_as(_P))
    return ko, vo


def decode(q, k_pages, v_pages, page_table, seq_lens, scale, k_scale=None, v_scale=None,
           num_splits=0):
    """Decode attention in fp64.  q: uint16 bf16 bits [B][Hq][D].

    num_splits == 0: returns (out [B][Hq][D], lse [B][Hq]).
    num_splits  > 0: returns the per-split results (o_part [S][B][Hq][D], lse_part [S][B][Hq]).
    """
    B, Hq, D = q.shape
    num_pages, Hk, P, D2 = k_pages.shape
    assert D2 == D and Hq % Hk == 0
    kd, dt = _kv(k_pages, v_pages)
    qq, q_p = _c(q, np.uint16)
    kp, kp_p = _c(k_pages, dt)
    vp, vp_p = _c(v_pages, dt)
    ks, ks_p = _opt(k_scale, np.float32)
    vs, vs_p = _opt(v_scale, np.float32)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    args = (q_p, kp_p, vp_p, ks_p, vs_p, kd, pt_p, pt.shape[1], sl_p, B, Hq, Hk, D, P,
            num_pages, float(scale))
    if num_splits == 0:
        out = np.zeros((B, Hq, D))
        lse = np.zeros((B, Hq))
        lib().oracle_decode(*args, out.ctypes.data_as(_P), lse.ctypes.data_as(_P))
        return out, lse
    o = np.zeros((num_splits, B, Hq, D))
    l = np.zeros((num_splits, B, Hq))
    lib().oracle_decode_split(*args, int(num_splits), o.ctypes.data_as(_P), l.ctypes.data_as(_P))
    return o, l


def lse_combine(o_part, lse_part):
    """Merge split results: o_part [S][rows][D], lse_part [S][rows] -> (out, lse)."""
    S, rows, D = o_part.shape
    o, o_p = _c(o_part, np.float64)
    l, l_p = _c(lse_part, np.float64)
    out = np.zeros((rows, D))
    lse = np.zeros(rows)
    lib().oracle_lse_combine(o_p, l_p, S, rows, D, out.ctypes.data_as(_P), lse.ctypes.data_as(_P))
    return out, lse


def prefill(q, cu_q, k_pages, v_pages, page_table, seq_lens, scale, causal=True, k_scale=None,
            v_scale=None):
    """Chunked prefill in fp64.  q: uint16 bf16 bits [total_q][Hq][D]; cu_q [B+1]."""
    T, Hq, D = q.shape
    num_pages, Hk, P, D2 = k_pages.shape
    assert D2 == D and Hq % Hk == 0
    kd, dt = _kv(k_pages, v_pages)
    B = len(seq_lens)
    qq, q_p = _c(q, np.uint16)
    cq, cq_p = _c(cu_q, np.int32)
    kp, kp_p = _c(k_pages, dt)
    vp, vp_p = _c(v_pages, dt)
    ks, ks_p = _opt(k_scale, np.float32)
    vs, vs_p = _opt(v_scale, np.float32)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    assert np.all(np.diff(cq) <= sl), "each sequence must hold its whole query chunk"
    out = np.zeros((T, Hq, D))
    lse = np.zeros((T, Hq))
    lib().oracle_prefill(q_p, cq_p, kp_p, vp_p, ks_p, vs_p, kd, pt_p, pt.shape[1], sl_p, B, Hq,
                         Hk, D, P, num_pages, float(scale), int(bool(causal)),
                         out.ctypes.data_as(_P), lse.ctypes.data_as(_P))
    return out, lse


class use_library:
    """Context manager: route every oracle call through another build of gqa_oracle.c
    (the mutation tests plant mistakes in a copy of the source and check a pin fails)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = None
        real = _build.build
        _build.build = lambda force=False: self.path
        try:
            lib()
        finally:
            _build.build = real
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def f32_to_e4m3(x):
    """e4m3 codes of fp32 values (round to nearest even, saturating at +-448)."""
    f = lib().oracle_f32_to_e4m3
    a = np.asarray(x, np.float32)
    return np.array([f(float(v)) for v in a.ravel()], np.uint8).reshape(a.shape)


def append_kv(k_pages, v_pages, page_table, seq_lens, k_new, v_new, k_scale=None, v_scale=None):
    """Copies of the pools (and scales) with token seq_lens[b] - 1 of every sequence
    written from k_new / v_new (bf16 bits [B][Hk][D]); e4m3 pools quantise it (see
    oracle_append_kv).  Returns (k_pages, v_pages, k_scale, v_scale)."""
    kp = np.array(k_pages, copy=True)
    vp = np.array(v_pages, copy=True)
    fp8 = kp.dtype == np.uint8
    ks = np.array(k_scale, dtype=np.float32, copy=True) if fp8 else None
    vs = np.array(v_scale, dtype=np.float32, copy=True) if fp8 else None
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    kn, knp = _c(k_new, np.uint16)
    vn, vnp = _c(v_new, np.uint16)
    num_pages, Hk, P, D = kp.shape
    lib().oracle_append_kv(kp.ctypes.data_as(_P), vp.ctypes.data_as(_P),
                           ks.ctypes.data_as(_P) if fp8 else None,
                           vs.ctypes.data_as(_P) if fp8 else None, 1 if fp8 else 0, ptp,
                           pt.shape[1], slp, len(sl), Hk, D, P, knp, vnp)
    return kp, vp, ks, vs


# ---------------------------------------------------------------------------------------
# Page-level top-K sparse decode (see the readings in gqa_oracle.c).

def kt_build(k_pages, page_table, seq_lens, kt=None):
    """KT cache entries (min, max of the keys over each referenced page's valid tokens):
    returns double [num_pages][Hk][D][2]; entries of unreferenced pages are NaN (or those
    of `kt` when given)."""
    num_pages, Hk, P, D = k_pages.shape
    if k_pages.dtype != np.uint16:
        raise TypeError("the KT cache is built from bf16 pools")
    out = np.full((num_pages, Hk, D, 2), np.nan) if kt is None else np.array(kt, np.float64, copy=True)
    kp, kp_p = _c(k_pages, np.uint16)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    lib().oracle_kt_build(kp_p, pt_p, pt.shape[1], sl_p, len(sl), Hk, D, P, out.ctypes.data_as(_P))
    return out


def page_scores(q, kt, page_table, seq_lens, page_size):
    """fp32 page scores [B][Hk][pt_stride] (-inf past each sequence's pages)."""
    B, Hq, D = q.shape
    Hk = kt.shape[1]
    qq, q_p = _c(q, np.uint16)
    k, k_p = _c(kt, np.float64)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    out = np.zeros((B, Hk, pt.shape[1]), np.float32)
    lib().oracle_page_scores(q_p, k_p, pt_p, pt.shape[1], sl_p, B, Hq, Hk, D, page_size,
                             out.ctypes.data_as(_P))
    return out


def sparse_select(scores, seq_lens, page_size, topk, window):
    """Chosen logical pages per (sequence, kv head): returns (sel int32 [B][Hk][pt_stride],
    nsel int32 [B][Hk]); sel[b][j][:nsel[b][j]] ascending."""
    B, Hk, pts = scores.shape
    sc, sc_p = _c(scores, np.float32)
    sl, sl_p = _c(seq_lens, np.int32)
    sel = np.full((B, Hk, pts), -1, np.int32)
    nsel = np.zeros((B, Hk), np.int32)
    lib().oracle_sparse_select(sc_p, sl_p, B, Hk, pts, page_size, int(topk), int(window),
                               sel.ctypes.data_as(_P), nsel.ctypes.data_as(_P))
    return sel, nsel


def sparse_decode(q, k_pages, v_pages, page_table, seq_lens, scale, sel, nsel):
    """fp64 attention over the chosen pages: returns (out [B][Hq][D], lse [B][Hq])."""
    B, Hq, D = q.shape
    num_pages, Hk, P, _ = k_pages.shape
    qq, q_p = _c(q, np.uint16)
    kp, kp_p = _c(k_pages, np.uint16)
    vp, vp_p = _c(v_pages, np.uint16)
    pt, pt_p = _c(page_table, np.int32)
    sl, sl_p = _c(seq_lens, np.int32)
    se = np.full((B, Hk, pt.shape[1]), -1, np.int32)
    se[:, :, :sel.shape[2]] = sel[:, :, :pt.shape[1]]
    se, se_p = _c(se, np.int32)
    ns, ns_p = _c(nsel, np.int32)
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    lib().oracle_sparse_decode(q_p, kp_p, vp_p, pt_p, pt.shape[1], sl_p, B, Hq, Hk, D, P,
                               float(scale), se_p, ns_p, out.ctypes.data_as(_P),
                               lse.ctypes.data_as(_P))
    return out, lse
