"""Plant plausible mistakes in a COPY of the oracle source and check that a pin catches
each one.  This shows the pins in test_oracle_pins.py and test_append_cpu.py constrain
every step of the oracle (head map, page/slot indexing, scale, softmax, lse, split
boundaries, merge, decoders, causal bound, KV append position, e4m3 encoding, the
append scale, and the sparse decode's KT entries, page scores, selection and gather).  The real oracle source is never modified."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import build as obuild
from oracle import oracle
from tests import test_append_cpu as append_pins
from tests import test_oracle_pins as pins
from tests import test_sparse_cpu as sparse_pins

MUTANTS = {
    "head_map_interleaved": ("int h = kvh * g + j;\n                    for (int d = 0; d < D; ++d)\n                        qd[d] = oracle_bf16_to_f64(q[((int64_t)b",
                             "int h = j * Hk + kvh;\n                    for (int d = 0; d < D; ++d)\n                        qd[d] = oracle_bf16_to_f64(q[((int64_t)b"),
    "slot_off_by_one": ("kv_value(pages, kv_dtype, scale, Hk, P, D, phys, kvh, t % P, d)",
                        "kv_value(pages, kv_dtype, scale, Hk, P, D, phys, kvh, (t + 1) % P, d)"),
    "page_index_wrong": ("page_table[(int64_t)b * pt_stride + t / P];\n        for (int d",
                         "page_table[(int64_t)b * pt_stride + t % pt_stride];\n        for (int d"),
    "scale_dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "lse_without_max": ("*lse = m + log(Z);", "*lse = log(Z);"),
    "exp_sign_flipped": ("double w = exp(s[t] - m) / Z;", "double w = exp(m - s[t]) / Z;"),
    "first_term_dropped_from_Z": ("for (int t = t0; t < t1; ++t)\n        Z += exp(s[t] - m);",
                                  "for (int t = t0 + 1; t < t1; ++t)\n        Z += exp(s[t] - m);"),
    "split_size_floor": ("int c = (np + num_splits - 1) / num_splits;",
                         "int c = np / num_splits + 1;"),
    "merge_weight_dropped": ("W += w;", "W += 1.0;"),
    "e4m3_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "bf16_subnormal": ("ldexp((double)f, -126 - 7)", "ldexp((double)f, -127 - 7)"),
    "causal_off_by_one": ("(L - Lq + i + 1) : L", "(L - Lq + i) : L"),
    "query_head_index": ("qd[d] = oracle_bf16_to_f64(q[((int64_t)b * Hq + h) * D + d]);",
                         "qd[d] = oracle_bf16_to_f64(q[((int64_t)b * Hq + j) * D + d]);"),
    "fp8_scale_ignored": ("* scale[phys * Hk + kvh];", ";"),
    "empty_split_weighed": ("if (lse_part[(int64_t)s * rows + r] == -INFINITY)\n                continue;", ""),
    "append_slot_off_by_one": ("int slot = t % P;\n        for (int kvh", "int slot = (t + 1) % P;\n        for (int kvh"),
    "append_at_L": ("int t = L - 1;\n        int64_t phys", "int t = L - 2 < 0 ? 0 : L - 2;\n        int64_t phys"),
    "e4m3_ties_up": ("if (d < bd || (d == bd && (c & 1) == 0)) {", "if (d <= bd) {"),
    "e4m3_inf_not_saturated": ("return (uint8_t)((sign << 7) | 0x7e);", "return 0x7f;"),
    "append_scale_not_448": ("scale[si] = amax > 0.0f ? amax / 448.0f : 1.0f;",
                             "scale[si] = amax > 0.0f ? amax / 240.0f : 1.0f;"),
    "append_keeps_no_scale": ("if (slot == 0) {\n                    float amax", "if (slot >= 0) {\n                    float amax"),
    "kt_over_all_slots": ("int n = L - p * P < P ? L - p * P : P;\n            for (int kvh",
                          "int n = P;\n            for (int kvh"),
    "kt_min_max_swapped": ("e[0] = mn;\n                    e[1] = mx;", "e[0] = mx;\n                    e[1] = mn;"),
    "score_min_corner_only": ("sh = sh + (lo > hi ? lo : hi);", "sh = sh + lo;"),
    "score_last_head_only": ("total = total + sh;", "total = sh;"),
    "ties_to_higher_page": ("if (best < 0 || s[p] > s[best])", "if (best < 0 || s[p] >= s[best])"),
    "window_one_token_short": ("int lo = L - window > 0 ? L - window : 0;",
                               "int lo = L - window + 1 > 0 ? L - window + 1 : 0;"),
    "topk_one_short": ("for (int k = 0; k < topk; ++k) {", "for (int k = 1; k < topk; ++k) {"),
    "sparse_last_token_dropped": ("int cnt = L - p * P < P ? L - p * P : P;",
                                  "int cnt = L - p * P < P ? L - p * P - 1 : P;"),
}


def _pins():
    """Every pin, as zero-argument callables (parametrized ones expanded)."""
    fns = []
    for mod, name in [(m, n) for m in (pins, append_pins, sparse_pins) for n in dir(m)]:
        if not name.startswith("test_"):
            continue
        f = getattr(mod, name)
        marks = getattr(f, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            fns.append((name, f, {}))
            continue
        (m,) = params
        argnames = [a.strip() for a in m.args[0].split(",")] if isinstance(m.args[0], str) else m.args[0]
        for vals in m.args[1]:
            vals = vals if len(argnames) > 1 else (vals,)
            fns.append((name, f, dict(zip(argnames, vals))))
    return fns


def _build_mutant(tmp, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    src = src.replace(old, new, 1)
    c = os.path.join(tmp, "mut.c")
    so = os.path.join(tmp, "libmut.so")
    open(c, "w").write(src)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", c, "-o", so, "-lm"],
                   check=True)
    return so


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_some_pin_catches_mutant(mutant):
    old, new = MUTANTS[mutant]
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, old, new)
        caught = []
        with oracle.use_library(so), np.errstate(all="ignore"):
            for name, f, kw in _pins():
                if name == "test_kv_bytes_model_matches_the_pages_figure":
                    continue
                try:
                    f(**kw)
                except (AssertionError, ValueError, FloatingPointError):
                    caught.append(name)
                    break
        assert caught, f"no pin fails for mutant {mutant}"


def test_unmutated_copy_passes_every_pin():
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, "s[t] = scale * acc;", "s[t] = scale * acc;")
        with oracle.use_library(so):
            for name, f, kw in _pins():
                if name != "test_kv_bytes_model_matches_the_pages_figure":
                    f(**kw)
