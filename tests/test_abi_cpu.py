"""Host-only checks of the C ABI (no GPU needed): the library loads, exports every function
include/gqa_paged.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from gqa_attention_paged_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                             src, flags=re.M):
            names.append(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ["gqa_paged_decode", "gqa_paged_prefill", "lse_combine", "gqa_paged_gather",
              "gqa_get_error", "gqa_pick_splits", "gqa_paged_decode_workspace_size",
              "gqa_paged_prefill_workspace_size", "gqa_status_string"]:
        assert n in names, n


def test_decode_kernel_launch_count():
    """Host-only policy: one launch, or two when a second kernel merges partial results."""
    f = binding.gqa_paged_decode_kernel_launches
    assert f(64, 32, 8, 128, 16, 2048, 0, 0) == 1          # balanced, in-launch merge
    assert f(4, 64, 8, 128, 64, 32768, 0, 0) == 2          # few long sequences: merge kernel
    assert f(64, 32, 8, 128, 16, 2048, 0, 1) == 1          # one split
    assert f(64, 32, 8, 128, 16, 2048, 0, 4) == 2          # splits + lse_combine
    assert f(0, 32, 8, 128, 16, 2048, 0, 0) == 0           # rejected sizes
    assert f(4, 30, 8, 128, 16, 2048, 0, 0) == 0


def test_library_exports_every_declared_symbol():
    lib = binding.load()
    for name in declared_functions():
        assert hasattr(lib, name), f"missing export {name}"
        assert name in binding.SIGNATURES, f"binding lacks {name}"


def test_library_has_no_oracle_or_torch_dependency():
    """The product library links neither the oracle nor torch."""
    lib_path = binding.LIB_PATH
    binding.load()
    data = open(lib_path, "rb").read()
    assert b"oracle_decode" not in data and b"liboracle" not in data
    assert b"libtorch" not in data and b"libc10" not in data


def _fake(n=0x10000):
    return ctypes.c_void_p(n)


def _decode(**kw):
    args = dict(q=_fake(), k=_fake(), v=_fake(), ks=None, vs=None, kvd=0, pt=_fake(), pts=8,
                sl=_fake(), B=2, Hq=8, Hk=2, D=64, P=16, npg=16, scale=0.125, S=1, pack=1,
                out=_fake(), lse=None, ws=_fake(), wsb=1 << 20, st=None)
    args.update(kw)
    return binding.load().gqa_paged_decode(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), -1), (dict(pt=None), -1), (dict(ws=None), -1),
    (dict(Hq=6, Hk=4), -2), (dict(D=96), -2), (dict(P=8), -2), (dict(P=128), -2),
    (dict(npg=0), -2), (dict(pts=0), -2), (dict(B=-1), -2), (dict(B=70000), -2),
    (dict(kvd=5), -3), (dict(kvd=1), -3), (dict(kvd=1, ks=_fake(), vs=_fake(), D=64), -3),
    (dict(S=-2), -4), (dict(S=65), -4),
    (dict(q=_fake(0x10008)), -9), (dict(k=_fake(0x10004)), -9),
    (dict(ws=_fake(0x10010)), -5), (dict(wsb=16), -5),
    (dict(S=4, wsb=256), -5),
])
def test_decode_rejects_bad_arguments_on_the_host(kw, status):
    assert _decode(**kw) == status


def _append_decode(**kw):
    args = dict(q=_fake(), kn=_fake(), vn=_fake(), k=_fake(), v=_fake(), ks=None, vs=None,
                kvd=0, pt=_fake(), pts=8, sl=_fake(), B=2, Hq=8, Hk=2, D=64, P=16, npg=16,
                scale=0.125, S=0, pack=1, out=_fake(), lse=None, ws=_fake(), wsb=1 << 26,
                st=None)
    args.update(kw)
    return binding.load().gqa_paged_append_decode(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), -1), (dict(kn=None), -1), (dict(ws=None), -1),
    (dict(Hq=6, Hk=4), -2), (dict(D=96), -2), (dict(P=8), -2), (dict(B=-1), -2),
    (dict(kvd=1), -3), (dict(S=65), -4), (dict(wsb=16), -5),
    (dict(q=_fake(0x10008)), -9), (dict(out=_fake(0x10004)), -9), (dict(k=_fake(0x10002)), -9),
])
def test_append_decode_rejects_before_writing(kw, status):
    """Every rejection happens on the host before the append kernel is enqueued (these
    pointers are never dereferenced), so a rejected call leaves the cache untouched."""
    assert _append_decode(**kw) == status


def test_host_helpers():
    lib = binding.load()
    assert lib.gqa_paged_decode_workspace_size(4, 8, 2, 64, 16, 256, 0, 1) == 256
    assert lib.gqa_paged_decode_workspace_size(4, 8, 2, 64, 16, 256, 0, 3) == \
        256 + 3 * 32 * 64 * 4 + 512
    for B in (1, 16, 64, 256):
        s = lib.gqa_pick_splits(B, 8, 2048, 16, 0)
        assert 1 <= s <= 64
    assert lib.gqa_pick_splits(1, 8, 16, 16, 0) == 1
    assert binding.status_string(-7).startswith("page-table")
    assert lib.lse_combine(None, _fake(), 2, 4, 64, _fake(), None, None) == -1
    assert lib.lse_combine(_fake(), _fake(), 0, 4, 64, _fake(), None, None) == -4
    assert lib.lse_combine(_fake(), _fake(), 2, 4, 32, _fake(), None, None) == -2
    assert lib.gqa_paged_gather(_fake(), _fake(), _fake(), 4, _fake(), _fake(), 2, 2, 64, 16, 8,
                                3, _fake(), _fake(), None) == -2
    assert lib.gqa_get_error(None, None) == -1
    for tq in (0, 1, 63, 64, 4096):
        assert lib.gqa_paged_prefill_workspace_size(tq, 32, 128) == 256 + (4 * (tq + 1) + 255) // 256 * 256


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    kp = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.gqa_paged_decode(q, kp, kp, torch.zeros(1, 4, dtype=torch.int32),
                                 torch.ones(1, dtype=torch.int32), 0.125)


def test_prefill_rejects_bad_arguments_on_the_host():
    lib = binding.load()
    def call(**kw):
        args = dict(q=_fake(), cu=_fake(), k=_fake(), v=_fake(), pt=_fake(), pts=8, sl=_fake(),
                    B=2, Hq=8, Hk=2, D=128, P=16, npg=16, scale=0.1, causal=1, tq=10, mq=5,
                    out=_fake(), lse=None, ws=_fake(), wsb=256, st=None)
        args.update(kw)
        return lib.gqa_paged_prefill(*args.values())
    assert call(q=None) == -1
    assert call(D=96) == -2
    assert call(D=256) == -2
    assert call(scale=0.0) == -2
    assert call(scale=-1.0) == -2
    assert call(Hq=6, Hk=4) == -2
    assert call(wsb=16) == -5
    assert call(q=_fake(0x10008)) == -9


def _static(**kw):
    args = dict(q=_fake(), k=_fake(), v=_fake(), ks=None, vs=None, kvd=0, pt=_fake(), pts=128,
                sl=_fake(), B=16, Hq=32, Hk=8, D=128, P=16, npg=4096, scale=0.088, S=0, pack=1,
                out=_fake(), lse=None, st=None)
    args.update(kw)
    return binding.load().gqa_paged_decode_static_scratch(*args.values())


@pytest.mark.parametrize("kw,status", [
    # gqa_paged_decode's own checks come first: nothing (not even the scratch memset) is
    # queued for a call it rejects
    (dict(q=None), -1), (dict(kvd=7), -3), (dict(Hq=30), -2), (dict(S=65), -4),
    (dict(out=_fake(0x10008)), -9),
    # then the size check: 64 splits of B=64 need more than the fixed array
    (dict(B=64, S=64), -5),
    # groups of more than 8 heads at head_dim 128 never fit the balanced schedule's pieces
    (dict(Hq=128, Hk=8, S=0), -5), (dict(B=256, Hq=16, Hk=1, S=0), -5),
])
def test_static_scratch_rejects_on_the_host(kw, status):
    """These pointers are never dereferenced: every rejection happens on the host."""
    assert _static(**kw) == status


def test_static_scratch_fits_groups_above_8_with_splits():
    lib = binding.load()
    assert lib.gqa_paged_decode_workspace_size(16, 128, 8, 128, 16, 2048, 0, 0) > 16 << 20
    assert lib.gqa_paged_decode_workspace_size(16, 128, 8, 128, 16, 2048, 0, 2) <= 16 << 20


def test_measured_split_table():
    """gqa_pick_splits reads the measured table (nearest cell, units scaled to the device;
    148 SMs on a host with no GPU), clamped to the pages; num_splits = 0 runs splits only
    where the sweep found them faster than the balanced schedule."""
    lib = binding.load()
    f = lib.gqa_pick_splits
    assert f(1, 8, 2048, 16, 0) == 16
    assert f(4, 8, 8192, 16, 0) == 8
    assert f(64, 8, 2048, 16, 0) == 4
    assert f(256, 8, 2048, 16, 0) == 1
    assert f(16, 8, 8192, 16, 1) == 16
    assert f(1, 8, 100, 16, 0) == 7          # clamped to ceil(100 / 16) pages
    launches = binding.gqa_paged_decode_kernel_launches
    assert launches(1, 32, 8, 128, 16, 512, 0, 0) == 2    # auto: 8 splits + lse_combine
    assert launches(1, 32, 8, 128, 16, 2048, 0, 0) == 2   # auto: 16 splits + lse_combine
    assert launches(4, 32, 8, 128, 16, 2048, 0, 0) == 2   # auto: 8 splits + lse_combine
    assert launches(4, 32, 8, 128, 16, 2048, 1, 0) == 2   # e4m3: 8 splits + lse_combine
    assert launches(64, 32, 8, 128, 16, 2048, 0, 0) == 1  # balanced, in-launch merge
    assert launches(16, 32, 8, 128, 16, 2048, 0, 0) == 2  # balanced, 9.25 grid workers per unit: merge kernel
    assert launches(32, 32, 8, 128, 16, 2048, 0, 0) == 1  # balanced, in-launch merge
    assert launches(16, 32, 8, 128, 16, 512, 0, -1) == 2  # balanced on request, merge kernel
    assert launches(32, 32, 8, 128, 16, 512, 0, -1) == 1  # balanced on request, in-launch merge
    assert launches(16, 32, 8, 128, 16, 512, 0, 0) == 2   # auto: 2 splits + lse_combine
    assert launches(64, 32, 2, 128, 16, 2048, 0, 0) == 2  # groups of 16: decode + merge kernel
    # the workspace follows the schedule: splits need their partials
    ws = lib.gqa_paged_decode_workspace_size
    # B=8: 4 splits at context 2048, the balanced schedule from context 4096 on
    assert ws(8, 32, 8, 128, 16, 2048, 0, 0) == ws(8, 32, 8, 128, 16, 2048, 0, 4)
    assert ws(8, 32, 8, 128, 16, 4096, 0, 0) == ws(8, 32, 8, 128, 16, 4096, 0, -1)
    assert ws(8, 32, 8, 128, 16, 4096, 0, 0) != ws(8, 32, 8, 128, 16, 4096, 0, 4)
    assert ws(1, 32, 8, 128, 16, 512, 0, 0) == 256 + (8 * 32 * 128 * 4 + 255) // 256 * 256 + 1024


def test_sparse_decode_runs_the_balanced_schedule_by_default():
    """num_splits = 0 in the sparse decode means the balanced schedule for the decode of the
    chosen pages (its workspace is the balanced one, not that of the split count the dense
    table gives for 32 one-kv-head sequences of ~2K tokens)."""
    lib = binding.load()
    f = lib.gqa_paged_sparse_decode_workspace_size
    args = (4, 64, 8, 128, 64, 512, 32, 32)
    assert f(*args, 0) == f(*args, -1)
    assert f(*args, 0) != f(*args, 8)
    ss = lib.gqa_paged_sparse_table_stride(512, 64, 32, 32)
    dec = lib.gqa_paged_decode_workspace_size
    assert dec(32, 8, 1, 128, 64, ss * 64, 0, -1) != dec(32, 8, 1, 128, 64, ss * 64, 0, 0)
