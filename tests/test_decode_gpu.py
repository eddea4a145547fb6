"""GPU parity of paged GQA decode (and its split merge) against the fp64 oracle, through
the C ABI.  Tolerance: |gpu - ref| <= 2e-3 + 1e-2 |ref| per element for bf16 KV.  fp8 KV:
the same bf16 tolerance against the oracle on the dequantised values (the kernel-bug
detector), and max |gpu - ref| <= 5e-2 against the oracle on the unquantised bf16 values
(the stated fp8 bound; quantisation alone moves the exact result by ~2e-2 there)."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from oracle import oracle
from tests._util import bf16_tol_ok, bits, err_report, np32, oracle_decode

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def to_dev(case):
    kv = case.kv
    d = dict(q=case.q.to(DEV), k=kv.k_pages.to(DEV), v=kv.v_pages.to(DEV),
             pt=kv.page_table.to(DEV), sl=kv.seq_lens.to(DEV))
    if kv.k_scale is not None:
        d["ks"] = kv.k_scale.to(DEV)
        d["vs"] = kv.v_scale.to(DEV)
    return d


def run_decode(case, num_splits=0, pack_gqa=True, dev=None, workspace=None):
    d = dev or to_dev(case)
    out, lse = binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"], case.scale,
                                        num_splits=num_splits, pack_gqa=pack_gqa,
                                        k_scale=d.get("ks"), v_scale=d.get("vs"),
                                        workspace=workspace)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check(out, lse, ref_o, ref_l, rtol=1e-2, what=""):
    ok, bad = bf16_tol_ok(out, ref_o, rtol=rtol)
    assert ok, f"{what} out: {err_report(out, ref_o)} bad={int(bad.sum())}"
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_l)), what
    np.testing.assert_allclose(lse[fin], ref_l[fin], rtol=1e-4, atol=2e-3, err_msg=what)


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("S", [1, 3])
def test_tiny_decode(seed, S):
    case = inputs.tiny_decode(seed=seed)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=S)
    check(out, lse, ref_o, ref_l, what=f"tiny seed={seed} S={S}")


@pytest.mark.parametrize("S", [0, 1, 2, 3, 4, 7, 64])
def test_llama7b_decode_splits(S):
    case = inputs.llama7b_decode(seed=0)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=S)
    check(out, lse, ref_o, ref_l, what=f"llama7b S={S}")


@pytest.mark.parametrize("seed", [1, 2])
def test_llama7b_decode_seeds(seed):
    case = inputs.llama7b_decode(seed=seed)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case)
    check(out, lse, ref_o, ref_l, what=f"llama7b seed={seed}")


def _sampled_oracle(case, rows):
    """Oracle on a subset of sequences (their page-table rows), same pool."""
    kv = case.kv
    return oracle.decode(bits(case.q[rows]), bits(kv.k_pages), bits(kv.v_pages),
                         kv.page_table[rows].numpy(), kv.seq_lens[rows].numpy(), case.scale,
                         np32(kv.k_scale), np32(kv.v_scale))


@pytest.mark.parametrize("B", [1, 16, 32, 64, 128, 256])
def test_sweep_decode_batch(B):
    case = inputs.sweep_decode(B, seed=B)
    rows = np.arange(B) if B <= 16 else np.sort(np.random.default_rng(B).choice(B, 8, replace=False))
    ref_o, ref_l = _sampled_oracle(case, rows)
    dev = to_dev(case)
    # num_splits 0 (the measured choice), the balanced schedule on request, and splits
    for S in ([0, binding.GQA_SPLITS_BALANCED, 1, 2, 4] if B in (1, 64) else [0]):
        out, lse = run_decode(case, num_splits=S, dev=dev)
        check(out[rows], lse[rows], ref_o, ref_l, what=f"sweep B={B} S={S}")


@pytest.mark.parametrize("S", [0, 1, 4])
def test_sweep_decode_pack_off(S):
    case = inputs.sweep_decode(16, seed=3)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=S, pack_gqa=False)
    check(out, lse, ref_o, ref_l, what=f"pack off S={S}")
    out2, lse2 = run_decode(case, num_splits=S, pack_gqa=True)
    check(out2, lse2, ref_o, ref_l, what=f"pack on S={S}")


@pytest.mark.parametrize("S", [0, 1, 8])
def test_long70b_decode_bf16(S):
    case = inputs.long70b_decode(seed=0)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=S)
    check(out, lse, ref_o, ref_l, what=f"long70b bf16 S={S}")


@pytest.mark.parametrize("S", [0, 1, 8])
def test_long70b_decode_fp8(S):
    case = inputs.long70b_decode(seed=0, kv_dtype="fp8_e4m3")
    out, lse = run_decode(case, num_splits=S)
    # kernel-bug detector: oracle on the same dequantised values
    deq_o, deq_l = oracle_decode(case)
    check(out, lse, deq_o, deq_l, what=f"fp8 vs dequantised S={S}")
    # stated fp8 bound: max |err| <= 5e-2 against the oracle on the unquantised values
    ref_o, _ = oracle_decode(case, use_bf16_pool=True)
    assert np.max(np.abs(out - ref_o)) <= 5e-2, f"fp8 vs bf16 oracle: {err_report(out, ref_o)}"


@pytest.mark.parametrize("P", [16, 32, 64])
@pytest.mark.parametrize("Hq,Hk", [(32, 8), (64, 8), (8, 8)])
def test_fp8_page_sizes_and_ragged_tiles(P, Hq, Hk):
    """e4m3 KV takes 32-token tiles on pages of 32+ tokens (and in the balanced schedule on
    any page): lengths that end inside either 16-token half of a tile, exactly on a tile
    edge, empty, and longer than a page; num_splits 0 (here the measured split count), the
    balanced schedule on request, splits, and PackGQA off."""
    lens = [1, 15, 16, 17, 31, 32, 33, 0, 63, 200]
    case = inputs.make_decode_case(len(lens), Hq, Hk, 128, P, lens, seed=P + Hq,
                                   kv_dtype="fp8_e4m3", outlier_p=0.01)
    ref_o, ref_l = oracle_decode(case)
    dev = to_dev(case)
    for S, pack in ((0, True), (binding.GQA_SPLITS_BALANCED, True), (1, True), (3, True), (1, False)):
        out, lse = run_decode(case, num_splits=S, pack_gqa=pack, dev=dev)
        check(out, lse, ref_o, ref_l, what=f"fp8 P={P} Hq={Hq} S={S} pack={pack}")


@pytest.mark.parametrize("Hq,Hk,D,P", [(8, 8, 64, 16), (8, 1, 64, 32), (32, 1, 128, 16),
                                       (12, 4, 128, 64), (40, 8, 128, 16), (16, 2, 64, 64)])
def test_head_layouts_mha_mqa_and_odd_groups(Hq, Hk, D, P):
    case = inputs.make_decode_case(3, Hq, Hk, D, P, [1, 150, 333], seed=Hq * D + P)
    ref_o, ref_l = oracle_decode(case)
    for S in (0, binding.GQA_SPLITS_BALANCED, 1, 3):
        out, lse = run_decode(case, num_splits=S)
        check(out, lse, ref_o, ref_l, what=f"Hq={Hq} Hk={Hk} D={D} P={P} S={S}")


def test_empty_and_single_token_sequences():
    case = inputs.make_decode_case(5, 8, 2, 128, 16, [0, 1, 0, 16, 17], seed=21)
    ref_o, ref_l = oracle_decode(case)
    for S in (0, binding.GQA_SPLITS_BALANCED, 1, 2, 5):
        out, lse = run_decode(case, num_splits=S)
        check(out, lse, ref_o, ref_l, what=f"empty S={S}")
        assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))


def test_page_permutation_is_bit_identical_on_gpu():
    case = inputs.llama7b_decode(seed=4, B=8)
    out, lse = run_decode(case, num_splits=2)
    kv = case.kv
    perm = torch.randperm(kv.num_pages, generator=torch.Generator().manual_seed(5))
    inv = torch.argsort(perm)
    case2 = inputs.DecodeCase(case.q, inputs.PagedKV(kv.k_pages[perm].contiguous(),
                                                     kv.v_pages[perm].contiguous(),
                                                     inv[kv.page_table.long()].to(torch.int32),
                                                     kv.seq_lens, kv.page_size),
                              case.Hq, case.Hk, case.head_dim, case.scale, case.seed)
    out2, lse2 = run_decode(case2, num_splits=2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_shared_prefix_pages():
    case = inputs.make_decode_case(3, 32, 8, 128, 16, [512, 300, 200], seed=9,
                                   alias_prefix=[0, 16, 12])
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=3)
    check(out, lse, ref_o, ref_l, what="aliased prefix")


def test_bad_page_entry_sets_the_error_word():
    case = inputs.make_decode_case(2, 8, 2, 64, 16, [40, 20], seed=3)
    d = to_dev(case)
    d["pt"][0, 1] = case.kv.num_pages + 5  # out of range: never dereferenced, flagged
    ws = binding.new_workspace(1 << 16, DEV)
    binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"], case.scale, num_splits=1,
                             workspace=ws)
    assert binding.gqa_get_error(ws) == -7
    assert binding.gqa_get_error(ws) == 0  # cleared by the read
    # the untouched sequence is still right
    ref_o, ref_l = oracle_decode(case)
    d["pt"][0, 1] = case.kv.page_table[0, 1]
    out, lse = run_decode(case, num_splits=1, dev=d, workspace=ws)
    check(out, lse, ref_o, ref_l, what="after bad page")
    assert binding.gqa_get_error(ws) == 0


def test_lse_combine_standalone():
    rng = np.random.default_rng(0)
    S, rows, D = 5, 37, 128
    o = rng.normal(size=(S, rows, D)).astype(np.float32)
    l = rng.normal(size=(S, rows)).astype(np.float32) * 3
    l[:, 3] = -np.inf          # an all-empty row
    l[2, 5] = -np.inf          # one empty split
    o[2, 5] = np.nan           # whose partial is garbage
    ref_o, ref_l = oracle.lse_combine(o.astype(np.float64), l.astype(np.float64))
    out, lse = binding.lse_combine(torch.from_numpy(o).to(DEV), torch.from_numpy(l).to(DEV))
    torch.cuda.synchronize()
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    ok, _ = bf16_tol_ok(out, ref_o)
    assert ok, err_report(out, ref_o)
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(lse[fin], ref_l[fin], rtol=1e-5, atol=1e-5)
    assert np.isneginf(lse[3]) and np.all(out[3] == 0)


@pytest.mark.parametrize("B,S", [(48, 0), (16, 0), (4, 3), (4, 0)])
def test_repeated_calls_are_deterministic(B, S):
    """B=48 with num_splits=0 runs the balanced schedule with the in-launch merge, B=16
    and B=4 the balanced schedule with the separate merge kernel; B=4 with 3 splits the
    split schedule and lse_combine."""
    case = inputs.llama7b_decode(seed=6, B=B)
    dev = to_dev(case)
    ws = binding.new_workspace(binding.gqa_paged_decode_workspace_size(B, 32, 8, 128, 16, 2048, 0, S), DEV)
    a = run_decode(case, num_splits=S, dev=dev, workspace=ws)
    b = run_decode(case, num_splits=S, dev=dev, workspace=ws)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    if B == 48 and S == 0:  # in-launch merge: counters are back to zero after every launch
        hdr = 256
        assert binding.gqa_paged_decode_kernel_launches(B, 32, 8, 128, 16, 2048, 0, 0) == 1
        assert int(ws[hdr:hdr + B * 32 * 4].view(torch.int32).abs().sum()) == 0


def test_chained_decodes_read_the_previous_output():
    """Balanced-schedule launches back to back on one stream, each taking the previous
    launch's output as its q and sharing one workspace.  A launch may start while the
    previous kernel is still running (programmatic stream serialization); it must still
    read the finished output and find the merge counters reset."""
    import dataclasses
    case = inputs.llama7b_decode(seed=3)
    d = to_dev(case)
    B, Hq, D = case.q.shape
    ws = binding.new_workspace(binding.gqa_paged_decode_workspace_size(
        B, Hq, case.Hk, D, 16, d["pt"].shape[1] * 16, 0, 0), DEV)
    outs, lses = [d["q"]], []
    for _ in range(3):
        o, l = binding.gqa_paged_decode(outs[-1], d["k"], d["v"], d["pt"], d["sl"], case.scale,
                                        workspace=ws)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert binding.gqa_get_error(ws) == 0
    for i in (1, 2):  # launch i + 1 against the oracle on launch i's output
        ref_o, ref_l = oracle_decode(dataclasses.replace(case, q=outs[i].cpu()))
        check(outs[i + 1].float().cpu().numpy(), lses[i].cpu().numpy(), ref_o, ref_l,
              what=f"chained launch {i + 1}")


@pytest.mark.parametrize("lens", [[64] * 64, [2048] * 2])
def test_decode_replays_in_a_cuda_graph(lens):
    """The balanced schedule captured in a CUDA graph (both merge variants: in-launch for
    many short units, the separate merge kernel for two long sequences) replays to the
    oracle's result within the bf16 gate, and to the eager result bit for bit."""
    case = inputs.make_decode_case(len(lens), 32, 8, 128, 16, lens, seed=21)
    d = to_dev(case)
    B = len(lens)
    ws = binding.new_workspace(binding.gqa_paged_decode_workspace_size(
        B, 32, 8, 128, 16, d["pt"].shape[1] * 16, 0, 0), DEV)
    out = torch.empty(B, 32, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, 32, dtype=torch.float32, device=DEV)
    binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"], case.scale, out=out,
                             lse=lse, workspace=ws)
    torch.cuda.synchronize()
    eager_o, eager_l = out.clone(), lse.clone()
    out.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        for _ in range(2):
            binding.gqa_paged_decode(d["q"], d["k"], d["v"], d["pt"], d["sl"], case.scale,
                                     out=out, lse=lse, workspace=ws, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    assert binding.gqa_get_error(ws) == 0
    ref_o, ref_l = oracle_decode(case)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, what=f"graph replay {lens[:2]}")
    assert torch.equal(out, eager_o) and torch.equal(lse, eager_l)
    del g


@pytest.mark.parametrize("lens", [[1], [2048], [16] * 37, [0, 0, 5], [3000, 1, 17, 0, 900, 4096]])
def test_balanced_schedule_shapes(lens):
    """The balanced persistent schedule (num_splits = 0) on batch shapes whose units are
    cut between workers in many ways: one tile, one long sequence, many tiny ones, empty
    sequences, a ragged mix."""
    case = inputs.make_decode_case(len(lens), 32, 8, 128, 16, lens, seed=sum(lens) % 97)
    ref_o, ref_l = oracle_decode(case)
    out, lse = run_decode(case, num_splits=0)
    check(out, lse, ref_o, ref_l, what=f"balanced {lens}")
