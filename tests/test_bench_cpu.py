"""Host-side models of bench.py: the prefill FLOP count against a brute-force count of the
unmasked (query, key) pairs, the decode byte model written out by hand, the timing
spread, and the DRAM-traffic lookup (an entry counts only while it was taken on the
current sources of its kernels)."""
import json
import os

import numpy as np
import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("prior,lq", [([0], [1]), ([0, 7, 300], [5, 1, 64]), ([4096, 0], [512, 512])])
def test_prefill_flops_count_the_causal_pairs(prior, lq):
    """Row i of a chunk of lq tokens after `prior` keys sees keys 0 .. prior + i: count the
    visible pairs of a boolean mask."""
    Hq, D = 32, 128
    pairs = 0
    for p, n in zip(prior, lq):
        L = p + n
        rows = np.arange(n)[:, None] + p          # query positions
        keys = np.arange(L)[None, :]
        pairs += int((keys <= rows).sum())
    assert bench.prefill_flops(prior, lq, Hq, D) == 4 * Hq * D * pairs


def test_decode_step_bytes_by_hand():
    # bf16: K and V rows of every token and kv head, q read and out written (bf16)
    lens, Hq, Hk, D = [3, 17], 8, 2, 64
    kv = 2 * (3 + 17) * Hk * D * 2
    assert bench.decode_step_bytes(lens, Hq, Hk, D, 2) == kv + 2 * 2 * Hq * D * 2
    # e4m3: one byte per element, plus one fp32 K and one V scale per (page, kv head) read
    pages = 1 + 2  # 3 tokens -> 1 page of 16, 17 tokens -> 2 pages
    want = 2 * (3 + 17) * Hk * D * 1 + 2 * 2 * Hq * D * 2 + 2 * 4 * Hk * pages
    assert bench.decode_step_bytes(lens, Hq, Hk, D, 1, P=16) == want


def test_headline_algorithmic_bytes():
    """B=64, ctx 2048, Hq=32, Hk=8, D=128, bf16: 536.9 MB of KV + 0.52 MB q + 0.52 MB out."""
    assert bench.decode_step_bytes([2048] * 64, 32, 8, 128, 2) == 537919488


def test_spread_reports_median_min_p90():
    s = bench.spread([3.0, 1.0, 2.0, 4.0, 5.0])
    assert s["median_ms"] == 3.0 and s["min_ms"] == 1.0 and s["samples"] == 5
    assert 4.0 <= s["p90_ms"] <= 5.0
    assert bench.spread([]) is None


def test_source_families():
    assert bench.src_family("prefill") == "prefill"
    assert bench.src_family("sparse70b") == "sparse"
    assert bench.src_family("B64_ctx2048_bf16_S0_pack1") == "decode"
    assert bench.src_family("long70b_fp8_e4m3_S0_pack1") == "decode"
    # a decode figure does not depend on the prefill source, and the reverse
    assert bench.kernel_src_sha("prefill") != bench.kernel_src_sha("B64_ctx2048_bf16_S0_pack1")


def test_traffic_lookup_needs_the_current_sources(tmp_path, monkeypatch):
    key = "B64_ctx2048_bf16_S0_pack1"
    prof = tmp_path / "profiles"
    prof.mkdir()
    (tmp_path / "gqa_attention_paged_b200").mkdir()
    (tmp_path / "gqa_attention_paged_b200" / "csrc").symlink_to(
        os.path.join(ROOT, "gqa_attention_paged_b200", "csrc"))
    entry = {"kernel_src_sha": bench.kernel_src_sha(key), "dram_bytes_per_launch": 541341696.0}
    (prof / "traffic.json").write_text(json.dumps({"workloads": {key: entry}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile(key) == 541341696.0
    assert bench.traffic_from_profile("prefill") is None          # no entry
    entry["kernel_src_sha"] = "0" * 16                              # taken on other code
    (prof / "traffic.json").write_text(json.dumps({"workloads": {key: entry}}))
    assert bench.traffic_from_profile(key) is None


def test_committed_traffic_was_taken_on_the_current_sources():
    """Every committed DRAM-traffic figure belongs to the kernels as they are now, and the
    decode figures stay within a few percent of the algorithmic bytes."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)["workloads"]
    assert d, "no committed traffic figures"
    for key, e in d.items():
        assert e["kernel_src_sha"] == bench.kernel_src_sha(key), f"{key}: counters predate the sources"
    alg = bench.decode_step_bytes([2048] * 64, 32, 8, 128, 2)
    ratio = d["B64_ctx2048_bf16_S0_pack1"]["dram_bytes_per_launch"] / alg
    assert 1.0 <= ratio <= 1.05
