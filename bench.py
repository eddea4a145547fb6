"""Benchmark: paged GQA decode on B200 -- HBM GB/s (% of peak) and queries/s at B=64, 2K ctx.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|long70b|prefill] [--B 64] [--ctx 2048] [--splits 0]
                    [--no-pack] [--kv bf16|fp8_e4m3] [--append] [--eager] [--no-secondary]

One step = one gqa_paged_decode call (the balanced decode kernel, plus the merge kernel
when the call merges separately) over a batch of B sequences, each with `ctx` tokens of
paged history (Hq=32, Hk=8, D=128, page_size=16, seeded synthetic N(0,1) data).  Under
torchrun every rank runs its own batch (weak scaling; no collective on the data path) and
rank 0 prints one JSON line.  With no flags, the line also carries a `secondary` list: the
causal chunked prefill (TFLOP/s) and the 70B-shaped long-context decode with e4m3 KV
(GB/s), each measured the same way in the same run.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "GQA paged decode: HBM GB/s (% of B200 peak) and queries/s at B=64, 2K ctx"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------------ byte / flop model

def decode_kv_bytes(seq_lens, Hk, D, elem):
    """Algorithmic K+V bytes of one decode step: every valid token's K and V row of every
    kv head, read once."""
    return 2 * sum(int(L) for L in seq_lens) * Hk * D * elem


def decode_step_bytes(seq_lens, Hq, Hk, D, elem, P=16):
    """KV (read once) + q (bf16, read) + out (bf16, written); fp8 adds the per-(page, kv
    head) K and V scales of every page read."""
    B = len(seq_lens)
    b = decode_kv_bytes(seq_lens, Hk, D, elem) + 2 * B * Hq * D * 2
    if elem == 1:
        b += 2 * 4 * Hk * sum((int(L) + P - 1) // P for L in seq_lens)
    return b


def prefill_flops(prior_lens, q_lens, Hq, D):
    """4*Hq*D per unmasked (query, key) pair: row i of a chunk of Lq after `prior` keys
    sees prior + i + 1 keys."""
    pairs = sum(int(Lq) * int(p) + int(Lq) * (int(Lq) + 1) // 2 for p, Lq in zip(prior_lens, q_lens))
    return 4 * Hq * D * pairs


def rank_seed(seed, rank):
    """Each rank of a weak-scaling run draws its own batch."""
    return seed + rank


def max_over_ranks(x, dist=None, device="cpu"):
    """Max of a per-rank scalar over all ranks (every rank gets it)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(step_bytes_per_rank, world, ms_max):
    """Whole-job GB/s: every rank moves step_bytes_per_rank per step; the job's step time
    is the slowest rank's."""
    return world * step_bytes_per_rank / (ms_max * 1e-3) / 1e9


def spread(ms_list):
    """median / min / p90 of per-step times (ms); None when nothing was repeated."""
    if not ms_list:
        return None
    s = sorted(ms_list)
    p90 = s[min(len(s) - 1, int(math.ceil(0.9 * len(s))) - 1)]
    return {"median_ms": round(statistics.median(s), 5), "min_ms": round(s[0], 5),
            "p90_ms": round(p90, 5), "samples": len(s)}


def _peaks_file():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return None


def peaks():
    p = _peaks_file()
    if p and "hbm_gbs" in p:
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    p = _peaks_file()
    if p and "bf16_tflops" in p:
        return float(p["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


# Device sources behind each workload's kernels (the shared device headers included).
SRC_COMMON = ("gqa_device.cuh", "gqa_internal.h")
SRC_OF = {"decode": ("decode.cu", "combine.cu"), "prefill": ("prefill.cu",),
          "sparse": ("sparse.cu", "decode.cu", "combine.cu")}


def src_family(workload_key):
    return "prefill" if workload_key == "prefill" else "sparse" if workload_key.startswith("sparse") else "decode"


def kernel_src_sha(workload_key="B64_ctx2048_bf16_S0_pack1"):
    """Hash of the device sources a workload's kernels are built from: the code a traffic
    figure belongs to."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gqa_attention_paged_b200", "csrc")
    for fn in sorted(SRC_COMMON + SRC_OF[src_family(workload_key)]):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload_key):
    """DRAM bytes (read + write) per call of the timed kernels, from the committed ncu
    summary, or None if absent or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get("workloads", {}).get(workload_key)
    if e is None or e.get("kernel_src_sha") != kernel_src_sha(workload_key):
        return None
    return float(e["dram_bytes_per_launch"])


# ------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        # samples under load: power well above idle
        loaded = [s for s, p in zip(sm, power) if p > 250.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "samples_under_load": len([p for p in power if p > 250.0])}


# ------------------------------------------------------------------------ timing helpers

def timed_graph(step, K, stream, dev, repeat_s=1.0):
    """Capture K steps as one CUDA graph and time its replay with CUDA events on `stream`:
    the contract timing (one replay, exactly K steps), then further replays for about
    `repeat_s` seconds, whose per-step times give median / min / p90."""
    import torch
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(K):
                step(side)
    stream.wait_stream(side)
    graph.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / K
    per = []
    t_end = time.perf_counter() + repeat_s
    while time.perf_counter() < t_end and len(per) < 2000:
        evs = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        per += [a.elapsed_time(b) / K for a, b in evs]
    del graph
    torch.cuda.synchronize(dev)
    return ms, spread(per)


def timed_eager(step, K, stream, dev, repeat_s=1.0):
    """Launch K steps one by one from the host between one pair of CUDA events, then
    repeat for about `repeat_s` seconds for median / min / p90."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K):
        step(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / K
    per = []
    t_end = time.perf_counter() + repeat_s
    while time.perf_counter() < t_end and len(per) < 200:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            step(stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        per.append(a.elapsed_time(b) / K)
    return ms, spread(per)


def e2e_pipelined(dev, stream, h_in, d_in, d_out, h_out, run, steps):
    """End-to-end time per step through the public API, as a serving loop would issue it:
    step i's inputs are copied from pinned host memory into one of two device input sets on
    a copy stream while step i-1 computes; the compute of step i (run(slot, stream)) waits
    for them; its results are copied back to one of two pinned host sets on a third stream
    while step i+1 computes.  Every step's copies are inside the timed region.

    h_in: pinned host tensors; d_in: per input, a pair of device buffers; d_out: per
    output, a pair of device buffers; h_out: per output, a pair of pinned host buffers."""
    import torch
    cp, dh = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    copied_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        s = i % 2
        if i >= 2:
            cp.wait_event(consumed[s])       # step i-2 has read this input set
        with torch.cuda.stream(cp):
            for h, d in zip(h_in, d_in):
                d[s].copy_(h, non_blocking=True)
        in_ready[s].record(cp)
        stream.wait_event(in_ready[s])
        if i >= 2:
            stream.wait_event(copied_out[s])  # step i-2's results have left this output set
        run(s, stream)
        consumed[s].record(stream)
        dh.wait_event(consumed[s])
        with torch.cuda.stream(dh):
            for d, h in zip(d_out, h_out):
                h[s].copy_(d[s], non_blocking=True)
        copied_out[s].record(dh)

    for i in range(4):  # warm
        one(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cp.wait_event(e0)
    dh.wait_event(e0)
    for i in range(steps):
        one(i)
    stream.wait_stream(dh)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / steps


# ------------------------------------------------------------------------ CPU oracle legs

def _bits(t):
    import numpy as np
    import torch
    t = t.contiguous()
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype.itemsize == 2 \
        else t.view(torch.uint8).numpy()


def run_oracle_sample(case, rows, min_seconds):
    """Time the fp64 oracle on sequences `rows` of `case`, repeating until min_seconds."""
    from oracle import oracle

    kv = case.kv
    q = _bits(case.q[rows])
    kp, vp = _bits(kv.k_pages), _bits(kv.v_pages)
    pt = kv.page_table[rows].numpy()
    sl = kv.seq_lens[rows].numpy()
    ks = None if kv.k_scale is None else kv.k_scale.numpy()
    vs = None if kv.v_scale is None else kv.v_scale.numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode(q, kp, vp, pt, sl, case.scale, ks, vs)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return el / reps, reps, oracle.num_threads()


def run_oracle_prefill_sample(case, rows_per_seq, min_seconds):
    """Time the fp64 oracle on the last `rows_per_seq` query rows of every chunk (same
    positions and keys as in the full chunk).  Returns (seconds per pass, flops of the
    sample, repeats, threads)."""
    import numpy as np
    from oracle import oracle

    kv = case.kv
    cu = case.cu_q.tolist()
    lens = kv.seq_lens.tolist()
    idx, cu_s, prior, qls = [], [0], [], []
    for b in range(len(lens)):
        n = min(rows_per_seq, cu[b + 1] - cu[b])
        idx += list(range(cu[b + 1] - n, cu[b + 1]))
        cu_s.append(cu_s[-1] + n)
        prior.append(lens[b] - n)
        qls.append(n)
    q = _bits(case.q[idx])
    kp, vp = _bits(kv.k_pages), _bits(kv.v_pages)
    pt, sl = kv.page_table.numpy(), kv.seq_lens.numpy()
    cu_np = np.array(cu_s, np.int32)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.prefill(q, cu_np, kp, vp, pt, sl, case.scale, True)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return el / reps, prefill_flops(prior, qls, case.Hq, case.head_dim), reps, oracle.num_threads()


# ------------------------------------------------------------------------ arguments

def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--B", type=int, default=64)
    ap.add_argument("--ctx", type=int, default=2048)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--no-pack", action="store_true")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8_e4m3"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="headline run: skip the prefill and e4m3 long-context lines")
    ap.add_argument("--repeat-seconds", type=float, default=1.0,
                    help="seconds of repeated replays behind median / min / p90")
    ap.add_argument("--eager", action="store_true",
                    help="decode workloads: launch the timed steps one by one from the host "
                         "instead of replaying them as one captured CUDA graph")
    ap.add_argument("--append", action="store_true",
                    help="decode workloads: time gqa_paged_append_decode (each step first "
                         "writes the new token's K/V into its page)")
    ap.add_argument("--sweep", default=None, choices=["config3", "splits"],
                    help="print one JSON document of a decode sweep instead of the bench line: "
                         "config3 = B x PackGQA x num_splits at ctx 2048 (bf16, e4m3); "
                         "splits = the split schedule's time per split count and (B, ctx)")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "long70b", "sparse70b"],
                    help="decode: the headline (paged GQA decode); prefill: causal chunked "
                         "prefill, B=8 chunks of 512 tokens after a prior context ~ U[0, 4096]; "
                         "long70b: B=4 decode at 8K/16K/24K/32K, Hq=64 Hk=8, page 64 (--kv)")
    return ap.parse_args(argv)


def decode_metric(a):
    """The metric string of a decode line: the headline's at B=64 / 2K with bf16 KV, and a
    string naming the workload everywhere else."""
    kv = "" if a.kv == "bf16" else ", e4m3 KV"
    what = "GQA paged KV append + decode" if a.append else "GQA paged decode"
    if a.workload == "long70b":
        return (f"{what}, 70B-shaped long context (B=4, ctx 8K-32K, Hq=64 Hk=8{kv}): "
                "HBM GB/s (% of B200 peak)")
    if not a.append and a.kv == "bf16" and a.B == 64 and a.ctx == 2048:
        return METRIC
    ctx = f"{a.ctx // 1024}K" if a.ctx % 1024 == 0 else str(a.ctx)
    return f"{what}: HBM GB/s (% of B200 peak) and queries/s at B={a.B}, {ctx} ctx{kv}"


PREFILL_METRIC = ("causal chunked prefill over a paged KV cache (B=8, 512-token chunks, "
                  "prior ~ U[0,4096]): TFLOP/s of unmasked pairs (% of bf16 peak)")


def workload_name(a):
    if a.workload == "long70b":
        return f"paged GQA decode, 70B-shaped long context: B=4 ctx={{8K,16K,24K,32K}} Hq=64 Hk=8 D=128 page_size=64 kv={a.kv}"
    return (f"paged GQA {'KV append + ' if a.append else ''}decode, B={a.B} ctx={a.ctx} Hq=32 "
            f"Hk=8 D=128 page_size=16 kv={a.kv}")


# ------------------------------------------------------------------------ prefill

def measure_prefill(a, dev, with_cpu):
    import torch
    from gqa_attention_paged_b200 import binding, inputs

    case = inputs.chunked_prefill(seed=a.seed)
    kv = case.kv
    q, cu = case.q.to(dev), case.cu_q.to(dev)
    kp, vp, pt, sl = kv.k_pages.to(dev), kv.v_pages.to(dev), kv.page_table.to(dev), kv.seq_lens.to(dev)
    T, Hq, D = case.q.shape
    out = torch.empty(T, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(T, Hq, dtype=torch.float32, device=dev)
    ws = binding.new_workspace(binding.gqa_paged_prefill_workspace_size(T, Hq, D), dev)
    stream = torch.cuda.current_stream(dev)

    def step(on=None, qq=None, cc=None, ptt=None, sll=None, oo=None, ll=None):
        binding.gqa_paged_prefill(q if qq is None else qq, cu if cc is None else cc, kp, vp,
                                  pt if ptt is None else ptt, sl if sll is None else sll,
                                  case.scale, case.max_q_len, out=out if oo is None else oo,
                                  lse=lse if ll is None else ll, workspace=ws,
                                  stream=stream if on is None else on)

    step()
    torch.cuda.synchronize(dev)
    assert binding.gqa_get_error(ws) == 0 and torch.isfinite(out.float()).all()
    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize(dev)
    # The step's K/V (84 MB) fit in L2, so L2 is flushed before every timed step by
    # writing a buffer twice its size; only the launch itself is inside the events.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()

    def timed(n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for e0, e1 in ev:
            flush.fill_(1)
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    per = timed(a.steps)
    ms = sum(per) / a.steps
    more, t_end = [], time.perf_counter() + a.repeat_seconds
    while time.perf_counter() < t_end and len(more) < 2000:
        more += timed(20)
    clk = clocks.stop()

    # end to end: q, cu_q, page table and seq_lens H2D from pinned memory, out and lse D2H
    # (the paged K/V, the chunk's included, are device-resident: written by the layers
    # that project them)
    hin = [case.q.pin_memory(), case.cu_q.pin_memory(), kv.page_table.pin_memory(),
           kv.seq_lens.pin_memory()]
    din = [(x.to(dev), x.to(dev)) for x in hin]
    dout = [(out, torch.empty_like(out)), (lse, torch.empty_like(lse))]
    hout = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
             torch.empty(out.shape, dtype=out.dtype).pin_memory()),
            (torch.empty(lse.shape).pin_memory(), torch.empty(lse.shape).pin_memory())]

    def run(s, on):
        step(on, din[0][s], din[1][s], din[2][s], din[3][s], dout[0][s], dout[1][s])

    e2e_ms = e2e_pipelined(dev, stream, hin, din, dout, hout, run, a.steps)
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = sum(p[0].numel() * p[0].element_size() for p in hout)

    q_lens = (case.cu_q[1:] - case.cu_q[:-1]).tolist()
    prior = [int(L) - int(x) for L, x in zip(kv.seq_lens.tolist(), q_lens)]
    flops = prefill_flops(prior, q_lens, Hq, D)
    tf = flops / (ms * 1e-3) / 1e12
    peak, kind = tensor_peak()
    cpu = None
    if with_cpu:
        sec, sflops, reps, cores = run_oracle_prefill_sample(case, 4, min(a.cpu_seconds, 8.0))
        cpu = {"value": round(sflops / sec / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
               "kind": "oracle",
               "sample": f"the last 4 query rows of each of the 8 chunks (same keys and "
                         f"positions as in the full chunk), {reps} repeats, "
                         f"{sec * reps:.1f} s of CPU work; TFLOP/s of the same flop model"}
    return {
        "metric": PREFILL_METRIC,
        "value": round(tf, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
        "steps": a.steps, "warmup": max(3, a.warmup), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) q/k/v)",
        "config": {"workload": "chunked prefill B=8 Lq=512 prior~U[0,4096] Hq=32 Hk=8 D=128 P=16",
                   "flops_per_step": flops, "prior_lens": prior,
                   "l2": "flushed before every timed step (256 MB write outside the events)"},
        "pct_of_bf16_peak": round(100 * tf / peak, 2),
        "tokens_per_s": round(sum(q_lens) / (ms * 1e-3), 1),
        "spread": spread(more) if more else None,
        "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tf / peak, 4), "traffic": traffic_from_profile("prefill"),
                     "traffic_key": "prefill",
                     "peak_source": f"{kind} (bf16_tflops, burst cuBLAS GEMM)",
                     "kernel": "prefill_kernel (plan kernel included in the step time)"},
        "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 5),
                "note": "q, cu_q, page table, seq_lens H2D from pinned memory on a copy stream, "
                        "out+lse D2H on a third stream, double-buffered so step i's copies "
                        "overlap steps i-1 / i+1; eager gqa_paged_prefill calls; L2 not flushed"},
        "gpu_launches": 2 * a.steps,  # the plan kernel and the prefill kernel per step
        "clocks": clk,
        "cpu_baseline": cpu,
    }


# ------------------------------------------------------------------------ decode

def measure_decode(a, dev, rank, world, dist, with_cpu):
    import torch
    from gqa_attention_paged_b200 import binding, inputs

    if a.workload == "long70b":
        case = inputs.long70b_decode(seed=rank_seed(a.seed, rank), kv_dtype=a.kv)
        a.B, a.ctx = 4, 32768
    else:
        case = inputs.sweep_decode(a.B, seed=rank_seed(a.seed, rank), ctx=a.ctx, kv_dtype=a.kv)
    kv = case.kv
    q = case.q.to(dev)
    kp, vp = kv.k_pages.to(dev), kv.v_pages.to(dev)
    ks = None if kv.k_scale is None else kv.k_scale.to(dev)
    vs = None if kv.v_scale is None else kv.v_scale.to(dev)
    pt, sl = kv.page_table.to(dev), kv.seq_lens.to(dev)
    elem = 1 if a.kv == "fp8_e4m3" else 2
    B, Hq, Hk, D, P = a.B, case.Hq, case.Hk, case.head_dim, kv.page_size
    kvc = binding.GQA_KV_FP8_E4M3 if elem == 1 else binding.GQA_KV_BF16
    balanced = a.splits == 0 and B <= 2048  # num_splits = 0: the balanced persistent schedule
    S = a.splits if a.splits > 0 else (0 if balanced else
                                      binding.gqa_pick_splits(B, Hk, pt.shape[1] * P, P, kvc))
    pack = not a.no_pack
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = binding.new_workspace(
        binding.gqa_paged_decode_workspace_size(B, Hq, Hk, D, P, pt.shape[1] * P, kvc, S), dev)
    stream = torch.cuda.current_stream(dev)
    launches = binding.gqa_paged_decode_kernel_launches(B, Hq, Hk, D, P, pt.shape[1] * P, kvc, S,
                                                        pack)
    if a.append:
        # the new token of every sequence (position seq_len - 1), written before each decode
        gk = torch.Generator().manual_seed(a.seed + 1)
        k_new = torch.randn(B, Hk, D, generator=gk).to(torch.bfloat16).to(dev)
        v_new = torch.randn(B, Hk, D, generator=gk).to(torch.bfloat16).to(dev)
        launches += 1

    def step(on=None, qq=None, ptt=None, sll=None, oo=None, ll=None):
        on = stream if on is None else on
        qq = q if qq is None else qq
        ptt = pt if ptt is None else ptt
        sll = sl if sll is None else sll
        oo = out if oo is None else oo
        ll = lse if ll is None else ll
        if a.append:
            binding.gqa_paged_append_decode(qq, k_new, v_new, kp, vp, ptt, sll, case.scale,
                                            num_splits=S, pack_gqa=pack, k_scale=ks, v_scale=vs,
                                            out=oo, lse=ll, workspace=ws, stream=on)
            return
        binding.gqa_paged_decode(qq, kp, vp, ptt, sll, case.scale, num_splits=S, pack_gqa=pack,
                                 k_scale=ks, v_scale=vs, out=oo, lse=ll, workspace=ws, stream=on)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # sanity check of this exact launch configuration before timing
    step()
    torch.cuda.synchronize(dev)
    assert binding.gqa_get_error(ws) == 0
    assert torch.isfinite(out.float()).all(), "non-finite output"

    for _ in range(max(3, a.warmup)):
        step()
    barrier()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    barrier()
    if a.eager:
        ms, sp = timed_eager(step, a.steps, stream, dev, a.repeat_seconds)
    else:
        ms, sp = timed_graph(step, a.steps, stream, dev, a.repeat_seconds)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(ms, dist, dev)

    # The dominant kernel alone: time the merge kernel by itself on the same partials and
    # subtract it (when the call splits), all with events on this stream.
    comb_ms = 0.0
    if S > 1:
        hdr = 256
        rows = B * Hq
        o_bytes = (S * rows * D * 4 + 255) // 256 * 256
        o_part = ws[hdr:hdr + S * rows * D * 4].view(torch.float32).view(S, rows, D)
        l_part = ws[hdr + o_bytes:hdr + o_bytes + S * rows * 4].view(torch.float32).view(S, rows)
        o2 = torch.empty(rows, D, dtype=torch.bfloat16, device=dev)
        l2 = torch.empty(rows, dtype=torch.float32, device=dev)
        for _ in range(3):
            binding.lse_combine(o_part, l_part, o2, l2, stream=stream)
        torch.cuda.synchronize(dev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(a.steps):
            binding.lse_combine(o_part, l_part, o2, l2, stream=stream)
        c1.record(stream)
        torch.cuda.synchronize(dev)
        comb_ms = c0.elapsed_time(c1) / a.steps
    kern_ms = max(ms - comb_ms, 1e-6)

    # end to end through the public API: per step, the step's inputs (q, page table,
    # sequence lengths) copied from pinned host memory, the decode, and the result (out,
    # lse) copied back; the KV cache is device-resident state.  Pipelined as a serving
    # loop issues it (see e2e_pipelined).
    hin = [case.q.pin_memory(), kv.page_table.pin_memory(), kv.seq_lens.pin_memory()]
    din = [(q, q.clone()), (pt, pt.clone()), (sl, sl.clone())]
    dout = [(out, torch.empty_like(out)), (lse, torch.empty_like(lse))]
    hout = [(torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory(),
             torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory()),
            (torch.empty(B, Hq).pin_memory(), torch.empty(B, Hq).pin_memory())]
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = sum(p[0].numel() * p[0].element_size() for p in hout)

    def run(s, on):
        step(on, din[0][s], din[1][s], din[2][s], dout[0][s], dout[1][s])

    barrier()
    e2e_ms = max_over_ranks(e2e_pipelined(dev, stream, hin, din, dout, hout, run, a.steps), dist, dev)

    lens = [int(x) for x in kv.seq_lens]
    step_bytes = decode_step_bytes(lens, Hq, Hk, D, elem, P)
    if a.append:  # the new tokens' K/V read (bf16) and written into the pages
        step_bytes += 2 * B * Hk * D * (2 + elem)
    peak, peak_kind = peaks()
    gbs = aggregate_gbs(step_bytes, world, ms)
    kern_gbs = step_bytes / (kern_ms * 1e-3) / 1e9
    e2e_gbs = aggregate_gbs(step_bytes, world, e2e_ms)
    wkey = (f"long70b_{a.kv}_S{S}_pack{int(pack)}" if a.workload == "long70b"
            else f"B{B}_ctx{a.ctx}_{a.kv}_S{S}_pack{int(pack)}")
    traffic = None if a.append else traffic_from_profile(wkey)

    cpu = None
    if with_cpu and rank == 0 and world == 1:
        rows = list(range(min(B, 8)))
        sec, reps, cores = run_oracle_sample(case, rows, a.cpu_seconds)
        sb = decode_step_bytes([lens[r] for r in rows], Hq, Hk, D, elem, P)
        cpu = {"value": sb / sec / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{len(rows)} of {B} sequences (ctx {a.ctx}), {reps} repeats, "
                         f"{sec * reps:.1f} s of CPU work; GB/s of the same byte model"}

    return {
        "metric": decode_metric(a),
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": a.steps,
        "warmup": max(3, a.warmup),
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if elem == 2 else "fp8_e4m3 KV, bf16 q/out, fp32 accumulate",
        "data": "synthetic (seeded N(0,1) q/k/v, shuffled page pool with 25% unused pages)",
        "config": {
            "workload": workload_name(a),
            "B_per_gpu": B, "global_batch": B * world, "ctx": a.ctx, "Hq": Hq, "Hk": Hk,
            "head_dim": D, "page_size": P, "num_splits": S, "pack_gqa": pack,
            "launch": "eager launches" if a.eager else "CUDA graph of the timed steps (captured once, replayed)",
            "schedule": ("balanced persistent (one launch)" if S == 0 and launches == 1 else
                         "balanced persistent + merge of cut units (two launches)" if S == 0 else
                         f"{S} splits + merge"),
            "parallelism": f"dp{world} (independent batches, no collective)",
            "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB per step per GPU vs 126 MB L2; "
                  "KV loads carry an L2 evict-first hint",
            "algorithmic_bytes_per_step": step_bytes,
        },
        "pct_of_hbm_peak": round(100 * gbs / world / peak, 2),
        "queries_per_s": round(world * B / (ms * 1e-3), 1),
        "head_queries_per_s": round(world * B * Hq / (ms * 1e-3), 1),
        "spread": sp,
        "roofline": {"bound": "hbm", "achieved": round(kern_gbs, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(kern_gbs / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": ("decode_sk_kernel (the whole call: one launch)" if S == 0 and launches == 1 else
                                "decode_sk_kernel + piece_merge_kernel (the whole call)" if S == 0 else
                                "decode_kernel (call time minus the separately timed lse_combine)"),
                     "kernel_ms": round(kern_ms, 5), "combine_ms": round(comb_ms, 5),
                     "traffic_key": wkey},
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
                "frac_of_device": round(ms / e2e_ms, 4),
                "note": "q, page table and seq_lens H2D from pinned memory on a copy stream, "
                        "out+lse D2H on a third stream, double-buffered so step i's copies "
                        "overlap steps i-1 / i+1; eager gqa_paged_decode calls; KV cache "
                        "device-resident"},
        "gpu_launches": a.steps * launches,
        "clocks": clk,
        "cpu_baseline": cpu,
    }


# ------------------------------------------------------------------------ sparse decode

SPARSE_TOPK, SPARSE_WINDOW = 32, 32
SPARSE_METRIC = ("page-level top-K sparse GQA decode, 70B-shaped long context (B=4, ctx 8K-32K, "
                 f"top {SPARSE_TOPK} pages of 64 + a {SPARSE_WINDOW}-token window): HBM GB/s of the "
                 "bytes it reads (KT entries + chosen KV + q + out)")


def sparse_step_bytes(sel_lens, seq_lens, Hq, Hk, D, P, topk, window):
    """Algorithmic bytes of one sparse decode step: the KT entries of every scored page
    (4*D bytes per (page, kv head); pages of the window are not scored, and nothing is
    scored when the earlier pages are at most topk), the chosen tokens' K and V (bf16),
    q and out."""
    kt = 0
    for L in seq_lens:
        L = int(L)
        np_ = (L + P - 1) // P
        wp = min(max(L - window, 0) // P, np_) if window > 0 else np_
        if wp > topk:
            kt += wp * Hk * 4 * D
    kv = 2 * sum(int(x) for x in sel_lens) * D * 2
    B = len(seq_lens)
    return kt + kv + 2 * B * Hq * D * 2, kt, kv


def measure_sparse(a, dev, with_cpu):
    import torch
    from gqa_attention_paged_b200 import binding, inputs

    case = inputs.long70b_decode(seed=a.seed, kv_dtype="bf16")
    kv = case.kv
    q, kp, vp = case.q.to(dev), kv.k_pages.to(dev), kv.v_pages.to(dev)
    pt, sl = kv.page_table.to(dev), kv.seq_lens.to(dev)
    B, Hq, D = case.q.shape
    Hk, P = case.Hk, kv.page_size
    topk, window = SPARSE_TOPK, SPARSE_WINDOW
    kt = binding.gqa_paged_kt_build(kp, pt, sl)
    ws = binding.new_workspace(binding.gqa_paged_sparse_decode_workspace_size(
        B, Hq, Hk, D, P, pt.shape[1], topk, window, 0), dev)
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(on=None, qq=None, ptt=None, sll=None, oo=None, ll=None):
        binding.gqa_paged_sparse_decode(q if qq is None else qq, kp, vp, kt,
                                        pt if ptt is None else ptt, sl if sll is None else sll,
                                        case.scale, topk, window, out=out if oo is None else oo,
                                        lse=lse if ll is None else ll, workspace=ws,
                                        stream=stream if on is None else on)

    step()
    torch.cuda.synchronize(dev)
    assert binding.gqa_get_error(ws) == 0 and torch.isfinite(out.float()).all()
    _, sel_lens, _ = binding.gqa_paged_sparse_select(q, kt, kp, pt, sl, topk, window)
    torch.cuda.synchronize(dev)
    step_bytes, kt_bytes, kv_bytes = sparse_step_bytes(sel_lens.tolist(), kv.seq_lens.tolist(),
                                                       Hq, Hk, D, P, topk, window)
    for _ in range(max(3, a.warmup)):
        step()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    ms, sp = timed_graph(step, a.steps, stream, dev, a.repeat_seconds)
    clk = clocks.stop()
    # the dense decode of the same inputs, for the speedup
    dws = binding.new_workspace(binding.gqa_paged_decode_workspace_size(
        B, Hq, Hk, D, P, pt.shape[1] * P, 0, 0), dev)

    def dense(on):
        binding.gqa_paged_decode(q, kp, vp, pt, sl, case.scale, out=out, lse=lse, workspace=dws,
                                 stream=on)

    dense(stream)
    dms, dsp = timed_graph(dense, a.steps, stream, dev, a.repeat_seconds)
    hin = [case.q.pin_memory(), kv.page_table.pin_memory(), kv.seq_lens.pin_memory()]
    din = [(q, q.clone()), (pt, pt.clone()), (sl, sl.clone())]
    dout = [(out, torch.empty_like(out)), (lse, torch.empty_like(lse))]
    hout = [(torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory(),
             torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory()),
            (torch.empty(B, Hq).pin_memory(), torch.empty(B, Hq).pin_memory())]

    def run(s_, on):
        step(on, din[0][s_], din[1][s_], din[2][s_], dout[0][s_], dout[1][s_])

    e2e_ms = e2e_pipelined(dev, stream, hin, din, dout, hout, run, a.steps)
    peak, kind = peaks()
    gbs = step_bytes / (ms * 1e-3) / 1e9
    # the decode of the chosen pages: B * Hk sequences of one kv head and Hq / Hk heads
    dec_launches = binding.gqa_paged_decode_kernel_launches(
        B * Hk, Hq // Hk, 1, D, P, binding.gqa_paged_sparse_table_stride(pt.shape[1], P, topk, window) * P,
        0, -1)
    cpu = None
    if with_cpu:
        from oracle import oracle
        t0, reps = time.perf_counter(), 0
        qb, kb, vb = _bits(case.q), _bits(kv.k_pages), _bits(kv.v_pages)
        ptn, sln = kv.page_table.numpy(), kv.seq_lens.numpy()
        while time.perf_counter() - t0 < min(a.cpu_seconds, 8.0):
            ktn = oracle.kt_build(kb, ptn, sln) if reps == 0 else ktn
            sc = oracle.page_scores(qb, ktn, ptn, sln, P)
            sel, nsel = oracle.sparse_select(sc, sln, P, topk, window)
            oracle.sparse_decode(qb, kb, vb, ptn, sln, case.scale, sel, nsel)
            reps += 1
        sec = (time.perf_counter() - t0) / reps
        cpu = {"value": round(step_bytes / sec / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
               "kind": "oracle", "sample": f"the whole step (scores, selection, attention), {reps} "
                                           "repeats (the first also builds the KT entries)"}
    return {
        "metric": SPARSE_METRIC, "value": round(gbs, 2), "unit": "GB/s",
        "ms_per_step": round(ms, 5), "steps": a.steps, "warmup": max(3, a.warmup),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded N(0,1) q/k/v, 1% outliers at 8 sigma)",
        "config": {"workload": f"sparse decode B=4 ctx={{8K,16K,24K,32K}} Hq=64 Hk=8 D=128 P=64 "
                               f"topk={topk} window={window}",
                   "algorithmic_bytes_per_step": step_bytes, "kt_bytes": kt_bytes,
                   "chosen_kv_bytes": kv_bytes, "chosen_tokens": int(sum(sel_lens.tolist())),
                   "dense_tokens": int(Hk * kv.seq_lens.sum())},
        "pct_of_hbm_peak": round(100 * gbs / peak, 2),
        "dense_ms_per_step": round(dms, 5), "speedup_over_dense": round(dms / ms, 3),
        "spread": sp,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": traffic_from_profile("sparse70b"),
                     "traffic_key": "sparse70b",
                     "kernel": "sparse_score_kernel + sparse_pick_kernel + the decode of the chosen pages on "
                               f"the balanced schedule ({dec_launches} launch(es)): the whole call"},
        "e2e": {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in hin),
                "d2h_bytes_per_step": sum(p_[0].numel() * p_[0].element_size() for p_ in hout),
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": a.steps * (2 + dec_launches),
        "clocks": clk, "cpu_baseline": cpu,
    }


# ------------------------------------------------------------------------ sweeps

L2_BYTES = 126 << 20


def device_decode_inputs(B, ctx, Hq, Hk, D, P, kv, dev, seed, min_bytes=3 * L2_BYTES):
    """Timing-only decode inputs made on the device (their values are N(0,1); parity is
    the tests' job): a shuffled pool holding `copies` disjoint copies of the batch, so
    that consecutive steps read different pages and the KV they touch (at least
    min_bytes over the copies) does not sit in L2.  Returns (q, k, v, ks, vs, tables,
    seq_lens, step_bytes)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(seed)
    npg = (ctx + P - 1) // P
    elem = 1 if kv == "fp8_e4m3" else 2
    kv_bytes = 2 * B * ctx * Hk * D * elem
    copies = max(1, -(-min_bytes // max(kv_bytes, 1)))
    used = B * npg * copies
    pool = -(-used * 4 // 3)
    perm = torch.randperm(pool, device=dev, generator=g).to(torch.int32)
    tables = [perm[c * B * npg:(c + 1) * B * npg].view(B, npg).contiguous() for c in range(copies)]
    k = torch.randn(pool, Hk, P, D, device=dev, generator=g, dtype=torch.bfloat16)
    v = torch.randn(pool, Hk, P, D, device=dev, generator=g, dtype=torch.bfloat16)
    ks = vs = None
    if elem == 1:
        def q8(x):
            amax = x.float().abs().amax(dim=(2, 3))
            sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            y = (x.float() / sc[:, :, None, None]).clamp(-448.0, 448.0)
            return y.to(torch.float8_e4m3fn).view(torch.uint8), sc.float().contiguous()
        k, ks = q8(k)
        v, vs = q8(v)
    q = torch.randn(B, Hq, D, device=dev, generator=g, dtype=torch.bfloat16)
    sl = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    return q, k, v, ks, vs, tables, sl, decode_step_bytes([ctx] * B, Hq, Hk, D, elem, P)


def sweep_point(binding, inp, S, pack, dev, K=20, repeat_s=0.25):
    """GB/s of one decode configuration: K steps (each on the next copy of the batch) as a
    CUDA graph, median of repeated replays."""
    import torch
    q, k, v, ks, vs, tables, sl, step_bytes = inp
    B, Hq, D = q.shape
    num_pages, Hk, P, _ = k.shape
    kvc = binding.GQA_KV_FP8_E4M3 if ks is not None else binding.GQA_KV_BF16
    pts = tables[0].shape[1]
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = binding.new_workspace(binding.gqa_paged_decode_workspace_size(B, Hq, Hk, D, P, pts * P,
                                                                       kvc, S), dev)
    stream = torch.cuda.current_stream(dev)
    K = max(K, len(tables))
    it = [0]

    def step(on):
        t = tables[it[0] % len(tables)]
        it[0] += 1
        binding.gqa_paged_decode(q, k, v, t, sl, 1.0 / math.sqrt(D), num_splits=S, pack_gqa=pack,
                                 k_scale=ks, v_scale=vs, out=out, lse=lse, workspace=ws, stream=on)

    for _ in range(3):
        step(stream)
    torch.cuda.synchronize(dev)
    assert binding.gqa_get_error(ws) == 0
    ms, sp = timed_graph(step, K, stream, dev, repeat_s)
    med = sp["median_ms"] if sp else ms
    return {"ms": round(med, 5), "us": round(med * 1e3, 2),
            "gbs": round(step_bytes / (med * 1e-3) / 1e9, 1),
            "pct_of_hbm_peak": round(100 * step_bytes / (med * 1e-3) / 1e9 / peaks()[0], 2),
            "copies": len(tables)}


def run_sweep(kind, a, dev):
    """config3: the batch-sensitivity grid (Hq=32, Hk=8, D=128, ctx 2048, page 16):
    B x PackGQA on/off x num_splits {1, 2, 4, auto}, bf16 and e4m3 KV.
    splits: the split schedule's best split count per (batch, context), the table
    gqa_pick_splits encodes."""
    import torch
    from gqa_attention_paged_b200 import binding
    Hq, Hk, D, P = 32, 8, 128, 16
    res = {"kind": kind, "peak_gbs": peaks()[0], "points": []}
    if kind == "config3":
        for kv in ("bf16", "fp8_e4m3"):
            for B in (1, 16, 32, 64, 128, 256):
                inp = device_decode_inputs(B, 2048, Hq, Hk, D, P, kv, dev, seed=B)
                for pack in (True, False):
                    for S in (1, 2, 4, 0):
                        if kv == "fp8_e4m3" and not pack and S != 0:
                            continue
                        r = sweep_point(binding, inp, S, pack, dev)
                        r.update({"B": B, "ctx": 2048, "kv": kv, "pack_gqa": pack,
                                  "num_splits": "auto" if S == 0 else S})
                        res["points"].append(r)
                        print(json.dumps(r), file=sys.stderr, flush=True)
                del inp
                torch.cuda.empty_cache()
    else:
        grid = [(B, ctx) for B in (1, 2, 4, 8, 16, 64, 256, 1024)
                for ctx in (512, 2048, 4096, 8192, 32768) if B * ctx <= (2 << 20)]
        for kv in ("bf16", "fp8_e4m3"):
            for B, ctx in grid:
                inp = device_decode_inputs(B, ctx, Hq, Hk, D, P, kv, dev, seed=B + ctx)
                for S in (-1, 0, 1, 2, 4, 8, 16, 32, 64):
                    if S > (ctx // P):
                        continue
                    r = sweep_point(binding, inp, S, True, dev)
                    r.update({"B": B, "ctx": ctx, "kv": kv,
                              "num_splits": {-1: "balanced", 0: "auto"}.get(S, S)})
                    res["points"].append(r)
                    print(json.dumps(r), file=sys.stderr, flush=True)
                del inp
                torch.cuda.empty_cache()
    return res


def _secondary_summary(line):
    keep = ("metric", "value", "unit", "ms_per_step", "spread", "roofline", "clocks", "e2e",
            "cpu_baseline", "gpu_launches", "pct_of_hbm_peak", "pct_of_bf16_peak", "dtype",
            "speedup_over_dense", "dense_ms_per_step")
    s = {k: line[k] for k in keep if k in line}
    s["workload"] = line["config"]["workload"]
    return s


def main():
    a = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if a.impl == "reference":
        if rank != 0:
            return 0
        return reference_arm(a, world)

    import torch

    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    if a.sweep:
        if rank == 0:
            print(json.dumps(run_sweep(a.sweep, a, dev)))
        return 0
    if a.workload in ("prefill", "sparse70b"):
        if rank != 0:
            return 0
        fn = measure_prefill if a.workload == "prefill" else measure_sparse
        line = fn(a, dev, with_cpu=not a.no_cpu_baseline)
        line.update({"n_gpus": 1, "scaling": "weak", "vs_baseline": None})
        print(json.dumps(line))
        return 0

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    headline = (a.workload == "decode" and not a.append and a.kv == "bf16" and a.B == 64
                and a.ctx == 2048 and a.splits == 0 and not a.no_pack)
    line = measure_decode(a, dev, rank, world, dist, with_cpu=not a.no_cpu_baseline)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    if headline and world == 1 and not a.no_secondary:
        sec = []
        pa = parse(["--steps", str(a.steps), "--warmup", str(a.warmup), "--workload", "prefill",
                    "--repeat-seconds", str(a.repeat_seconds), "--cpu-seconds", str(a.cpu_seconds)])
        sec.append(_secondary_summary(measure_prefill(pa, dev, with_cpu=not a.no_cpu_baseline)))
        la = parse(["--steps", str(a.steps), "--warmup", str(a.warmup), "--workload", "long70b",
                    "--kv", "fp8_e4m3", "--repeat-seconds", str(a.repeat_seconds)])
        sec.append(_secondary_summary(measure_decode(la, dev, 0, 1, None, with_cpu=False)))
        sa = parse(["--steps", str(a.steps), "--warmup", str(a.warmup), "--workload", "sparse70b",
                    "--repeat-seconds", str(a.repeat_seconds), "--cpu-seconds", str(a.cpu_seconds)])
        sec.append(_secondary_summary(measure_sparse(sa, dev, with_cpu=not a.no_cpu_baseline)))
        line["secondary"] = sec
    print(json.dumps(line))
    return 0


def reference_arm(a, world):
    """The fp64 CPU oracle, timed on the host cores, on a bounded sample of the same
    workload (rank 0 only)."""
    import torch  # noqa: F401  (input generation)
    from gqa_attention_paged_b200 import inputs

    case = inputs.sweep_decode(a.B, seed=a.seed, ctx=a.ctx, kv_dtype=a.kv)
    elem = 1 if a.kv == "fp8_e4m3" else 2
    rows = [0, 1]
    per_step = []
    cores = 1
    for _ in range(max(1, a.warmup) // 3):
        run_oracle_sample(case, rows, 0.0)
    for _ in range(a.steps):
        sec, reps, cores = run_oracle_sample(case, rows, 0.0)
        per_step.append(sec)
    sec = sum(per_step) / len(per_step)
    lens = [int(x) for x in case.kv.seq_lens]
    sb = decode_step_bytes([lens[r] for r in rows], 32, 8, 128, elem, 16)
    v = sb / sec / 1e9
    line = {
        "impl": "reference",
        "metric": decode_metric(a), "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(sec * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": workload_name(a), "B_per_gpu": a.B, "ctx": a.ctx,
                   "sample": f"{len(rows)} of {a.B} sequences per step"},
        "spread": spread([s * 1e3 for s in per_step]),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{len(rows)} of {a.B} sequences per step, {a.steps} steps"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
