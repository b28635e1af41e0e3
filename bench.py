#!/usr/bin/env python
"""Benchmark of one MLRA / MLA latent-KV decode step on B200.

A step is the whole hot path: absorb_q -> decode_attn (plan + split-KV
attention) -> combine_out_proj (split-KV merge fused with the output
projection), through the C ABI, on one batch of synthetic seeded inputs
already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--no-cpu-baseline]
                  [--per-config all|none|NAME,NAME...] [--batch N]

Prints ONE JSON line (rank 0).  The headline is the largest single-GPU
workload (the ragged batch of 128 sequences, 4.9 GB of cache): value = decode
tokens/s (sequences decoded per second: one new token each) aggregated over
all ranks; the roofline object reports the attention kernel's achieved HBM
GB/s against the measured copy bandwidth.  ``per_config`` repeats the same
measurements on every workload (the fp32 one, the contiguous one, the paged
one, the ragged one, MLA and MLRA-4 at 128 heads).

Timing: W untimed warm-up steps, then regions of exactly K steps, each
bracketed by a barrier and a device synchronisation, each timed with CUDA
events on the launching stream and maxed over ranks; regions repeat until
0.5 s of device time has accumulated and the median region is reported.
Between timed steps the KV cache rotates over several identical copies whose
total exceeds the 126 MB L2 (or a single copy is already larger), so every
step reads its cache from HBM.  Multi-GPU runs are independent replicas (weak
scaling): the step has no exchange between sequences.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("latent-KV decode attn: achieved HBM GB/s & % roofline; decode tokens/s at 1 B200")
DEFAULT_WORKLOAD = "mlra4_bf16_b128_h16_ragged1k_64k_paged"
PER_CONFIG = ["mlra4_f32_b1_h4_l256", "mlra4_bf16_b16_h16_l4096_contig",
              "mlra4_bf16_b64_h32_l16384_paged", "mlra4_bf16_b128_h16_ragged1k_64k_paged",
              "mla_bf16_b8_h128_l131072_paged", "mlra4_bf16_b8_h128_l131072_paged"]
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
MIN_TIMED_S = 0.5


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--per-config", default="all",
                   help="workloads measured besides the headline: all, none, or a comma list")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="bound on the oracle's CPU work for the baseline sample")
    p.add_argument("--batch", type=int, default=0,
                   help="run the workload with this many sequences instead (same lengths, "
                        "same layout): a smaller case of the same kernels, for profiling")
    return p.parse_args(argv)


def workload_spec(W, args):
    """The named workload, or (--batch) a smaller case of it with that many sequences."""
    spec = W.WORKLOADS[args.workload]
    batch = getattr(args, "batch", 0)
    if batch > 0 and batch != spec.batch:
        spec = W.scaled_down(spec, batch, seqlen=spec.seqlen, ragged=spec.ragged)
    return spec


def kernels_per_step(spec) -> int:
    """Launches of the library per decode step: absorb, plan, attention, merge +
    projection, and for the 128-head kernels (fp16 tile) the bf16 launch that
    recomputes the call if a cache value left the fp16 range (it returns at
    once otherwise)."""
    wide = spec.dtype == "bf16" and spec.n_heads % 128 == 0 and (
        (spec.n_blocks == 1 and spec.d_cb == 512) or (spec.d_cb == 128 and spec.n_heads == 128))
    return 5 if wide else 4


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------------------
# workload description shared by both arms
# ---------------------------------------------------------------------------
def cache_elems(spec) -> int:
    """Elements of the cache tensor the workload allocates (paged or contiguous)."""
    import workloads as W
    sl = W.seqlens_for(spec)
    if spec.paged:
        _, total = W.page_layout(spec, sl)
        return max(total, 1) * W.PAGE_SIZE * spec.D
    return spec.batch * max(int(sl.max()), 1) * spec.D


def cache_copies(spec) -> int:
    """Identical cache copies the timed loop rotates over: together (and each,
    when one is already larger) more than three times the L2.  0 when eight
    copies would not be enough: such a small workload is timed step by step
    with a write of twice the L2 between steps instead."""
    nbytes = cache_elems(spec) * spec.elem_bytes
    need = int(np.ceil(3 * L2_BYTES / max(nbytes, 1)))
    return max(1, need) if need <= 8 else 0


def workload_config(spec, world: int) -> dict:
    """The ``config`` object of the JSON line (identical in both arms)."""
    import workloads as W
    sl = W.seqlens_for(spec)
    copies = cache_copies(spec)
    mib = max(copies, 1) * cache_elems(spec) * spec.elem_bytes / 2 ** 20
    if copies == 0:
        l2 = (f"KV cache of {mib:.2f} MiB: L2 flushed before every step (a {2 * L2_BYTES >> 20} "
              "MiB write outside the step's event pair), each step timed alone")
    elif copies == 1:
        l2 = f"KV cache of {mib:.0f} MiB > 126 MB L2, read once per step"
    else:
        l2 = f"KV cache rotated over {copies} copies ({mib:.0f} MiB > 126 MB L2)"
    return {
        "workload": spec.name, "batch": spec.batch, "heads": spec.n_heads,
        "n_blocks": spec.n_blocks, "d_cb": spec.d_cb, "d_r": spec.d_r,
        "seqlen": spec.seqlen if spec.ragged is None else f"U{list(spec.ragged)}",
        "cached_tokens": int(sl.sum()), "paged": spec.paged,
        "parallelism": f"replicas x{world}", "l2": l2,
    }


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample of the workload
# ---------------------------------------------------------------------------
_SEQ_CACHE = {}


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # pragma: no cover
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(spec, seconds: float):
    """Time the fp64 oracle, as it stands, on whole (sequence, head) pairs.

    Pairs are taken in order (sequence 0 head 0, head 1, ...) until ``seconds``
    of oracle time have accumulated (at least one pair).  Value = sequences per
    second, where a sequence counts as the fraction of its heads done.  Input
    generation is excluded and cached between calls.
    """
    import oracle
    import workloads as W
    from oracle.mlra_oracle import split_cache_rows

    key = spec.name
    if key not in _SEQ_CACHE:
        w_uk, w_uv = W.weights(spec)
        q_nope, q_rope = W.queries(spec)
        _SEQ_CACHE[key] = dict(w=(w_uk, w_uv), q=(q_nope, q_rope), seqlens=W.seqlens_for(spec),
                               rows={})
    C = _SEQ_CACHE[key]
    w_uk, w_uv = C["w"]
    q_nope, q_rope = C["q"]
    elapsed, pairs, tokens, seqs = 0.0, 0, 0, 0.0
    for s in range(spec.batch):
        L = int(C["seqlens"][s])
        if s not in C["rows"]:
            C["rows"] = {s: split_cache_rows(W.token_rows(spec, s, 0, L), spec.n_blocks, spec.d_cb)}
        c, kr = C["rows"][s]
        for hh in range(spec.n_heads):
            t0 = time.perf_counter()
            oracle.decode_sequence(q_nope[s], q_rope[s], c, kr, w_uk, w_uv, spec.softmax_scale,
                                   spec.branch_scale, heads=[hh])
            elapsed += time.perf_counter() - t0
            pairs += 1
            seqs += 1.0 / spec.n_heads
            tokens += L
            if elapsed >= seconds:
                break
        if elapsed >= seconds:
            break
    sample = (f"{pairs} (sequence, head) pairs, all {spec.n_blocks} branches each = {seqs:.3g} "
              f"sequences of workload {spec.name} ({tokens} cached tokens x head); fp64 numpy, "
              f"input generation excluded")
    return dict(value=seqs / elapsed, unit="tokens/s", cores=_blas_threads(), kind="oracle",
                sample=sample, seconds=elapsed)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling every 25 ms in one long-running process; each line is
    stamped with the host clock when it arrives."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._proc = None
        self._th = None

    def _read(self):
        for line in self._proc.stdout:
            line = line.strip()
            if line:
                self.samples.append((time.perf_counter(), [x.strip() for x in line.split(",")]))

    def start(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self._proc = None
            return
        self._th = threading.Thread(target=self._read, daemon=True)
        self._th.start()

    def stop(self):
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        if self._th:
            self._th.join(timeout=5)

    def summary(self, windows):
        """Clock summary over the samples inside the wall-clock ``windows``
        [(t0, t1), ...] (all samples when none falls inside)."""
        inside = [s for t, s in self.samples if any(a <= t <= b for a, b in windows)]
        use = inside or [s for _, s in self.samples]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        sm = [float(s[1]) for s in use if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in use if s[2].replace(".", "").isdigit()]
        pw = [float(s[3]) for s in use if s[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in use for i in range(4)
                          if len(s) > 5 + i and s[5 + i].strip().lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w_max": max(pw) if pw else None,
                "samples": len(use), "samples_in_timed_region": len(inside)}


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the process group (identity
    on one rank).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def aggregate_rate(world: int, batch: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank decodes `batch` sequences per step (weak
    scaling, independent replicas); the step time is the slowest rank's."""
    return world * batch / (ms_per_step * 1e-3)


def measured_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu capture, or None.

    Each workload's figure is used only while the sources of the kernel it was
    measured on are unchanged (their sha256 is stored beside it).
    """
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        w = t["workloads"].get(workload)
        if w is None:
            return None, "no ncu capture for this workload"
        h = hashlib.sha256()
        csrc = os.path.join(ROOT, "decode_attention_rank_mlra_b200", "csrc")
        for name in w["sources"]:
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != w["sources_sha256"]:
            return None, "kernel changed since the ncu capture"
        return int(w["dram_bytes_per_launch"]), w["profile"]
    except Exception as e:  # pragma: no cover
        return None, f"unavailable ({type(e).__name__})"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def split_workloads(arg: str, headline: str):
    if arg == "none":
        return []
    names = PER_CONFIG if arg == "all" else [n for n in arg.split(",") if n]
    return [n for n in names if n != headline]


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Timer:
    """Repeated regions of exactly K steps, each bracketed by a barrier and a
    device synchronisation and timed with one CUDA event pair on ``stream``;
    each region's time is the max over ranks.  Regions repeat until
    MIN_TIMED_S of device time has accumulated (at least ``min_regions``).
    A body that returns event pairs (steps timed one by one, with an L2 flush
    between them) is timed by their sum."""

    def __init__(self, stream, world, dev):
        self.stream, self.world, self.dev = stream, world, dev
        self.windows = []

    def run(self, body, min_regions=1, max_regions=400):
        import torch
        import torch.distributed as dist
        times = []
        while (len(times) < min_regions or sum(times) < MIN_TIMED_S * 1e3) \
                and len(times) < max_regions:
            if self.world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            w0 = time.perf_counter()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            pairs = body()
            e1.record(self.stream)
            torch.cuda.synchronize()
            if self.world > 1:
                dist.barrier()
            self.windows.append((w0, time.perf_counter()))
            t = e0.elapsed_time(e1) if pairs is None else sum(a.elapsed_time(b) for a, b in pairs)
            times.append(max_over_ranks([t], self.dev)[0])
        return float(np.median(times)), len(times)


def measure(spec, args, dev, world, timer, full: bool):
    """Time one workload: the step (device-resident inputs), the attention
    call alone (per launch and back to back) and the one-call step from
    page-locked host buffers.  ``full`` adds the per-call breakdown."""
    import torch

    import decode_attention_rank_mlra_b200 as mlra
    import workloads as W

    inp = W.make_inputs(spec, dev)
    cfg = mlra.make_config(spec.n_blocks, spec.d_cb, spec.d_r, spec.n_heads, spec.d_h,
                           dtype=spec.torch_dtype, softmax_scale=spec.softmax_scale,
                           branch_scale=spec.branch_scale)
    B = spec.batch
    K = args.steps
    tokens = int(inp.seqlens.sum().item())
    cache_bytes = tokens * spec.D * spec.elem_bytes           # algorithmic bytes per launch
    flush = cache_copies(spec) == 0
    copies = max(cache_copies(spec), 1)
    assert flush or copies * inp.kv_cache.numel() * spec.elem_bytes > 3 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None

    def flush_l2():
        flush_buf.fill_(1.0)

    def one_by_one(fn):
        """K steps timed one by one, L2 flushed before each (outside its pair)."""
        pairs = []
        for i in range(K):
            flush_l2()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn(i)
            b.record(stream)
            pairs.append((a, b))
        return pairs

    cycle = copies * max(1, (4 + copies - 1) // copies)  # steps per captured cycle, >= 4
    caches = [inp.kv_cache] + [inp.kv_cache.clone() for _ in range(copies - 1)]
    max_pages = inp.page_table.shape[1] if inp.page_table is not None else inp.max_len
    dec = mlra.Decoder(cfg, B, dev)
    stream = torch.cuda.current_stream()
    kind = mlra.decode_kernel_kind(cfg)

    def step(i):
        mlra.absorb_q(cfg, inp.q_nope, inp.w_uk, dec.q_abs)
        mlra.decode_attn(cfg, dec.q_abs, inp.q_rope, caches[i % copies], inp.page_table,
                         inp.seqlens, max_pages, dec.workspace)
        return mlra.combine_out_proj(cfg, dec.workspace, B, inp.w_uv, dec.out, dec.o_latent,
                                     dec.lse)

    def attn(i):
        mlra.decode_attn(cfg, dec.q_abs, inp.q_rope, caches[i % copies], inp.page_table,
                         inp.seqlens, max_pages, dec.workspace)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if mlra.get_device_error(dec.workspace) != 0:
        raise RuntimeError(f"{spec.name}: device error during warm-up")

    # CUDA graphs: the step per cache copy, the attention call alone per copy,
    # `cycle` consecutive steps (the decode loop as served: consecutive steps
    # overlap their launch prologues like the kernels inside a step do), and
    # n_rep attention calls back to back
    n_rep = 2 * copies
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g_step, g_attn = [], []
    with torch.cuda.stream(side):
        for i in range(copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                step(i)
            g_step.append(g)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                attn(i)
            g_attn.append(g)
        g_cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_cycle, stream=side):
            for i in range(cycle):
                step(i)
        g_b2b = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_b2b, stream=side):
            for i in range(n_rep):
                attn(i)
    stream.wait_stream(side)
    for i in range(max(2 * copies, args.warmup)):
        g_step[i % copies].replay()
        g_attn[i % copies].replay()
    g_cycle.replay()
    g_b2b.replay()
    torch.cuda.synchronize()

    # ---- the step: regions of exactly K steps --------------------------------
    def k_steps():
        if flush:
            return one_by_one(lambda i: g_step[0].replay())
        for _ in range(K // cycle):
            g_cycle.replay()
        for i in range(K % cycle):
            g_step[i % copies].replay()

    ms_region, n_regions = timer.run(k_steps)
    ms_step = ms_region / K
    # ---- the attention call alone: one event pair per launch -----------------
    n_launch = max(K, 20)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_launch)]
    for i in range(n_launch):
        if flush:
            flush_l2()
        kev[i][0].record(stream)
        g_attn[i % copies].replay()
        kev[i][1].record(stream)
    torch.cuda.synchronize()
    k_mean = float(np.mean([a.elapsed_time(b) for a, b in kev]))
    # ... and back to back (n_rep calls in one graph, no launch gaps)
    reps = max(3, min(200, int(np.ceil(0.2e3 / max(k_mean * n_rep, 1e-3)))))
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for _ in range(reps):
        g_b2b.replay()
    b1.record(stream)
    torch.cuda.synchronize()
    # (a cache smaller than L2 stays there across these calls: an L2 figure then)
    k_b2b = b0.elapsed_time(b1) / (reps * n_rep)
    k_mean, k_b2b = max_over_ranks([k_mean, k_b2b], dev)

    # ---- per-call breakdown (headline only) ----------------------------------
    breakdown = None
    if full:
        g_app = torch.Generator().manual_seed(1)
        app_c = torch.randn(B, spec.n_blocks * spec.d_cb, generator=g_app).to(spec.torch_dtype).to(dev)
        app_kr = torch.randn(B, spec.d_r, generator=g_app).to(spec.torch_dtype).to(dev)
        app_gamma = torch.ones(spec.n_blocks * spec.d_cb, dtype=torch.float32, device=dev)
        app_pos = (inp.seqlens - 1).clamp(min=0)
        calls = {
            "absorb_q": lambda i: mlra.absorb_q(cfg, inp.q_nope, inp.w_uk, dec.q_abs),
            "decode_attn": attn,
            "combine_out_proj": lambda i: mlra.combine_out_proj(cfg, dec.workspace, B, inp.w_uv,
                                                                dec.out, dec.o_latent, dec.lse),
            # the same two steps unfused (the step above uses the fused call)
            "splitkv_combine": lambda i: mlra.splitkv_combine(cfg, dec.workspace, B,
                                                              dec.o_latent, dec.lse),
            "out_proj": lambda i: mlra.out_proj(cfg, dec.o_latent, inp.w_uv, dec.out),
            # the cache write (not part of the step): every sequence's last row
            # rewritten from a normalised latent and a rotated RoPE key
            "cache_append": lambda i: mlra.cache_append(cfg, app_c, app_kr, app_gamma, 2.0,
                                                        caches[i % copies], inp.page_table,
                                                        app_pos, max_pages),
        }
        breakdown = {}
        for name, fn in calls.items():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(side):
                with torch.cuda.graph(g, stream=side):
                    for i in range(n_rep):
                        fn(i)
            stream.wait_stream(side)
            g.replay()
            torch.cuda.synchronize()
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            r = max(3, min(50, K // n_rep))
            c0.record(stream)
            for _ in range(r):
                g.replay()
            c1.record(stream)
            torch.cuda.synchronize()
            breakdown[name] = c0.elapsed_time(c1) * 1e3 / (r * n_rep)
            del g

    # ---- end to end: host buffers, transfers inside the timed region ----------
    # One library call per step (mlra_decode_step with host buffers): a staging
    # kernel reads the step's queries and lengths from page-locked host memory,
    # then absorb -> plan + attention -> merge + projection, whose kernel
    # stores the output into page-locked host memory.
    h_qn = inp.q_nope.cpu().pin_memory()
    h_qr = inp.q_rope.cpu().pin_memory()
    h_sl = inp.seqlens.cpu().pin_memory()
    h_out = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()

    def e2e_step(i):
        dec.step(h_qn, h_qr, h_sl, inp.w_uk, inp.w_uv, caches[i % copies], inp.page_table,
                 max_pages, out=h_out)

    for i in range(max(3, 2 * copies)):
        e2e_step(i)
    torch.cuda.synchronize()

    def k_e2e():
        if flush:
            return one_by_one(e2e_step)
        for i in range(K):
            e2e_step(i)

    e2e_region, e2e_regions = timer.run(k_e2e)
    if mlra.get_device_error(dec.workspace) != 0:
        raise RuntimeError(f"{spec.name}: device error during timing")
    # the result read back in the last step is the oracle-checked computation
    assert torch.isfinite(h_out).all().item()

    peak, peak_kind = measured_peak()
    achieved = cache_bytes / (k_mean * 1e-3) / 1e9
    achieved_b2b = cache_bytes / (k_b2b * 1e-3) / 1e9
    traffic, traffic_src = measured_traffic(spec.name) if kind == "tcgen05" else (None, "SIMT kernel")
    res = {
        "kernel": kind,
        "step_us": ms_step * 1e3,
        "step_tokens_per_s": aggregate_rate(world, B, ms_step),
        "timed_regions": n_regions,
        "attn_us_per_launch": k_mean * 1e3,
        "attn_us_back_to_back": k_b2b * 1e3,
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic,
            "achieved_back_to_back": achieved_b2b, "frac_back_to_back": achieved_b2b / peak,
            "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "traffic_source": traffic_src,
            "algorithmic_bytes_per_launch": cache_bytes,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
            if peak_kind == "measured" else "fallback 6.65 TB/s",
        },
        "e2e": {"value": aggregate_rate(world, B, e2e_region / K), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h_qn.numel() * h_qn.element_size()
                                          + h_qr.numel() * h_qr.element_size()
                                          + h_sl.numel() * h_sl.element_size()),
                "d2h_bytes_per_step": int(h_out.numel() * h_out.element_size()),
                "timed_regions": e2e_regions},
        "_cycle": cycle, "_copies": copies,
    }
    if breakdown is not None:
        res["breakdown_us"] = breakdown
    del g_step, g_attn, g_cycle, g_b2b, caches, inp, dec
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    import workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    spec = workload_spec(W, args)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(0.3)
    timer = Timer(stream, world, dev)
    head = measure(spec, args, dev, world, timer, full=True)
    head_windows = list(timer.windows)
    per = {}
    for name in split_workloads(args.per_config, spec.name):
        timer.windows = []
        r = measure(W.WORKLOADS[name], args, dev, world, timer, full=False)
        r["clocks"] = sampler.summary(timer.windows)
        r.pop("_cycle"), r.pop("_copies")
        per[name] = r
    sampler.stop()
    result = None
    if rank == 0:
        cycle, copies = head.pop("_cycle"), head.pop("_copies")
        K = args.steps
        e2e = head["e2e"]
        e2e["note"] = ("one mlra_decode_step call per step with page-locked host buffers, "
                       "host-launched: a staging kernel reads the queries and seqlens from "
                       "mapped host memory and the projection kernel stores the output into it, "
                       "every step; the KV cache is device-resident state; median of "
                       f"{e2e['timed_regions']} regions of exactly K steps")
        head_entry = {k: v for k, v in head.items() if k != "breakdown_us"}
        head_entry["clocks"] = sampler.summary(head_windows)
        per = {spec.name: head_entry, **per}
        result = {
            "metric": METRIC, "value": head["step_tokens_per_s"], "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": head["step_us"] * 1e-3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if spec.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(spec, world),
            "decode_kernel": head["kernel"],
            "hbm_gbs_step": head["roofline"]["algorithmic_bytes_per_launch"]
            / (head["step_us"] * 1e-6) / 1e9,
            "roofline": dict(head["roofline"], kernel=(
                "mlra_decode_attn (plan + attention kernel): one CUDA-graph launch per event "
                "pair on the launching stream; achieved = algorithmic bytes / mean launch time")),
            "e2e": e2e,
            "clocks": head_entry["clocks"],
            "breakdown_us": head["breakdown_us"],
            "gpu_launches": kernels_per_step(spec) * K,
            "e2e_gpu_launches": (kernels_per_step(spec) + 1) * K,
            "timing": (f"median of {head['timed_regions']} regions of exactly K={K} steps (each "
                       f"bracketed by barrier + synchronize, CUDA events, max over ranks), "
                       f"repeated until {MIN_TIMED_S} s of device time; a region = K // {cycle} "
                       f"replays of a CUDA graph of {cycle} consecutive steps "
                       f"({kernels_per_step(spec)} kernels each, "
                       f"cache copy step % {copies}) + K % {cycle} single-step graph replays; "
                       "gpu_launches counts one region"),
            "per_config": per,
        }
        if not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(spec, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_reference(args):
    """The oracle timed on the host cores, as it stands, on a bounded sample.

    Each step is a bounded sample of the workload; the whole run is kept to
    about two minutes of oracle time whatever K and W are.
    """
    import workloads as W
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    spec = workload_spec(W, args)
    per_step = min(3.0, max(0.02, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(spec, per_step)
    vals, info, total = [], None, 0.0
    for _ in range(args.steps):
        info = cpu_baseline(spec, per_step)
        vals.append(info["value"])
        total += info["seconds"]
    value = len(vals) / sum(1.0 / v for v in vals)  # sequences / total seconds
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(vals),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(spec, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle",
                         "sample": "per step, on rank 0 only: " + info["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
