#!/usr/bin/env python
"""Benchmark of one MLRA / MLA latent-KV decode step on B200.

A step is the whole hot path: absorb_q -> decode_attn (plan + split-KV
attention) -> combine_out_proj (split-KV merge fused with the output
projection), through the C ABI, on one batch of synthetic seeded inputs
already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--no-cpu-baseline]

Prints ONE JSON line (rank 0).  value = decode tokens/s (sequences decoded per
second: one new token each) aggregated over all ranks; the roofline object
reports the attention kernel's achieved HBM GB/s against the measured copy
bandwidth.  Between timed steps the KV cache rotates over several identical
copies whose total exceeds the 126 MB L2, so every step reads its cache from
HBM.  Multi-GPU runs are independent replicas (weak scaling): the step has no
exchange between sequences.
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
DEFAULT_WORKLOAD = "mlra4_bf16_b16_h16_l4096_contig"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="bound on the oracle's CPU work for the baseline sample")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


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

    def summary(self, t0: float, t1: float):
        inside = [s for t, s in self.samples if t0 <= t <= t1]
        use = inside or [s for _, s in self.samples]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        sm = [float(s[1]) for s in use if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in use if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in use for i in range(4)
                          if len(s) > 5 + i and s[5 + i].strip().lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
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

    The figure is used only while the attention kernel's sources are the ones
    it was measured on (their sha256 is stored beside it).
    """
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        h = hashlib.sha256()
        csrc = os.path.join(ROOT, "decode_attention_rank_mlra_b200", "csrc")
        for name in t["sources"]:
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != t["sources_sha256"]:
            return None, "kernel changed since the ncu capture"
        w = t["workloads"].get(workload)
        if w is None:
            return None, "no ncu capture for this workload"
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


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    import decode_attention_rank_mlra_b200 as mlra
    import workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    spec = W.WORKLOADS[args.workload]
    inp = W.make_inputs(spec, dev)
    cfg = mlra.make_config(spec.n_blocks, spec.d_cb, spec.d_r, spec.n_heads, spec.d_h,
                           dtype=spec.torch_dtype, softmax_scale=spec.softmax_scale,
                           branch_scale=spec.branch_scale)
    B = spec.batch
    seqlens_np = inp.seqlens.cpu().numpy()
    tokens = int(seqlens_np.sum())
    cache_bytes = tokens * spec.D * spec.elem_bytes           # algorithmic bytes per launch
    copies = max(1, min(8, int(np.ceil(3 * L2_BYTES / max(inp.kv_cache.numel() * spec.elem_bytes, 1)))))
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

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if mlra.get_device_error(dec.workspace) != 0:
        raise RuntimeError("device error during warm-up")

    # One CUDA graph per cache copy for the whole step, and one for the
    # attention call alone (plan + attention kernel) to time that kernel.
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
                mlra.decode_attn(cfg, dec.q_abs, inp.q_rope, caches[i], inp.page_table,
                                 inp.seqlens, max_pages, dec.workspace)
            g_attn.append(g)
        # the decode loop as served: one graph holds `cycle` consecutive steps
        # (cache copy i % copies; every copy, and every set of copies, is larger
        # than L2), so consecutive steps overlap their launch prologues like the
        # kernels inside a step do
        g_cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_cycle, stream=side):
            for i in range(cycle):
                step(i)
    stream.wait_stream(side)
    # every captured graph is launched at least twice before anything is timed
    for i in range(max(2 * copies, args.warmup)):
        g_step[i % copies].replay()
        g_attn[i % copies].replay()
    g_cycle.replay()
    g_cycle.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(0.3)
    # ---- timed region: exactly K steps --------------------------------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    # exactly K steps: K // cycle cycles, then the remaining single steps
    for _ in range(args.steps // cycle):
        g_cycle.replay()
    for i in range(args.steps % cycle):
        g_step[i % copies].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.perf_counter()
    ms_total = e0.elapsed_time(e1)
    # ---- the attention kernel alone: one event pair per launch ---------------
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        kev[i][0].record(stream)
        g_attn[i % copies].replay()
        kev[i][1].record(stream)
    torch.cuda.synchronize()
    k_ms = [a.elapsed_time(b) for a, b in kev]
    # ---- per-call breakdown: each call captured N times back to back in one
    # CUDA graph (device time per call, no host launch gaps) -------------------
    calls = {
        "absorb_q": lambda i: mlra.absorb_q(cfg, inp.q_nope, inp.w_uk, dec.q_abs),
        "decode_attn": lambda i: mlra.decode_attn(cfg, dec.q_abs, inp.q_rope, caches[i % copies],
                                                  inp.page_table, inp.seqlens, max_pages,
                                                  dec.workspace),
        "combine_out_proj": lambda i: mlra.combine_out_proj(cfg, dec.workspace, B, inp.w_uv,
                                                            dec.out, dec.o_latent, dec.lse),
        # the same two steps unfused (the step above uses the fused call)
        "splitkv_combine": lambda i: mlra.splitkv_combine(cfg, dec.workspace, B, dec.o_latent,
                                                          dec.lse),
        "out_proj": lambda i: mlra.out_proj(cfg, dec.o_latent, inp.w_uv, dec.out),
        # the cache-write step (not part of the step above): every sequence's
        # last row rewritten from a normalised latent and a rotated RoPE key
        "cache_append": lambda i: mlra.cache_append(cfg, app_c, app_kr, app_gamma, 2.0,
                                                    caches[i % copies], inp.page_table, app_pos,
                                                    max_pages),
    }
    g_app = torch.Generator().manual_seed(1)
    app_c = torch.randn(B, spec.n_blocks * spec.d_cb, generator=g_app).to(spec.torch_dtype).to(dev)
    app_kr = torch.randn(B, spec.d_r, generator=g_app).to(spec.torch_dtype).to(dev)
    app_gamma = torch.ones(spec.n_blocks * spec.d_cb, dtype=torch.float32, device=dev)
    app_pos = (inp.seqlens - 1).clamp(min=0)
    breakdown = {}
    n_rep = 2 * copies
    for name, fn in calls.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(n_rep):
                    fn(i)
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        b0 = torch.cuda.Event(enable_timing=True)
        b1 = torch.cuda.Event(enable_timing=True)
        reps = max(3, min(50, args.steps // n_rep))
        b0.record(stream)
        for _ in range(reps):
            g.replay()
        b1.record(stream)
        torch.cuda.synchronize()
        breakdown[name] = b0.elapsed_time(b1) * 1e3 / (reps * n_rep)
        del g
    # ---- end-to-end: host buffers, copies inside the timed region ------------
    # One library call per step (mlra_decode_step with host buffers): a
    # staging kernel reads the step's queries and seqlens from page-locked
    # host memory, then absorb -> plan + attention -> merge + projection, whose
    # kernel stores the output into page-locked host memory.
    h_qn = inp.q_nope.cpu().pin_memory()
    h_qr = inp.q_rope.cpu().pin_memory()
    h_sl = inp.seqlens.cpu().pin_memory()
    h_out = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    e2e_steps = max(1, args.steps)

    def e2e_step(i):
        dec.step(h_qn, h_qr, h_sl, inp.w_uk, inp.w_uv, caches[i % copies], inp.page_table,
                 max_pages, out=h_out)

    for i in range(max(3, min(args.warmup, 2 * copies))):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)
    sampler.stop()
    if mlra.get_device_error(dec.workspace) != 0:
        raise RuntimeError("device error during timing")

    # max over ranks
    ms_total, e2e_ms, k_mean = max_over_ranks([ms_total, e2e_ms, float(np.mean(k_ms))], dev)
    ms_step = ms_total / args.steps
    value = aggregate_rate(world, B, ms_step)
    peak, peak_kind = measured_peak()
    achieved = cache_bytes / (k_mean * 1e-3) / 1e9
    traffic, traffic_src = measured_traffic(spec.name) if kind == "tcgen05" else (None, "SIMT kernel")
    result = None
    if rank == 0:
        clocks = sampler.summary(t_wall0, t_wall1)
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if spec.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {
                "workload": spec.name, "batch": B, "heads": spec.n_heads,
                "n_blocks": spec.n_blocks, "d_cb": spec.d_cb, "d_r": spec.d_r,
                "seqlen": spec.seqlen if spec.ragged is None else f"U{list(spec.ragged)}",
                "cached_tokens": tokens, "paged": spec.paged, "parallelism": f"replicas x{world}",
                "decode_kernel": kind,
                "l2": f"KV cache rotated over {copies} copies "
                      f"({copies * inp.kv_cache.numel() * spec.elem_bytes / 2**20:.0f} MiB > 126 MB L2)",
            },
            "hbm_gbs_step": cache_bytes / (ms_step * 1e-3) / 1e9,
            "roofline": {
                "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_src,
                "kernel": "mlra_decode_attn (plan + attention kernel): one CUDA-graph launch per event pair on the launch stream, K launches",
                "algorithmic_bytes_per_launch": cache_bytes,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
            },
            "e2e": {"value": aggregate_rate(world, B, e2e_ms / e2e_steps), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h_qn.numel() * h_qn.element_size()
                                              + h_qr.numel() * h_qr.element_size()
                                              + h_sl.numel() * h_sl.element_size()),
                    "d2h_bytes_per_step": int(h_out.numel() * h_out.element_size()),
                    "note": "one mlra_decode_step call per step with page-locked host buffers, "
                            "host-launched (no graph): a staging kernel reads the queries and "
                            "seqlens from mapped host memory and the projection kernel stores "
                            "the output into it, every step; the KV cache is device-resident "
                            "state"},
            "clocks": clocks,
            "breakdown_us": breakdown,
            "gpu_launches": 4 * args.steps,
            "e2e_gpu_launches": 5 * e2e_steps,
            "timing": (f"K steps = K // {cycle} replays of a CUDA graph of {cycle} consecutive steps "
                       f"(4 kernels each, cache copy step % {copies}) + K % {cycle} single-step "
                       "graph replays; one event pair around all K"),
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
    spec = W.WORKLOADS[args.workload]
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
        "config": {"workload": spec.name, "batch": spec.batch, "heads": spec.n_heads,
                   "n_blocks": spec.n_blocks, "parallelism": "none (host cores, rank 0)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle", "sample": "per step: " + info["sample"]},
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
