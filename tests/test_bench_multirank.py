"""The bench's multi-rank plumbing on CPU: two gloo ranks, max over ranks,
whole-job aggregation, and rank-0-only output of the reference arm."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) ms in total and 10 - r ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank])
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(",".join(repr(v) for v in got))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        vals = [float(x) for x in (tmp_path / f"rank{r}.txt").read_text().split(",")]
        assert vals == [2.0, 10.0, 0.5]


def test_single_rank_is_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]


def test_aggregate_is_whole_job_weak_scaling():
    import bench
    # 8 replicas x 16 sequences each, 0.05 ms per step (slowest rank)
    assert bench.aggregate_rate(8, 16, 0.05) == pytest.approx(8 * 16 / 0.05e-3)
    assert bench.aggregate_rate(1, 16, 0.05) * 8 == pytest.approx(bench.aggregate_rate(8, 16, 0.05))


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    import bench

    class Args:
        workload = "mlra4_f32_b1_h4_l256"
        steps = 1
        warmup = 0
        impl = "reference"

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(Args()) is None
    monkeypatch.setenv("RANK", "0")
    res = bench.run_reference(Args())
    assert res["impl"] == "reference" and res["value"] > 0
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["cpu_baseline"]["kind"] == "oracle"


def test_traffic_only_for_the_captured_kernel_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from an ncu capture only while the sources of the
    kernel it was measured on hash to the captured ones: a matching entry gives
    the figure, an unknown workload none, an edited source none (for the
    workloads that depend on it only)."""
    import hashlib
    import json
    import shutil

    import bench
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    csrc = fake / "decode_attention_rank_mlra_b200" / "csrc"
    csrc.mkdir(parents=True)
    names = ["k_decode_tc.cu", "k_decode_wide.cu", "tc_common.cuh"]
    for n in names:
        shutil.copy(os.path.join(ROOT, "decode_attention_rank_mlra_b200", "csrc", n), csrc)

    def sha(files):
        h = hashlib.sha256()
        for n in files:
            h.update((csrc / n).read_bytes())
        return h.hexdigest()

    a_src, b_src = ["k_decode_tc.cu", "tc_common.cuh"], ["k_decode_wide.cu", "tc_common.cuh"]
    json.dump({"workloads": {
        "a": {"dram_bytes_per_launch": 123, "profile": "p.md", "sources": a_src,
              "sources_sha256": sha(a_src)},
        "b": {"dram_bytes_per_launch": 456, "profile": "q.md", "sources": b_src,
              "sources_sha256": sha(b_src)}}},
        open(fake / "profiles" / "traffic.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.measured_traffic("a") == (123, "p.md")
    assert bench.measured_traffic("b") == (456, "q.md")
    got, src = bench.measured_traffic("no_such_workload")
    assert got is None and "no ncu capture" in src
    with open(csrc / "k_decode_tc.cu", "a") as f:
        f.write("\n// edited\n")
    got, src = bench.measured_traffic("a")
    assert got is None and "changed" in src
    assert bench.measured_traffic("b") == (456, "q.md")


def test_committed_traffic_entries_name_their_kernel_sources():
    """Every committed entry lists the files its figure depends on."""
    import json
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for w, e in t["workloads"].items():
        assert e["sources"] and len(e["sources_sha256"]) == 64, w
        for n in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "decode_attention_rank_mlra_b200", "csrc", n))


def test_both_arms_print_the_same_config(monkeypatch):
    """The reference arm's config object is the one our arm prints (built from
    the workload alone, no device needed), for every workload."""
    import bench
    import workloads as W
    for name in bench.PER_CONFIG:
        spec = W.WORKLOADS[name]
        c = bench.workload_config(spec, 1)
        assert c["workload"] == name and c["cached_tokens"] == int(W.seqlens_for(spec).sum())
        copies = bench.cache_copies(spec)
        nbytes = bench.cache_elems(spec) * spec.elem_bytes
        # rotating copies exceed three L2s, else one copy already does, else flush
        assert (copies > 1 and copies * nbytes > 3 * bench.L2_BYTES) or \
            (copies == 1 and nbytes > 3 * bench.L2_BYTES) or (copies == 0 and 8 * nbytes <= 3 * bench.L2_BYTES)
        assert ("flushed" in c["l2"]) == (copies == 0)

    class Args:
        workload = "mlra4_f32_b1_h4_l256"
        steps = 1
        warmup = 0
        impl = "reference"

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    res = bench.run_reference(Args())
    assert res["config"] == bench.workload_config(W.WORKLOADS[Args.workload], 1)


def test_default_headline_is_the_largest_workload():
    import bench
    import workloads as W
    sizes = {n: int(W.seqlens_for(W.WORKLOADS[n]).sum()) * W.WORKLOADS[n].D
             * W.WORKLOADS[n].elem_bytes for n in bench.PER_CONFIG}
    assert bench.DEFAULT_WORKLOAD == max(sizes, key=sizes.get)
    assert bench.parse([]).workload == bench.DEFAULT_WORKLOAD
    assert bench.split_workloads("all", bench.DEFAULT_WORKLOAD) == [
        n for n in bench.PER_CONFIG if n != bench.DEFAULT_WORKLOAD]
    assert bench.split_workloads("none", bench.DEFAULT_WORKLOAD) == []


def test_batch_option_runs_a_smaller_case_of_the_same_workload():
    """--batch N keeps the workload's shape, layout and length law with N sequences."""
    import bench
    import workloads as W
    a = bench.parse(["--workload", "mlra4_bf16_b128_h16_ragged1k_64k_paged", "--batch", "16"])
    full, small = W.WORKLOADS[a.workload], bench.workload_spec(W, a)
    assert small.batch == 16 and small.ragged == full.ragged and small.paged == full.paged
    assert (small.n_heads, small.n_blocks, small.d_cb, small.d_r) == (
        full.n_heads, full.n_blocks, full.d_cb, full.d_r)
    assert bench.workload_spec(W, bench.parse(["--workload", a.workload])) is full


def test_launch_count_includes_the_range_recompute_launch_at_128_heads():
    import bench
    import workloads as W
    counts = {n: bench.kernels_per_step(W.WORKLOADS[n]) for n in bench.PER_CONFIG}
    assert counts["mla_bf16_b8_h128_l131072_paged"] == 5
    assert counts["mlra4_bf16_b8_h128_l131072_paged"] == 5
    assert counts["mlra4_bf16_b128_h16_ragged1k_64k_paged"] == 4
