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
    """roofline.traffic comes from an ncu capture only while the attention
    kernels' sources hash to the captured ones: a tree whose capture matches
    gives the figure, an unknown workload none, an edited source none."""
    import hashlib
    import json
    import shutil

    import bench
    names = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["sources"]
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    csrc = fake / "decode_attention_rank_mlra_b200" / "csrc"
    csrc.mkdir(parents=True)
    h = hashlib.sha256()
    for n in names:
        shutil.copy(os.path.join(ROOT, "decode_attention_rank_mlra_b200", "csrc", n), csrc)
        h.update((csrc / n).read_bytes())
    json.dump({"sources": names, "sources_sha256": h.hexdigest(),
               "workloads": {"w": {"dram_bytes_per_launch": 123, "profile": "p.md"}}},
              open(fake / "profiles" / "traffic.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.measured_traffic("w") == (123, "p.md")
    got, src = bench.measured_traffic("no_such_workload")
    assert got is None and "no ncu capture" in src
    with open(csrc / names[0], "a") as f:
        f.write("\n// edited\n")
    got, src = bench.measured_traffic("w")
    assert got is None and "changed" in src
