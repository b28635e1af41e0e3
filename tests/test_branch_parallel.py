"""Branch-parallel decoding on CPU: the shard helpers and the sum over ranks.

Four gloo ranks each hold one latent branch of an MLRA-4 layer (its cache
columns plus the shared RoPE key, its slices of W_uk / W_uv, the layer's
branch rescale), compute their share with the fp64 oracle, and sum over the
group with the module's all-reduce: the result must be the oracle's
single-device MLRA-4 output ("Multi-Head Low-Rank Attention", Key
Contributions #2; Main Findings, second bullet).  The CUDA kernels are not
involved here; tests/test_gpu_branch_parallel.py runs the shards through them.
"""
import os
import socket
import sys

import numpy as np
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


def _inputs():
    import workloads as W
    base = W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"]
    spec = W.scaled_down(base, 3, seqlen=300, n_heads=4, seed=51)
    return W.make_inputs(spec, "cpu", seqlens=np.asarray([300, 65, 1], np.int32))


def _cfg(spec):
    import decode_attention_rank_mlra_b200 as mlra
    return mlra.make_config(spec.n_blocks, spec.d_cb, spec.d_r, spec.n_heads, spec.d_h,
                            dtype=spec.torch_dtype, softmax_scale=spec.softmax_scale,
                            branch_scale=spec.branch_scale)


def _local_oracle(inp, cfg, world, rank):
    """This rank's partial output [B, h, d_h] from the oracle on its shard."""
    import oracle
    import workloads as W
    from decode_attention_rank_mlra_b200 import branch_parallel as bp
    from oracle.mlra_oracle import split_cache_rows
    lc = bp.local_config(cfg, world)
    cache = bp.shard_cache(inp.kv_cache, cfg, world, rank)
    w_uk = bp.shard_weights(inp.w_uk, cfg, world, rank)
    w_uv = bp.shard_weights(inp.w_uv, cfg, world, rank)
    local = W.DecodeInputs(spec=inp.spec.replace(n_blocks=lc.n_blocks), seqlens=inp.seqlens,
                           q_nope=inp.q_nope, q_rope=inp.q_rope, w_uk=w_uk, w_uv=w_uv,
                           kv_cache=cache, page_table=inp.page_table, max_len=inp.max_len)
    outs = []
    for s in range(inp.spec.batch):
        rows = W.sequence_cache(local, s)
        c, kr = split_cache_rows(rows, lc.n_blocks, lc.d_cb)
        # (the layer's scales in fp64: the config struct holds them as fp32)
        r = oracle.decode_sequence(inp.q_nope[s], inp.q_rope[s], c, kr, w_uk, w_uv,
                                   inp.spec.softmax_scale, inp.spec.branch_scale)
        outs.append(r.out)
    return torch.from_numpy(np.stack(outs))


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from decode_attention_rank_mlra_b200 import branch_parallel as bp
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs()
        out = _local_oracle(inp, _cfg(inp.spec), world, rank)
        bp.reduce_branch_outputs(out)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), out.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [4, 2])
def test_branch_shards_sum_to_the_single_device_output(tmp_path, world):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import oracle
    inp = _inputs()
    ref = np.stack([r.out for r in oracle.decode_batch(inp)])
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npy")
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_shards_hold_their_blocks_and_the_rope_key():
    from decode_attention_rank_mlra_b200 import branch_parallel as bp
    inp = _inputs()
    cfg = _cfg(inp.spec)
    d_cb, nb = cfg.d_cb, cfg.n_blocks
    bits = lambda t: t.view(torch.int16)   # rows past a sequence's end are uninitialised
    for world in (1, 2, 4):
        cols = []
        for r in range(world):
            sh = bp.shard_cache(inp.kv_cache, cfg, world, r)
            per = nb // world
            assert sh.shape == inp.kv_cache.shape[:-1] + (per * d_cb + cfg.d_r,)
            assert torch.equal(bits(sh[..., per * d_cb:]), bits(inp.kv_cache[..., nb * d_cb:]))
            cols.append(sh[..., : per * d_cb])
            w = bp.shard_weights(inp.w_uk, cfg, world, r)
            assert torch.equal(w, inp.w_uk[r * per:(r + 1) * per])
            lc = bp.local_config(cfg, world)
            assert lc.n_blocks == per and lc.branch_scale == cfg.branch_scale
            assert lc.softmax_scale == cfg.softmax_scale and lc.D == per * d_cb + cfg.d_r
        assert torch.equal(bits(torch.cat(cols, -1)), bits(inp.kv_cache[..., : nb * d_cb]))
    with pytest.raises(ValueError):
        bp.blocks_of(4, 3, 0)
    with pytest.raises(ValueError):
        bp.shard_cache(inp.kv_cache[..., :-1], cfg, 2, 0)


def test_one_branch_per_rank_carries_one_and_a_half_d_h():
    """At 4-way branch parallelism each rank stores d_h + d_h / 2 per token for
    MLRA-4 with d_h = 128 (192 bf16 = 384 B), a third of the 4.5 d_h row."""
    import workloads as W
    from decode_attention_rank_mlra_b200 import branch_parallel as bp
    spec = W.WORKLOADS["mlra4_bf16_b8_h128_l131072_paged"]
    cfg = _cfg(spec)
    lc = bp.local_config(cfg, 4)
    assert lc.D == 192 == 1.5 * spec.d_h and cfg.D == 576 == 4.5 * spec.d_h
