"""GPU: branch-parallel shards through the CUDA kernels, summed, against the
fp64 MLRA-4 oracle.

Each shard (one or two latent blocks of 128 plus the shared RoPE key, the
layer's branch rescale) runs the ordinary step through the C ABI on one GPU,
one after the other; their outputs are summed as the all-reduce would sum
them across GPUs ("Multi-Head Low-Rank Attention", Key Contributions #2; Main
Findings, second bullet).  No shard waits on another: the sum is taken on the
host side of the calls.  The multi-process all-reduce itself is tested with
gloo ranks on CPU (tests/test_branch_parallel.py).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from decode_attention_rank_mlra_b200 import branch_parallel as bp
from parity_util import check_close, config_of, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


@pytest.mark.parametrize("name,heads", [("mlra4_bf16_b8_h128_l131072_paged", 128),
                                        ("mlra4_bf16_b64_h32_l16384_paged", 32),
                                        ("mlra4_bf16_b128_h16_ragged1k_64k_paged", 16)])
@pytest.mark.parametrize("world", [4, 2])
def test_branch_shards_sum_to_the_mlra4_output(name, heads, world):
    seqlens = np.asarray([900, 64, 1, 333], np.int32)
    spec = W.scaled_down(W.WORKLOADS[name], len(seqlens), seqlen=int(seqlens.max()),
                         n_heads=heads, seed=53)
    inp = W.make_inputs(spec, "cuda", seqlens=seqlens)
    cfg = config_of(spec)
    mp = inp.page_table.shape[1]
    total = torch.zeros((spec.batch, heads, spec.d_h), dtype=torch.float32, device="cuda")
    for r in range(world):
        dec = bp.BranchParallelDecoder(cfg, spec.batch, "cuda", world, r)
        out = dec.step(inp.q_nope, inp.q_rope, bp.shard_weights(inp.w_uk, cfg, world, r),
                       bp.shard_weights(inp.w_uv, cfg, world, r),
                       bp.shard_cache(inp.kv_cache, cfg, world, r), inp.page_table, inp.seqlens,
                       mp)
        total += out
    torch.cuda.synchronize()
    hs = sorted({0, heads // 2, heads - 1})
    refs = oracle.decode_batch(inp, heads=hs)
    ref = np.stack([x.out[hs] for x in refs])
    check_close(total.cpu().double().numpy()[:, hs], ref, "bf16", f"{world} shards")
    # and the single-device step on the whole cache
    full = run_gpu(inp, fused=True)["out"]
    check_close(total.cpu().double().numpy()[:, hs], full.double().numpy()[:, hs], "bf16",
                "shards vs one device")
