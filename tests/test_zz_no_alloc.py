"""The allocation-free entry point against the workspace path.

mlra_decode_attn_noalloc exists for callers that cannot call cudaMalloc (a
plugin whose host framework owns every device allocation, or a server that
reserves all free HBM for the KV cache and may not allocate afterwards).  It
runs the same attention + combine with the library's fixed scratch array; its
results must match mlra_decode_attn + mlra_splitkv_combine on the same inputs,
call after call, although the array keeps each call's leftovers.

This file is collected last on purpose: it must pass on its own in a fresh
process and after every other test.
"""
import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import workloads as W
from parity_util import check_close, config_of

pytestmark = pytest.mark.gpu


def _inputs(name, seqlens, seed):
    spec = W.scaled_down(W.WORKLOADS[name], len(seqlens), seqlen=int(max(seqlens)), seed=seed)
    return W.make_inputs(spec, "cuda", seqlens=np.asarray(seqlens, np.int32))


def _both_paths(inp):
    spec = inp.spec
    cfg = config_of(spec)
    max_pages = inp.page_table.shape[1] if inp.page_table is not None else inp.max_len
    q_abs = mlra.absorb_q(cfg, inp.q_nope, inp.w_uk)
    ws = mlra.alloc_workspace(cfg, spec.batch, inp.device)
    mlra.decode_attn(cfg, q_abs, inp.q_rope, inp.kv_cache, inp.page_table, inp.seqlens,
                     max_pages, ws)
    ref_lat, ref_lse = mlra.splitkv_combine(cfg, ws, spec.batch)
    o_lat = torch.full_like(ref_lat, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=inp.device)
    mlra.decode_attn_noalloc(cfg, q_abs, inp.q_rope, inp.kv_cache, inp.page_table, inp.seqlens,
                             max_pages, o_lat, lse, status)
    torch.cuda.synchronize()
    return ref_lat.cpu(), ref_lse.cpu(), o_lat.cpu(), lse.cpu(), int(status.item())


def test_noalloc_matches_workspace_path_twice():
    # two calls in a row, different shapes and kernels, sharing the scratch array
    cases = [("mlra4_bf16_b64_h32_l16384_paged", [700, 1, 2049], 21),
             ("mlra4_bf16_b16_h16_l4096_contig", [300, 64, 1000, 5], 22)]
    for name, seqlens, seed in cases:
        inp = _inputs(name, seqlens, seed)
        ref_lat, ref_lse, got_lat, got_lse, status = _both_paths(inp)
        assert status == 0
        check_close(got_lat.double().numpy(), ref_lat.double().numpy(), inp.spec.dtype, "o_latent")
        fin = torch.isfinite(ref_lse)
        assert torch.equal(fin, torch.isfinite(got_lse))
        assert torch.max(torch.abs(got_lse[fin] - ref_lse[fin])).item() < 1e-4


def test_noalloc_rejects_batches_beyond_its_scratch():
    inp = _inputs("mlra4_bf16_b64_h32_l16384_paged", [64], 23)
    cfg = config_of(inp.spec)
    big = 20000  # needs far more than the fixed 16 MiB scratch
    seqlens = torch.zeros(big, dtype=torch.int32, device="cuda")
    q_abs = torch.zeros((big, cfg.n_heads, cfg.n_blocks, cfg.d_cb), dtype=torch.float32,
                        device="cuda")
    q_rope = torch.zeros((big, cfg.n_heads, cfg.d_r), dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros((big, 1), dtype=torch.int32, device="cuda")
    o_lat = torch.zeros_like(q_abs)
    with pytest.raises(mlra.MlraError) as e:
        mlra.decode_attn_noalloc(cfg, q_abs, q_rope, inp.kv_cache, pt, seqlens, 1, o_lat)
    assert e.value.status == 4  # MLRA_ERR_WORKSPACE
