"""The allocation-free entry point against the workspace path.

mlra_decode_attn_noalloc exists for callers that cannot call cudaMalloc (a
plugin whose host framework owns every device allocation, or a server that
reserves all free HBM for the KV cache and may not allocate afterwards).  It
runs the same plan, attention and combine kernels, in the same order, with the
library's fixed scratch array instead of a workspace: its results must equal
mlra_decode_attn + mlra_splitkv_combine on the same inputs bit for bit, call
after call, although the array keeps each call's leftovers.

This file is collected last on purpose: it must pass on its own in a fresh
process and after every other test.
"""
import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import workloads as W
from parity_util import config_of

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20   # the array's fixed size (include/mlra.h)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


def _inputs(name, seqlens, seed):
    spec = W.scaled_down(W.WORKLOADS[name], len(seqlens), seqlen=int(max(max(seqlens), 1)),
                         seed=seed)
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
    ref_err = mlra.get_device_error(ws)
    o_lat = torch.full_like(ref_lat, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=inp.device)
    mlra.decode_attn_noalloc(cfg, q_abs, inp.q_rope, inp.kv_cache, inp.page_table, inp.seqlens,
                             max_pages, o_lat, lse, status)
    torch.cuda.synchronize()
    return ref_lat.cpu(), ref_lse.cpu(), ref_err, o_lat.cpu(), lse.cpu(), int(status.item())


def _assert_same(inp):
    ref_lat, ref_lse, ref_err, got_lat, got_lse, status = _both_paths(inp)
    assert ref_err == 0 and status == 0
    assert torch.equal(got_lat, ref_lat), "o_latent differs from the workspace path"
    assert torch.equal(got_lse, ref_lse), "lse differs from the workspace path"


def test_noalloc_equals_workspace_path_twice():
    # two calls in a row, different shapes and kernels, sharing the scratch array
    cases = [("mlra4_bf16_b64_h32_l16384_paged", [700, 1, 2049], 21),
             ("mlra4_bf16_b16_h16_l4096_contig", [300, 64, 1000, 5], 22)]
    for name, seqlens, seed in cases:
        _assert_same(_inputs(name, seqlens, seed))


def _largest_batch(cfg) -> int:
    """Largest batch whose workspace fits the 16 MiB array (bisection)."""
    lo, hi = 1, 1
    while mlra.workspace_size(cfg, hi) <= SCRATCH_BYTES:
        lo, hi = hi, hi * 2
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if mlra.workspace_size(cfg, mid) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


def test_noalloc_at_its_scratch_limit():
    """The largest batch that fits the array runs and equals the workspace path;
    one more sequence is rejected (MLRA_ERR_WORKSPACE) before any launch."""
    name = "mlra4_bf16_b64_h32_l16384_paged"
    spec0 = W.WORKLOADS[name]
    cfg = config_of(spec0)
    n = _largest_batch(cfg)
    assert mlra.workspace_size(cfg, n) <= SCRATCH_BYTES < mlra.workspace_size(cfg, n + 1)
    rng = np.random.default_rng(24)
    seqlens = rng.integers(0, 130, size=n)
    seqlens[0] = 130
    _assert_same(_inputs(name, seqlens, 24))
    # batch n + 1: small tensors suffice, nothing is read before the size check
    inp = _inputs(name, [64], 25)
    B = n + 1
    seqlens = torch.zeros(B, dtype=torch.int32, device="cuda")
    q_abs = torch.zeros((B, cfg.n_heads, cfg.n_blocks, cfg.d_cb), dtype=torch.float32,
                        device="cuda")
    q_rope = torch.zeros((B, cfg.n_heads, cfg.d_r), dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    o_lat = torch.zeros_like(q_abs)
    with pytest.raises(mlra.MlraError) as e:
        mlra.decode_attn_noalloc(cfg, q_abs, q_rope, inp.kv_cache, pt, seqlens, 1, o_lat)
    assert e.value.status == 4  # MLRA_ERR_WORKSPACE
    # and the array still serves the next call
    _assert_same(_inputs("mlra4_bf16_b16_h16_l4096_contig", [129, 3], 26))
