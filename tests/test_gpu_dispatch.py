"""GPU: every kernel a caller can reach, against the fp64 oracle.

The tensor-core kernels take the bf16 shapes of the workloads (16, 32, 64 or a
multiple of 128 heads; latent blocks of 128, or one of 512; d_h = 128 for the
weight contractions).  Other bf16 shapes, the fp32 cache and under-aligned
operands run on the fp32 SIMT kernels; each of those paths is checked here
against the oracle, within the same bf16 bounds as the tensor-core path.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import oracle
import workloads as W
from parity_util import check_close, compare_batch, config_of, run_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


def _spec(heads, n_blocks=4, d_cb=128, d_h=128, d_r=64, seqlens=(1, 64, 300, 1000), seed=41):
    base = W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"]
    s = W.scaled_down(base, len(seqlens), seqlen=max(seqlens), n_heads=heads, seed=seed)
    return s.replace(n_blocks=n_blocks, d_cb=d_cb, d_h=d_h, d_r=d_r,
                     name=f"{s.name}_h{heads}_nb{n_blocks}_cb{d_cb}_dh{d_h}")


@pytest.mark.parametrize("heads", [8, 48, 96])
@pytest.mark.parametrize("fused", [False, True])
def test_bf16_head_counts_outside_the_tensor_core_layouts(heads, fused):
    """bf16 MLRA-4 with 8, 48 or 96 heads: the SIMT attention kernel, the
    tensor-core weight contractions (d_h = 128)."""
    spec = _spec(heads)
    cfg = config_of(spec)
    assert mlra.decode_kernel_kind(cfg) == "simt"
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([1, 64, 300, 1000], np.int32))
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=sorted({0, heads // 2, heads - 1}))


@pytest.mark.parametrize("fused", [False, True])
def test_bf16_small_head_dim_all_simt(fused):
    """bf16 with d_h = 64 (blocks of 64, RoPE key of 32): SIMT attention and
    SIMT absorption / output projection (the tensor-core contractions need
    d_h = 128)."""
    spec = _spec(16, d_cb=64, d_h=64, d_r=32)
    assert mlra.decode_kernel_kind(config_of(spec)) == "simt"
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([1, 64, 300, 1000], np.int32))
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    compare_batch(inp, got)


def test_unaligned_operands_take_the_simt_contractions():
    """q_nope and o_latent that start 2 / 4 bytes past a 16-byte boundary cannot
    be read by TMA: absorption and projection run on the SIMT kernels and agree
    with the oracle (and with the tensor-core results on aligned copies)."""
    spec = _spec(32, seqlens=(200, 70))
    cfg = config_of(spec)
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([200, 70], np.int32))
    B, h = spec.batch, spec.n_heads
    # absorb: q_nope one bf16 element past an aligned start
    buf = torch.empty(inp.q_nope.numel() + 8, dtype=torch.bfloat16, device="cuda")
    q_mis = buf[1: 1 + inp.q_nope.numel()].view_as(inp.q_nope)
    q_mis.copy_(inp.q_nope)
    assert q_mis.data_ptr() % 16 != 0
    qa_simt = mlra.absorb_q(cfg, q_mis, inp.w_uk)
    qa_tc = mlra.absorb_q(cfg, inp.q_nope, inp.w_uk)
    torch.cuda.synchronize()
    for s in range(B):
        ref = oracle.absorb_query(inp.q_nope[s].cpu(), inp.w_uk.cpu())
        check_close(qa_simt[s].double().cpu().numpy(), ref, "f32", "q_abs (SIMT)")
        check_close(qa_tc[s].double().cpu().numpy(), ref, "f32", "q_abs (tcgen05)")
    # out-proj: o_latent one fp32 element past an aligned start
    ws = mlra.alloc_workspace(cfg, B, inp.device)
    mp = inp.page_table.shape[1]
    mlra.decode_attn(cfg, qa_tc, inp.q_rope, inp.kv_cache, inp.page_table, inp.seqlens, mp, ws)
    o_lat, lse = mlra.splitkv_combine(cfg, ws, B)
    obuf = torch.empty(o_lat.numel() + 4, dtype=torch.float32, device="cuda")
    o_mis = obuf[1: 1 + o_lat.numel()].view_as(o_lat)
    o_mis.copy_(o_lat)
    assert o_mis.data_ptr() % 16 != 0
    out_simt = mlra.out_proj(cfg, o_mis, inp.w_uv)
    torch.cuda.synchronize()
    refs = oracle.decode_batch(inp)
    ref = np.stack([r.out for r in refs])
    check_close(out_simt.double().cpu().numpy(), ref, "bf16", "out (SIMT projection)")


def test_fp32_paged_cache():
    """The fp32 cache through a page table (the fp32 workload is contiguous)."""
    base = W.WORKLOADS["mlra4_f32_b1_h4_l256"]
    spec = W.scaled_down(base, 3, seqlen=700, seed=43).replace(paged=True)
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([700, 65, 1], np.int32))
    assert mlra.decode_kernel_kind(config_of(spec)) == "simt"
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    compare_batch(inp, got)


CHILD_ROWS = r"""
import sys, numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import decode_attention_rank_mlra_b200 as mlra
import workloads as W
from parity_util import compare_batch, run_gpu
spec = W.scaled_down(W.WORKLOADS["mlra4_bf16_b8_h128_l131072_paged"], 2, seqlen=500, seed=47)
inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([500, 90], np.int32))
flat = inp.kv_cache.view(-1, spec.D)
row = int(inp.page_table[0, 1].item()) * 64 + 3
flat[row, 5] = 70000.0      # beyond the fp16 range of the 128-head kernel
flat[row, 130] = -250000.0
got = run_gpu(inp, fused=True)
compare_batch(inp, got, heads=[0, 1, 64, 127])
print("status", got["device_error"])
""".replace("ROOT", repr(ROOT))


def test_rows_layout_takes_caches_beyond_fp16_at_128_heads():
    """MLRA_TC_LAYOUT=rows keeps 128 heads on the head-rows kernel (two head
    groups of 64, bf16 operands throughout): cache values beyond the fp16
    range give the oracle's result there (in a child process: the variable is
    read once per process)."""
    env = dict(os.environ, MLRA_TC_LAYOUT="rows")
    r = subprocess.run([sys.executable, "-c", CHILD_ROWS], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "status 0" in r.stdout, r.stdout[-2000:]


def test_binding_rejects_mismatched_shapes_before_the_library():
    """Outputs smaller than [B, h, nb, d_cb] / [B, h, nb] (which the kernels
    would write past) and inputs of the wrong shape are refused by the
    binding with ValueError; nothing is launched."""
    spec = _spec(16, seqlens=(100, 30))
    cfg = config_of(spec)
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([100, 30], np.int32))
    mp = inp.page_table.shape[1]
    q_abs = mlra.absorb_q(cfg, inp.q_nope, inp.w_uk)
    small = torch.zeros((1, 16, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        mlra.decode_attn_noalloc(cfg, q_abs, inp.q_rope, inp.kv_cache, inp.page_table,
                                 inp.seqlens, mp, small)
    o_lat = torch.zeros((2, 16, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        mlra.decode_attn_noalloc(cfg, q_abs, inp.q_rope, inp.kv_cache, inp.page_table,
                                 inp.seqlens, mp, o_lat, torch.zeros(5, device="cuda"))
    with pytest.raises(ValueError):
        mlra.decode_attn(cfg, q_abs[:1].contiguous(), inp.q_rope, inp.kv_cache, inp.page_table,
                         inp.seqlens, mp, mlra.alloc_workspace(cfg, 2, inp.device))
    with pytest.raises(ValueError):
        mlra.out_proj(cfg, o_lat, inp.w_uv, torch.zeros((2, 16, 64), device="cuda"))
    with pytest.raises(ValueError):
        mlra.absorb_q(cfg, inp.q_nope, inp.w_uk[:, :8].contiguous())
