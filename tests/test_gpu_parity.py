"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Oracle-sized cases span several 64-token tiles and a ragged tail; full-size
workloads are checked on sampled (sequence, head) outputs regenerated alone.
"""
import math

import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import oracle
import workloads as W
from parity_util import (check_close, check_lse, compare_batch, config_of, query_unit, run_gpu,
                         rows_logit_magnitude)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


def _small(name, batch, seqlens, heads=None, seed=11):
    spec = W.WORKLOADS[name]
    s = W.scaled_down(spec, batch, seqlen=int(max(seqlens)), n_heads=heads, seed=seed)
    return W.make_inputs(s, "cuda", seqlens=np.asarray(seqlens, np.int32))


def test_fp32_workload_full():
    """B=1, h=4, d_h=64, L=256, fp32: max relative error <= 1e-5."""
    spec = W.WORKLOADS["mlra4_f32_b1_h4_l256"]
    inp = W.make_inputs(spec, "cuda")
    got = run_gpu(inp)
    assert got["device_error"] == 0
    compare_batch(inp, got)
    # the absorbed query against the oracle's absorption
    qa = oracle.absorb_query(inp.q_nope[0].cpu(), inp.w_uk.cpu())
    check_close(got["q_abs"][0].double().numpy(), qa, "f32", "q_abs")


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("name,seqlens", [
    ("mlra4_bf16_b16_h16_l4096_contig", [1, 63, 64, 65, 700, 1500]),
    ("mlra4_bf16_b64_h32_l16384_paged", [129, 1000, 2049]),
    ("mlra4_bf16_b128_h16_ragged1k_64k_paged", [1, 64, 333, 1024, 2500, 77]),
])
def test_bf16_oracle_sized(name, seqlens, fused):
    inp = _small(name, len(seqlens), seqlens)
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    compare_batch(inp, got)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("name", ["mla_bf16_b8_h128_l131072_paged",
                                  "mlra4_bf16_b8_h128_l131072_paged"])
def test_bf16_h128_oracle_sized(name, fused):
    inp = _small(name, 2, [1100, 190])
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=[0, 1, 63, 100, 127])


@pytest.mark.parametrize("name", ["mlra4_bf16_b8_h128_l131072_paged", "mla_bf16_b8_h128_l131072_paged"])
def test_bf16_two_groups_of_128_heads(name):
    """256 heads: two groups of 128 (two head groups of 128-head CTAs per branch
    for MLRA-4, two head groups of clusters for MLA), heads on both sides of the
    group boundary."""
    inp = _small(name, 2, [700, 129], heads=256, seed=23)
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=[0, 127, 128, 200, 255])


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("batch", [17, 70, 300])
def test_batches_spanning_several_sequence_tiles(batch, fused):
    """Batches that fill several N tiles of the weight contractions (16..256
    sequences per CTA) with a partial last tile, and many short sequences."""
    rng = np.random.default_rng(batch)
    seqlens = rng.integers(0, 150, size=batch)
    seqlens[0] = 150
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", batch, seqlens)
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    pick = sorted({0, 1, batch // 2, batch - 17, batch - 1})
    compare_batch(inp, got, seqs=pick, heads=[0, 13, 31])


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("heads", [16, 32, 64, 128])
def test_mlra2_two_branches(heads, fused):
    """MLRA-2 (two latent blocks of 128, branch rescale 1/sqrt(2)): the same
    kernels with two branches per CTA (h <= 32), one (h = 64), or 128 heads of
    one branch (h = 128)."""
    base = W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"]
    seqlens = [1, 64, 700, 1300, 333]
    spec = W.scaled_down(base, len(seqlens), seqlen=max(seqlens), n_heads=heads, seed=23)
    spec = spec.replace(n_blocks=2, name=spec.name + "_mlra2")
    assert spec.D == 320 and abs(spec.branch_scale - 2 ** -0.5) < 1e-12
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray(seqlens, np.int32))
    got = run_gpu(inp, fused=fused)
    assert got["device_error"] == 0
    assert mlra.decode_kernel_kind(config_of(spec)) == "tcgen05"
    compare_batch(inp, got, heads=sorted({0, heads // 2, heads - 1}))


@pytest.mark.parametrize("heads", [128, 256])
def test_single_128_channel_block_h128(heads):
    """One latent block of 128 channels (n_blocks = 1, D = 192) with 128 and 256
    heads: the 128-head kernel with one branch, one or two head groups."""
    base = W.WORKLOADS["mlra4_bf16_b8_h128_l131072_paged"]
    seqlens = [65, 1000, 129]
    spec = W.scaled_down(base, len(seqlens), seqlen=max(seqlens), n_heads=heads, seed=29)
    spec = spec.replace(n_blocks=1, name=spec.name + "_nb1")
    assert spec.D == 192 and spec.branch_scale == 1.0
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray(seqlens, np.int32))
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=sorted({0, 77, heads - 1}))


def test_fused_projection_without_latent_outputs():
    """combine_out_proj with o_latent = lse = None gives the same out."""
    inp = _small("mlra4_bf16_b16_h16_l4096_contig", 3, [500, 64, 1])
    ref = run_gpu(inp, fused=True)
    spec = inp.spec
    cfg = config_of(spec)
    dec = mlra.Decoder(cfg, spec.batch, inp.device)
    mlra.absorb_q(cfg, inp.q_nope, inp.w_uk, dec.q_abs)
    mlra.decode_attn(cfg, dec.q_abs, inp.q_rope, inp.kv_cache, None, inp.seqlens, inp.max_len,
                     dec.workspace)
    out = mlra.combine_out_proj(cfg, dec.workspace, spec.batch, inp.w_uv)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), ref["out"])


def test_empty_and_single_token_sequences():
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", 4, [0, 1, 0, 130])
    got = run_gpu(inp)
    assert got["device_error"] == 0
    assert torch.all(got["out"][0] == 0) and torch.all(got["out"][2] == 0)
    assert torch.all(torch.isneginf(got["lse"][0]))
    compare_batch(inp, got, seqs=[1, 3])


def test_tail_rows_never_matter():
    """Rows at or past seqlen hold NaN / huge values: the result must not change."""
    inp = _small("mlra4_bf16_b16_h16_l4096_contig", 3, [100, 64, 190])
    ref = run_gpu(inp)
    inp.kv_cache[0, 100:] = float("nan")
    inp.kv_cache[1, 64:] = 3.0e38
    got = run_gpu(inp)
    for k in ("out", "o_lat", "lse"):
        assert torch.equal(got[k], ref[k]), k


def test_paged_tail_rows_never_matter():
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", 2, [70, 5])
    ref = run_gpu(inp)
    flat = inp.kv_cache.view(-1, inp.spec.D)
    pt = inp.page_table.cpu()
    flat[int(pt[0, 1]) * 64 + 6: int(pt[0, 1]) * 64 + 64] = float("nan")
    flat[int(pt[1, 0]) * 64 + 5: int(pt[1, 0]) * 64 + 64] = float("inf")
    got = run_gpu(inp)
    for k in ("out", "o_lat", "lse"):
        assert torch.equal(got[k], ref[k]), k


def test_h128_paged_tail_rows_never_matter():
    """The 128-head kernel converts each tile to fp16 in shared memory: rows past
    seqlen hold NaN / inf and must still not change the result."""
    inp = _small("mlra4_bf16_b8_h128_l131072_paged", 2, [70, 5])
    ref = run_gpu(inp)
    flat = inp.kv_cache.view(-1, inp.spec.D)
    pt = inp.page_table.cpu()
    flat[int(pt[0, 1]) * 64 + 6: int(pt[0, 1]) * 64 + 64] = float("nan")
    flat[int(pt[1, 0]) * 64 + 5: int(pt[1, 0]) * 64 + 64] = float("inf")
    got = run_gpu(inp)
    assert got["device_error"] == 0
    for k in ("out", "o_lat", "lse"):
        assert torch.equal(got[k], ref[k]), k


def test_h128_cache_values_beyond_fp16_range_are_recomputed():
    """The 128-head MLRA-4 kernel carries the latent tile into the MMAs as fp16:
    59904 (bf16) is still exact there; a valid cache value of magnitude >= 65520
    makes it report MLRA_ERR_RANGE, and the head-rows kernel launched after it
    recomputes the call in bf16, which then matches the oracle with no error."""
    inp = _small("mlra4_bf16_b8_h128_l131072_paged", 2, [200, 90])
    flat = inp.kv_cache.view(-1, inp.spec.D)
    row = int(inp.page_table[0, 1].item()) * 64 + 3
    flat[row, 5] = 60000.0          # bf16 59904: inside the fp16 range
    got = run_gpu(inp)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=[0, 1, 64, 127])
    flat[row, 5] = 70000.0          # bf16 70144: outside
    row2 = int(inp.page_table[1, 0].item()) * 64 + 7
    flat[row2, 300] = -250000.0
    for fused in (False, True):
        got = run_gpu(inp, fused=fused)
        assert got["device_error"] == 0
        compare_batch(inp, got, heads=[0, 1, 64, 127])


def test_mla_h128_cache_values_beyond_fp16_range_are_recomputed():
    """The same for the paired MLA kernel: a cache value beyond the fp16 range
    is recomputed by the 64-head MLA kernel (bf16 hi + lo), no error left."""
    inp = _small("mla_bf16_b8_h128_l131072_paged", 2, [150, 70], seed=7)
    flat = inp.kv_cache.view(-1, inp.spec.D)
    flat[int(inp.page_table[0, 1].item()) * 64 + 9, 17] = 70000.0
    flat[int(inp.page_table[1, 0].item()) * 64 + 2, 400] = -250000.0
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    compare_batch(inp, got, heads=[0, 63, 64, 127])


def test_mla_tile_boundaries():
    """MLA: lengths on both sides of the 32- and 64-token boundaries (a last
    tile holding 1, 31, 32, 33 or 63 tokens), then NaN / inf in the rows past
    seqlen must leave every output unchanged."""
    seqlens = [1, 31, 32, 33, 63, 64, 65, 96, 97, 128]
    inp = _small("mla_bf16_b8_h128_l131072_paged", len(seqlens), seqlens, seed=31)
    ref = run_gpu(inp)
    assert ref["device_error"] == 0
    compare_batch(inp, ref, heads=[0, 37, 64, 127])
    flat = inp.kv_cache.view(-1, inp.spec.D)
    pt = inp.page_table.cpu()
    for s, L in enumerate(seqlens):
        if L % 64:
            r0 = int(pt[s, L // 64]) * 64
            flat[r0 + L % 64: r0 + 64] = float("nan") if s % 2 else float("inf")
    got = run_gpu(inp)
    assert got["device_error"] == 0
    for k in ("out", "o_lat", "lse"):
        assert torch.equal(got[k], ref[k]), k


def test_scores_rising_far_above_the_first_tile():
    """Later tiles score hundreds of log2 units above the first tile's max: the
    running reference point of the exponentials must move (no overflow)."""
    inp = _small("mlra4_bf16_b16_h16_l4096_contig", 2, [700, 130])
    inp.kv_cache[0, 64:700] *= 3000.0
    inp.kv_cache[1, 100:130] *= 3000.0
    got = run_gpu(inp)
    assert got["device_error"] == 0
    compare_batch(inp, got)


def _boost_tokens(inp, seq, first_token, factor):
    """Multiply the cache rows of tokens >= first_token of one sequence."""
    L = int(inp.seqlens[seq])
    if inp.page_table is None:
        inp.kv_cache[seq, first_token:L] *= factor
        return
    flat = inp.kv_cache.view(-1, inp.spec.D)
    pt = inp.page_table.cpu()
    for t0 in range(first_token, L, 64):
        r0 = int(pt[seq, t0 // 64]) * 64
        flat[r0 + t0 % 64: r0 + 64] *= factor


@pytest.mark.parametrize("name,factor", [
    ("mla_bf16_b8_h128_l131072_paged", 3000.0),
    ("mla_bf16_b8_h128_l131072_paged", 20.0),
    ("mlra4_bf16_b64_h32_l16384_paged", 20.0),
    ("mlra4_bf16_b128_h16_ragged1k_64k_paged", 20.0),
])
def test_scores_rising_in_some_heads_only(name, factor):
    """Later tiles overflow the first tile's reference point in all heads
    (x3000) or only in some heads of a warp (x20): the rescale of O is taken
    by whole warps either way.  Pieces span several tiles."""
    inp = _small(name, 2, [3000, 2000])
    _boost_tokens(inp, 0, 200, factor)
    _boost_tokens(inp, 1, 1000, factor)
    got = run_gpu(inp)
    assert got["device_error"] == 0
    heads = sorted({0, 1, inp.spec.n_heads // 2 + 1, inp.spec.n_heads - 1})
    compare_batch(inp, got, heads=heads)


def test_scores_falling_far_below_the_first_tile():
    """The first tile holds the largest scores by far: later weights underflow."""
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", 2, [300, 129])
    flat = inp.kv_cache.view(-1, inp.spec.D)
    pt = inp.page_table.cpu()
    for s in range(2):
        p0 = int(pt[s, 0]) * 64
        flat[p0 + 3: p0 + 9] *= 3000.0
    got = run_gpu(inp)
    assert got["device_error"] == 0
    compare_batch(inp, got)


def test_page_permutation_invariance():
    """Moving pages together with the page table leaves every output unchanged."""
    inp = _small("mlra4_bf16_b128_h16_ragged1k_64k_paged", 3, [300, 1000, 65])
    ref = run_gpu(inp)
    n = inp.kv_cache.shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(5)).to("cuda")
    new_cache = torch.empty_like(inp.kv_cache)
    new_cache[perm] = inp.kv_cache
    inp.page_table = torch.where(inp.page_table >= 0, perm[inp.page_table.clamp(min=0).long()].int(),
                                 inp.page_table)
    inp.kv_cache = new_cache
    got = run_gpu(inp)
    for k in ("out", "o_lat", "lse"):
        torch.testing.assert_close(got[k], ref[k], rtol=0, atol=0)


def test_ragged_isolation():
    """A sequence's output does not depend on the other sequences in the batch
    (nor on how the split planner cuts the batch)."""
    big = _small("mlra4_bf16_b128_h16_ragged1k_64k_paged", 5, [3000, 17, 1200, 4100, 640])
    one = W.DecodeInputs(spec=big.spec.replace(batch=1), seqlens=big.seqlens[3:4],
                         q_nope=big.q_nope[3:4], q_rope=big.q_rope[3:4],
                         w_uk=big.w_uk, w_uv=big.w_uv, kv_cache=big.kv_cache,
                         page_table=big.page_table[3:4], max_len=big.max_len)
    a = run_gpu(big)
    b = run_gpu(one)
    check_close(b["out"][0].double().numpy(), a["out"][3].double().numpy(), "f32", "isolation")


def test_bad_page_sets_error_word():
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", 2, [200, 100])
    inp.page_table[1, 0] = inp.kv_cache.shape[0] + 5
    got = run_gpu(inp)
    assert got["device_error"] == 6
    ok = run_gpu(_small("mlra4_bf16_b64_h32_l16384_paged", 2, [200, 100]))
    assert ok["device_error"] == 0


def test_seqlen_beyond_capacity_sets_error_word():
    inp = _small("mlra4_bf16_b16_h16_l4096_contig", 2, [100, 50])
    inp.seqlens[0] = 10_000
    got = run_gpu(inp)
    assert got["device_error"] == 1


def test_determinism():
    inp = _small("mlra4_bf16_b64_h32_l16384_paged", 2, [2000, 999])
    a = run_gpu(inp)
    b = run_gpu(inp)
    for k in ("out", "o_lat", "lse"):
        assert torch.equal(a[k], b[k])


# ---- full workload sizes, sampled outputs --------------------------------

FULL = [
    ("mlra4_bf16_b16_h16_l4096_contig", [(0, [0, 15]), (9, [7])]),
    ("mlra4_bf16_b64_h32_l16384_paged", [(0, [0, 31]), (63, [5])]),
    ("mlra4_bf16_b128_h16_ragged1k_64k_paged", [(5, [3]), (127, [0, 15])]),
    ("mla_bf16_b8_h128_l131072_paged", [(0, [0, 127]), (7, [64])]),
    ("mlra4_bf16_b8_h128_l131072_paged", [(0, [0, 127]), (7, [64])]),
]


@pytest.mark.slow
@pytest.mark.parametrize("name,samples", FULL)
def test_full_size_sampled(name, samples):
    spec = W.WORKLOADS[name]
    inp = W.make_inputs(spec, "cuda")
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    assert torch.all(torch.isfinite(got["out"]))
    L_all = inp.seqlens.cpu().numpy()
    for seq, heads in samples:
        ref = oracle.decode_sampled(spec, seq, heads, int(L_all[seq]))
        check_close(got["out"][seq, heads].double().numpy(), ref.out[heads], spec.dtype,
                    f"{name} seq {seq}")
        check_close(got["o_lat"][seq, heads].double().numpy(), ref.o_lat[heads], spec.dtype,
                    f"{name} seq {seq} o_lat")
        rows = W.token_rows(spec, seq, 0, int(L_all[seq]))
        w_uk, _ = W.weights(spec)
        q_nope, q_rope = W.queries(spec)
        mag = rows_logit_magnitude(spec, rows, q_nope[seq], q_rope[seq], w_uk, heads)
        check_lse(got["lse"][seq, heads].double().numpy(), ref.lse[heads], spec.dtype, mag,
                  query_unit(spec))
