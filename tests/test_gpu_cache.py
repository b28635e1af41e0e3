"""GPU parity of the cache-write step against the fp64 oracle."""
import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import workloads as W
import oracle
from oracle import cache_rows, kv_scale, q_scale, query_side
from parity_util import check_close, compare_batch, config_of, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


def _new_token_inputs(spec, B, seed):
    g = torch.Generator().manual_seed(seed)
    K = spec.n_blocks * spec.d_cb
    c_new = (torch.randn(B, K, generator=g) * 3.0).to(spec.torch_dtype)
    kr_new = torch.randn(B, spec.d_r, generator=g).to(spec.torch_dtype)
    gamma = (1.0 + 0.1 * torch.randn(K, generator=g)).float()
    return c_new, kr_new, gamma


def _rows_of(inp, seqs, positions):
    rows = []
    for s, p in zip(seqs, positions):
        if inp.page_table is None:
            rows.append(inp.kv_cache[s, p])
        else:
            pg = int(inp.page_table[s, p // 64])
            rows.append(inp.kv_cache[pg, p % 64])
    return torch.stack(rows).double().cpu().numpy()


@pytest.mark.parametrize("name", ["mlra4_bf16_b64_h32_l16384_paged", "mla_bf16_b8_h128_l131072_paged",
                                  "mlra4_f32_b1_h4_l256"])
def test_cache_append_rows_match_oracle(name):
    base = W.WORKLOADS[name]
    seqlens = [5, 64, 300, 129] if base.paged else [200]
    B = len(seqlens)
    spec = W.scaled_down(base, B, seqlen=max(seqlens) + 1, seed=31)
    # room for one more token per sequence; the new row goes at position seqlens[s]
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray(seqlens, np.int32) + 1)
    inp.seqlens -= 1
    before = inp.kv_cache.clone()
    c_new, kr_new, gamma = _new_token_inputs(spec, B, 7)
    positions = torch.tensor(seqlens, dtype=torch.int32)  # the next free slot
    alpha = kv_scale(4096, spec.d_cb)
    cfg = config_of(spec)
    max_pages = inp.page_table.shape[1] if inp.page_table is not None else inp.max_len
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mlra.cache_append(cfg, c_new.cuda(), kr_new.cuda(), gamma.cuda(), alpha, inp.kv_cache,
                      inp.page_table, positions.cuda(), max_pages, rms_eps=1e-6,
                      rope_theta=10000.0, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = _rows_of(inp, range(B), seqlens)
    ref = cache_rows(c_new, kr_new, gamma, spec.n_blocks, alpha, 1e-6, np.asarray(seqlens), 1e4)
    if spec.dtype == "f32":
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)
    else:  # fp32 arithmetic, then one rounding to bf16 (relative step 2^-8)
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    # nothing else in the cache changed (bit patterns: rows past a sequence's
    # end are uninitialised and may hold NaN, which never equals itself)
    bits = torch.int16 if spec.dtype == "bf16" else torch.int32
    changed = (inp.kv_cache.view(bits) != before.view(bits)).reshape(-1, spec.D).any(dim=1)
    changed = changed.nonzero().flatten().cpu()
    if inp.page_table is None:
        want = sorted(s * inp.max_len + p for s, p in enumerate(seqlens))
    else:
        want = sorted(int(inp.page_table[s, p // 64]) * 64 + p % 64 for s, p in enumerate(seqlens))
    assert set(changed.tolist()) <= set(want)


def test_cache_append_rejects_bad_positions_and_pages():
    base = W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"]
    spec = W.scaled_down(base, 2, seqlen=131, seed=3)
    inp = W.make_inputs(spec, "cuda", seqlens=np.asarray([131, 11], np.int32))
    c_new, kr_new, gamma = _new_token_inputs(spec, 2, 1)
    cfg = config_of(spec)
    max_pages = inp.page_table.shape[1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = inp.kv_cache.clone()
    bad_pos = torch.tensor([max_pages * 64, 10], dtype=torch.int32, device="cuda")
    mlra.cache_append(cfg, c_new.cuda(), kr_new.cuda(), gamma.cuda(), 2.0, inp.kv_cache,
                      inp.page_table, bad_pos, max_pages, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1                      # MLRA_ERR_INVALID_ARG
    assert not torch.equal(inp.kv_cache, before)        # sequence 1's row was still written
    status.zero_()
    inp.page_table[1, 0] = inp.kv_cache.shape[0] + 3
    mlra.cache_append(cfg, c_new.cuda(), kr_new.cuda(), gamma.cuda(), 2.0, inp.kv_cache,
                      inp.page_table, torch.tensor([0, 5], dtype=torch.int32, device="cuda"),
                      max_pages, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6                      # MLRA_ERR_BAD_PAGE


def test_append_then_attend():
    """Write the new token's row, then decode over seqlen + 1 tokens: the
    attention result matches the oracle on the cache with the row the oracle
    itself computes for that token (no oracle input comes from the GPU)."""
    base = W.WORKLOADS["mlra4_bf16_b128_h16_ragged1k_64k_paged"]
    seqlens = np.asarray([700, 63, 1000], np.int32)
    spec = W.scaled_down(base, 3, seqlen=int(seqlens.max()) + 1, seed=9)
    inp = W.make_inputs(spec, "cuda", seqlens=seqlens + 1)
    ref_cache = inp.kv_cache.clone()
    inp.seqlens -= 1
    c_new, kr_new, gamma = _new_token_inputs(spec, 3, 5)
    cfg = config_of(spec)
    alpha = kv_scale(4096, spec.d_cb)
    mlra.cache_append(cfg, c_new.cuda(), kr_new.cuda(), gamma.cuda(), alpha, inp.kv_cache,
                      inp.page_table, inp.seqlens.clone(), inp.page_table.shape[1])
    inp.seqlens += 1
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    # the oracle's own rows for the new tokens, rounded to the storage dtype
    rows = cache_rows(c_new, kr_new, gamma, spec.n_blocks, alpha, 1e-6, seqlens, 10000.0)
    rows_t = torch.from_numpy(rows).to(spec.torch_dtype).cuda()
    for s, p in enumerate(seqlens):
        pg = int(inp.page_table[s, p // 64])
        ref_cache[pg, p % 64] = rows_t[s]
    ref = W.DecodeInputs(spec=spec, seqlens=inp.seqlens, q_nope=inp.q_nope, q_rope=inp.q_rope,
                         w_uk=inp.w_uk, w_uv=inp.w_uv, kv_cache=ref_cache,
                         page_table=inp.page_table, max_len=inp.max_len)
    compare_batch(ref, got)


def _raw_queries(spec, B, seed):
    g = torch.Generator().manual_seed(seed)
    qn = torch.randn(B, spec.n_heads, spec.d_h, generator=g).to(spec.torch_dtype)
    qr = torch.randn(B, spec.n_heads, spec.d_r, generator=g).to(spec.torch_dtype)
    return qn, qr


@pytest.mark.parametrize("name", ["mlra4_bf16_b64_h32_l16384_paged", "mla_bf16_b8_h128_l131072_paged",
                                  "mlra4_f32_b1_h4_l256"])
def test_absorb_q_rope_matches_oracle(name):
    """q_abs = alpha_q W_uk q_nope and q_rope' = RoPE(alpha_q q_rope) at each
    sequence's position, against the fp64 oracle: q_abs within the fp32 bound,
    q_rope' within one rounding to the storage dtype plus the fp32 rotation."""
    spec = W.WORKLOADS[name]
    B = 5
    pos = np.asarray([0, 1, 4095, 65535, 131071], np.int32)
    qn, qr = _raw_queries(spec, B, 31)
    w_uk, _ = W.weights(spec)
    cfg = config_of(spec)
    alpha = 1.75
    q_abs, q_rope_out = mlra.absorb_q_rope(cfg, qn.cuda(), qr.cuda(),
                                           torch.from_numpy(pos).cuda(), alpha, w_uk.cuda())
    torch.cuda.synchronize()
    qn2, qr2 = query_side(qn, qr, pos[:, None], alpha, 10000.0)
    for s in range(B):
        check_close(q_abs[s].double().cpu().numpy(), oracle.absorb_query(qn2[s], w_uk), "f32",
                    f"q_abs seq {s}")
    got = q_rope_out.double().cpu().numpy()
    half = spec.d_r // 2
    a = np.abs(alpha * qr.double().numpy())
    pair = np.concatenate([a[..., :half] + a[..., half:]] * 2, axis=-1)
    unit = 2.0 ** -8 if spec.dtype == "bf16" else 2.0 ** -24   # half an ulp, relative
    tol = unit * np.abs(qr2) + 2.0 ** -21 * pair
    assert np.all(np.abs(got - qr2) <= tol), float(np.max(np.abs(got - qr2) - tol))
    # alpha_q = 1 gives mlra_absorb_q's q_abs bit for bit; in place gives the same rope
    q1, _ = mlra.absorb_q_rope(cfg, qn.cuda(), qr.cuda(), torch.from_numpy(pos).cuda(), 1.0,
                               w_uk.cuda())
    q0 = mlra.absorb_q(cfg, qn.cuda(), w_uk.cuda())
    inplace = qr.clone().cuda()
    mlra.absorb_q_rope(cfg, qn.cuda(), inplace, torch.from_numpy(pos).cuda(), alpha, w_uk.cuda(),
                       q_rope_out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(q1, q0)
    assert torch.equal(inplace.cpu(), q_rope_out.cpu())


def test_query_side_then_attend():
    """The query side (alpha_q, RoPE at the query's position) then attention,
    merge and projection, against the oracle given the same raw query: the
    oracle applies its own query side and rounds the rotated RoPE query to the
    storage dtype, as the step stores it."""
    base = W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"]
    seqlens = np.asarray([700, 64, 1500], np.int32)
    spec = W.scaled_down(base, 3, seqlen=int(seqlens.max()), seed=33)
    inp = W.make_inputs(spec, "cuda", seqlens=seqlens)
    cfg = config_of(spec)
    qn, qr = _raw_queries(spec, 3, 35)
    pos = torch.from_numpy(seqlens - 1).cuda()
    alpha = q_scale(4096, 1024)
    dec = mlra.Decoder(cfg, 3, inp.device)
    q_rope_out = torch.empty_like(inp.q_rope)
    mlra.absorb_q_rope(cfg, qn.cuda(), qr.cuda(), pos, alpha, inp.w_uk, dec.q_abs, q_rope_out)
    mlra.decode_attn(cfg, dec.q_abs, q_rope_out, inp.kv_cache, inp.page_table, inp.seqlens,
                     inp.page_table.shape[1], dec.workspace)
    mlra.combine_out_proj(cfg, dec.workspace, 3, inp.w_uv, dec.out, dec.o_latent, dec.lse)
    assert mlra.get_device_error(dec.workspace) == 0
    torch.cuda.synchronize()
    qn2, qr2 = query_side(qn, qr, (seqlens - 1)[:, None], alpha, 10000.0)
    qr2 = torch.from_numpy(qr2).to(spec.torch_dtype)     # stored in the cache's dtype
    ref_in = W.DecodeInputs(spec=spec, seqlens=inp.seqlens, q_nope=torch.from_numpy(qn2),
                            q_rope=qr2, w_uk=inp.w_uk, w_uv=inp.w_uv, kv_cache=inp.kv_cache,
                            page_table=inp.page_table, max_len=inp.max_len)
    refs = oracle.decode_batch(ref_in)
    check_close(dec.out.double().cpu().numpy(), np.stack([r.out for r in refs]), "bf16", "out")
