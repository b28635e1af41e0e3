"""GPU parity of the cache-write step against the fp64 oracle."""
import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import workloads as W
from oracle import cache_rows, kv_scale
from parity_util import compare_batch, config_of, run_gpu

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
    # nothing else in the cache changed
    changed = (inp.kv_cache != before).reshape(-1, spec.D).any(dim=1).nonzero().flatten().cpu()
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
    attention result matches the oracle on the updated cache."""
    base = W.WORKLOADS["mlra4_bf16_b128_h16_ragged1k_64k_paged"]
    seqlens = np.asarray([700, 63, 1000], np.int32)
    spec = W.scaled_down(base, 3, seqlen=int(seqlens.max()) + 1, seed=9)
    inp = W.make_inputs(spec, "cuda", seqlens=seqlens + 1)
    inp.seqlens -= 1
    c_new, kr_new, gamma = _new_token_inputs(spec, 3, 5)
    cfg = config_of(spec)
    mlra.cache_append(cfg, c_new.cuda(), kr_new.cuda(), gamma.cuda(), kv_scale(4096, spec.d_cb),
                      inp.kv_cache, inp.page_table, inp.seqlens.clone(), inp.page_table.shape[1])
    inp.seqlens += 1
    got = run_gpu(inp, fused=True)
    assert got["device_error"] == 0
    compare_batch(inp, got)
