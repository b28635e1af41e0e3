"""GPU: the one-call decode step (mlra_decode_step) from device and host buffers.

It must equal the three separate calls (absorb -> attention -> merge and
projection) bit for bit, and so the oracle within the stated tolerances.
"""
import numpy as np
import pytest
import torch

import decode_attention_rank_mlra_b200 as mlra
import oracle
import workloads as W
from parity_util import check_close, config_of, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    torch.cuda.init()


def _inputs(name, seqlens, heads=None, seed=23):
    spec = W.WORKLOADS[name]
    s = W.scaled_down(spec, len(seqlens), seqlen=int(max(seqlens)), n_heads=heads, seed=seed)
    return W.make_inputs(s, "cuda", seqlens=np.asarray(seqlens, np.int32))


def _max_pages(inp):
    return inp.page_table.shape[1] if inp.page_table is not None else inp.max_len


def _step(inp, host: bool, pinned: bool = True):
    cfg = config_of(inp.spec)
    dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)
    if host:
        def h(t):
            t = t.cpu()
            return t.pin_memory() if pinned else t
        qn, qr, sl = h(inp.q_nope), h(inp.q_rope), h(inp.seqlens)
        out = torch.empty(dec.out.shape, dtype=torch.float32)
        out = out.pin_memory() if pinned else out
        out.fill_(float("nan"))
    else:
        qn, qr, sl = inp.q_nope, inp.q_rope, inp.seqlens
        out = torch.full(dec.out.shape, float("nan"), dtype=torch.float32, device=inp.device)
    dec.step(qn, qr, sl, inp.w_uk, inp.w_uv, inp.kv_cache, inp.page_table, _max_pages(inp),
             out=out)
    err = mlra.get_device_error(dec.workspace)
    torch.cuda.synchronize()
    return out.cpu(), err


@pytest.mark.parametrize("name,seqlens", [
    ("mlra4_bf16_b16_h16_l4096_contig", [1, 63, 64, 65, 700, 1500]),
    ("mlra4_bf16_b64_h32_l16384_paged", [129, 1000, 0, 2049]),
    ("mla_bf16_b8_h128_l131072_paged", [300, 1]),
    ("mlra4_bf16_b8_h128_l131072_paged", [200, 64, 5]),
    ("mlra4_f32_b1_h4_l256", [256, 17, 5]),
])
@pytest.mark.parametrize("host", [False, True])
def test_step_equals_separate_calls(name, seqlens, host):
    heads = 64 if name.startswith("mla") else None  # (the MLRA-4 h = 128 case keeps 128)
    inp = _inputs(name, seqlens, heads=heads)
    got, err = _step(inp, host)
    assert err == 0
    ref = run_gpu(inp, fused=True)
    assert torch.equal(got, ref["out"]), "decode_step differs from the separate calls"
    # and the oracle on a few (sequence, head) pairs
    hs = sorted({0, inp.spec.n_heads // 2, inp.spec.n_heads - 1})
    refs = oracle.decode_batch(inp, heads=hs, seqs=list(range(inp.spec.batch)))
    out_ref = np.stack([r.out[hs] for r in refs])
    check_close(got.double().numpy()[:, hs], out_ref, inp.spec.dtype, "out")


def test_step_from_pageable_host_memory():
    inp = _inputs("mlra4_bf16_b16_h16_l4096_contig", [900, 64, 1])
    got, err = _step(inp, host=True, pinned=False)
    assert err == 0
    pinned, _ = _step(inp, host=True, pinned=True)
    assert torch.equal(got, pinned)


def test_step_host_buffers_unaligned_and_mixed():
    """Page-locked inputs at 2- and 4-byte offsets (the staging kernel's narrow
    units), one pageable input (a copy) and an offset page-locked output."""
    inp = _inputs("mlra4_bf16_b64_h32_l16384_paged", [700, 64, 1, 1999, 3])
    cfg = config_of(inp.spec)
    dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)

    def pinned_at(t, offset):
        flat = torch.empty(t.numel() + offset, dtype=t.dtype).pin_memory()
        v = flat[offset:].view(t.shape)
        v.copy_(t.cpu())
        return v

    qn = pinned_at(inp.q_nope, 1)          # bf16: 2-byte aligned
    qr = inp.q_rope.cpu()                  # pageable
    sl = pinned_at(inp.seqlens, 3)         # int32: 4-byte aligned
    out = pinned_at(torch.zeros(dec.out.shape), 1)
    dec.step(qn, qr, sl, inp.w_uk, inp.w_uv, inp.kv_cache, inp.page_table, _max_pages(inp),
             out=out)
    assert mlra.get_device_error(dec.workspace) == 0
    torch.cuda.synchronize()
    ref, _ = _step(inp, host=False)
    assert torch.equal(out.clone(), ref)


def test_step_rejects_mixed_buffers_and_empty_batch():
    inp = _inputs("mlra4_bf16_b16_h16_l4096_contig", [128, 5])
    cfg = config_of(inp.spec)
    ws = mlra.alloc_step_workspace(cfg, 2)
    out = torch.empty((2, cfg.n_heads, cfg.d_h), dtype=torch.float32)
    with pytest.raises(ValueError):
        mlra.decode_step(cfg, inp.q_nope, inp.q_rope, inp.seqlens, inp.w_uk, inp.w_uv,
                         inp.kv_cache, inp.page_table, _max_pages(inp), out, ws)
    # a workspace one byte short is refused before anything is launched
    short = ws[: ws.numel() - 1]
    with pytest.raises(mlra.MlraError, match="WORKSPACE"):
        mlra.decode_step(cfg, inp.q_nope, inp.q_rope, inp.seqlens, inp.w_uk, inp.w_uv,
                         inp.kv_cache, inp.page_table, _max_pages(inp), out.cuda(), short)
    # batch 0 launches nothing and succeeds
    z = inp.seqlens[:0]
    mlra.decode_step(cfg, inp.q_nope[:0], inp.q_rope[:0], z, inp.w_uk, inp.w_uv, inp.kv_cache,
                     inp.page_table, _max_pages(inp), out.cuda()[:0], ws)
    torch.cuda.synchronize()


def test_step_workspace_holds_decode_workspace():
    cfg = config_of(W.WORKLOADS["mlra4_bf16_b64_h32_l16384_paged"])
    for b in (1, 64, 300):
        assert mlra.step_workspace_size(cfg, b) >= mlra.workspace_size(cfg, b) \
            + 2 * b * cfg.n_heads * cfg.n_blocks * cfg.d_cb * 4


@pytest.mark.parametrize("host", [False, True])
def test_repeated_steps_with_new_lengths(host):
    """The same buffers called again and again (the first call runs directly,
    the second is recorded, later ones replay the recording) with new sequence
    lengths each time: every result equals the separate calls on those lengths."""
    inp = _inputs("mlra4_bf16_b64_h32_l16384_paged", [1999] * 4)  # pages for 1999 tokens each
    base = [700, 64, 1999, 3]
    cfg = config_of(inp.spec)
    dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)
    ref_dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)
    if host:
        qn, qr = inp.q_nope.cpu().pin_memory(), inp.q_rope.cpu().pin_memory()
        sl = inp.seqlens.cpu().pin_memory()
        out = torch.empty(dec.out.shape, dtype=torch.float32).pin_memory()
    else:
        qn, qr, sl = inp.q_nope, inp.q_rope, inp.seqlens.clone()
        out = dec.out
    for i, lens in enumerate([base, [5, 1999, 64, 700], [1, 1, 1, 1], [640, 0, 129, 1000],
                              base]):
        sl.copy_(torch.tensor(lens, dtype=torch.int32))
        d_sl = sl.to(inp.device)
        dec.step(qn, qr, sl, inp.w_uk, inp.w_uv, inp.kv_cache, inp.page_table, _max_pages(inp),
                 out=out)
        ref_dec.run(inp.q_nope, inp.q_rope, inp.w_uk, inp.w_uv, inp.kv_cache, inp.page_table,
                    d_sl, _max_pages(inp), fused=True)
        torch.cuda.synchronize()
        assert mlra.get_device_error(dec.workspace) == 0
        assert torch.equal(out.cpu(), ref_dec.out.cpu()), f"call {i}"


def test_step_inside_a_caller_graph():
    """A caller that captures the step into its own CUDA graph gets the launches
    themselves in that graph (the library does not record into a capturing
    stream); replays match the direct result."""
    inp = _inputs("mlra4_bf16_b16_h16_l4096_contig", [900, 64, 1, 333])
    cfg = config_of(inp.spec)
    dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)
    args = (inp.q_nope, inp.q_rope, inp.seqlens, inp.w_uk, inp.w_uv, inp.kv_cache,
            inp.page_table, _max_pages(inp))
    ref = dec.step(*args).clone()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            dec.step(*args)
    torch.cuda.current_stream().wait_stream(s)
    dec.out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(dec.out, ref)
    assert mlra.get_device_error(dec.workspace) == 0


def test_released_graphs_record_again():
    """The same call (same pointers) runs directly, is recorded, is replayed;
    after mlra_release_step_graphs it records afresh: the same result bit for
    bit every time."""
    inp = _inputs("mlra4_bf16_b64_h32_l16384_paged", [300, 70])
    cfg = config_of(inp.spec)
    dec = mlra.Decoder(cfg, inp.spec.batch, inp.device)
    out = torch.empty(dec.out.shape, dtype=torch.float32, device=inp.device)
    outs = []
    for k in range(6):
        if k == 3:
            torch.cuda.synchronize()
            mlra.release_step_graphs()
        out.fill_(float("nan"))
        dec.step(inp.q_nope, inp.q_rope, inp.seqlens, inp.w_uk, inp.w_uv, inp.kv_cache,
                 inp.page_table, _max_pages(inp), out=out)
        assert mlra.get_device_error(dec.workspace) == 0
        outs.append(out.cpu().clone())
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
