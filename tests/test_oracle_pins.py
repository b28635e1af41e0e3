"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Source: "Multi-Head Low-Rank Attention" (ai.info AI summary), Key
Contributions #1-#3, Main Findings ("three absorbable steps"), Methodology.
None of these tests call the CUDA library.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import mlra_oracle as om

mp = pytest.importorskip("mpmath")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, h=2, nb=4, d_cb=3, d_h=2, d_r=2, L=5, wscale=0.7):
    return dict(
        q_nope=rng.standard_normal((h, d_h)),
        q_rope=rng.standard_normal((h, d_r)),
        c_lat=rng.standard_normal((L, nb, d_cb)),
        k_rope=rng.standard_normal((L, d_r)),
        w_uk=rng.standard_normal((nb, h, d_cb, d_h)) * wscale,
        w_uv=rng.standard_normal((nb, h, d_cb, d_h)) * wscale,
        softmax_scale=1.0 / math.sqrt(d_h + d_r),
        branch_scale=1.0 / math.sqrt(nb),
    )


def _brute_force(P):
    """Scalar loops at 50 significant digits, written from the definition.

    For each head h and block b: k[t][j] = sum_i c[t][b][i] W_uk[b][h][i][j],
    v likewise with W_uv, z_t = (sum_j q_nope[h][j] k[t][j] + sum_r
    q_rope[h][r] k_rope[t][r]) * scale, p = exp(z) / sum exp(z),
    v_b = sum_t p_t v[t]; out = branch_scale * sum_b v_b.
    """
    mp.mp.dps = 50
    q_nope, q_rope, c, kr = P["q_nope"], P["q_rope"], P["c_lat"], P["k_rope"]
    w_uk, w_uv = P["w_uk"], P["w_uv"]
    nb, h, d_cb, d_h = w_uk.shape
    L, d_r = kr.shape
    M = mp.mpf
    out = [[M(0)] * d_h for _ in range(h)]
    lse = [[None] * nb for _ in range(h)]
    for hh in range(h):
        for b in range(nb):
            zs = []
            vs = []
            for t in range(L):
                k = [sum(M(c[t][b][i]) * M(w_uk[b][hh][i][j]) for i in range(d_cb)) for j in range(d_h)]
                v = [sum(M(c[t][b][i]) * M(w_uv[b][hh][i][j]) for i in range(d_cb)) for j in range(d_h)]
                z = sum(M(q_nope[hh][j]) * k[j] for j in range(d_h))
                z += sum(M(q_rope[hh][r]) * M(kr[t][r]) for r in range(d_r))
                zs.append(z * M(P["softmax_scale"]))
                vs.append(v)
            den = sum(mp.exp(z) for z in zs)
            lse[hh][b] = mp.log(den)
            for j in range(d_h):
                vb = sum(mp.exp(zs[t]) / den * vs[t][j] for t in range(L))
                out[hh][j] += M(P["branch_scale"]) * vb
    return (np.array([[float(x) for x in row] for row in out]),
            np.array([[float(x) for x in row] for row in lse]))


def _oracle(P, fn=None):
    fn = fn or oracle.decode_sequence
    return fn(P["q_nope"], P["q_rope"], P["c_lat"], P["k_rope"], P["w_uk"], P["w_uv"],
              P["softmax_scale"], P["branch_scale"])


@pytest.mark.parametrize("L", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("nb", [1, 2, 4])
def test_brute_force_small(L, nb):
    rng = np.random.default_rng(100 + 10 * L + nb)
    P = _rand_problem(rng, nb=nb, L=L)
    out_bf, lse_bf = _brute_force(P)
    r = _oracle(P)
    np.testing.assert_allclose(r.out, out_bf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r.lse, lse_bf, rtol=1e-12, atol=1e-13)


def test_mla_equals_textbook_sdpa():
    """n_blocks = 1 is MLA: standard attention with K = [C W_uk, k_rope], V = C W_uv."""
    rng = np.random.default_rng(7)
    h, d_c, d_h, d_r, L = 4, 16, 8, 4, 37
    q_nope = rng.standard_normal((h, d_h))
    q_rope = rng.standard_normal((h, d_r))
    c = rng.standard_normal((L, d_c))
    kr = rng.standard_normal((L, d_r))
    w_uk = rng.standard_normal((h, d_c, d_h)) / 4
    w_uv = rng.standard_normal((h, d_c, d_h)) / 4
    scale = 1.0 / math.sqrt(d_h + d_r)
    r = oracle.mla_decode_sequence(q_nope, q_rope, c, kr, w_uk, w_uv, scale)
    T = lambda x: torch.from_numpy(np.ascontiguousarray(x))  # noqa: E731
    K = torch.cat([torch.einsum("ti,hij->htj", T(c), T(w_uk)),
                   T(kr)[None].expand(h, L, d_r)], dim=-1)          # [h, L, d_h+d_r]
    V = torch.einsum("ti,hij->htj", T(c), T(w_uv))                   # [h, L, d_h]
    Q = torch.cat([T(q_nope), T(q_rope)], dim=-1)[:, None, :]        # [h, 1, d_h+d_r]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[:, 0]
    np.testing.assert_allclose(r.out, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_block_decomposition_identity():
    """Key Contributions #1: the up-projection of a block-split latent is the sum
    of the four block-wise projections (same for K and V)."""
    rng = np.random.default_rng(11)
    nb, d_cb, d_h, L = 4, 8, 6, 9
    c = rng.standard_normal((L, nb, d_cb))
    w = rng.standard_normal((nb, d_cb, d_h))
    full = om.up_project(c.reshape(L, nb * d_cb), w.reshape(nb * d_cb, d_h))
    summed = sum(om.up_project(c[:, b], w[b]) for b in range(nb))
    np.testing.assert_allclose(full, summed, rtol=1e-13, atol=1e-13)


def test_mlra_is_not_mla():
    """Methodology: moving the block sum from K/V to the outputs is not the same
    computation (softmax is nonlinear).  MLA on the concatenated latent with
    stacked weights must differ from MLRA on random data."""
    rng = np.random.default_rng(12)
    P = _rand_problem(rng, h=3, nb=4, d_cb=4, d_h=3, d_r=2, L=16)
    r = _oracle(P)
    nb, h, d_cb, d_h = P["w_uk"].shape
    L = P["c_lat"].shape[0]
    w_uk_full = P["w_uk"].transpose(1, 0, 2, 3).reshape(h, nb * d_cb, d_h)
    w_uv_full = P["w_uv"].transpose(1, 0, 2, 3).reshape(h, nb * d_cb, d_h)
    mla = oracle.mla_decode_sequence(P["q_nope"], P["q_rope"], P["c_lat"].reshape(L, -1),
                                     P["k_rope"], w_uk_full, w_uv_full, P["softmax_scale"])
    assert np.max(np.abs(mla.out - r.out / P["branch_scale"])) > 1e-2
    # ...but with one token both reduce to the plain sum of value projections.
    P1 = dict(P, c_lat=P["c_lat"][:1], k_rope=P["k_rope"][:1])
    r1 = _oracle(P1)
    mla1 = oracle.mla_decode_sequence(P1["q_nope"], P1["q_rope"], P1["c_lat"].reshape(1, -1),
                                      P1["k_rope"], w_uk_full, w_uv_full, P1["softmax_scale"])
    np.testing.assert_allclose(mla1.out, r1.out / P["branch_scale"], rtol=1e-12, atol=1e-13)


def test_single_token_closed_form():
    """L = 1: softmax of one logit is 1, so out = (1/sqrt(nb)) sum_b W_uv[b,h]^T c_b[0]
    (Key Contributions #3: 1/2 for four branches) and lse is the logit itself."""
    rng = np.random.default_rng(13)
    P = _rand_problem(rng, h=3, nb=4, d_cb=5, d_h=4, d_r=2, L=1)
    r = _oracle(P)
    assert P["branch_scale"] == 0.5
    for hh in range(3):
        expect = 0.5 * sum(P["w_uv"][b, hh].T @ P["c_lat"][0, b] for b in range(4))
        np.testing.assert_allclose(r.out[hh], expect, rtol=1e-13, atol=1e-14)
        for b in range(4):
            k = P["c_lat"][0, b] @ P["w_uk"][b, hh]
            z = (k @ P["q_nope"][hh] + P["k_rope"][0] @ P["q_rope"][hh]) * P["softmax_scale"]
            assert abs(r.lse[hh, b] - z) < 1e-13


def test_two_token_sigmoid_form():
    """Two tokens: p_1 = 1 / (1 + exp(z_0 - z_1)) (logistic form of a 2-way softmax)."""
    rng = np.random.default_rng(14)
    P = _rand_problem(rng, h=2, nb=2, d_cb=3, d_h=3, d_r=2, L=2, wscale=1.5)
    r = _oracle(P)
    for hh in range(2):
        acc = np.zeros(3)
        for b in range(2):
            c0, c1 = P["c_lat"][0, b], P["c_lat"][1, b]
            z = [((c @ P["w_uk"][b, hh]) @ P["q_nope"][hh] + kr @ P["q_rope"][hh]) * P["softmax_scale"]
                 for c, kr in ((c0, P["k_rope"][0]), (c1, P["k_rope"][1]))]
            p1 = 1.0 / (1.0 + math.exp(z[0] - z[1]))
            v = (1 - p1) * (c0 @ P["w_uv"][b, hh]) + p1 * (c1 @ P["w_uv"][b, hh])
            np.testing.assert_allclose(r.v[hh, b], v, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(r.o_lat[hh, b], (1 - p1) * c0 + p1 * c1, rtol=1e-12)
            acc += v
        np.testing.assert_allclose(r.out[hh], acc / math.sqrt(2), rtol=1e-12, atol=1e-13)


def test_constant_cache_gives_the_latent_itself():
    """If every token carries the same c_b, o_b = c_b whatever the logits."""
    rng = np.random.default_rng(15)
    P = _rand_problem(rng, h=2, nb=4, d_cb=4, d_h=3, d_r=2, L=11)
    P["c_lat"][:] = P["c_lat"][0]
    r = _oracle(P)
    for hh in range(2):
        for b in range(4):
            np.testing.assert_allclose(r.o_lat[hh, b], P["c_lat"][0, b], rtol=1e-12)


def test_zero_query_is_uniform_mean():
    """Zero queries give equal logits: o_b is the plain mean of c_b, lse = log L."""
    rng = np.random.default_rng(16)
    P = _rand_problem(rng, h=2, nb=4, d_cb=4, d_h=3, d_r=2, L=13)
    P["q_nope"][:] = 0.0
    P["q_rope"][:] = 0.0
    r = _oracle(P)
    np.testing.assert_allclose(r.o_lat[0, 2], P["c_lat"][:, 2].mean(axis=0), rtol=1e-12)
    np.testing.assert_allclose(r.lse, np.log(13.0), rtol=1e-14)


def test_shift_invariance_through_rope():
    """A token-independent RoPE key adds the same amount to every logit of a head:
    the outputs are unchanged and each lse moves by exactly that amount."""
    rng = np.random.default_rng(17)
    P = _rand_problem(rng, h=2, nb=4, d_cb=4, d_h=3, d_r=2, L=9)
    P["k_rope"][:] = P["k_rope"][0]
    r0 = _oracle(P)
    dq = rng.standard_normal(P["q_rope"].shape)
    r1 = _oracle(dict(P, q_rope=P["q_rope"] + dq))
    np.testing.assert_allclose(r1.out, r0.out, rtol=1e-11, atol=1e-12)
    shift = (dq @ P["k_rope"][0]) * P["softmax_scale"]
    np.testing.assert_allclose(r1.lse - r0.lse, np.repeat(shift[:, None], 4, axis=1),
                               rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("nb", [1, 2, 4])
def test_absorbed_equals_unabsorbed(nb):
    """Main Findings: decoding reduces to absorbable steps, so the absorbed form
    (query absorption, attention over the latent, output up-projection) gives
    the same result as explicit per-head keys and values."""
    rng = np.random.default_rng(18 + nb)
    P = _rand_problem(rng, h=3, nb=nb, d_cb=7, d_h=5, d_r=3, L=40)
    a = _oracle(P)
    b = _oracle(P, fn=oracle.absorbed_decode)
    for x, y in ((a.out, b.out), (a.lse, b.lse), (a.o_lat, b.o_lat), (a.v, b.v)):
        np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-12)


def test_absorb_query_definition():
    """q_abs . c_b = q_nope . (c_b W_uk[b,h]) for every block and head."""
    rng = np.random.default_rng(19)
    nb, h, d_cb, d_h = 4, 3, 6, 5
    w = rng.standard_normal((nb, h, d_cb, d_h))
    q = rng.standard_normal((h, d_h))
    c = rng.standard_normal((d_cb,))
    qa = oracle.absorb_query(q, w)
    for b in range(nb):
        for hh in range(h):
            assert abs(qa[hh, b] @ c - q[hh] @ (c @ w[b, hh])) < 1e-12


def test_empty_sequence():
    rng = np.random.default_rng(20)
    P = _rand_problem(rng, L=0)
    P["c_lat"] = np.zeros((0, 4, 3))
    P["k_rope"] = np.zeros((0, 2))
    r = _oracle(P)
    assert np.all(r.out == 0) and np.all(np.isneginf(r.lse))


def _ev(s):
    s = s.replace("sqrt", "math.sqrt").replace("log", "math.log")
    return float(eval(s, {"math": math, "Fraction": Fraction}))


def _arr(x):
    if isinstance(x, str):
        return _ev(x)
    return np.array([_arr(y) for y in x], dtype=np.float64)


def test_golden_tiny_two_branch():
    with open(os.path.join(GOLDEN, "tiny_two_branch.json")) as f:
        G = json.load(f)
    P = dict(q_nope=_arr(G["q_nope"]), q_rope=_arr(G["q_rope"]), c_lat=_arr(G["c_lat"]),
             k_rope=_arr(G["k_rope"]), w_uk=_arr(G["w_uk"]), w_uv=_arr(G["w_uv"]),
             softmax_scale=_ev(G["softmax_scale"]), branch_scale=_ev(G["branch_scale"]))
    r = _oracle(P)
    E = G["expected"]
    np.testing.assert_allclose(r.out, _arr(E["out"]), rtol=1e-14)
    np.testing.assert_allclose(r.lse, _arr(E["lse"]), rtol=1e-14)
    np.testing.assert_allclose(r.o_lat, _arr(E["o_lat"]), rtol=1e-14)
    np.testing.assert_allclose(r.v, _arr(E["v"]), rtol=1e-14)
    L = P["c_lat"].shape[0]
    w_uk_full = P["w_uk"].transpose(1, 0, 2, 3).reshape(1, 2, 1)
    w_uv_full = P["w_uv"].transpose(1, 0, 2, 3).reshape(1, 2, 1)
    mla = oracle.mla_decode_sequence(P["q_nope"], P["q_rope"], P["c_lat"].reshape(L, -1),
                                     P["k_rope"], w_uk_full, w_uv_full, P["softmax_scale"])
    np.testing.assert_allclose(mla.out, _arr(E["mla_out"]), rtol=1e-14)
    np.testing.assert_allclose(mla.lse, _arr(E["mla_lse"]), rtol=1e-14)


# ---- planted mistakes: each must be caught by at least one pin -------------

def _planted_variants():
    def no_rope(q_nope_h, q_rope_h, k_nope, k_rope, v, scale):
        return _orig_branch(q_nope_h, 0 * q_rope_h, k_nope, k_rope, v, scale)

    def no_scale(q_nope_h, q_rope_h, k_nope, k_rope, v, scale):
        return _orig_branch(q_nope_h, q_rope_h, k_nope, k_rope, v, 1.0)

    def wrong_sign(q_nope_h, q_rope_h, k_nope, k_rope, v, scale):
        return _orig_branch(q_nope_h, -q_rope_h, k_nope, k_rope, v, scale)

    def transposed_w(c_b, w):
        return c_b @ (w.T if w.shape[0] == w.shape[1] else w)

    return [("branch_attention", no_rope), ("branch_attention", no_scale),
            ("branch_attention", wrong_sign), ("up_project", transposed_w)]


_orig_branch = om.branch_attention


@pytest.mark.parametrize("which", range(4))
def test_planted_mistake_is_caught(which, monkeypatch):
    name, fn = _planted_variants()[which]
    monkeypatch.setattr(om, name, fn)
    rng = np.random.default_rng(21)
    P = _rand_problem(rng, h=2, nb=2, d_cb=3, d_h=3, d_r=2, L=4)
    out_bf, lse_bf = _brute_force(P)
    r = _oracle(P)
    assert not (np.allclose(r.out, out_bf, rtol=1e-9) and np.allclose(r.lse, lse_bf, rtol=1e-9))


# ---- the oracle's input plumbing: cache-row split and sampled regeneration ----

def test_split_cache_rows_takes_blocks_then_the_rope_key():
    """A cache row is [c_0 | c_1 | ... | c_{nb-1} | k_rope] (4.5 d_h per token at
    d_h = 128: Key Contributions #2).  Rows built from known blocks with
    distinct integer values split back into exactly those blocks, the RoPE
    key taken from offset nb * d_cb."""
    L, nb, d_cb, d_r = 3, 4, 5, 2
    c = np.arange(L * nb * d_cb, dtype=np.float64).reshape(L, nb, d_cb)
    kr = -1.0 - np.arange(L * d_r, dtype=np.float64).reshape(L, d_r)
    rows = np.concatenate([np.concatenate([c[t, b] for b in range(nb)] + [kr[t]])[None]
                           for t in range(L)])
    assert rows.shape == (L, nb * d_cb + d_r)
    c2, kr2 = om.split_cache_rows(rows, nb, d_cb)
    assert np.array_equal(c2, c) and np.array_equal(kr2, kr)
    # block b of token t starts at column b * d_cb; the RoPE key at nb * d_cb
    assert c2[2, 3, 0] == rows[2, 3 * d_cb] and kr2[1, 0] == rows[1, nb * d_cb]
    # the cache-write oracle lays a row out the same way
    g = np.ones(nb * d_cb)
    new = oracle.cache_rows(c.reshape(L, -1), kr, g, nb, 1.0, 0.0, np.zeros(L), 10000.0)
    c3, kr3 = om.split_cache_rows(new, nb, d_cb)
    np.testing.assert_allclose(kr3, kr, rtol=0, atol=0)   # RoPE at position 0 is the identity
    norm = c / np.sqrt(np.mean(c * c, axis=-1, keepdims=True))
    np.testing.assert_allclose(c3, norm, rtol=1e-15)


def test_split_cache_rows_same_latent_for_mla_and_mlra4():
    """MLA (one block of 512 + 64) and MLRA-4 (4 x 128 + 64) read the same 576
    columns: the latent part of a row is the same bytes either way."""
    rng = np.random.default_rng(3)
    rows = rng.standard_normal((7, 576))
    c4, kr4 = om.split_cache_rows(rows, 4, 128)
    c1, kr1 = om.split_cache_rows(rows, 1, 512)
    assert np.array_equal(c4.reshape(7, 512), c1.reshape(7, 512))
    assert np.array_equal(kr4, kr1) and kr4.shape == (7, 64)


@pytest.mark.parametrize("name,seq,L", [
    ("mlra4_bf16_b64_h32_l16384_paged", 2, 300),
    ("mlra4_bf16_b128_h16_ragged1k_64k_paged", 1, 4100),
    ("mla_bf16_b8_h128_l131072_paged", 0, 130),
    ("mlra4_bf16_b16_h16_l4096_contig", 1, 70),
])
def test_decode_sampled_equals_decode_batch(name, seq, L):
    """decode_sampled (one sequence's inputs redrawn from their seeds, used at
    full sizes) gives exactly what decode_batch gives on the same sequence of
    the whole generated batch (paged or contiguous, other sequences present)."""
    import workloads as W
    base = W.WORKLOADS[name]
    heads = [0, base.n_heads - 1]
    lens = np.array([L + 7 * s for s in range(seq + 2)], np.int32)
    spec = W.scaled_down(base, len(lens), seqlen=int(lens.max()), seed=9)
    inp = W.make_inputs(spec, "cpu", seqlens=lens)
    whole = oracle.decode_batch(inp, heads=heads, seqs=[seq])[0]
    one = oracle.decode_sampled(spec, seq, heads, int(lens[seq]))
    for k in ("out", "lse", "o_lat", "v"):
        assert np.array_equal(getattr(one, k)[heads], getattr(whole, k)[heads]), k
