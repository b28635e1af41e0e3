"""Pins of the cache-write oracle (per-block RMSNorm with gain, alpha_kv, RoPE)
against what the mathematics and the pages fix, independent of the oracle's
own formulas."""
import math

import numpy as np
import pytest

from oracle import cache_rows, kv_scale, rms_norm_blocks, rope


def test_rope_at_position_zero_is_identity():
    x = np.random.default_rng(0).normal(size=(3, 64))
    np.testing.assert_array_equal(rope(x, np.zeros(3), 10000.0), x)


def test_rope_two_channels_closed_form():
    # one pair, inverse frequency theta^0 = 1: a plain rotation by pos radians
    x = np.array([[0.3, -1.7]])
    got = rope(x, np.array([2]), 10000.0)[0]
    c, s = math.cos(2.0), math.sin(2.0)
    np.testing.assert_allclose(got, [0.3 * c + 1.7 * s, 0.3 * s - 1.7 * c], rtol=0, atol=1e-15)


def test_rope_pairs_channel_i_with_i_plus_half():
    # only channels 5 and 5 + 32 are non-zero: the rotation must stay on that pair
    x = np.zeros((1, 64))
    x[0, 5], x[0, 37] = 1.0, 2.0
    got = rope(x, np.array([7]), 10000.0)[0]
    others = np.delete(got, [5, 37])
    assert np.all(others == 0.0)
    assert abs(np.hypot(got[5], got[37]) - math.hypot(1.0, 2.0)) < 1e-14
    ang = 7 * 10000.0 ** (-2 * 5 / 64)
    assert abs(math.atan2(got[37], got[5]) - math.atan2(2.0, 1.0) - ang) % (2 * math.pi) < 1e-12


def test_rope_preserves_norm_and_adds_angles():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(4, 64))
    a, b = np.array([3, 100, 4096, 131071]), np.array([1, 77, 5, 2])
    np.testing.assert_allclose(np.linalg.norm(rope(x, a, 1e4), axis=1), np.linalg.norm(x, axis=1),
                               rtol=1e-13)
    np.testing.assert_allclose(rope(rope(x, a, 1e4), b, 1e4), rope(x, a + b, 1e4), rtol=0,
                               atol=1e-9)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    q, k = rng.normal(size=64), rng.normal(size=64)
    s1 = rope(q[None], np.array([900]), 1e4)[0] @ rope(k[None], np.array([850]), 1e4)[0]
    s2 = rope(q[None], np.array([50]), 1e4)[0] @ rope(k[None], np.array([0]), 1e4)[0]
    assert abs(s1 - s2) < 1e-10


def test_rms_norm_of_constant_block_is_its_sign_times_gain():
    c = np.concatenate([np.full(128, 3.0), np.full(128, -0.5)])
    gamma = np.linspace(0.5, 2.0, 256)
    got = rms_norm_blocks(c, gamma, 2, eps=0.0)
    np.testing.assert_allclose(got, np.concatenate([np.ones(128), -np.ones(128)]) * gamma, rtol=1e-14)


def test_rms_norm_is_per_block_and_scale_free():
    rng = np.random.default_rng(3)
    c = rng.normal(size=512)
    gamma = np.ones(512)
    base = rms_norm_blocks(c, gamma, 4, eps=0.0)
    c2 = c.copy()
    c2[128:256] *= 37.0  # rescale block 1 only
    got = rms_norm_blocks(c2, gamma, 4, eps=0.0)
    np.testing.assert_allclose(got, base, rtol=1e-13)
    # unit RMS per block
    np.testing.assert_allclose(np.sqrt(np.mean(base.reshape(4, 128) ** 2, axis=1)), 1.0, rtol=1e-13)


def test_kv_scale_matches_the_pages_formula():
    d, d_c = 4096, 512
    # four branches: sqrt(4 d / d_c) with d_c the whole latent (Main Findings)
    assert abs(kv_scale(d, d_c // 4) - math.sqrt(4 * d / d_c)) < 1e-12
    # MLA, one block: sqrt(d / d_c)
    assert abs(kv_scale(d, d_c) - math.sqrt(d / d_c)) < 1e-12


def test_cache_rows_layout():
    rng = np.random.default_rng(4)
    c, kr = rng.normal(size=(2, 512)), rng.normal(size=(2, 64))
    rows = cache_rows(c, kr, np.ones(512), 4, 2.0, 1e-6, np.array([0, 9]), 1e4)
    assert rows.shape == (2, 576)
    np.testing.assert_allclose(rows[0, 512:], kr[0], rtol=0, atol=0)  # position 0: unrotated
    np.testing.assert_allclose(np.sqrt(np.mean(rows[:, :128] ** 2, axis=1)), 2.0, rtol=1e-5)


# ---- the query side: alpha_q and RoPE at the query's position ----------------

def test_q_scale_matches_the_pages_formula():
    """alpha_q = sqrt(d / d_c') (Main Findings, variance bullet)."""
    from oracle import q_scale
    assert q_scale(4096, 1024) == 2.0
    assert q_scale(2048, 512) == 2.0
    assert abs(q_scale(7168, 1536) - math.sqrt(7168 / 1536)) < 1e-15
    assert q_scale(512, 512) == 1.0


def test_query_side_at_position_zero_is_a_plain_scale():
    from oracle import query_side
    rng = np.random.default_rng(5)
    qn, qr = rng.normal(size=(3, 4, 128)), rng.normal(size=(3, 4, 64))
    a, b = query_side(qn, qr, np.zeros((3, 1)), 1.5, 10000.0)
    np.testing.assert_array_equal(a, 1.5 * qn)
    np.testing.assert_array_equal(b, 1.5 * qr)


def test_query_alpha_scales_every_logit():
    """Both parts of the query carry alpha_q, so the decode with the scaled query
    equals the decode with the unscaled query and softmax scale * alpha_q."""
    import oracle
    from oracle import query_side
    rng = np.random.default_rng(6)
    h, nb, d_cb, d_h, d_r, L = 2, 4, 8, 8, 4, 9
    qn, qr = rng.normal(size=(h, d_h)), rng.normal(size=(h, d_r))
    c, kr = rng.normal(size=(L, nb, d_cb)), rng.normal(size=(L, d_r))
    wk, wv = rng.normal(size=(nb, h, d_cb, d_h)), rng.normal(size=(nb, h, d_cb, d_h))
    a = 1.7
    qn2, qr2 = query_side(qn, qr, np.zeros(h), a, 10000.0)
    r1 = oracle.decode_sequence(qn2, qr2, c, kr, wk, wv, 0.3, 0.5)
    r2 = oracle.decode_sequence(qn, qr, c, kr, wk, wv, 0.3 * a, 0.5)
    np.testing.assert_allclose(r1.out, r2.out, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(r1.lse, r2.lse, rtol=1e-13)


def test_query_and_key_rotations_meet_at_their_distance():
    """The RoPE logit of a query rotated at position p against a cache key
    written at position t depends on p - t alone (the query side and the cache
    write use the same rotation)."""
    from oracle import query_side
    rng = np.random.default_rng(7)
    q, k = rng.normal(size=64), rng.normal(size=64)
    g = np.ones(8)

    def logit(p, t):
        _, qr = query_side(np.zeros(4), q[None], np.array([p]), 1.0, 10000.0)
        row = cache_rows(np.ones((1, 8)), k[None], g, 1, 1.0, 0.0, np.array([t]), 10000.0)
        return float(qr[0] @ row[0, 8:])

    for p, t, dp in [(10, 3, 50), (131071, 131000, -5000), (7, 7, 123)]:
        assert abs(logit(p, t) - logit(p + dp, t + dp)) < 1e-9
    # and it is not position-free: a different distance gives a different logit
    assert abs(logit(10, 3) - logit(11, 3)) > 1e-6
