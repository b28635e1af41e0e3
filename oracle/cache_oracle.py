"""fp64 reference of the cache-write step (CPU, numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The step that produces a token's cache row before decode attention reads it
("Multi-Head Low-Rank Attention", ai.info AI summary):

* Methodology, third paragraph: the latent states are RMS-normalised before
  the up-projection, which is why the RoPE key would otherwise dominate the
  NoPE key's variance.
* Main Findings, variance bullet: the KV latent is rescaled by
  alpha_kv = sqrt(d / d_c), applied as sqrt(4 d / d_c) for the four branches.

Readings (the pages give no formulas for them):

* The normalisation is per latent block of d_cb channels (n_blocks of them),
  with a learned per-channel gain: c_b <- gamma_b * c_b / sqrt(mean(c_b^2) + eps).
  With d_c = n_blocks * d_cb, "sqrt(4 d / d_c)" for four blocks is
  sqrt(d / d_cb): the same rule for every block, and sqrt(d / d_c) for MLA.
* RoPE on the decoupled key is the usual rotary embedding with the
  rotate-half pairing: channel i is paired with channel i + d_r / 2, angle
  pos * theta^(-2 i / d_r).
"""
from __future__ import annotations

import numpy as np

from .mlra_oracle import _f64


def kv_scale(d_model: int, d_cb: int) -> float:
    """alpha_kv for one latent block of d_cb channels (reading above)."""
    return float(np.sqrt(d_model / d_cb))


def rms_norm_blocks(c, gamma, n_blocks: int, eps: float):
    """Per-block RMSNorm with gain: c [..., n_blocks * d_cb] -> same shape."""
    c, gamma = _f64(c), _f64(gamma)
    shp = c.shape
    blocks = c.reshape(shp[:-1] + (n_blocks, shp[-1] // n_blocks))
    rms = np.sqrt(np.mean(blocks * blocks, axis=-1, keepdims=True) + eps)
    return (blocks / rms).reshape(shp) * gamma


def rope(x, pos, theta: float):
    """Rotary embedding of x [..., d_r] at integer positions pos [...]."""
    x = _f64(x)
    d_r = x.shape[-1]
    half = d_r // 2
    inv_freq = theta ** (-2.0 * np.arange(half) / d_r)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


def q_scale(d_model: int, d_cq: int) -> float:
    """alpha_q = sqrt(d / d_c') (Main Findings, variance bullet), d_c' the
    query latent's width."""
    return float(np.sqrt(d_model / d_cq))


def query_side(q_nope, q_rope, pos, alpha_q: float, theta: float):
    """The query's share of the calibration and of RoPE (reading: alpha_q scales
    the normalised query latent, and the query up-projection is linear, so it
    scales both q_nope and q_rope; RoPE then rotates q_rope at the query's
    position with the cache key's rotation).  q_nope [..., d_h], q_rope
    [..., d_r], pos broadcast over the leading axes -> (q_nope', q_rope')."""
    q_nope, q_rope = _f64(q_nope), _f64(q_rope)
    return alpha_q * q_nope, rope(alpha_q * q_rope, pos, theta)


def cache_rows(c_new, k_rope_new, gamma, n_blocks: int, alpha_kv: float, eps: float,
               pos, theta: float):
    """The new tokens' cache rows [B, n_blocks * d_cb + d_r] (fp64)."""
    lat = rms_norm_blocks(c_new, gamma, n_blocks, eps) * alpha_kv
    return np.concatenate([lat, rope(k_rope_new, pos, theta)], axis=-1)
