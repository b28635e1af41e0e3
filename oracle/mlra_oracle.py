"""fp64 reference of one decode step of MLRA / MLA attention (CPU, numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg, never by the
product path.

All arrays are converted to float64 on entry; inputs are the exact values the
GPU receives (already rounded to their storage dtype).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch  # local: only for dtype conversion of torch inputs
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def up_project(c_b: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Explicit per-head NoPE key or value of one latent block.

    "Multi-Head Low-Rank Attention" (ai.info summary), Methodology: a head's
    NoPE key / value is the latent multiplied by its up-projection matrix.
    ``c_b`` [L, d_cb], ``w`` [d_cb, d_h] -> [L, d_h].
    """
    return c_b @ w


def branch_attention(q_nope_h: np.ndarray, q_rope_h: np.ndarray, k_nope: np.ndarray,
                     k_rope: np.ndarray, v: np.ndarray, scale: float
                     ) -> Tuple[np.ndarray, float, np.ndarray]:
    """Standard softmax attention of one query over one branch.

    logits z_t = (q_nope . k_nope[t] + q_rope . k_rope[t]) * scale (Key
    Contributions #2: NoPE key of the branch plus the shared decoupled RoPE
    key); p = softmax(z); returns (p @ v, logsumexp(z), p).
    An empty branch (L = 0) returns zeros and lse = -inf.
    """
    L = k_nope.shape[0]
    if L == 0:
        return np.zeros(v.shape[1]), -np.inf, np.zeros(0)
    z = (k_nope @ q_nope_h + k_rope @ q_rope_h) * scale
    m = np.max(z)
    e = np.exp(z - m)
    s = np.sum(e)
    p = e / s
    return p @ v, float(m + np.log(s)), p


@dataclass
class SeqResult:
    out: np.ndarray    # [h, d_h]      (1/sqrt(nb)) * sum_b v_b
    lse: np.ndarray    # [h, nb]       natural-log logsumexp of each branch's logits
    o_lat: np.ndarray  # [h, nb, d_cb] p_b @ c_b: the latent output of each branch
    v: np.ndarray      # [h, nb, d_h]  p_b @ (c_b W_uv[b,h]): each branch's value output


def decode_sequence(q_nope, q_rope, c_lat, k_rope, w_uk, w_uv, softmax_scale: float,
                    branch_scale: float, heads: Optional[Iterable[int]] = None) -> SeqResult:
    """Unabsorbed MLRA decode of one sequence (MLA when n_blocks == 1).

    q_nope [h, d_h], q_rope [h, d_r], c_lat [L, nb, d_cb], k_rope [L, d_r],
    w_uk / w_uv [nb, h, d_cb, d_h].  For every head and block: explicit NoPE
    key and value through W_uk_b / W_uv_b, softmax attention on that branch
    alone, then the branch outputs are summed and scaled by ``branch_scale``
    (Methodology, second paragraph; Key Contributions #2, #3).
    ``heads`` restricts the work to a subset of heads (others stay zero).
    """
    q_nope, q_rope, c_lat, k_rope = map(_f64, (q_nope, q_rope, c_lat, k_rope))
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    nb, h, d_cb, d_h = w_uk.shape
    L = c_lat.shape[0]
    assert c_lat.shape == (L, nb, d_cb) and k_rope.shape[0] == L
    out = np.zeros((h, d_h))
    lse = np.full((h, nb), -np.inf)
    o_lat = np.zeros((h, nb, d_cb))
    v_all = np.zeros((h, nb, d_h))
    hs = range(h) if heads is None else heads
    for hh in hs:
        for b in range(nb):
            c_b = c_lat[:, b, :]
            k_nope = up_project(c_b, w_uk[b, hh])
            v = up_project(c_b, w_uv[b, hh])
            vb, lb, p = branch_attention(q_nope[hh], q_rope[hh], k_nope, k_rope, v,
                                         softmax_scale)
            v_all[hh, b] = vb
            lse[hh, b] = lb
            o_lat[hh, b] = p @ c_b if L else 0.0
        out[hh] = branch_scale * v_all[hh].sum(axis=0)
    return SeqResult(out=out, lse=lse, o_lat=o_lat, v=v_all)


def absorb_query(q_nope, w_uk) -> np.ndarray:
    """Query-side weight absorption (Main Findings, "three absorbable steps").

    q_abs[h, b, i] = sum_j W_uk[b, h, i, j] q_nope[h, j], so that
    q_abs . c_b[t] = q_nope . k_nope[t].  q_nope [h, d_h] -> [h, nb, d_cb].
    """
    q_nope, w_uk = _f64(q_nope), _f64(w_uk)
    return np.einsum("bhij,hj->hbi", w_uk, q_nope)


def absorbed_decode(q_nope, q_rope, c_lat, k_rope, w_uk, w_uv, softmax_scale: float,
                    branch_scale: float) -> SeqResult:
    """The absorbed form (Main Findings, "three absorbable steps").

    1. absorb the query into the latent space of each block;
    2. MQA-style attention of every (head, block) directly over the shared
       latent c_b plus the RoPE key, one softmax per branch;
    3. output up-projection of each branch's latent output through W_uv_b,
       summed over blocks and scaled by ``branch_scale``.
    No per-head key or value is formed.  Used to pin the unabsorbed oracle.
    """
    q_rope, c_lat, k_rope, w_uv = map(_f64, (q_rope, c_lat, k_rope, w_uv))
    q_abs = absorb_query(q_nope, w_uk)
    nb, h, d_cb, d_h = w_uv.shape
    L = c_lat.shape[0]
    out = np.zeros((h, d_h))
    lse = np.full((h, nb), -np.inf)
    o_lat = np.zeros((h, nb, d_cb))
    v_all = np.zeros((h, nb, d_h))
    for hh in range(h):
        for b in range(nb):
            if L == 0:
                continue
            z = (c_lat[:, b, :] @ q_abs[hh, b] + k_rope @ q_rope[hh]) * softmax_scale
            m = z.max()
            e = np.exp(z - m)
            lse[hh, b] = m + np.log(e.sum())
            o_lat[hh, b] = (e / e.sum()) @ c_lat[:, b, :]
            v_all[hh, b] = o_lat[hh, b] @ w_uv[b, hh]
        out[hh] = branch_scale * v_all[hh].sum(axis=0)
    return SeqResult(out=out, lse=lse, o_lat=o_lat, v=v_all)


def mla_decode_sequence(q_nope, q_rope, c_full, k_rope, w_uk_full, w_uv_full,
                        softmax_scale: float) -> SeqResult:
    """MLA: one latent head, one softmax (the n_blocks = 1 comparison mode).

    c_full [L, d_c], w_*_full [h, d_c, d_h].  This is ``decode_sequence`` with a
    single block and branch scale 1.
    """
    c_full = _f64(c_full)
    return decode_sequence(q_nope, q_rope, c_full[:, None, :], k_rope,
                           _f64(w_uk_full)[None], _f64(w_uv_full)[None],
                           softmax_scale, 1.0)


def split_cache_rows(rows, n_blocks: int, d_cb: int) -> Tuple[np.ndarray, np.ndarray]:
    """Cache rows [L, nb*d_cb + d_r] -> (c_lat [L, nb, d_cb], k_rope [L, d_r])."""
    rows = _f64(rows)
    L = rows.shape[0]
    c = rows[:, : n_blocks * d_cb].reshape(L, n_blocks, d_cb)
    return c, rows[:, n_blocks * d_cb:]


def decode_batch(inp, heads: Optional[Iterable[int]] = None,
                 seqs: Optional[Sequence[int]] = None) -> List[SeqResult]:
    """Oracle over a ``workloads.DecodeInputs`` batch (or a subset of sequences)."""
    import workloads  # inputs only: no arithmetic of the method lives there

    spec = inp.spec
    out = []
    seq_ids = range(spec.batch) if seqs is None else seqs
    for s in seq_ids:
        rows = workloads.sequence_cache(inp, s)
        c, kr = split_cache_rows(rows, spec.n_blocks, spec.d_cb)
        out.append(decode_sequence(inp.q_nope[s], inp.q_rope[s], c, kr, inp.w_uk, inp.w_uv,
                                   spec.softmax_scale, spec.branch_scale, heads=heads))
    return out


def decode_sampled(spec, seq: int, heads: Sequence[int], seqlen: int) -> SeqResult:
    """Oracle for a few heads of one sequence, regenerating its inputs alone.

    Used at full workload sizes, where the whole batch is too large for the
    CPU: the sequence's cache rows are redrawn from their seeds.
    """
    import workloads

    w_uk, w_uv = workloads.weights(spec)
    q_nope, q_rope = workloads.queries(spec)
    rows = workloads.token_rows(spec, seq, 0, seqlen)
    c, kr = split_cache_rows(rows, spec.n_blocks, spec.d_cb)
    return decode_sequence(q_nope[seq], q_rope[seq], c, kr, w_uk, w_uv,
                           spec.softmax_scale, spec.branch_scale, heads=heads)
