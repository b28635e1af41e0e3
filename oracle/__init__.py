"""CPU fp64 oracle for MLRA / MLA latent-KV decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library or its Python binding.

What it computes (the unabsorbed form, "Multi-Head Low-Rank Attention",
ai.info AI summary):

* Methodology, first paragraph: a head's NoPE key and value are the latent
  times an up-projection matrix; sliced into channel blocks the result is the
  sum of the block products (block-decomposition identity, Key Contributions
  #1).
* Methodology, second paragraph and Key Contributions #2: MLRA runs attention
  separately on every latent block (each block up-projected on its own to a
  NoPE key / value), one softmax per branch, and sums the branch outputs; this
  is not the same as MLA's single attention over the summed key/value, because
  softmax is nonlinear.
* Key Contributions #2: the logit of a branch combines its NoPE key with the
  decoupled RoPE key (after absorption, d_h + d_h/2 = 1.5 d_h per head).
* Key Contributions #3: the branch outputs are rescaled by the branch count
  (1/sqrt(2) for two branches, 1/2 for four), read as 1/sqrt(n_blocks).
* Main Findings, "three absorbable steps": the same result in absorbed form
  (query absorption, attention over the shared latent, output up-projection);
  ``absorbed_decode`` writes that form out so the two can be compared.

Index convention (the pages give none): ``W[b, h, i, j]`` maps latent channel
``i`` of block ``b`` to head-dim channel ``j`` of head ``h``:
``k_nope[t, j] = sum_i c_b[t, i] W_uk[b, h, i, j]``.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
brute-force high-precision loops (mpmath), ``torch`` SDPA for the MLA case,
closed forms (one token, two tokens, constant cache, zero query), the
block-decomposition identity and a golden fixture in ``tests/golden/``.
"""
from .mlra_oracle import (  # noqa: F401
    up_project,
    branch_attention,
    decode_sequence,
    absorbed_decode,
    absorb_query,
    mla_decode_sequence,
    decode_batch,
    decode_sampled,
    SeqResult,
)
from .cache_oracle import (  # noqa: F401
    q_scale,
    query_side,
    kv_scale,
    rms_norm_blocks,
    rope,
    cache_rows,
)
