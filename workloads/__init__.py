"""Seeded synthetic inputs for MLRA / MLA latent-KV decode attention.

This module is shared by the CPU oracle (``oracle/``), the tests, ``bench.py``
and ``__graft_entry__.smoke()``.  It draws random numbers, rounds them to the
storage dtype and lays them out (contiguous or paged cache, page table,
sequence lengths).  It holds none of the attention arithmetic.

Shapes and value distributions follow the workloads the method is studied on
("Multi-Head Low-Rank Attention", ai.info summary: Key Contributions #2 and
Methodology; MLA-scale dims d_h=128, d_h^R=64, latent 4x128 = 512):

* latent block ``c_b`` of width ``d_cb`` per block, ``n_blocks`` blocks, plus a
  shared RoPE key of width ``d_r = d_h/2``; one cache row per token is
  ``[c_0 | c_1 | ... | c_{nb-1} | k_rope]`` (``D = nb*d_cb + d_r`` elements);
* W_uk, W_uv: ``[nb, h, d_cb, d_h]`` i.i.d. N(0,1)/sqrt(d_cb);
* q_nope ``[B, h, d_h]``, q_rope ``[B, h, d_r]``: N(0, q_std^2);
* cache rows: i.i.d. N(0, 1);
* paged caches use 64-token pages placed by a seeded random permutation.

Every random draw comes from a ``torch.Generator`` (CPU, Mersenne Twister)
seeded from (workload seed, purpose, sequence, 4096-token chunk), so any one
sequence can be regenerated on its own and the result does not depend on how
the cache is batched or on the device it is uploaded to.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Dict, Iterator, List, Optional, Tuple

import numpy as np
import torch

PAGE_SIZE = 64
TOKEN_CHUNK = 4096  # tokens per independently seeded block of cache rows

_P = 1_000_003


def _seed(*parts: int) -> int:
    """Deterministic 63-bit seed from a tuple of small integers."""
    s = 0x5EED
    for p in parts:
        s = (s * _P + int(p) + 1) & ((1 << 63) - 1)
    return s


@dataclass(frozen=True)
class WorkloadSpec:
    """One decode-attention workload (one layer, one decode step)."""

    name: str
    dtype: str                 # "f32" or "bf16": storage dtype of cache, weights, queries
    batch: int
    n_heads: int
    n_blocks: int              # 4 = MLRA-4, 1 = MLA
    d_cb: int                  # latent block width
    d_h: int                   # per-head NoPE key / value width
    d_r: int                   # shared RoPE key width
    seqlen: int = 0            # fixed length (when ragged is None)
    ragged: Optional[Tuple[int, int]] = None  # inclusive [lo, hi] uniform lengths
    paged: bool = False
    q_std: float = 1.0
    identity_w_uk: bool = False  # queries given pre-absorbed: W_uk = I, q_nope := q_abs
    seed: int = 0

    @property
    def D(self) -> int:
        return self.n_blocks * self.d_cb + self.d_r

    @property
    def softmax_scale(self) -> float:
        # per-branch key width after absorption is d_h (NoPE) + d_r (RoPE)
        return 1.0 / math.sqrt(self.d_h + self.d_r)

    @property
    def branch_scale(self) -> float:
        # 1/sqrt(n_blocks): 1/2 for four branches, 1/sqrt(2) for two, 1 for MLA
        return 1.0 / math.sqrt(self.n_blocks)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


# The five workloads (plus the MLA/MLRA-4 pair of the long-context comparison).
WORKLOADS: Dict[str, WorkloadSpec] = {
    "mlra4_f32_b1_h4_l256": WorkloadSpec(
        name="mlra4_f32_b1_h4_l256", dtype="f32", batch=1, n_heads=4, n_blocks=4,
        d_cb=64, d_h=64, d_r=32, seqlen=256),
    "mlra4_bf16_b16_h16_l4096_contig": WorkloadSpec(
        name="mlra4_bf16_b16_h16_l4096_contig", dtype="bf16", batch=16, n_heads=16,
        n_blocks=4, d_cb=128, d_h=128, d_r=64, seqlen=4096,
        q_std=1.0 / math.sqrt(512.0), identity_w_uk=True),
    "mlra4_bf16_b64_h32_l16384_paged": WorkloadSpec(
        name="mlra4_bf16_b64_h32_l16384_paged", dtype="bf16", batch=64, n_heads=32,
        n_blocks=4, d_cb=128, d_h=128, d_r=64, seqlen=16384, paged=True),
    "mlra4_bf16_b128_h16_ragged1k_64k_paged": WorkloadSpec(
        name="mlra4_bf16_b128_h16_ragged1k_64k_paged", dtype="bf16", batch=128,
        n_heads=16, n_blocks=4, d_cb=128, d_h=128, d_r=64, ragged=(1024, 65536),
        paged=True),
    "mla_bf16_b8_h128_l131072_paged": WorkloadSpec(
        name="mla_bf16_b8_h128_l131072_paged", dtype="bf16", batch=8, n_heads=128,
        n_blocks=1, d_cb=512, d_h=128, d_r=64, seqlen=131072, paged=True),
    "mlra4_bf16_b8_h128_l131072_paged": WorkloadSpec(
        name="mlra4_bf16_b8_h128_l131072_paged", dtype="bf16", batch=8, n_heads=128,
        n_blocks=4, d_cb=128, d_h=128, d_r=64, seqlen=131072, paged=True),
}


def seqlens_for(spec: WorkloadSpec) -> np.ndarray:
    """Per-sequence cache lengths (int32)."""
    if spec.ragged is None:
        return np.full(spec.batch, spec.seqlen, dtype=np.int32)
    lo, hi = spec.ragged
    g = torch.Generator().manual_seed(_seed(spec.seed, 7))
    return torch.randint(lo, hi + 1, (spec.batch,), generator=g,
                         dtype=torch.int64).numpy().astype(np.int32)


def _normal(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    x = torch.empty(shape, dtype=torch.float32)
    x.normal_(0.0, 1.0, generator=g)
    if std != 1.0:
        x.mul_(std)
    return x


def weights(spec: WorkloadSpec) -> Tuple[torch.Tensor, torch.Tensor]:
    """W_uk, W_uv: [nb, h, d_cb, d_h] in the storage dtype (CPU)."""
    shp = (spec.n_blocks, spec.n_heads, spec.d_cb, spec.d_h)
    w_std = 1.0 / math.sqrt(spec.d_cb)
    if spec.identity_w_uk:
        assert spec.d_cb == spec.d_h
        w_uk = torch.eye(spec.d_cb, dtype=torch.float32).expand(shp).contiguous()
    else:
        w_uk = _normal(shp, _seed(spec.seed, 1), w_std)
    w_uv = _normal(shp, _seed(spec.seed, 2), w_std)
    return w_uk.to(spec.torch_dtype), w_uv.to(spec.torch_dtype)


def queries(spec: WorkloadSpec) -> Tuple[torch.Tensor, torch.Tensor]:
    """q_nope [B, h, d_h], q_rope [B, h, d_r] in the storage dtype (CPU)."""
    qn = _normal((spec.batch, spec.n_heads, spec.d_h), _seed(spec.seed, 3), spec.q_std)
    qr = _normal((spec.batch, spec.n_heads, spec.d_r), _seed(spec.seed, 4), spec.q_std)
    return qn.to(spec.torch_dtype), qr.to(spec.torch_dtype)


def token_rows(spec: WorkloadSpec, seq: int, t0: int, t1: int,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Cache rows of tokens [t0, t1) of sequence ``seq``: [t1-t0, D], storage dtype.

    ``t0`` must be a multiple of TOKEN_CHUNK; each chunk has its own seed.
    """
    assert t0 % TOKEN_CHUNK == 0 and t1 >= t0
    n = t1 - t0
    if out is None:
        out = torch.empty((n, spec.D), dtype=spec.torch_dtype)
    buf = _scratch(spec.D)
    for c0 in range(t0, t1, TOKEN_CHUNK):
        c1 = min(c0 + TOKEN_CHUNK, t1)
        g = torch.Generator().manual_seed(_seed(spec.seed, 5, seq, c0 // TOKEN_CHUNK))
        # always draw a full chunk, so a short tail gets the same values as a long one
        buf.normal_(0.0, 1.0, generator=g)
        out[c0 - t0: c1 - t0].copy_(buf[: c1 - c0])
    return out


_SCRATCH: Dict[int, torch.Tensor] = {}


def _scratch(D: int) -> torch.Tensor:
    """Reused fp32 host buffer of one chunk (first touch of host pages is slow)."""
    if D not in _SCRATCH:
        _SCRATCH[D] = torch.empty((TOKEN_CHUNK, D), dtype=torch.float32)
    return _SCRATCH[D]


def page_layout(spec: WorkloadSpec, seqlens: np.ndarray) -> Tuple[np.ndarray, int]:
    """Page table [B, max_pages] (int32, -1 = unused) and the number of pages."""
    n_pages = [(int(L) + PAGE_SIZE - 1) // PAGE_SIZE for L in seqlens]
    total = int(sum(n_pages))
    max_pages = max(1, max(n_pages) if n_pages else 1)
    g = torch.Generator().manual_seed(_seed(spec.seed, 6))
    perm = torch.randperm(max(total, 1), generator=g).numpy().astype(np.int32)[:total]
    table = np.full((spec.batch, max_pages), -1, dtype=np.int32)
    off = 0
    for s, n in enumerate(n_pages):
        table[s, :n] = perm[off: off + n]
        off += n
    return table, total


@dataclass
class DecodeInputs:
    """All inputs of one decode-attention call, on one device."""

    spec: WorkloadSpec
    seqlens: torch.Tensor       # [B] int32
    q_nope: torch.Tensor        # [B, h, d_h]
    q_rope: torch.Tensor        # [B, h, d_r]
    w_uk: torch.Tensor          # [nb, h, d_cb, d_h]
    w_uv: torch.Tensor          # [nb, h, d_cb, d_h]
    kv_cache: torch.Tensor      # paged [pages, 64, D] / contiguous [B, L_max, D]
    page_table: Optional[torch.Tensor]  # [B, max_pages] int32 or None
    max_len: int                # contiguous row stride in tokens (L_max)

    @property
    def device(self) -> torch.device:
        return self.kv_cache.device


def make_inputs(spec: WorkloadSpec, device: str | torch.device = "cpu",
                seqlens: Optional[np.ndarray] = None) -> DecodeInputs:
    """Generate every input of ``spec`` and place it on ``device``.

    The cache is drawn on the host chunk by chunk (bounded host memory) and
    copied into a device buffer; pages are scattered with an index copy.
    """
    device = torch.device(device)
    if seqlens is None:
        seqlens = seqlens_for(spec)
    seqlens = np.asarray(seqlens, dtype=np.int32)
    assert seqlens.shape == (spec.batch,)
    w_uk, w_uv = weights(spec)
    q_nope, q_rope = queries(spec)
    dt = spec.torch_dtype
    L_max = int(seqlens.max()) if spec.batch else 0
    chunk_host = torch.empty((TOKEN_CHUNK, spec.D), dtype=dt)
    if device.type == "cuda":
        chunk_host = chunk_host.pin_memory()
    if spec.paged:
        table, total = page_layout(spec, seqlens)
        cache = torch.empty((max(total, 1), PAGE_SIZE, spec.D), dtype=dt, device=device)
        flat = cache.view(-1, spec.D)
        for s in range(spec.batch):
            L = int(seqlens[s])
            for c0 in range(0, L, TOKEN_CHUNK):
                c1 = min(c0 + TOKEN_CHUNK, L)
                rows = token_rows(spec, s, c0, c1, out=chunk_host[: c1 - c0])
                t = torch.arange(c0, c1, dtype=torch.int64)
                pg = torch.from_numpy(table[s]).to(torch.int64)[t // PAGE_SIZE]
                dst = (pg * PAGE_SIZE + t % PAGE_SIZE).to(device)
                flat.index_copy_(0, dst, rows.to(device, non_blocking=False))
        page_table = torch.from_numpy(table).to(device)
    else:
        cache = torch.zeros((spec.batch, max(L_max, 1), spec.D), dtype=dt, device=device)
        for s in range(spec.batch):
            L = int(seqlens[s])
            for c0 in range(0, L, TOKEN_CHUNK):
                c1 = min(c0 + TOKEN_CHUNK, L)
                rows = token_rows(spec, s, c0, c1, out=chunk_host[: c1 - c0])
                cache[s, c0:c1].copy_(rows)
        page_table = None
    return DecodeInputs(
        spec=spec,
        seqlens=torch.from_numpy(seqlens).to(device),
        q_nope=q_nope.to(device), q_rope=q_rope.to(device),
        w_uk=w_uk.to(device), w_uv=w_uv.to(device),
        kv_cache=cache, page_table=page_table, max_len=max(L_max, 1))


def sequence_cache(inp: DecodeInputs, seq: int) -> torch.Tensor:
    """Cache rows [L_s, D] of one sequence gathered from ``inp`` (on its device)."""
    L = int(inp.seqlens[seq])
    if inp.page_table is None:
        return inp.kv_cache[seq, :L]
    t = torch.arange(L, device=inp.device)
    pg = inp.page_table[seq].to(torch.int64)[t // PAGE_SIZE]
    return inp.kv_cache.view(-1, inp.spec.D)[pg * PAGE_SIZE + t % PAGE_SIZE]


def scaled_down(spec: WorkloadSpec, batch: int, seqlen: int = 0,
                ragged: Optional[Tuple[int, int]] = None, n_heads: Optional[int] = None,
                seed: Optional[int] = None) -> WorkloadSpec:
    """Same shape family with fewer sequences / tokens (for oracle-sized parity)."""
    kw = dict(batch=batch, seqlen=seqlen, ragged=ragged,
              name=f"{spec.name}__b{batch}_" + (f"l{seqlen}" if ragged is None else f"r{ragged[0]}_{ragged[1]}"))
    if n_heads is not None:
        kw["n_heads"] = n_heads
    if seed is not None:
        kw["seed"] = seed
    return spec.replace(**kw)


__all__ = [
    "PAGE_SIZE", "TOKEN_CHUNK", "WorkloadSpec", "WORKLOADS", "DecodeInputs",
    "seqlens_for", "weights", "queries", "token_rows", "page_layout",
    "make_inputs", "sequence_cache", "scaled_down",
]
