"""Branch-parallel decoding: the latent branches of one layer split across GPUs.

"Multi-Head Low-Rank Attention" (ai.info summary), Key Contributions #2 and
Main Findings, second bullet: because MLRA attends over each latent block
separately and sums the block outputs, the blocks can live on different
devices.  With 4-way tensor parallelism every device holds one latent block of
d_h channels plus the shared RoPE key of d_h / 2 -- 1.5 d_h per token instead
of MLA's 4.5 d_h -- runs the decode step over its own block, and the devices
sum their outputs.

Rank r of a group of W ranks (W divides n_blocks) holds blocks
[r * nb / W, (r + 1) * nb / W):
  * its cache rows: those blocks' columns followed by the RoPE key
    (``shard_cache``), i.e. a cache of D_local = nb / W * d_cb + d_r columns;
  * W_uk and W_uv of those blocks (``shard_weights``);
  * a config with n_blocks = nb / W and the branch rescale of the whole
    layer, 1 / sqrt(nb) (``local_config``): the rescale multiplies the sum
    over all blocks, so each rank applies it to its share.
Each rank runs the ordinary step (absorb, attention, merge + projection)
through the C ABI on its shard; ``reduce_branch_outputs`` sums the [B, h, d_h]
partial outputs over the group (one all-reduce, NCCL over NVLink on GPUs).
The sum over ranks equals the single-GPU step over all blocks up to fp32
rounding order.  The all-reduce moves B * h * d_h * 4 bytes per layer (512 KB
at B = 8, h = 128): latency-bound, so one NCCL call is the whole exchange.

Argument marshalling and tensor slicing only: every arithmetic step runs in
libmlra.so's kernels or inside NCCL.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import Config, Decoder, make_config


def blocks_of(n_blocks: int, world: int, rank: int) -> range:
    """The latent blocks rank ``rank`` holds (``world`` must divide n_blocks)."""
    if world < 1 or n_blocks % world != 0 or not 0 <= rank < world:
        raise ValueError(f"{world} ranks cannot share {n_blocks} latent blocks evenly")
    per = n_blocks // world
    return range(rank * per, (rank + 1) * per)


def local_config(cfg: Config, world: int) -> Config:
    """The config of one rank's shard: n_blocks / world blocks, the layer's
    own softmax scale and branch rescale."""
    nb = len(blocks_of(cfg.n_blocks, world, 0))
    dt = torch.bfloat16 if cfg.torch_dtype == torch.bfloat16 else torch.float32
    return make_config(nb, cfg.d_cb, cfg.d_r, cfg.n_heads, cfg.d_h, dtype=dt,
                       softmax_scale=cfg.softmax_scale, branch_scale=cfg.branch_scale,
                       page_size=cfg.page_size)


def shard_cache(kv_cache: torch.Tensor, cfg: Config, world: int, rank: int) -> torch.Tensor:
    """Rank ``rank``'s cache: its blocks' columns, then the RoPE key.

    ``kv_cache`` is [..., D] with D = n_blocks * d_cb + d_r (paged or
    contiguous); the result is a new contiguous [..., D_local] tensor."""
    if kv_cache.shape[-1] != cfg.D:
        raise ValueError(f"cache rows hold {kv_cache.shape[-1]} columns, the config {cfg.D}")
    bl = blocks_of(cfg.n_blocks, world, rank)
    lat = kv_cache[..., bl.start * cfg.d_cb: bl.stop * cfg.d_cb]
    rope = kv_cache[..., cfg.n_blocks * cfg.d_cb:]
    return torch.cat([lat, rope], dim=-1).contiguous()


def shard_weights(w: torch.Tensor, cfg: Config, world: int, rank: int) -> torch.Tensor:
    """Rank ``rank``'s slice of W_uk or W_uv [n_blocks, h, d_cb, d_h]."""
    if w.shape[0] != cfg.n_blocks:
        raise ValueError(f"weights hold {w.shape[0]} blocks, the config {cfg.n_blocks}")
    bl = blocks_of(cfg.n_blocks, world, rank)
    return w[bl.start: bl.stop].contiguous()


def reduce_branch_outputs(out: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (all-reduce over ``group``)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


class BranchParallelDecoder:
    """One rank's share of a branch-parallel decode step.

    Holds the rank's shard config and buffers; ``step`` runs absorb ->
    attention -> merge + projection on the shard through the C ABI and sums
    the partial outputs over the group."""

    def __init__(self, cfg: Config, batch: int, device, world: int, rank: int, group=None):
        self.cfg = cfg
        self.world, self.rank, self.group = world, rank, group
        self.local_cfg = local_config(cfg, world)
        self.decoder = Decoder(self.local_cfg, batch, torch.device(device))

    def step(self, q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk_local: torch.Tensor,
             w_uv_local: torch.Tensor, cache_local: torch.Tensor,
             page_table: Optional[torch.Tensor], seqlens: torch.Tensor, max_pages: int,
             stream=None) -> torch.Tensor:
        out = self.decoder.run(q_nope, q_rope, w_uk_local, w_uv_local, cache_local, page_table,
                               seqlens, max_pages, stream=stream, fused=True)
        return reduce_branch_outputs(out, self.group)

    def latent_outputs(self) -> Tuple[torch.Tensor, torch.Tensor]:
        """This rank's branches' latent outputs and lse from the last step."""
        return self.decoder.o_latent, self.decoder.lse


__all__ = ["blocks_of", "local_config", "shard_cache", "shard_weights", "reduce_branch_outputs",
           "BranchParallelDecoder"]
