"""Python binding of libmlra.so: MLRA / MLA latent-KV decode attention on B200.

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels (see ``include/mlra.h`` for the operations, layouts and error
behaviour).  PyTorch supplies device memory and the current stream.  There is
no fallback: if the shared library is missing this module raises on import of
the library handle, and every call requires CUDA tensors.

Steps of one decode call ("Multi-Head Low-Rank Attention", Main Findings:
decoding reduces to three absorbable steps):
``absorb_q`` -> ``decode_attn`` -> ``splitkv_combine`` -> ``out_proj``.
``Decoder`` bundles the four with preallocated buffers.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlra.so")

F32 = 0
BF16 = 1

STATUS = {
    0: "MLRA_OK", 1: "MLRA_ERR_INVALID_ARG", 2: "MLRA_ERR_UNSUPPORTED", 3: "MLRA_ERR_ALIGNMENT",
    4: "MLRA_ERR_WORKSPACE", 5: "MLRA_ERR_CUDA", 6: "MLRA_ERR_BAD_PAGE", 7: "MLRA_ERR_TIMEOUT",
    8: "MLRA_ERR_NO_DEVICE", 9: "MLRA_ERR_RANGE",
}

# Every symbol the C header declares (checked by the CPU tests).
EXPORTS = [
    "mlra_status_string", "mlra_version", "mlra_absorb_q", "mlra_workspace_size",
    "mlra_decode_attn", "mlra_splitkv_combine", "mlra_out_proj", "mlra_get_device_error",
    "mlra_decode_kernel_kind", "mlra_decode_attn_noalloc", "mlra_combine_out_proj",
    "mlra_cache_append", "mlra_step_workspace_size", "mlra_decode_step", "mlra_absorb_q_rope",
    "mlra_release_step_graphs",
]


class MlraError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status_string(status)})")


class Config(ctypes.Structure):
    """mirror of mlra_config_t"""
    _fields_ = [
        ("n_blocks", ctypes.c_int32), ("d_cb", ctypes.c_int32), ("d_r", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("d_h", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
        ("branch_scale", ctypes.c_float),
    ]

    @property
    def D(self) -> int:
        return self.n_blocks * self.d_cb + self.d_r

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == BF16 else torch.float32


def make_config(n_blocks: int, d_cb: int, d_r: int, n_heads: int, d_h: int,
                dtype: torch.dtype = torch.bfloat16, softmax_scale: Optional[float] = None,
                branch_scale: Optional[float] = None, page_size: int = 64) -> Config:
    """Config with the paper's default scales: 1/sqrt(d_h + d_r) and 1/sqrt(n_blocks)."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_h + d_r)
    if branch_scale is None:
        branch_scale = 1.0 / math.sqrt(n_blocks)
    dt = {torch.bfloat16: BF16, torch.float32: F32}[dtype]
    return Config(n_blocks, d_cb, d_r, n_heads, d_h, page_size, dt, softmax_scale, branch_scale)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmlra.so from this package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} not found: build it with "
                          "`python -m decode_attention_rank_mlra_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    CP = ctypes.POINTER(Config)
    sig = {
        "mlra_status_string": (ctypes.c_char_p, [I32]),
        "mlra_version": (I32, []),
        "mlra_absorb_q": (I32, [CP, P, P, P, I32, P]),
        "mlra_absorb_q_rope": (I32, [CP, P, P, P, ctypes.c_float, ctypes.c_float, P, P, P, I32, P]),
        "mlra_workspace_size": (I32, [CP, I32, ctypes.POINTER(SZ)]),
        "mlra_decode_attn": (I32, [CP, P, P, P, I64, P, I32, P, I32, P, SZ, P]),
        "mlra_splitkv_combine": (I32, [CP, P, SZ, I32, P, P, P]),
        "mlra_out_proj": (I32, [CP, P, P, P, I32, P]),
        "mlra_combine_out_proj": (I32, [CP, P, SZ, I32, P, P, P, P, P]),
        "mlra_cache_append": (I32, [CP, P, P, P, ctypes.c_float, ctypes.c_float, ctypes.c_float, P,
                                    I64, P, I32, P, I32, P, P]),
        "mlra_get_device_error": (I32, [P, SZ, ctypes.POINTER(I32), P]),
        "mlra_decode_kernel_kind": (I32, [CP]),
        "mlra_decode_attn_noalloc": (I32, [CP, P, P, P, I64, P, I32, P, I32, P, P, P, P]),
        "mlra_step_workspace_size": (I32, [CP, I32, ctypes.POINTER(SZ)]),
        "mlra_decode_step": (I32, [CP, P, P, P, I32, P, P, P, I64, P, I32, P, I32, P, SZ, P]),
        "mlra_release_step_graphs": (I32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().mlra_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    """cudaStream_t of ``stream`` (default: the current stream of the current device)."""
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch._C._cuda_getDevice())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t: torch.Tensor, name: str, dtype: Optional[torch.dtype] = None, shape=None):
    """A contiguous CUDA tensor on the current device (the library launches there),
    of ``dtype`` and, when given, of ``shape`` (-1 matches any extent)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None:
        shape = tuple(int(x) for x in shape)
        if t.dim() != len(shape) or any(w != -1 and w != g for w, g in zip(shape, t.shape)):
            raise ValueError(f"{name} must have shape {shape} (-1: any), got {tuple(t.shape)}")


def _contig_cache(kv_cache: torch.Tensor, cfg: Config, batch: int, max_len: int):
    """A contiguous cache [>= batch, max_len, D]: row s * max_len + t is token t
    of sequence s (a cache allocated for more sequences than the call's batch
    is fine)."""
    _need(kv_cache, "kv_cache", cfg.torch_dtype, (-1, max_len, cfg.D))
    if kv_cache.shape[0] < batch:
        raise ValueError(f"kv_cache holds {kv_cache.shape[0]} sequences, the batch is {batch}")


def _check(fn: str, status: int):
    if status != 0:
        raise MlraError(fn, status)


def absorb_q(cfg: Config, q_nope: torch.Tensor, w_uk: torch.Tensor,
             q_abs: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Step 1: q_abs[s,h,b,i] = sum_j W_uk[b,h,i,j] q_nope[s,h,j] (fp32 out)."""
    _need(q_nope, "q_nope", cfg.torch_dtype, (-1, cfg.n_heads, cfg.d_h))
    _need(w_uk, "w_uk", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    B = q_nope.shape[0]
    if q_abs is None:
        q_abs = torch.empty((B, cfg.n_heads, cfg.n_blocks, cfg.d_cb), dtype=torch.float32,
                            device=q_nope.device)
    _need(q_abs, "q_abs", torch.float32, (B, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    _check("mlra_absorb_q", lib().mlra_absorb_q(ctypes.byref(cfg), _ptr(q_nope), _ptr(w_uk),
                                                _ptr(q_abs), B, _stream(stream)))
    return q_abs


def absorb_q_rope(cfg: Config, q_nope: torch.Tensor, q_rope: torch.Tensor,
                  positions: torch.Tensor, alpha_q: float, w_uk: torch.Tensor,
                  q_abs: Optional[torch.Tensor] = None, q_rope_out: Optional[torch.Tensor] = None,
                  rope_theta: float = 10000.0, stream=None):
    """Step 1 with the query-side calibration: q_abs = alpha_q W_uk q_nope (fp32)
    and q_rope_out = RoPE(alpha_q q_rope) at ``positions[s]`` (storage dtype).
    Returns (q_abs, q_rope_out)."""
    _need(positions, "positions", torch.int32, (-1,))
    B = positions.shape[0]
    _need(q_nope, "q_nope", cfg.torch_dtype, (B, cfg.n_heads, cfg.d_h))
    _need(q_rope, "q_rope", cfg.torch_dtype, (B, cfg.n_heads, cfg.d_r))
    _need(w_uk, "w_uk", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    if q_abs is None:
        q_abs = torch.empty((B, cfg.n_heads, cfg.n_blocks, cfg.d_cb), dtype=torch.float32,
                            device=q_nope.device)
    if q_rope_out is None:
        q_rope_out = torch.empty_like(q_rope)
    _need(q_abs, "q_abs", torch.float32, (B, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    _need(q_rope_out, "q_rope_out", cfg.torch_dtype, (B, cfg.n_heads, cfg.d_r))
    _check("mlra_absorb_q_rope", lib().mlra_absorb_q_rope(
        ctypes.byref(cfg), _ptr(q_nope), _ptr(q_rope), _ptr(positions), float(alpha_q),
        float(rope_theta), _ptr(w_uk), _ptr(q_abs), _ptr(q_rope_out), B, _stream(stream)))
    return q_abs, q_rope_out


def workspace_size(cfg: Config, batch: int) -> int:
    n = ctypes.c_size_t(0)
    _check("mlra_workspace_size", lib().mlra_workspace_size(ctypes.byref(cfg), batch,
                                                            ctypes.byref(n)))
    return int(n.value)


def alloc_workspace(cfg: Config, batch: int, device=None) -> torch.Tensor:
    """Caller-owned workspace (uint8, 256-byte aligned)."""
    return _aligned_bytes(workspace_size(cfg, batch), device)


def _attn_inputs(cfg: Config, q_abs, q_rope, kv_cache, page_table, seqlens, max_pages) -> int:
    """Checks shared by the attention calls; returns the batch."""
    _need(seqlens, "seqlens", torch.int32, (-1,))
    B = seqlens.shape[0]
    _need(q_abs, "q_abs", torch.float32, (B, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    _need(q_rope, "q_rope", cfg.torch_dtype, (B, cfg.n_heads, cfg.d_r))
    if page_table is not None:
        _need(page_table, "page_table", torch.int32, (B, max_pages))
        _need(kv_cache, "kv_cache", cfg.torch_dtype, (-1, cfg.page_size, cfg.D))
    else:
        _contig_cache(kv_cache, cfg, B, max_pages)
    return B


def decode_attn(cfg: Config, q_abs: torch.Tensor, q_rope: torch.Tensor, kv_cache: torch.Tensor,
                page_table: Optional[torch.Tensor], seqlens: torch.Tensor, max_pages: int,
                workspace: torch.Tensor, stream=None) -> None:
    """Step 2a: split-KV attention into the workspace.

    Paged: kv_cache [num_pages, 64, D], page_table [B, max_pages] int32.
    Contiguous: page_table None, kv_cache [B, max_len, D], max_pages = max_len.
    """
    B = _attn_inputs(cfg, q_abs, q_rope, kv_cache, page_table, seqlens, max_pages)
    _need(workspace, "workspace", torch.uint8)
    num_pages = kv_cache.shape[0] if page_table is not None else 0
    _check("mlra_decode_attn", lib().mlra_decode_attn(
        ctypes.byref(cfg), _ptr(q_abs), _ptr(q_rope), _ptr(kv_cache), num_pages, _ptr(page_table),
        int(max_pages), _ptr(seqlens), B, _ptr(workspace), workspace.numel(), _stream(stream)))


def splitkv_combine(cfg: Config, workspace: torch.Tensor, batch: int,
                    o_latent: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    stream=None):
    """Step 2b: merge split partials -> o_latent [B,h,nb,d_cb], lse [B,h,nb] (fp32)."""
    dev = workspace.device
    if o_latent is None:
        o_latent = torch.empty((batch, cfg.n_heads, cfg.n_blocks, cfg.d_cb), dtype=torch.float32,
                               device=dev)
    if lse is None:
        lse = torch.empty((batch, cfg.n_heads, cfg.n_blocks), dtype=torch.float32, device=dev)
    _need(workspace, "workspace", torch.uint8)
    _need(o_latent, "o_latent", torch.float32, (batch, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    _need(lse, "lse", torch.float32, (batch, cfg.n_heads, cfg.n_blocks))
    _check("mlra_splitkv_combine", lib().mlra_splitkv_combine(
        ctypes.byref(cfg), _ptr(workspace), workspace.numel(), batch, _ptr(o_latent), _ptr(lse),
        _stream(stream)))
    return o_latent, lse


def out_proj(cfg: Config, o_latent: torch.Tensor, w_uv: torch.Tensor,
             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Step 3: out[s,h,:] = branch_scale * sum_b W_uv[b,h]^T o_latent[s,h,b] (fp32)."""
    _need(o_latent, "o_latent", torch.float32, (-1, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    _need(w_uv, "w_uv", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    B = o_latent.shape[0]
    if out is None:
        out = torch.empty((B, cfg.n_heads, cfg.d_h), dtype=torch.float32, device=o_latent.device)
    _need(out, "out", torch.float32, (B, cfg.n_heads, cfg.d_h))
    _check("mlra_out_proj", lib().mlra_out_proj(ctypes.byref(cfg), _ptr(o_latent), _ptr(w_uv),
                                                _ptr(out), B, _stream(stream)))
    return out


def combine_out_proj(cfg: Config, workspace: torch.Tensor, batch: int, w_uv: torch.Tensor,
                     out: Optional[torch.Tensor] = None, o_latent: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Steps 2b + 3 fused: merge the split partials and project (fp32 out).

    ``o_latent`` / ``lse`` are written when given (needed when the fused
    tensor-core kernel does not apply).
    """
    _need(workspace, "workspace", torch.uint8)
    _need(w_uv, "w_uv", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    if out is None:
        out = torch.empty((batch, cfg.n_heads, cfg.d_h), dtype=torch.float32,
                          device=workspace.device)
    _need(out, "out", torch.float32, (batch, cfg.n_heads, cfg.d_h))
    if o_latent is not None:
        _need(o_latent, "o_latent", torch.float32, (batch, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    if lse is not None:
        _need(lse, "lse", torch.float32, (batch, cfg.n_heads, cfg.n_blocks))
    _check("mlra_combine_out_proj", lib().mlra_combine_out_proj(
        ctypes.byref(cfg), _ptr(workspace), workspace.numel(), batch, _ptr(w_uv), _ptr(out),
        _ptr(o_latent), _ptr(lse), _stream(stream)))
    return out


def cache_append(cfg: Config, c_new: torch.Tensor, k_rope_new: torch.Tensor,
                 rms_gamma: torch.Tensor, alpha_kv: float, kv_cache: torch.Tensor,
                 page_table: Optional[torch.Tensor], positions: torch.Tensor, max_pages: int,
                 rms_eps: float = 1e-6, rope_theta: float = 10000.0,
                 device_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Cache write: each sequence's new row (per-block RMSNorm x gain x alpha_kv,
    rotated RoPE key) at token ``positions[s]``, in place in ``kv_cache``."""
    _need(positions, "positions", torch.int32, (-1,))
    B = positions.shape[0]
    _need(c_new, "c_new", cfg.torch_dtype, (B, cfg.n_blocks * cfg.d_cb))
    _need(k_rope_new, "k_rope_new", cfg.torch_dtype, (B, cfg.d_r))
    _need(rms_gamma, "rms_gamma", torch.float32, (cfg.n_blocks * cfg.d_cb,))
    num_pages = 0
    if page_table is not None:
        _need(page_table, "page_table", torch.int32, (B, max_pages))
        _need(kv_cache, "kv_cache", cfg.torch_dtype, (-1, cfg.page_size, cfg.D))
        num_pages = kv_cache.shape[0]
    else:
        _contig_cache(kv_cache, cfg, B, max_pages)
    if device_status is not None:
        _need(device_status, "device_status", torch.int32, (-1,))
    _check("mlra_cache_append", lib().mlra_cache_append(
        ctypes.byref(cfg), _ptr(c_new), _ptr(k_rope_new), _ptr(rms_gamma), float(alpha_kv),
        float(rms_eps), float(rope_theta), _ptr(kv_cache), num_pages, _ptr(page_table),
        int(max_pages), _ptr(positions), B, _ptr(device_status), _stream(stream)))


def step_workspace_size(cfg: Config, batch: int) -> int:
    n = ctypes.c_size_t(0)
    _check("mlra_step_workspace_size", lib().mlra_step_workspace_size(ctypes.byref(cfg), batch,
                                                                      ctypes.byref(n)))
    return int(n.value)


def _aligned_bytes(n: int, device) -> torch.Tensor:
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    return ws[off: off + n]


def alloc_step_workspace(cfg: Config, batch: int, device=None) -> torch.Tensor:
    """Caller-owned workspace for ``decode_step`` (its first
    ``workspace_size`` bytes serve as the decode workspace)."""
    return _aligned_bytes(step_workspace_size(cfg, batch), device)


def decode_step(cfg: Config, q_nope: torch.Tensor, q_rope: torch.Tensor, seqlens: torch.Tensor,
                w_uk: torch.Tensor, w_uv: torch.Tensor, kv_cache: torch.Tensor,
                page_table: Optional[torch.Tensor], max_pages: int, out: torch.Tensor,
                workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """Steps 1, 2a, 2b and 3 in one library call (absorb, attention, merge,
    output projection), bitwise equal to the three separate calls.

    ``q_nope``, ``q_rope``, ``seqlens`` and ``out`` are either all CUDA
    tensors or all host tensors (page-locked for an asynchronous call).  With
    host tensors the library moves them on ``stream`` (page-locked memory by
    one staging kernel and in-place output stores, other memory by copies);
    ``out`` is valid once the stream has passed the call.
    """
    on_host = not q_nope.is_cuda
    if q_rope.is_cuda == on_host or seqlens.is_cuda == on_host or out.is_cuda == on_host:
        raise ValueError("q_nope, q_rope, seqlens and out must all be on the host "
                         "or all on the device")
    if not (q_nope.is_contiguous() and q_rope.is_contiguous() and seqlens.is_contiguous()
            and out.is_contiguous()):
        raise ValueError("q_nope, q_rope, seqlens and out must be contiguous")
    dt = cfg.torch_dtype
    if q_nope.dtype != dt or q_rope.dtype != dt or seqlens.dtype != torch.int32 \
            or out.dtype != torch.float32:
        raise ValueError(f"dtypes must be q_nope/q_rope {dt}, seqlens int32, out float32")
    B = seqlens.shape[0]
    h = cfg.n_heads
    if q_nope.shape != (B, h, cfg.d_h) or q_rope.shape != (B, h, cfg.d_r) \
            or out.shape != (B, h, cfg.d_h):
        raise ValueError("q_nope / q_rope / out shapes do not match seqlens and cfg")
    _need(w_uk, "w_uk", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    _need(w_uv, "w_uv", cfg.torch_dtype, (cfg.n_blocks, cfg.n_heads, cfg.d_cb, cfg.d_h))
    _need(workspace, "workspace", torch.uint8)
    num_pages = 0
    if page_table is not None:
        _need(page_table, "page_table", torch.int32, (B, max_pages))
        _need(kv_cache, "kv_cache", cfg.torch_dtype, (-1, cfg.page_size, cfg.D))
        num_pages = kv_cache.shape[0]
    else:
        _contig_cache(kv_cache, cfg, B, max_pages)
    _check("mlra_decode_step", lib().mlra_decode_step(
        ctypes.byref(cfg), _ptr(q_nope), _ptr(q_rope), _ptr(seqlens), B, _ptr(w_uk), _ptr(w_uv),
        _ptr(kv_cache), num_pages, _ptr(page_table), int(max_pages), _ptr(out), int(on_host),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def release_step_graphs() -> None:
    """Destroy the CUDA graphs ``decode_step`` recorded; call only with no step
    executing on the GPU (synchronise first)."""
    _check("mlra_release_step_graphs", lib().mlra_release_step_graphs())


def decode_attn_noalloc(cfg: Config, q_abs: torch.Tensor, q_rope: torch.Tensor,
                        kv_cache: torch.Tensor, page_table: Optional[torch.Tensor],
                        seqlens: torch.Tensor, max_pages: int, o_latent: torch.Tensor,
                        lse: Optional[torch.Tensor] = None,
                        device_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Steps 2a + 2b with the library's own fixed scratch (no workspace).

    For callers that cannot allocate device memory (a plugin whose host owns
    the device allocator, or a server that reserved all free HBM up front):
    nothing is allocated here or in the library.  All calls share one 16 MiB
    array inside libmlra.so, so calls that overlap on the GPU race; batches
    needing more scratch are rejected with MLRA_ERR_WORKSPACE.  Outputs as
    ``splitkv_combine``; ``device_status`` (one int32 on the device) receives
    the call's device error word.
    """
    B = _attn_inputs(cfg, q_abs, q_rope, kv_cache, page_table, seqlens, max_pages)
    _need(o_latent, "o_latent", torch.float32, (B, cfg.n_heads, cfg.n_blocks, cfg.d_cb))
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, cfg.n_heads, cfg.n_blocks))
    if device_status is not None:
        _need(device_status, "device_status", torch.int32, (-1,))
        if device_status.numel() < 1:
            raise ValueError("device_status must hold at least one int32")
    num_pages = kv_cache.shape[0] if page_table is not None else 0
    _check("mlra_decode_attn_noalloc", lib().mlra_decode_attn_noalloc(
        ctypes.byref(cfg), _ptr(q_abs), _ptr(q_rope), _ptr(kv_cache), num_pages, _ptr(page_table),
        int(max_pages), _ptr(seqlens), B, _ptr(o_latent), _ptr(lse), _ptr(device_status),
        _stream(stream)))


def get_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Device-side status recorded in the workspace (synchronises the stream)."""
    v = ctypes.c_int32(0)
    _check("mlra_get_device_error", lib().mlra_get_device_error(
        _ptr(workspace), workspace.numel(), ctypes.byref(v), _stream(stream)))
    return int(v.value)


def decode_kernel_kind(cfg: Config) -> str:
    k = lib().mlra_decode_kernel_kind(ctypes.byref(cfg))
    return {0: "unsupported", 1: "tcgen05", 2: "simt"}[k]


@dataclass
class Decoder:
    """One layer's decode step with preallocated outputs and workspace.

    ``run`` launches absorb -> decode_attn -> splitkv_combine -> out_proj on
    the current stream and returns ``out`` [B, h, d_h] fp32; with
    ``fused=True`` the last two are one combine_out_proj call.  ``step`` makes
    the same computation one library call (``decode_step``), from device or
    host buffers.
    """

    cfg: Config
    batch: int
    device: torch.device

    def __post_init__(self):
        c, B, dev = self.cfg, self.batch, self.device
        self.step_workspace = alloc_step_workspace(c, B, dev)
        self.workspace = self.step_workspace[: workspace_size(c, B)]
        self.q_abs = torch.empty((B, c.n_heads, c.n_blocks, c.d_cb), dtype=torch.float32, device=dev)
        self.o_latent = torch.empty((B, c.n_heads, c.n_blocks, c.d_cb), dtype=torch.float32,
                                    device=dev)
        self.lse = torch.empty((B, c.n_heads, c.n_blocks), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, c.n_heads, c.d_h), dtype=torch.float32, device=dev)

    def run(self, q_nope, q_rope, w_uk, w_uv, kv_cache, page_table, seqlens, max_pages,
            stream=None, fused: bool = False) -> torch.Tensor:
        absorb_q(self.cfg, q_nope, w_uk, self.q_abs, stream)
        decode_attn(self.cfg, self.q_abs, q_rope, kv_cache, page_table, seqlens, max_pages,
                    self.workspace, stream)
        if fused:
            combine_out_proj(self.cfg, self.workspace, self.batch, w_uv, self.out, self.o_latent,
                             self.lse, stream)
        else:
            splitkv_combine(self.cfg, self.workspace, self.batch, self.o_latent, self.lse, stream)
            out_proj(self.cfg, self.o_latent, w_uv, self.out, stream)
        return self.out

    def step(self, q_nope, q_rope, seqlens, w_uk, w_uv, kv_cache, page_table, max_pages,
             out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = self.out
        return decode_step(self.cfg, q_nope, q_rope, seqlens, w_uk, w_uv, kv_cache, page_table,
                           max_pages, out, self.step_workspace, stream)


__all__ = [
    "Config", "make_config", "lib", "absorb_q", "absorb_q_rope", "workspace_size", "alloc_workspace",
    "decode_attn", "splitkv_combine", "out_proj", "combine_out_proj", "cache_append",
    "get_device_error",
    "decode_kernel_kind", "decode_attn_noalloc", "step_workspace_size", "alloc_step_workspace",
    "decode_step", "release_step_graphs",
    "Decoder", "MlraError", "EXPORTS", "F32", "BF16",
]
