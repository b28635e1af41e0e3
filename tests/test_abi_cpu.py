"""The C-ABI library loads and exports every symbol include/mlra.h declares.

No compute calls: these run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

import decode_attention_rank_mlra_b200 as mlra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"MLRA_API\s+[\w\s\*]+?\b(mlra_\w+)\s*\(", txt)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from decode_attention_rank_mlra_b200 import build
    build.build()
    return mlra.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert len(declared) >= 9
    for n in declared:
        assert hasattr(L, n), n
    assert sorted(mlra.EXPORTS) == declared


def test_config_struct_layout():
    assert ctypes.sizeof(mlra.Config) == 9 * 4


def test_status_strings(L):
    assert mlra.status_string(0) == "ok"
    assert "page" in mlra.status_string(6)
    assert mlra.status_string(99) == "unknown status"
    # every status the header declares has its own string and Python name
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "mlra.h")).read()
    codes = {int(v): k for k, v in re.findall(r"(MLRA_\w+)\s*=\s*(\d+)", hdr.split("mlra_status_t;")[0])
             if k.startswith("MLRA_ERR") or k == "MLRA_OK"}
    assert codes[9] == "MLRA_ERR_RANGE"
    for v, k in codes.items():
        assert mlra.STATUS[v] == k
        assert mlra.status_string(v) != "unknown status"
    assert L.mlra_version() == 10000


def test_host_validation_without_device(L):
    cfg = mlra.make_config(4, 128, 64, 16, 128)
    # null config / pointers are rejected before any CUDA call
    assert L.mlra_absorb_q(None, None, None, None, 1, None) == 1
    assert L.mlra_absorb_q(ctypes.byref(cfg), None, None, None, 1, None) == 1
    assert L.mlra_absorb_q(ctypes.byref(cfg), None, None, None, 0, None) == 0  # empty batch
    assert L.mlra_absorb_q(ctypes.byref(cfg), None, None, None, -1, None) == 1
    bad = mlra.make_config(4, 128, 64, 16, 256)  # d_h > 128
    assert L.mlra_out_proj(ctypes.byref(bad), None, None, None, 1, None) == 2
    assert L.mlra_decode_attn(ctypes.byref(cfg), None, None, None, 0, None, 1, None, 1, None, 0,
                              None) == 1
    # misaligned workspace
    assert L.mlra_decode_attn(ctypes.byref(cfg), None, None, None, 0, None, 1, None, 0,
                              ctypes.c_void_p(16), 0, None) == 4
    v = ctypes.c_int32(0)
    assert L.mlra_get_device_error(None, 0, ctypes.byref(v), None) == 1


def test_no_cpu_path():
    import torch
    cfg = mlra.make_config(4, 128, 64, 16, 128)
    with pytest.raises(ValueError):
        mlra.absorb_q(cfg, torch.zeros(1, 16, 128, dtype=torch.bfloat16),
                      torch.zeros(4, 16, 128, 128, dtype=torch.bfloat16))


def test_decode_step_validation_without_device(L):
    """mlra_decode_step rejects bad arguments before it touches the device or the
    workspace (a dummy, never dereferenced address stands in for it)."""
    cfg = mlra.make_config(4, 128, 64, 16, 128)
    ws = ctypes.c_void_p(256)

    def call(batch, host_io, workspace):
        return L.mlra_decode_step(ctypes.byref(cfg), None, None, None, batch, None, None, None,
                                  0, None, 1, None, host_io, workspace, 1 << 20, None)

    assert call(1, 2, ws) == 1                      # host_io neither 0 nor 1
    assert call(-1, 0, ws) == 1                     # negative batch
    assert call(1, 0, None) == 1                    # no workspace
    assert call(1, 0, ctypes.c_void_p(16)) == 4     # workspace not 256-byte aligned
    assert call(0, 1, ws) == 0                      # empty batch: nothing is launched
    assert call(1, 0, ws) == 1                      # null inputs
    assert L.mlra_decode_step(None, None, None, None, 1, None, None, None, 0, None, 1, None, 0,
                              ws, 1 << 20, None) == 1


def test_no_device_no_result(L):
    """Without a usable GPU the library computes nothing on the host: a call that
    needs the device reports MLRA_ERR_NO_DEVICE (after its argument checks)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = mlra.make_config(4, 128, 64, 16, 128)
    sz = ctypes.c_size_t(0)
    assert L.mlra_workspace_size(ctypes.byref(cfg), 4, None) == 1
    assert L.mlra_step_workspace_size(None, 4, ctypes.byref(sz)) == 1
    assert L.mlra_workspace_size(ctypes.byref(cfg), 4, ctypes.byref(sz)) == 8
    assert L.mlra_step_workspace_size(ctypes.byref(cfg), 4, ctypes.byref(sz)) == 8
