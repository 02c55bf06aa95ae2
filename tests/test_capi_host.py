"""The C-ABI library on the host: it loads, exports every declared symbol, and
rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import transformer_denoiser_b200 as kb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"KIMODO_API\s+[\w\s\*]*?\b(kimodo_\w+)\s*\(", txt))
    return names


@pytest.fixture(scope="module")
def lib():
    from transformer_denoiser_b200.build import build
    build()
    return kb.load_library()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), name
    bound = {n for n, _, _ in kb.SIGNATURES}
    assert bound == declared


def test_header_constants_match_binding():
    h = open(os.path.join(ROOT, "include", "kimodo.h")).read()
    assert f"KIMODO_N_PARAMS {kb.N_PARAMS}u" in h
    from oracle import kimodo_oracle as ko
    assert ko.param_count() == kb.N_PARAMS


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        kb.load_library(str(tmp_path / "nope.so"))


def test_null_and_size_errors(lib):
    ctx = ctypes.c_void_p()
    buf = np.zeros(16, np.float32)
    assert lib.kimodo_load_weights(None, buf.ctypes.data, 16, 1, 0) == -1
    assert lib.kimodo_load_weights(ctypes.byref(ctx), None, kb.N_PARAMS, 1, 0) == -1
    assert lib.kimodo_load_weights(ctypes.byref(ctx), buf.ctypes.data, 16, 1, 0) == -1
    assert b"expected 281963799" in lib.kimodo_last_error()
    assert lib.kimodo_load_weights(ctypes.byref(ctx), buf.ctypes.data, kb.N_PARAMS, 7, 0) == -1
    assert lib.kimodo_ddim_sample(None, None, None, 1, None, None, 1, 1, 50, 2.0, None, None) == -1
    assert lib.kimodo_denoiser_forward(None, 0, None, None, 999, None, 1, 1, None, None) == -1
    assert lib.kimodo_sync_status(None, None) == -1
    assert lib.kimodo_last_launch_count(None) == 0
    lib.kimodo_free(None)


def test_kernel_entry_argument_checks(lib):
    p = ctypes.c_void_p(16)
    # NULL operands, bad sizes, unknown epilogue: all rejected on the host
    assert lib.kimodo_gemm_bf16(None, 64, p, 64, p, None, 0, p, 64, 1, 1, 64, 0, 0, 0, None) == -1
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 0, 1, 64, 0, 0, 0, None) == -1
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 1, 1, 64, 9, 0, 0, None) == -1
    assert lib.kimodo_gemm_bf16(p, 60, p, 64, p, None, 0, p, 64, 1, 1, 60, 0, 0, 0, None) == -1
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 1, 1, 64, 3, 1, 0, None) == -1  # resid missing
    assert lib.kimodo_gemm_f32(p, 64, p, 64, p, None, 0, p, 64, 1, 1, 40, 0, None) == -1       # K % 16
    # output tiles: 32, 64, 128, 256 or 0; the narrow ones exist for bias / GELU (bf16) and residual only
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 1, 64, 64, 0, 0, 48, None) == -1
    assert b"tile_n must be" in lib.kimodo_last_error()
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 1, 64, 64, 2, 0, 32, None) == -1  # SiLU
    assert b"not built" in lib.kimodo_last_error()
    assert lib.kimodo_gemm_bf16(p, 64, p, 64, p, None, 0, p, 64, 1, 64, 64, 0, 1, 64, None) == -1  # fp32 bias
    assert b"not built" in lib.kimodo_last_error()
    # pair GEMM: N a multiple of 16; tile_n 144, 160, 208, 256 or 0
    assert lib.kimodo_gemm_bf16_pair(p, 64, p, 64, p, None, 0, p, 64, 1, 40, 64, 0, 0, 0, None) == -1
    assert b"N % 16" in lib.kimodo_last_error()
    assert lib.kimodo_gemm_bf16_pair(p, 64, p, 64, p, None, 0, p, 64, 1, 64, 64, 0, 0, 48, None) == -1
    assert b"tile_n must be" in lib.kimodo_last_error()
    assert lib.kimodo_attention_bf16(p, p, p, 1, 302, None) == -1
    assert lib.kimodo_layernorm(p, p, 1, p, p, 0, None) == -1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_no_device_is_reported(lib):
    ctx = ctypes.c_void_p()
    buf = np.zeros(4, np.float32)   # never read: the device check comes first
    rc = lib.kimodo_load_weights(ctypes.byref(ctx), buf.ctypes.data, kb.N_PARAMS, 1, 0)
    assert rc == -4 and b"no CUDA device" in lib.kimodo_last_error()
    assert ctx.value is None
