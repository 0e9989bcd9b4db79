"""Host-only checks of the C ABI (no GPU needed).

The library must load, export every function include/mla.h declares, and
reject bad arguments with the documented status codes before it touches the
device. Fake non-null device addresses are used: argument validation runs
before any CUDA call, so they are never dereferenced.
"""
import ctypes
import os
import re

import pytest
import torch

from mla_causal_attention_attn_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")

OK, INVALID, SHAPE, MISALIGNED, UNSUPPORTED, WORKSPACE, CUDA, TIMEOUT = 0, -1, -2, -3, -4, -5, -6, -7
A = 0x7f0000000000  # a 16-byte aligned fake device address, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("mla_attn_prefill", "mla_o_proj", "mla_attn_oproj"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding._SIGNATURES), "binding signatures drift from the header"


def test_abi_version_and_status_strings(lib):
    assert lib.mla_abi_version() == 4
    for code, name in binding.STATUS.items():
        assert lib.mla_status_string(code).decode() == name
    assert lib.mla_status_string(12345).decode() == "MLA_ERR_UNKNOWN"


ST = binding.WORKSPACE_STATUS_BYTES  # the status word's block at the start of a workspace


def test_workspace_sizes(lib):
    assert ST == 256
    assert lib.mla_attn_prefill_workspace_bytes(1, 4096, 0) == ST
    assert lib.mla_attn_prefill_workspace_bytes(8, 4096, 1) == ST + 8 * 32 * 32
    assert lib.mla_attn_prefill_workspace_bytes(2, 129, 1) == ST + 2 * 2 * 2
    assert lib.mla_attn_prefill_workspace_bytes(0, 10, 1) == 0
    attn = 1 * 4096 * 8192 * 2
    assert lib.mla_attn_oproj_workspace_bytes(1, 4096, 0) == ST + attn
    assert lib.mla_attn_oproj_workspace_bytes(8, 4096, 1) == ST + 8 * 4096 * 8192 * 2 + 8 * 32 * 32
    assert lib.mla_attn_oproj_workspace_bytes(1, 3, 0) == ST + 49152  # 3*8192*2 rounded to 256
    assert lib.mla_attn_oproj_workspace_bytes(-1, 3, 0) == 0


def prefill(lib, q=A, qp=A, k=A, kp=A, v=A, mask=None, ld=0, B=1, T=64, scale=0.07,
            ws=None, ws_bytes=0, out=A):
    return lib.mla_attn_prefill(q, qp, k, kp, v, mask, ld, B, T, scale, ws, ws_bytes, out, None)


def fused(lib, q=A, qp=A, k=A, kp=A, v=A, mask=None, ld=0, B=1, T=64, scale=0.07, W=A,
          ws=A, ws_bytes=1 << 40, out=A):
    return lib.mla_attn_oproj(q, qp, k, kp, v, mask, ld, B, T, scale, W, ws, ws_bytes, out, None)


def test_prefill_argument_errors(lib):
    assert prefill(lib, q=None) == INVALID
    assert prefill(lib, kp=None) == INVALID
    assert prefill(lib, out=None) == INVALID
    assert prefill(lib, scale=float("nan")) == INVALID
    assert prefill(lib, scale=float("inf")) == INVALID
    assert prefill(lib, B=0) == SHAPE
    assert prefill(lib, T=0) == SHAPE
    assert prefill(lib, T=-5) == SHAPE
    assert prefill(lib, B=65536) == SHAPE
    assert prefill(lib, T=65535 * 128 + 1) == SHAPE
    assert prefill(lib, mask=A, ld=32, T=64, ws=A, ws_bytes=ST + 64) == SHAPE  # ld < T
    assert prefill(lib, q=A + 8) == MISALIGNED
    assert prefill(lib, v=A + 2) == MISALIGNED
    assert prefill(lib, out=A + 4) == MISALIGNED
    assert prefill(lib, mask=A + 1, ld=64, ws=A, ws_bytes=ST + 64) == MISALIGNED  # odd address
    assert prefill(lib, mask=A, ld=64) == WORKSPACE                       # none given
    assert prefill(lib, mask=A, ld=304, B=2, T=300, ws=A, ws_bytes=ST + 17) == WORKSPACE  # 18
    assert prefill(lib, ws=A, ws_bytes=ST - 1) == WORKSPACE  # optional, but then whole
    assert prefill(lib, ws=A + 8, ws_bytes=ST) == MISALIGNED


def test_oproj_argument_errors(lib):
    assert lib.mla_o_proj(None, A, 4, A, None) == INVALID
    assert lib.mla_o_proj(A, None, 4, A, None) == INVALID
    assert lib.mla_o_proj(A, A, 4, None, None) == INVALID
    assert lib.mla_o_proj(A, A, 0, A, None) == SHAPE
    assert lib.mla_o_proj(A, A, -1, A, None) == SHAPE
    assert lib.mla_o_proj(A, A, 1 << 31, A, None) == SHAPE
    assert lib.mla_o_proj(A + 2, A, 4, A, None) == MISALIGNED
    assert lib.mla_o_proj(A, A + 8, 4, A, None) == MISALIGNED


def test_fused_argument_errors(lib):
    assert fused(lib, W=None) == INVALID
    assert fused(lib, q=None) == INVALID
    assert fused(lib, B=0) == SHAPE
    assert fused(lib, W=A + 2) == MISALIGNED
    assert fused(lib, ws=None) == WORKSPACE
    assert fused(lib, ws_bytes=ST + 64 * 8192 * 2 - 1) == WORKSPACE
    assert fused(lib, ws=A + 8) == MISALIGNED
    assert fused(lib, mask=A, ld=64, ws_bytes=ST + 64 * 8192 * 2) == WORKSPACE  # no class bytes


def varlen(lib, q=A, qp=A, k=A, kp=A, v=A, vl=A, B=1, T=64, scale=0.07, out=A):
    return lib.mla_attn_prefill_varlen(q, qp, k, kp, v, vl, B, T, scale, out, None)


def fused_varlen(lib, q=A, qp=A, k=A, kp=A, v=A, vl=A, B=1, T=64, scale=0.07, W=A, ws=A,
                 ws_bytes=1 << 40, out=A):
    return lib.mla_attn_oproj_varlen(q, qp, k, kp, v, vl, B, T, scale, W, ws, ws_bytes, out, None)


def test_varlen_argument_errors(lib):
    assert varlen(lib, vl=None) == INVALID
    assert varlen(lib, q=None) == INVALID
    assert varlen(lib, scale=float("nan")) == INVALID
    assert varlen(lib, B=0) == SHAPE
    assert varlen(lib, T=0) == SHAPE
    assert varlen(lib, vl=A + 2) == MISALIGNED  # int32 array must be 4-byte aligned
    assert varlen(lib, k=A + 8) == MISALIGNED
    assert fused_varlen(lib, vl=None) == INVALID
    assert fused_varlen(lib, W=None) == INVALID
    assert fused_varlen(lib, W=A + 2) == MISALIGNED
    assert fused_varlen(lib, vl=A + 1) == MISALIGNED
    assert fused_varlen(lib, ws=None) == WORKSPACE
    assert fused_varlen(lib, ws_bytes=ST + 64 * 8192 * 2 - 1) == WORKSPACE
    assert fused_varlen(lib, ws=A + 8) == MISALIGNED


def fused_fp8(lib, q=A, qp=A, k=A, kp=A, v=A, mask=None, ld=0, B=1, T=64, scale=0.07, Wq=A,
              Ws=A, ws=A, ws_bytes=1 << 40, out=A):
    return lib.mla_attn_oproj_fp8(q, qp, k, kp, v, mask, ld, B, T, scale, Wq, Ws, ws, ws_bytes,
                                  out, None)


def test_fp8_workspace_sizes(lib):
    M = 4096
    assert lib.mla_attn_oproj_fp8_workspace_bytes(1, M, 0) == \
        ST + M * 8192 * 2 + M * 8192 + 64 * M * 4
    # 3 tokens: 49152 + 24576 + 768, each already a multiple of 256; mask classes 1 -> 256
    assert lib.mla_attn_oproj_fp8_workspace_bytes(1, 3, 0) == ST + 49152 + 24576 + 768
    assert lib.mla_attn_oproj_fp8_workspace_bytes(1, 3, 1) == ST + 49152 + 24576 + 768 + 256
    assert lib.mla_attn_oproj_fp8_workspace_bytes(0, 3, 0) == 0


def test_fp8_argument_errors(lib):
    assert lib.mla_quantize_act_fp8(None, 4, A, A, None) == INVALID
    assert lib.mla_quantize_act_fp8(A, 4, None, A, None) == INVALID
    assert lib.mla_quantize_act_fp8(A, 4, A, None, None) == INVALID
    assert lib.mla_quantize_act_fp8(A, 0, A, A, None) == SHAPE
    assert lib.mla_quantize_act_fp8(A, 1 << 31, A, A, None) == SHAPE
    assert lib.mla_quantize_act_fp8(A + 8, 4, A, A, None) == MISALIGNED
    assert lib.mla_quantize_act_fp8(A, 4, A + 4, A, None) == MISALIGNED
    assert lib.mla_quantize_act_fp8(A, 4, A, A + 2, None) == MISALIGNED
    assert lib.mla_quantize_weight_fp8(None, A, A, None) == INVALID
    assert lib.mla_quantize_weight_fp8(A, A + 8, A, None) == MISALIGNED
    assert lib.mla_quantize_weight_fp8(A, A, A + 1, None) == MISALIGNED
    assert lib.mla_o_proj_fp8(None, A, A, A, 4, A, None) == INVALID
    assert lib.mla_o_proj_fp8(A, A, A, None, 4, A, None) == INVALID
    assert lib.mla_o_proj_fp8(A, A, A, A, 0, A, None) == SHAPE
    assert lib.mla_o_proj_fp8(A + 8, A, A, A, 4, A, None) == MISALIGNED
    assert lib.mla_o_proj_fp8(A, A + 2, A, A, 4, A, None) == MISALIGNED
    assert lib.mla_o_proj_fp8(A, A, A, A, 4, A + 2, None) == MISALIGNED
    assert fused_fp8(lib, Wq=None) == INVALID
    assert fused_fp8(lib, Ws=None) == INVALID
    assert fused_fp8(lib, B=0) == SHAPE
    assert fused_fp8(lib, Wq=A + 8) == MISALIGNED
    assert fused_fp8(lib, ws=None) == WORKSPACE
    assert fused_fp8(lib, ws_bytes=ST + 64 * 8192 * 3 + 64 * 64 * 4 - 1) == WORKSPACE
    assert fused_fp8(lib, ws=A + 8) == MISALIGNED


def test_last_device_status_argument_errors(lib):
    """The per-call status read checks its workspace before any CUDA call."""
    detail = ctypes.c_uint32(123)
    assert lib.mla_last_device_status(None, None, ctypes.byref(detail)) == INVALID
    assert detail.value == 0
    assert lib.mla_last_device_status(A + 4, None, None) == MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path only")
def test_valid_call_without_device_reports_cuda_error(lib):
    """With no usable device a well-formed call fails cleanly (MLA_ERR_CUDA)
    instead of launching anything."""
    assert prefill(lib) in (CUDA, UNSUPPORTED)
    assert lib.mla_o_proj(A, A, 4, A, None) in (CUDA, UNSUPPORTED)
    assert varlen(lib) in (CUDA, UNSUPPORTED)
    assert lib.mla_o_proj_fp8(A, A, A, A, 4, A, None) in (CUDA, UNSUPPORTED)
    assert lib.mla_quantize_act_fp8(A, 4, A, A, None) in (CUDA, UNSUPPORTED)


def test_binding_refuses_missing_library(tmp_path):
    with pytest.raises(RuntimeError):
        old = binding._lib
        try:
            binding._lib = None
            binding.load(str(tmp_path / "nope.so"))
        finally:
            binding._lib = old


def rope_call(lib, q=A, qp=A, k=A, kp=A, v=A, pos=None, rope="k2", mask=None, ld=0, B=1, T=64,
              scale=0.07, ws=A, ws_bytes=1 << 40, out=A):
    r = None if rope is None else ctypes.byref(
        binding._yarn(None) if rope == "k2" else binding.YarnRope(*rope))
    return lib.mla_attn_prefill_rope(q, qp, k, kp, v, pos, r, mask, ld, B, T, scale, ws,
                                     ws_bytes, out, None)


def test_rope_workspace_sizes(lib):
    # status | rotated key (B*T*128) | cos/sin table (B*T*256) | classes
    assert lib.mla_attn_prefill_rope_workspace_bytes(1, 4096, 0) == ST + 4096 * 128 + 4096 * 256
    assert lib.mla_attn_prefill_rope_workspace_bytes(2, 3, 1) == ST + 768 + 1536 + 256
    assert lib.mla_attn_oproj_rope_workspace_bytes(1, 3, 0) == ST + 512 + 768 + 49152  # 384 -> 512
    assert lib.mla_attn_prefill_rope_workspace_bytes(0, 3, 0) == 0


def test_rope_argument_errors(lib):
    k2 = (50000.0, 32.0, 4096.0, 1.0, 1.0, 1.0, 1.0)
    assert rope_call(lib, rope=None) == INVALID
    assert rope_call(lib, rope=(1.0,) + k2[1:]) == INVALID             # theta must exceed 1
    assert rope_call(lib, rope=k2[:1] + (0.0,) + k2[2:]) == INVALID    # factor > 0
    assert rope_call(lib, rope=k2[:3] + (-1.0,) + k2[4:]) == INVALID   # beta_fast > 0
    assert rope_call(lib, rope=k2[:5] + (float("nan"),) + k2[6:]) == INVALID
    assert rope_call(lib, q=None) == INVALID
    assert rope_call(lib, B=0) == SHAPE
    assert rope_call(lib, pos=A + 2) == MISALIGNED
    assert rope_call(lib, ws=None) == WORKSPACE                          # always required
    assert rope_call(lib, ws_bytes=ST + 64 * 128 + 64 * 256 - 1) == WORKSPACE
    assert rope_call(lib, ws=A + 8) == MISALIGNED
    assert lib.mla_attn_oproj_rope(A, A, A, A, A, None, ctypes.byref(binding._yarn(None)), None,
                                   0, 1, 64, 0.07, None, A, 1 << 40, A, None) == INVALID


def test_latent_workspace_sizes_and_argument_errors(lib):
    kv = 64 * 64 * 128 * 2  # k_nope or v of B=1, T=64
    assert lib.mla_attn_oproj_latent_workspace_bytes(1, 64, 0) == ST + 64 * 8192 * 2 + 2 * kv
    assert lib.mla_attn_oproj_latent_workspace_bytes(0, 64, 0) == 0
    up = lib.mla_kv_up_proj
    assert up(None, A, 1, 64, A, A, None) == INVALID
    assert up(A, A, 1, 64, A, None, None) == INVALID
    assert up(A, A, 0, 64, A, A, None) == SHAPE
    assert up(A, A, 1, 0, A, A, None) == SHAPE
    assert up(A + 2, A, 1, 64, A, A, None) == MISALIGNED
    assert up(A, A, 1, 64, A + 8, A, None) == MISALIGNED
    lat = lib.mla_attn_oproj_latent
    assert lat(A, A, None, A, A, None, 0, 1, 64, 0.07, A, A, 1 << 40, A, None) == INVALID
    assert lat(A, A, A, A, A, None, 0, 1, 64, 0.07, None, A, 1 << 40, A, None) == INVALID
    assert lat(A, A, A, A, A, None, 0, 1, 64, 0.07, A, A, ST + 64 * 8192 * 2, A, None) == WORKSPACE
    assert lat(A, A, A, A, A + 2, None, 0, 1, 64, 0.07, A, A, 1 << 40, A, None) == MISALIGNED
