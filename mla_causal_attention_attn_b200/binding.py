"""ctypes binding of ``libmla_b200.so`` (declared in ``include/mla.h``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI. PyTorch provides device memory and streams. There
is no fallback: if the library is missing or fails to load, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import inputs as _inputs

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

H = _inputs.H
DN, DR, DV = _inputs.DN, _inputs.DR, _inputs.DV
D_MODEL = _inputs.D_MODEL
K_OPROJ = _inputs.K_OPROJ

STATUS = {
    0: "MLA_OK",
    -1: "MLA_ERR_INVALID_ARG",
    -2: "MLA_ERR_SHAPE",
    -3: "MLA_ERR_MISALIGNED",
    -4: "MLA_ERR_UNSUPPORTED_DEVICE",
    -5: "MLA_ERR_WORKSPACE",
    -6: "MLA_ERR_CUDA",
    -7: "MLA_ERR_TIMEOUT",
}
MLA_OK = 0
WORKSPACE_STATUS_BYTES = 256  # MLA_WORKSPACE_STATUS_BYTES: the status word's block

class YarnRope(ctypes.Structure):
    """mla_yarn_rope_t: config.json's rope_theta and rope_scaling fields."""
    _fields_ = [("rope_theta", ctypes.c_double), ("factor", ctypes.c_double),
                ("original_max_position_embeddings", ctypes.c_double),
                ("beta_fast", ctypes.c_double), ("beta_slow", ctypes.c_double),
                ("mscale", ctypes.c_double), ("mscale_all_dim", ctypes.c_double)]


def _yarn(rope) -> YarnRope:
    r = _inputs.KIMI_K2_ROPE if rope is None else rope
    return YarnRope(*[float(r[f]) for f, _ in YarnRope._fields_])


# Every symbol include/mla.h declares, with its ctypes signature.
_VP = ctypes.c_void_p
_ROPE_P = ctypes.POINTER(YarnRope)
_SIGNATURES = {
    "mla_attn_prefill_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_prefill": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_float, _VP, ctypes.c_size_t, _VP,
                                        _VP]),
    "mla_o_proj": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, _VP, _VP]),
    "mla_attn_oproj_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_oproj": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_float, _VP, _VP, ctypes.c_size_t, _VP,
                                      _VP]),
    "mla_attn_oproj_noalloc": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_float, _VP,
                                              _VP, _VP]),
    "mla_attn_prefill_varlen": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_float, _VP, _VP]),
    "mla_attn_oproj_varlen": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_float, _VP, _VP,
                                             ctypes.c_size_t, _VP, _VP]),
    "mla_attn_prefill_rope_workspace_bytes": (ctypes.c_size_t,
                                              [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_prefill_rope": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _ROPE_P, _VP,
                                             ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_float, _VP, ctypes.c_size_t, _VP, _VP]),
    "mla_attn_oproj_rope_workspace_bytes": (ctypes.c_size_t,
                                            [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_oproj_rope": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _ROPE_P, _VP,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_float, _VP, _VP, ctypes.c_size_t, _VP, _VP]),
    "mla_kv_up_proj": (ctypes.c_int, [_VP, _VP, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP]),
    "mla_attn_oproj_latent_workspace_bytes": (ctypes.c_size_t,
                                              [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_oproj_latent": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_float, _VP,
                                             _VP, ctypes.c_size_t, _VP, _VP]),
    "mla_quantize_act_fp8": (ctypes.c_int, [_VP, ctypes.c_int64, _VP, _VP, _VP]),
    "mla_quantize_weight_fp8": (ctypes.c_int, [_VP, _VP, _VP, _VP]),
    "mla_o_proj_fp8": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP]),
    "mla_attn_oproj_fp8_workspace_bytes": (ctypes.c_size_t,
                                           [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_attn_oproj_fp8": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_float, _VP, _VP,
                                          _VP, ctypes.c_size_t, _VP, _VP]),
    "mla_last_device_status": (ctypes.c_int, [_VP, _VP, ctypes.POINTER(ctypes.c_uint32)]),
    "mla_device_status": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_uint32)]),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_abi_version": (ctypes.c_int, []),
}

_lock = threading.Lock()
_lib = None


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once). Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise RuntimeError(
                    f"{p} is missing: build it with `python -m mla_causal_attention_attn_b200.build`")
            lib = ctypes.CDLL(p)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(fn: str, status: int):
    if status != MLA_OK:
        raise MLAError(fn, status)


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _req(t, shape, name):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bf16, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def attn_prefill_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_prefill_workspace_bytes(B, T, int(bool(has_mask))))


def attn_oproj_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_oproj_workspace_bytes(B, T, int(bool(has_mask))))


def _mask_ld(mask, B, T):
    """Row stride of a [B,1,T,T] mask view whose rows are ``ld`` elements apart
    and whose batches are ``T*ld`` apart (a dense [B,1,T,ld] buffer)."""
    if mask is None:
        return 0
    if mask.dtype != torch.bfloat16 or not mask.is_cuda:
        raise TypeError("mask must be a bf16 CUDA tensor")
    if mask.dim() != 4 or tuple(mask.shape) != (B, 1, T, T):
        raise ValueError(f"mask must be [B,1,T,T] = {(B, 1, T, T)}, got {tuple(mask.shape)}")
    ld = int(mask.stride(2)) if T > 1 else max(int(mask.stride(2)), T)
    if mask.stride(3) != 1 or ld < T or (B > 1 and mask.stride(0) != T * ld):
        raise ValueError("mask must be a view of a dense [B,1,T,ld] buffer")
    return ld


def attn_prefill(q_nope, q_pe, k_nope, k_pe, v, mask=None, softmax_scale=None, out=None,
                 workspace=None, stream=None):
    """Merged-head attention output [B, T, 8192] (bf16) via ``mla_attn_prefill``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, K_OPROJ), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, K_OPROJ), "out")
    # Without a mask the workspace is optional (timeouts then go to the
    # device-wide status word); with one it holds the mask-tile classes.
    if mask is not None and workspace is None:
        need = attn_prefill_workspace_bytes(B, T, True)
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.mla_attn_prefill(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                              _ptr(mask), mask_ld, B, T, scale, _ptr(workspace), ws_bytes,
                              _ptr(out), _stream_handle(stream))
    _check("mla_attn_prefill", st)
    return out


def o_proj(attn, W_o, out=None, stream=None):
    """``attn [M, 8192] . W_o^T`` -> [M, 7168] (bf16) via ``mla_o_proj``."""
    lib = load()
    a2 = attn.reshape(-1, K_OPROJ)
    M = a2.shape[0]
    _req(a2, (M, K_OPROJ), "attn")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    if out is None:
        out = torch.empty((M, D_MODEL), dtype=torch.bfloat16, device=attn.device)
    _req(out.view(-1, D_MODEL), (M, D_MODEL), "out")
    st = lib.mla_o_proj(_ptr(a2), _ptr(W_o), M, _ptr(out), _stream_handle(stream))
    _check("mla_o_proj", st)
    return out


def attn_oproj(q_nope, q_pe, k_nope, k_pe, v, W_o, mask=None, softmax_scale=None, out=None,
               workspace=None, stream=None):
    """Whole path: attention then o_proj, [B, T, 7168] bf16, via ``mla_attn_oproj``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    need = attn_oproj_workspace_bytes(B, T, mask is not None)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.mla_attn_oproj(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                            _ptr(mask), mask_ld, B, T, scale, _ptr(W_o), _ptr(workspace),
                            ws_bytes, _ptr(out), _stream_handle(stream))
    _check("mla_attn_oproj", st)
    return out


def _valid_len(valid_len, B):
    if valid_len.dtype != torch.int32 or not valid_len.is_cuda:
        raise TypeError("valid_len must be an int32 CUDA tensor")
    if tuple(valid_len.shape) != (B,) or not valid_len.is_contiguous():
        raise ValueError(f"valid_len must be a contiguous [{B}] tensor")
    return valid_len


def attn_prefill_varlen(q_nope, q_pe, k_nope, k_pe, v, valid_len, softmax_scale=None, out=None,
                        stream=None):
    """Causal attention with key padding (keys j >= valid_len[b] excluded),
    [B, T, 8192] bf16, via ``mla_attn_prefill_varlen``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _valid_len(valid_len, B)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, K_OPROJ), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, K_OPROJ), "out")
    st = lib.mla_attn_prefill_varlen(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                     _ptr(valid_len), B, T, scale, _ptr(out),
                                     _stream_handle(stream))
    _check("mla_attn_prefill_varlen", st)
    return out


def attn_oproj_varlen(q_nope, q_pe, k_nope, k_pe, v, valid_len, W_o, softmax_scale=None,
                      out=None, workspace=None, stream=None):
    """Whole path with key padding given as valid lengths, [B, T, 7168] bf16,
    via ``mla_attn_oproj_varlen``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    _valid_len(valid_len, B)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    need = attn_oproj_workspace_bytes(B, T, False)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.mla_attn_oproj_varlen(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                   _ptr(valid_len), B, T, scale, _ptr(W_o), _ptr(workspace),
                                   ws_bytes, _ptr(out), _stream_handle(stream))
    _check("mla_attn_oproj_varlen", st)
    return out


def _positions(position_ids, B, T):
    if position_ids is None:
        return None
    if position_ids.dtype != torch.int32 or not position_ids.is_cuda:
        raise TypeError("position_ids must be an int32 CUDA tensor")
    if tuple(position_ids.shape) != (B, T) or not position_ids.is_contiguous():
        raise ValueError(f"position_ids must be a contiguous [{B}, {T}] tensor")
    return position_ids


def attn_prefill_rope_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_prefill_rope_workspace_bytes(B, T, int(bool(has_mask))))


def attn_oproj_rope_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_oproj_rope_workspace_bytes(B, T, int(bool(has_mask))))


def attn_prefill_rope(q_nope, q_pe, k_nope, k_pe, v, position_ids=None, rope=None, mask=None,
                      softmax_scale=None, out=None, workspace=None, stream=None):
    """Attention with unrotated q_pe / k_pe (YaRN rotation at position_ids
    [B, T] int32, None = 0..T-1; rope = a mapping of config.json's rotary
    fields, None = the printed Kimi K2 values), [B, T, 8192] bf16, via
    ``mla_attn_prefill_rope``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    pos = _positions(position_ids, B, T)
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, K_OPROJ), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, K_OPROJ), "out")
    if workspace is None:
        workspace = torch.empty(attn_prefill_rope_workspace_bytes(B, T, mask is not None),
                                dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    yr = _yarn(rope)
    st = lib.mla_attn_prefill_rope(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                   _ptr(pos), ctypes.byref(yr), _ptr(mask), mask_ld, B, T, scale,
                                   _ptr(workspace), ws_bytes, _ptr(out), _stream_handle(stream))
    _check("mla_attn_prefill_rope", st)
    return out


def attn_oproj_rope(q_nope, q_pe, k_nope, k_pe, v, W_o, position_ids=None, rope=None, mask=None,
                    softmax_scale=None, out=None, workspace=None, stream=None):
    """Whole path with unrotated q_pe / k_pe, [B, T, 7168] bf16, via
    ``mla_attn_oproj_rope``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    pos = _positions(position_ids, B, T)
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    if workspace is None:
        workspace = torch.empty(attn_oproj_rope_workspace_bytes(B, T, mask is not None),
                                dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    yr = _yarn(rope)
    st = lib.mla_attn_oproj_rope(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                 _ptr(pos), ctypes.byref(yr), _ptr(mask), mask_ld, B, T, scale,
                                 _ptr(W_o), _ptr(workspace), ws_bytes, _ptr(out),
                                 _stream_handle(stream))
    _check("mla_attn_oproj_rope", st)
    return out


KV_RANK = 512  # MLA_KV_RANK


def kv_up_proj(c_kv, W_kv_b, k_nope=None, v=None, stream=None):
    """k_nope, v [B, 64, T, 128] (bf16) from the latent c_kv [B, T, 512] and
    W_kv_b [16384, 512] via ``mla_kv_up_proj``."""
    lib = load()
    B, T, _ = c_kv.shape
    _req(c_kv, (B, T, KV_RANK), "c_kv")
    _req(W_kv_b, (H * (DN + DV), KV_RANK), "W_kv_b")
    if k_nope is None:
        k_nope = torch.empty((B, H, T, DN), dtype=torch.bfloat16, device=c_kv.device)
    if v is None:
        v = torch.empty((B, H, T, DV), dtype=torch.bfloat16, device=c_kv.device)
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(v, (B, H, T, DV), "v")
    st = lib.mla_kv_up_proj(_ptr(c_kv), _ptr(W_kv_b), B, T, _ptr(k_nope), _ptr(v),
                            _stream_handle(stream))
    _check("mla_kv_up_proj", st)
    return k_nope, v


def attn_oproj_latent_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_oproj_latent_workspace_bytes(B, T, int(bool(has_mask))))


def attn_oproj_latent(q_nope, q_pe, c_kv, k_pe, W_kv_b, W_o, mask=None, softmax_scale=None,
                      out=None, workspace=None, stream=None):
    """Whole path from the latent (up-projection, attention, o_proj),
    [B, T, 7168] bf16, via ``mla_attn_oproj_latent``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(c_kv, (B, T, KV_RANK), "c_kv")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(W_kv_b, (H * (DN + DV), KV_RANK), "W_kv_b")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    if workspace is None:
        workspace = torch.empty(attn_oproj_latent_workspace_bytes(B, T, mask is not None),
                                dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.mla_attn_oproj_latent(_ptr(q_nope), _ptr(q_pe), _ptr(c_kv), _ptr(k_pe),
                                   _ptr(W_kv_b), _ptr(mask), mask_ld, B, T, scale, _ptr(W_o),
                                   _ptr(workspace), ws_bytes, _ptr(out), _stream_handle(stream))
    _check("mla_attn_oproj_latent", st)
    return out


NOALLOC_MAX_TOKENS = 4096  # MLA_NOALLOC_MAX_TOKENS


def attn_oproj_noalloc(q_nope, q_pe, k_nope, k_pe, v, W_o, mask=None, softmax_scale=None,
                       out=None, stream=None):
    """Whole path through ``mla_attn_oproj_noalloc``: no workspace; the library
    uses its own fixed scratch (B*T <= 4096 tokens). Meant for callers that
    cannot allocate device memory; ``out`` should then be passed in."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    st = lib.mla_attn_oproj_noalloc(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                    _ptr(mask), mask_ld, B, T, scale, _ptr(W_o), _ptr(out),
                                    _stream_handle(stream))
    _check("mla_attn_oproj_noalloc", st)
    return out


# ------------------------------------------------------------------ FP8 o_proj
FP8_GROUP = 128
FP8_K_GROUPS = K_OPROJ // FP8_GROUP
FP8_N_BLOCKS = D_MODEL // FP8_GROUP


def _req_t(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def quantize_act_fp8(x, q=None, scale=None, stream=None):
    """Dynamic e4m3 quantisation of ``x [M, 8192]`` (bf16) via
    ``mla_quantize_act_fp8``: codes [M, 8192] (uint8), scales [64, M] (fp32)."""
    lib = load()
    x2 = x.reshape(-1, K_OPROJ)
    M = x2.shape[0]
    _req(x2, (M, K_OPROJ), "x")
    if q is None:
        q = torch.empty((M, K_OPROJ), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((FP8_K_GROUPS, M), dtype=torch.float32, device=x.device)
    _req_t(q, torch.uint8, (M, K_OPROJ), "q")
    _req_t(scale, torch.float32, (FP8_K_GROUPS, M), "scale")
    st = lib.mla_quantize_act_fp8(_ptr(x2), M, _ptr(q), _ptr(scale), _stream_handle(stream))
    _check("mla_quantize_act_fp8", st)
    return q, scale


def quantize_weight_fp8(W_o, stream=None):
    """128 x 128 block e4m3 quantisation of ``W_o [7168, 8192]`` via
    ``mla_quantize_weight_fp8``: codes [7168, 8192], scales [56, 64]."""
    lib = load()
    _req(W_o, (D_MODEL, K_OPROJ), "W_o")
    q = torch.empty((D_MODEL, K_OPROJ), dtype=torch.uint8, device=W_o.device)
    scale = torch.empty((FP8_N_BLOCKS, FP8_K_GROUPS), dtype=torch.float32, device=W_o.device)
    st = lib.mla_quantize_weight_fp8(_ptr(W_o), _ptr(q), _ptr(scale), _stream_handle(stream))
    _check("mla_quantize_weight_fp8", st)
    return q, scale


def o_proj_fp8(attn_q, attn_scale, W_q, W_scale, out=None, stream=None):
    """Block-scaled e4m3 o_proj -> [M, 7168] bf16 via ``mla_o_proj_fp8``."""
    lib = load()
    M = attn_q.shape[0]
    _req_t(attn_q, torch.uint8, (M, K_OPROJ), "attn_q")
    _req_t(attn_scale, torch.float32, (FP8_K_GROUPS, M), "attn_scale")
    _req_t(W_q, torch.uint8, (D_MODEL, K_OPROJ), "W_q")
    _req_t(W_scale, torch.float32, (FP8_N_BLOCKS, FP8_K_GROUPS), "W_scale")
    if out is None:
        out = torch.empty((M, D_MODEL), dtype=torch.bfloat16, device=attn_q.device)
    _req(out.view(-1, D_MODEL), (M, D_MODEL), "out")
    st = lib.mla_o_proj_fp8(_ptr(attn_q), _ptr(attn_scale), _ptr(W_q), _ptr(W_scale), M,
                            _ptr(out), _stream_handle(stream))
    _check("mla_o_proj_fp8", st)
    return out


def attn_oproj_fp8_workspace_bytes(B: int, T: int, has_mask: bool) -> int:
    return int(load().mla_attn_oproj_fp8_workspace_bytes(B, T, int(bool(has_mask))))


def attn_oproj_fp8(q_nope, q_pe, k_nope, k_pe, v, W_q, W_scale, mask=None, softmax_scale=None,
                   out=None, workspace=None, stream=None):
    """Attention, dynamic e4m3 quantisation of its output, FP8 o_proj:
    [B, T, 7168] bf16 via ``mla_attn_oproj_fp8``."""
    lib = load()
    B, _, T, _ = q_nope.shape
    _req(q_nope, (B, H, T, DN), "q_nope")
    _req(q_pe, (B, H, T, DR), "q_pe")
    _req(k_nope, (B, H, T, DN), "k_nope")
    _req(k_pe, (B, 1, T, DR), "k_pe")
    _req(v, (B, H, T, DV), "v")
    _req_t(W_q, torch.uint8, (D_MODEL, K_OPROJ), "W_q")
    _req_t(W_scale, torch.float32, (FP8_N_BLOCKS, FP8_K_GROUPS), "W_scale")
    mask_ld = _mask_ld(mask, B, T)
    scale = _inputs.DEFAULT_SCALE if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty((B, T, D_MODEL), dtype=torch.bfloat16, device=q_nope.device)
    _req(out, (B, T, D_MODEL), "out")
    need = attn_oproj_fp8_workspace_bytes(B, T, mask is not None)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.mla_attn_oproj_fp8(_ptr(q_nope), _ptr(q_pe), _ptr(k_nope), _ptr(k_pe), _ptr(v),
                                _ptr(mask), mask_ld, B, T, scale, _ptr(W_q), _ptr(W_scale),
                                _ptr(workspace), ws_bytes, _ptr(out), _stream_handle(stream))
    _check("mla_attn_oproj_fp8", st)
    return out


def device_status(stream=None):
    """Synchronise the stream; take the device-wide status word (the one the
    calls without a workspace report to). Returns (status, raw word)."""
    lib = load()
    detail = ctypes.c_uint32(0)
    st = lib.mla_device_status(_stream_handle(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


def last_device_status(workspace, stream=None):
    """Synchronise the stream; return (status, raw word) of the last call that
    used ``workspace`` (``mla_last_device_status``)."""
    lib = load()
    if workspace is None or not workspace.is_cuda:
        raise TypeError("workspace must be a CUDA tensor")
    detail = ctypes.c_uint32(0)
    st = lib.mla_last_device_status(_ptr(workspace), _stream_handle(stream),
                                    ctypes.byref(detail))
    return int(st), int(detail.value)
