"""fp64 CPU oracle for the MLA prefill core and its output projection.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use it; the product library never does.

The arithmetic lives in ``mla_oracle.c`` (plain loops, double precision, a
two-pass exact softmax). This module only compiles that file with gcc,
loads it with ctypes and marshals numpy / torch arrays. It shares nothing
with the CUDA path: the same seeded inputs are handed to both, and neither
imports the other.

What it follows: page "Kimi K2 · Mix and project", code excerpts
modeling_deepseek.py 799-840 (query/key assembly, scaled scores, additive
mask, fp32 softmax over keys, value mix) and 848-852 (head merge, o_proj);
the rotary step of the same excerpt (rotary_emb / apply_rotary_pos_emb) with
the YaRN parameters of the configuration printed on "Kimi K2 · Block input";
for the FP8 o_proj, page "Kimi K2 · Transformer blocks", configuration
excerpt (quantization_config: e4m3 codes, dynamic activation scales,
128 x 128 weight blocks), with the readings stated in mla_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmla_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libmla_oracle.so`` (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u16p = ctypes.POINTER(ctypes.c_uint16)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            u8p = ctypes.POINTER(ctypes.c_uint8)
            lib.mla_oracle_attn_rows.restype = ctypes.c_int
            lib.mla_oracle_attn_rows.argtypes = [
                u16p, u16p, u16p, u16p, u16p, u16p, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, i64p,
                ctypes.c_int64, f64p, f64p, u8p]
            lib.mla_oracle_oproj_rows.restype = ctypes.c_int
            lib.mla_oracle_oproj_rows.argtypes = [
                f64p, u16p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, f64p]
            f32p = ctypes.POINTER(ctypes.c_float)
            lib.mla_oracle_e4m3_decode.restype = ctypes.c_double
            lib.mla_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.mla_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.mla_oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.mla_oracle_quant_rows_fp8.restype = ctypes.c_int
            lib.mla_oracle_quant_rows_fp8.argtypes = [u16p, ctypes.c_int64, ctypes.c_int, u8p,
                                                      f32p]
            lib.mla_oracle_quant_weight_fp8.restype = ctypes.c_int
            lib.mla_oracle_quant_weight_fp8.argtypes = [u16p, ctypes.c_int, ctypes.c_int, u8p,
                                                        f32p]
            lib.mla_oracle_oproj_fp8_rows.restype = ctypes.c_int
            lib.mla_oracle_oproj_fp8_rows.argtypes = [
                u8p, f32p, ctypes.c_int64, i64p, ctypes.c_int64, u8p, f32p, ctypes.c_int,
                ctypes.c_int, f64p]
            lib.mla_oracle_yarn_inv_freq.restype = ctypes.c_int
            lib.mla_oracle_yarn_inv_freq.argtypes = [ctypes.c_int] + [ctypes.c_double] * 5 + [f64p]
            lib.mla_oracle_yarn_attn_factor.restype = ctypes.c_double
            lib.mla_oracle_yarn_attn_factor.argtypes = [ctypes.c_double] * 3
            lib.mla_oracle_rope_rotate.restype = ctypes.c_int
            lib.mla_oracle_rope_rotate.argtypes = [u16p, ctypes.c_int64, ctypes.c_int, i64p, f64p,
                                                   ctypes.c_double, f64p]
            lib.mla_oracle_attn_rows_rope.restype = ctypes.c_int
            lib.mla_oracle_attn_rows_rope.argtypes = [
                u16p, u16p, u16p, u16p, u16p, u16p, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, f64p, ctypes.c_double,
                i64p, i64p, ctypes.c_int64, f64p, f64p, u8p]
            lib.mla_oracle_kv_up.restype = ctypes.c_int
            lib.mla_oracle_kv_up.argtypes = [u16p, u16p] + [ctypes.c_int] * 6 + [f64p, f64p]
            lib.mla_oracle_attn_rows_kv64.restype = ctypes.c_int
            lib.mla_oracle_attn_rows_kv64.argtypes = [
                u16p, u16p, f64p, u16p, f64p, u16p, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_double, i64p, i64p,
                ctypes.c_int64, f64p, f64p, u8p]
            lib.mla_oracle_num_threads.restype = ctypes.c_int
            lib.mla_oracle_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().mla_oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().mla_oracle_set_num_threads(int(n))


def _bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor -> contiguous uint16 numpy array of its bit patterns."""
    import torch
    if isinstance(x, torch.Tensor):
        if x.dtype != torch.bfloat16:
            raise TypeError(f"expected a bf16 tensor, got {x.dtype}")
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16)
                                    .numpy().view(np.uint16))
    a = np.asarray(x)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns as uint16")
    return np.ascontiguousarray(a)


def bf16_to_f64(x) -> np.ndarray:
    """Exact widening of a bf16 tensor (or its uint16 bits) to float64."""
    bits = _bf16_bits(x).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def attn_rows(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale, rows=None,
              want_probs=False):
    """Merged head outputs ``attn[b, i, h*Dv + e]`` for the requested rows.

    Tensors are bf16 with shapes q_nope/k_nope [B,H,T,Dn], q_pe [B,H,T,Dr],
    k_pe [B,1,T,Dr], v [B,H,T,Dv], mask [B,1,T,T] or None (None = causal).
    ``rows`` is a sequence of (b, i) pairs, or None for every row in order.
    ``softmax_scale`` is widened from fp32 to double, the precision the
    kernels receive it in.

    Returns ``(out [R, H*Dv] float64, fully_masked [R, H] bool[, probs])``.
    """
    B, H, T, Dn = q_nope.shape
    Dr = q_pe.shape[-1]
    Dv = v.shape[-1]
    if tuple(q_pe.shape) != (B, H, T, Dr) or tuple(k_nope.shape) != (B, H, T, Dn):
        raise ValueError("q_pe / k_nope shape mismatch")
    if tuple(k_pe.shape) != (B, 1, T, Dr) or tuple(v.shape) != (B, H, T, Dv):
        raise ValueError("k_pe / v shape mismatch")
    if mask is not None and tuple(mask.shape) != (B, 1, T, T):
        raise ValueError("mask must be [B,1,T,T]")
    if rows is None:
        rb = np.repeat(np.arange(B, dtype=np.int64), T)
        ri = np.tile(np.arange(T, dtype=np.int64), B)
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        rb = np.ascontiguousarray(rows[:, 0])
        ri = np.ascontiguousarray(rows[:, 1])
    R = rb.shape[0]
    arrays = [_bf16_bits(t) for t in (q_nope, q_pe, k_nope, k_pe, v)]
    m = _bf16_bits(mask) if mask is not None else None
    out = np.zeros((R, H * Dv), dtype=np.float64)
    probs = np.zeros((R, H, T), dtype=np.float64) if want_probs else None
    fm = np.zeros((R, H), dtype=np.uint8)
    scale = float(np.float32(softmax_scale))
    rc = _load().mla_oracle_attn_rows(
        *[_ptr(a, ctypes.c_uint16) for a in arrays],
        _ptr(m, ctypes.c_uint16) if m is not None else None,
        ctypes.c_int64(T), B, H, T, Dn, Dr, Dv, scale,
        _ptr(rb, ctypes.c_int64), _ptr(ri, ctypes.c_int64), ctypes.c_int64(R),
        _ptr(out, ctypes.c_double),
        _ptr(probs, ctypes.c_double) if probs is not None else None,
        _ptr(fm, ctypes.c_uint8))
    if rc != 0:
        raise RuntimeError(f"oracle attn_rows failed ({rc})")
    if want_probs:
        return out, fm.astype(bool), probs
    return out, fm.astype(bool)


def oproj_rows(attn: np.ndarray, W_o) -> np.ndarray:
    """``attn [R, K] float64 . W_o^T`` with W_o bf16 ``[N, K]`` -> [R, N] float64."""
    a = np.ascontiguousarray(np.asarray(attn, dtype=np.float64))
    w = _bf16_bits(W_o)
    N, K = w.shape
    if a.ndim != 2 or a.shape[1] != K:
        raise ValueError("attn must be [R, K] with K = W_o.shape[1]")
    R = a.shape[0]
    out = np.zeros((R, N), dtype=np.float64)
    rc = _load().mla_oracle_oproj_rows(_ptr(a, ctypes.c_double),
                                       _ptr(w, ctypes.c_uint16),
                                       ctypes.c_int64(R), N, K,
                                       _ptr(out, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle oproj_rows failed ({rc})")
    return out


def attn_oproj_rows(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale, W_o,
                    rows=None):
    """Full path for the requested rows: attention, head merge, o_proj.

    Returns ``(out [R, N] float64, fully_masked_row [R] bool)``; a row is
    flagged when any of its heads had no allowed key.
    """
    attn, fm = attn_rows(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale,
                         rows=rows)
    return oproj_rows(attn, W_o), fm.any(axis=1)


# ------------------------------------------------------------------ rotary (YaRN)
# The readings (pair layout, YaRN frequencies, attention factor) are stated in
# mla_oracle.c. A parameter set is a mapping with the keys of config.json's
# rope_scaling plus rope_theta.

def yarn_inv_freq(Dr, rope) -> np.ndarray:
    """The Dr/2 rotation frequencies (radians per position) of a YaRN set."""
    out = np.zeros(Dr // 2, dtype=np.float64)
    rc = _load().mla_oracle_yarn_inv_freq(
        int(Dr), float(rope["rope_theta"]), float(rope["factor"]),
        float(rope["original_max_position_embeddings"]), float(rope["beta_fast"]),
        float(rope["beta_slow"]), _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle yarn_inv_freq rejected {rope}")
    return out


def yarn_attn_factor(rope) -> float:
    """The factor YaRN multiplies cos and sin by."""
    return float(_load().mla_oracle_yarn_attn_factor(
        float(rope["factor"]), float(rope["mscale"]), float(rope["mscale_all_dim"])))


def _positions(position_ids, B, T) -> np.ndarray:
    if position_ids is None:
        return np.ascontiguousarray(np.tile(np.arange(T, dtype=np.int64), B))
    import torch
    p = position_ids
    if isinstance(p, torch.Tensor):
        p = p.detach().cpu().numpy()
    p = np.asarray(p, dtype=np.int64)
    if p.shape != (B, T):
        raise ValueError(f"position_ids must be [B, T] = {(B, T)}, got {p.shape}")
    return np.ascontiguousarray(p.reshape(-1))


def rope_rotate(x, positions, rope) -> np.ndarray:
    """Rotated copy (float64) of bf16 rotary vectors x [..., Dr] at integer
    positions of shape x.shape[:-1]."""
    bits = _bf16_bits(x)
    Dr = bits.shape[-1]
    n = int(np.prod(bits.shape[:-1]))
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64).reshape(-1))
    if pos.shape[0] != n:
        raise ValueError("one position per rotary vector")
    inv = yarn_inv_freq(Dr, rope)
    out = np.zeros((n, Dr), dtype=np.float64)
    rc = _load().mla_oracle_rope_rotate(_ptr(bits, ctypes.c_uint16), ctypes.c_int64(n), Dr,
                                        _ptr(pos, ctypes.c_int64), _ptr(inv, ctypes.c_double),
                                        yarn_attn_factor(rope), _ptr(out, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle rope_rotate failed ({rc})")
    return out.reshape(bits.shape)


def attn_rows_rope(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale, position_ids, rope,
                   rows=None):
    """attn_rows with q_pe and k_pe given unrotated: both are rotated (YaRN,
    at position_ids [B, T], or 0..T-1 when None) before the scores."""
    B, H, T, Dn = q_nope.shape
    Dr = q_pe.shape[-1]
    Dv = v.shape[-1]
    if tuple(q_pe.shape) != (B, H, T, Dr) or tuple(k_pe.shape) != (B, 1, T, Dr) or \
            tuple(k_nope.shape) != (B, H, T, Dn) or tuple(v.shape) != (B, H, T, Dv):
        raise ValueError("input shapes do not match")
    if mask is not None and tuple(mask.shape) != (B, 1, T, T):
        raise ValueError("mask must be [B,1,T,T]")
    if rows is None:
        rb = np.repeat(np.arange(B, dtype=np.int64), T)
        ri = np.tile(np.arange(T, dtype=np.int64), B)
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        rb = np.ascontiguousarray(rows[:, 0])
        ri = np.ascontiguousarray(rows[:, 1])
    R = rb.shape[0]
    arrays = [_bf16_bits(t) for t in (q_nope, q_pe, k_nope, k_pe, v)]
    m = _bf16_bits(mask) if mask is not None else None
    pos = _positions(position_ids, B, T)
    inv = yarn_inv_freq(Dr, rope)
    out = np.zeros((R, H * Dv), dtype=np.float64)
    fm = np.zeros((R, H), dtype=np.uint8)
    scale = float(np.float32(softmax_scale))
    rc = _load().mla_oracle_attn_rows_rope(
        *[_ptr(a, ctypes.c_uint16) for a in arrays],
        _ptr(m, ctypes.c_uint16) if m is not None else None,
        ctypes.c_int64(T), B, H, T, Dn, Dr, Dv, scale, _ptr(pos, ctypes.c_int64),
        _ptr(inv, ctypes.c_double), yarn_attn_factor(rope),
        _ptr(rb, ctypes.c_int64), _ptr(ri, ctypes.c_int64), ctypes.c_int64(R),
        _ptr(out, ctypes.c_double), None, _ptr(fm, ctypes.c_uint8))
    if rc != 0:
        raise RuntimeError(f"oracle attn_rows_rope failed ({rc})")
    return out, fm.astype(bool)


def attn_oproj_rows_rope(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale, position_ids, rope,
                         W_o, rows=None):
    """Full path with unrotated q_pe / k_pe: rotation, attention, o_proj."""
    attn, fm = attn_rows_rope(q_nope, q_pe, k_nope, k_pe, v, mask, softmax_scale, position_ids,
                              rope, rows=rows)
    return oproj_rows(attn, W_o), fm.any(axis=1)


# ------------------------------------------------------------------ latent up-projection
# Reading (mla_oracle.c, section "latent"): one bias-free linear map of each
# token's latent to 64 heads x (128 non-rotary key + 128 value), the key part
# first within each head's block of rows of W.

def kv_up(c_kv, W_kv, H, Dn, Dv):
    """k_nope [B,H,T,Dn] and v [B,H,T,Dv] (float64) from the bf16 latent
    c_kv [B,T,R] and the bf16 weight W_kv [H*(Dn+Dv), R]."""
    x = _bf16_bits(c_kv)
    w = _bf16_bits(W_kv)
    B, T, R = x.shape
    if w.shape != (H * (Dn + Dv), R):
        raise ValueError(f"W_kv must be [{H * (Dn + Dv)}, {R}], got {w.shape}")
    k = np.zeros((B, H, T, Dn), dtype=np.float64)
    v = np.zeros((B, H, T, Dv), dtype=np.float64)
    rc = _load().mla_oracle_kv_up(_ptr(x, ctypes.c_uint16), _ptr(w, ctypes.c_uint16), B, T, R, H,
                                  Dn, Dv, _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle kv_up failed ({rc})")
    return k, v


def attn_rows_kv64(q_nope, q_pe, k_nope64, k_pe, v64, mask, softmax_scale, rows=None):
    """attn_rows with the non-rotary keys and the values given in float64."""
    B, H, T, Dn = q_nope.shape
    Dr = q_pe.shape[-1]
    Dv = v64.shape[-1]
    k_nope64 = np.ascontiguousarray(k_nope64, dtype=np.float64)
    v64 = np.ascontiguousarray(v64, dtype=np.float64)
    if k_nope64.shape != (B, H, T, Dn) or v64.shape[:3] != (B, H, T) or \
            tuple(k_pe.shape) != (B, 1, T, Dr) or tuple(q_pe.shape) != (B, H, T, Dr):
        raise ValueError("input shapes do not match")
    if mask is not None and tuple(mask.shape) != (B, 1, T, T):
        raise ValueError("mask must be [B,1,T,T]")
    if rows is None:
        rb = np.repeat(np.arange(B, dtype=np.int64), T)
        ri = np.tile(np.arange(T, dtype=np.int64), B)
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        rb = np.ascontiguousarray(rows[:, 0])
        ri = np.ascontiguousarray(rows[:, 1])
    R = rb.shape[0]
    qn, qp, kp = (_bf16_bits(t) for t in (q_nope, q_pe, k_pe))
    m = _bf16_bits(mask) if mask is not None else None
    out = np.zeros((R, H * Dv), dtype=np.float64)
    fm = np.zeros((R, H), dtype=np.uint8)
    rc = _load().mla_oracle_attn_rows_kv64(
        _ptr(qn, ctypes.c_uint16), _ptr(qp, ctypes.c_uint16), _ptr(k_nope64, ctypes.c_double),
        _ptr(kp, ctypes.c_uint16), _ptr(v64, ctypes.c_double),
        _ptr(m, ctypes.c_uint16) if m is not None else None, ctypes.c_int64(T), B, H, T, Dn, Dr,
        Dv, float(np.float32(softmax_scale)), _ptr(rb, ctypes.c_int64), _ptr(ri, ctypes.c_int64),
        ctypes.c_int64(R), _ptr(out, ctypes.c_double), None, _ptr(fm, ctypes.c_uint8))
    if rc != 0:
        raise RuntimeError(f"oracle attn_rows_kv64 failed ({rc})")
    return out, fm.astype(bool)


def attn_oproj_rows_latent(q_nope, q_pe, c_kv, W_kv, k_pe, mask, softmax_scale, W_o, rows=None):
    """Full path from the latent: up-projection, attention, head merge, o_proj."""
    H, Dn = q_nope.shape[1], q_nope.shape[3]
    Dv = W_kv.shape[0] // H - Dn
    k, v = kv_up(c_kv, W_kv, H, Dn, Dv)
    attn, fm = attn_rows_kv64(q_nope, q_pe, k, k_pe, v, mask, softmax_scale, rows=rows)
    return oproj_rows(attn, W_o), fm.any(axis=1)


# ------------------------------------------------------------------ FP8 o_proj
# Page "Kimi K2 · Transformer blocks", configuration excerpt (config.json,
# quantization_config: fp8, e4m3, dynamic activation scales, 128 x 128 weight
# blocks). The arithmetic and the readings are in mla_oracle.c.

FP8_GROUP = 128


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of e4m3 codes (uint8 array-like)."""
    c = np.asarray(codes, dtype=np.uint8)
    lib = _load()
    flat = np.array([lib.mla_oracle_e4m3_decode(int(x)) for x in c.reshape(-1)],
                    dtype=np.float64)
    return flat.reshape(c.shape)


def e4m3_encode(y) -> np.ndarray:
    """Nearest e4m3 codes (ties to even, saturating at 448) of fp32 values."""
    a = np.asarray(y, dtype=np.float32)
    lib = _load()
    flat = np.array([lib.mla_oracle_e4m3_encode(float(x)) for x in a.reshape(-1)],
                    dtype=np.uint8)
    return flat.reshape(a.shape)


def quant_rows_fp8(x):
    """Dynamic per-token quantisation of a bf16 [M, K] tensor.

    Returns ``(q [M, K] uint8, scale [K/128, M] float32)``."""
    bits = _bf16_bits(x)
    if bits.ndim != 2:
        raise ValueError("x must be [M, K]")
    M, K = bits.shape
    q = np.zeros((M, K), dtype=np.uint8)
    s = np.zeros((K // FP8_GROUP, M), dtype=np.float32)
    rc = _load().mla_oracle_quant_rows_fp8(_ptr(bits, ctypes.c_uint16), ctypes.c_int64(M), K,
                                           _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle quant_rows_fp8 failed ({rc})")
    return q, s


def quant_weight_fp8(W):
    """128 x 128 block quantisation of a bf16 [N, K] weight.

    Returns ``(q [N, K] uint8, scale [N/128, K/128] float32)``."""
    bits = _bf16_bits(W)
    if bits.ndim != 2:
        raise ValueError("W must be [N, K]")
    N, K = bits.shape
    q = np.zeros((N, K), dtype=np.uint8)
    s = np.zeros((N // FP8_GROUP, K // FP8_GROUP), dtype=np.float32)
    rc = _load().mla_oracle_quant_weight_fp8(_ptr(bits, ctypes.c_uint16), N, K,
                                             _ptr(q, ctypes.c_uint8), _ptr(s, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle quant_weight_fp8 failed ({rc})")
    return q, s


def _u8(a) -> np.ndarray:
    import torch
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().contiguous().view(torch.uint8).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def _f32(a) -> np.ndarray:
    import torch
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def oproj_fp8_rows(qa, a_scale, qw, w_scale, rows=None) -> np.ndarray:
    """Block-scaled e4m3 product for the requested rows of qa.

    qa [M, K] codes, a_scale [K/128, M]; qw [N, K] codes, w_scale
    [N/128, K/128]; rows: row indices or None for all. Returns [R, N] float64.
    """
    qa, qw = _u8(qa), _u8(qw)
    a_scale, w_scale = _f32(a_scale), _f32(w_scale)
    M, K = qa.shape
    N = qw.shape[0]
    if qw.shape[1] != K or a_scale.shape != (K // FP8_GROUP, M) or \
            w_scale.shape != (N // FP8_GROUP, K // FP8_GROUP):
        raise ValueError("fp8 operand shapes do not match")
    r = (np.arange(M, dtype=np.int64) if rows is None
         else np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1)))
    out = np.zeros((r.shape[0], N), dtype=np.float64)
    rc = _load().mla_oracle_oproj_fp8_rows(
        _ptr(qa, ctypes.c_uint8), _ptr(a_scale, ctypes.c_float), ctypes.c_int64(M),
        _ptr(r, ctypes.c_int64), ctypes.c_int64(r.shape[0]), _ptr(qw, ctypes.c_uint8),
        _ptr(w_scale, ctypes.c_float), N, K, _ptr(out, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle oproj_fp8_rows failed ({rc})")
    return out
