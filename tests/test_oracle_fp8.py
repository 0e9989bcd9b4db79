"""Pins for the oracle's FP8 o_proj functions, CPU only.

The configuration excerpt on page "Kimi K2 · Transformer blocks" names the
format (e4m3, dynamic activation scales, 128 x 128 weight blocks) and prints
no values. The oracle's e4m3 arithmetic is pinned against an independent
implementation of the format, torch's float8_e4m3fn type (its decoding of
every code and its round-to-nearest-even conversion), against the format's
landmark values, and by brute force. The quantisers are pinned against a
numpy/torch restatement that shares no code with the C oracle, and the
block-scaled product against exact integer and float64 library matmuls.
Each case names the mistake it is there to catch.
"""
import numpy as np
import pytest
import torch

import oracle

G = oracle.FP8_GROUP


def torch_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_encode(y32):
    """torch's nearest-even cast; valid for |y| <= 464 (beyond that torch
    gives NaN where the e4m3 reading saturates)."""
    return torch.from_numpy(np.ascontiguousarray(y32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_every_code_matches_torch():
    """All 256 codes: a wrong exponent bias, subnormal rule or NaN code fails."""
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))  # -0 at 0x80


def test_decode_landmarks():
    """The format's fixed points: largest finite, smallest subnormal and
    normal, one, and the sign bit."""
    v = oracle.e4m3_decode(np.array([0x7E, 0x01, 0x07, 0x08, 0x38, 0x39, 0xB8, 0xFE],
                                    dtype=np.uint8))
    assert list(v) == [448.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.125, -1.0, -448.0]


def test_encode_matches_torch_on_random_and_tie_values():
    """Random magnitudes over the whole range and every exact midpoint
    between neighbouring codes (the ties): a wrong tie rule or an off-by-one
    in the search fails."""
    rng = np.random.default_rng(0)
    mag = np.exp2(rng.uniform(-12, np.log2(448.0), 20000))
    y = (mag * rng.choice([-1.0, 1.0], mag.shape)).astype(np.float32)
    vals = torch_decode(np.arange(127, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)  # exact in fp32
    y = np.concatenate([y, mids, -mids, np.float32([0.0, -0.0, 448.0, -448.0, 460.0])])
    assert np.array_equal(oracle.e4m3_encode(y), torch_encode(y))


def test_encode_is_the_nearest_code_by_brute_force():
    """Nearest by exhaustive search over the 127 finite magnitudes (ties to
    the even code), a different algorithm from the oracle's bisection."""
    rng = np.random.default_rng(1)
    y = (np.exp2(rng.uniform(-11, 9, 3000)) * rng.choice([-1.0, 1.0], 3000)).astype(np.float32)
    table = torch_decode(np.arange(127, dtype=np.uint8))
    got = oracle.e4m3_encode(y)
    for yi, gi in zip(y, got):
        a = min(abs(float(yi)), 448.0)
        d = np.abs(table - a)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        assert gi == (code | (0x80 if yi < 0 else 0)), (yi, gi, code)


def test_encode_saturates_and_keeps_the_sign_of_zero():
    y = np.float32([449.0, 464.0, 465.0, 1e30, -500.0, 2.0 ** -11, -(2.0 ** -11), -0.0,
                    2.0 ** -10, 2.0 ** -10 * 1.0001])
    assert list(oracle.e4m3_encode(y)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80, 0x80,
                                           0x00, 0x01]


def reference_quant(x32, groups_axis_last):
    """numpy/torch restatement of the quantiser for [.., G] groups: fp32
    amax, fp32 scale amax/448 (1 for zeros), fp32 quotient, torch's
    nearest-even cast."""
    amax = np.abs(x32).max(axis=-1, keepdims=True).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    y = (x32 / s).astype(np.float32)
    assert np.abs(y).max() <= 464.0
    return torch_encode(y), s[..., 0]


def bf16_tensor(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_quant_rows_matches_restatement():
    """Per-token, per-128-feature groups with group-major scales: a group
    taken along the wrong axis, a scale layout transposed, or a scale in the
    wrong precision fails bit-exactly."""
    rng = np.random.default_rng(2)
    M, K = 37, 4 * G
    x = rng.standard_normal((M, K)) * np.exp2(rng.integers(-8, 8, (M, 1)))
    x[3, G:2 * G] = 0.0                     # a group of zeros: scale 1
    x[4, :G] = -0.0
    x[5, 5] = 1e4                           # one large value in a group
    xb = bf16_tensor(x)
    q, s = oracle.quant_rows_fp8(xb)
    x32 = xb.float().numpy().reshape(M, K // G, G)
    rq, rs = reference_quant(x32, True)
    assert np.array_equal(q, rq.reshape(M, K))
    assert np.array_equal(s, rs.T)          # [K/128, M]
    assert s[1, 3] == 1.0 and np.all(q[3, G:2 * G] == 0)
    assert np.all(q[4, :G] == 0x80)


def test_quant_rows_group_maximum_maps_to_448_and_error_bound():
    """The largest magnitude of each group becomes +-448, and every element is
    within half a step of the e4m3 grid (of the fp32 quotient)."""
    rng = np.random.default_rng(3)
    xb = bf16_tensor(rng.standard_normal((16, 2 * G)))
    q, s = oracle.quant_rows_fp8(xb)
    x32 = xb.float().numpy().reshape(16, 2, G)
    idx = np.abs(x32).argmax(axis=-1)
    qg = q.reshape(16, 2, G)
    top = np.take_along_axis(qg, idx[..., None], axis=-1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)
    y = (x32 / s.T[..., None]).astype(np.float32).astype(np.float64)
    v = oracle.e4m3_decode(qg)
    e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
    half_step = np.exp2(e - 4)              # half of 2^(e-3)
    assert np.all(np.abs(v - y) <= half_step)


def test_quant_weight_blocks_match_restatement():
    """128 x 128 blocks, scales [N/128, K/128]: a block taken as 1 x 128 or
    a transposed scale grid fails."""
    rng = np.random.default_rng(4)
    N, K = 2 * G, 3 * G
    W = rng.standard_normal((N, K)) * 0.02
    W[:G, 2 * G:] *= 50.0                   # one block with a much larger scale
    Wb = bf16_tensor(W)
    q, s = oracle.quant_weight_fp8(Wb)
    w32 = Wb.float().numpy().reshape(N // G, G, K // G, G).transpose(0, 2, 1, 3)
    rq, rs = reference_quant(w32.reshape(N // G, K // G, G * G), True)
    assert np.array_equal(s, rs)
    rq = rq.reshape(N // G, K // G, G, G).transpose(0, 2, 1, 3).reshape(N, K)
    assert np.array_equal(q, rq)


def random_codes(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38            # no NaN codes
    return c


def test_oproj_fp8_integer_case_is_exact():
    """Codes whose values are small integers and unit scales: the product is
    an integer matmul, exactly (a dropped block or a wrong code table fails)."""
    rng = np.random.default_rng(5)
    ints = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48, -1: 0xB8, -2: 0xC0, -3: 0xC4}
    keys = np.array(list(ints.keys()))
    M, N, K = 5, 2 * G, 3 * G
    ia = rng.choice(keys, (M, K))
    iw = rng.choice(keys, (N, K))
    qa = np.vectorize(ints.get)(ia).astype(np.uint8)
    qw = np.vectorize(ints.get)(iw).astype(np.uint8)
    out = oracle.oproj_fp8_rows(qa, np.ones((K // G, M), np.float32), qw,
                                np.ones((N // G, K // G), np.float32))
    assert np.array_equal(out, (ia.astype(np.int64) @ iw.astype(np.int64).T).astype(np.float64))


def test_oproj_fp8_matches_dequantised_float64_matmul():
    """Random codes and scales against numpy's float64 matmul of the
    dequantised operands (torch's decoding, scales expanded elementwise): a
    scale applied to the wrong row, column or block fails."""
    rng = np.random.default_rng(6)
    M, N, K = 9, 3 * G, 4 * G
    qa, qw = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    a_s = np.exp2(rng.uniform(-10, 0, (K // G, M))).astype(np.float32)
    w_s = np.exp2(rng.uniform(-12, -4, (N // G, K // G))).astype(np.float32)
    A = torch_decode(qa) * np.repeat(a_s.T.astype(np.float64), G, axis=1)
    W = torch_decode(qw) * np.repeat(np.repeat(w_s.astype(np.float64), G, axis=0), G, axis=1)
    ref = A @ W.T
    out = oracle.oproj_fp8_rows(qa, a_s, qw, w_s)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = [8, 0, 3]
    assert np.array_equal(oracle.oproj_fp8_rows(qa, a_s, qw, w_s, rows=rows), out[rows])


def test_oproj_fp8_shape_checks():
    qa = np.zeros((2, G), np.uint8)
    with pytest.raises(ValueError):
        oracle.oproj_fp8_rows(qa, np.ones((1, 3), np.float32), np.zeros((G, G), np.uint8),
                              np.ones((1, 1), np.float32))
    with pytest.raises(RuntimeError):
        oracle.oproj_fp8_rows(qa, np.ones((1, 2), np.float32), np.zeros((G, G), np.uint8),
                              np.ones((1, 1), np.float32), rows=[2])
