"""Pins of the oracle's rotary step (YaRN frequencies, attention factor,
rotation) and of attention with unrotated rotary inputs, on the CPU.

What the oracle follows: the rotary step of page "Kimi K2 · Mix and project"
(excerpt modeling_deepseek.py 799-840: rotary_emb, apply_rotary_pos_emb)
with rope_theta and the rope_scaling block of config.json on page "Kimi K2 ·
Block input"; the readings are in oracle/mla_oracle.c, section "rotary".
Each pin below is chosen so that a plausible mistake fails it: a swapped
sign in the rotation, sin/cos swapped, the ramp reversed or floor/ceil
swapped, the factor multiplied instead of divided, the key rotated with the
wrong positions, the rotation applied to the non-rotary part.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "rope_cases.json")
K2 = inputs.KIMI_K2_ROPE


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def rope(**kw):
    r = dict(K2)
    r.update(kw)
    return r


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------ frequencies
def test_factor_one_is_plain_rope():
    """With factor 1 interpolation and extrapolation coincide: the
    frequencies are the textbook RoPE ones, theta^(-2i/Dr), whatever the ramp."""
    for theta, Dr in ((50000.0, 64), (10000.0, 8)):
        f = oracle.yarn_inv_freq(Dr, rope(rope_theta=theta, factor=1.0))
        want = theta ** (-np.arange(Dr // 2) * 2.0 / Dr)
        np.testing.assert_allclose(f, want, rtol=1e-15)


def test_kimi_k2_frequency_cut(golden):
    """The printed set (beta_fast = beta_slow = 1) puts the ramp between pair
    19 and pair 20: worked by hand in the golden file."""
    g = golden["kimi_k2_frequency_cut"]
    f = oracle.yarn_inv_freq(64, K2)
    base = 50000.0 ** (-np.arange(32) * 2.0 / 64)
    ratio = f / base
    np.testing.assert_allclose(ratio[: g["high"]], 1.0, rtol=1e-14)
    np.testing.assert_allclose(ratio[g["high"]:], 1.0 / g["factor"], rtol=1e-14)
    assert g["low"] == math.floor(g["correction_index"]) and g["high"] == g["low"] + 1


def test_ramp_between_low_and_high(golden):
    """beta_fast = 32, beta_slow = 1 (a wide ramp): extrapolated below pair
    10, interpolated from pair 23, linear in between (hand-worked bounds)."""
    g = golden["ramp_example"]
    r = rope(rope_theta=g["theta"], factor=g["factor"], beta_fast=g["beta_fast"],
             beta_slow=g["beta_slow"])
    f = oracle.yarn_inv_freq(64, r)
    base = g["theta"] ** (-np.arange(32) * 2.0 / 64)
    lo, hi, s = g["low"], g["high"], g["factor"]
    for i in range(32):
        t = min(max((i - lo) / (hi - lo), 0.0), 1.0)
        assert f[i] / base[i] == pytest.approx(1.0 - t + t / s, rel=1e-13), i
    assert np.all(np.diff(f) < 0)   # frequencies fall with the pair index


def test_attention_factor(golden):
    g = golden["attention_factor"]
    assert oracle.yarn_attn_factor(K2) == 1.0
    assert oracle.yarn_attn_factor(rope(factor=g["factor"], mscale=g["mscale"],
                                        mscale_all_dim=g["mscale_all_dim"])) == \
        pytest.approx(g["expect"], abs=2e-7)
    assert oracle.yarn_attn_factor(rope(factor=1.0, mscale=3.0)) == 1.0  # no scaling at s <= 1


# ------------------------------------------------------------------ rotation
def test_hand_worked_rotations(golden):
    for c in golden["rotation"]:
        got = oracle.rope_rotate(bf16([c["x"]]), [c["position"]], rope())
        np.testing.assert_allclose(got[0], c["expect"], atol=1e-9, err_msg=c["what"])


def test_rotation_is_complex_multiplication():
    """An independent formulation: pair (x0, x1) as the complex number
    x0 + i x1 times f * exp(i * position * inv_freq)."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(50, 64, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, 40000, (50,), generator=g)
    for r in (K2, rope(mscale=2.0)):
        got = oracle.rope_rotate(x, pos.numpy(), r)
        w = oracle.yarn_inv_freq(64, r)
        f = oracle.yarn_attn_factor(r)
        xf = oracle.bf16_to_f64(x)
        z = (xf[:, 0::2] + 1j * xf[:, 1::2]) * f * np.exp(1j * pos.numpy()[:, None] * w[None, :])
        want = np.empty_like(xf)
        want[:, 0::2], want[:, 1::2] = z.real, z.imag
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=1e-12)


def test_position_zero_identity_and_pair_norms():
    g = torch.Generator().manual_seed(4)
    x = torch.randn(20, 64, generator=g).to(torch.bfloat16)
    xf = oracle.bf16_to_f64(x)
    assert np.array_equal(oracle.rope_rotate(x, np.zeros(20, dtype=np.int64), K2), xf)
    y = oracle.rope_rotate(x, np.arange(20) * 977, rope(mscale=2.0))
    f = oracle.yarn_attn_factor(rope(mscale=2.0))
    np.testing.assert_allclose(np.hypot(y[:, 0::2], y[:, 1::2]),
                               f * np.hypot(xf[:, 0::2], xf[:, 1::2]), rtol=1e-13)


def test_scores_depend_on_relative_position_only():
    """q at position m against k at position n: the same number for (m + s,
    n + s), for the printed set and for a ramped one."""
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 64, generator=g).to(torch.bfloat16)
    for r in (K2, rope(beta_fast=32.0, factor=40.0)):
        for m, n, s in ((5, 2, 1000), (300, 299, 77777), (4096, 0, 12345)):
            a = oracle.rope_rotate(q, [m], r)[0] @ oracle.rope_rotate(k, [n], r)[0]
            b = oracle.rope_rotate(q, [m + s], r)[0] @ oracle.rope_rotate(k, [n + s], r)[0]
            assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


def test_half_split_layout_gives_the_same_scores():
    """Storing rotated pair i at (i, i + Dr/2) instead of (2i, 2i + 1) (the
    first-halves-then-second-halves layout) changes no dot product, so the
    reading of the layout cannot move any score."""
    g = torch.Generator().manual_seed(6)
    q = torch.randn(8, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(8, 64, generator=g).to(torch.bfloat16)
    pq, pk = np.arange(8) * 31 + 3, np.arange(8) * 7
    rq, rk = oracle.rope_rotate(q, pq, K2), oracle.rope_rotate(k, pk, K2)
    perm = np.concatenate([np.arange(0, 64, 2), np.arange(1, 64, 2)])
    np.testing.assert_allclose(rq[:, perm] @ rk[:, perm].T, rq @ rk.T, rtol=1e-14, atol=1e-13)


# ------------------------------------------------------------------ attention
def _numpy_attention(d, pos, r):
    """softmax(Q K^T * scale + causal) V per head in numpy, with the rotary
    parts rotated as complex numbers: a second implementation of the whole
    rotary path for tiny shapes."""
    f64 = oracle.bf16_to_f64
    qn, qp, kn, kp, v = (f64(d[n]) for n in ("q_nope", "q_pe", "k_nope", "k_pe", "v"))
    B, H, T, _ = qn.shape
    Dr = qp.shape[-1]
    w = oracle.yarn_inv_freq(Dr, r)
    f = oracle.yarn_attn_factor(r)

    def rot(x, p):
        z = (x[..., 0::2] + 1j * x[..., 1::2]) * f * np.exp(1j * p[..., None] * w)
        y = np.empty_like(x)
        y[..., 0::2], y[..., 1::2] = z.real, z.imag
        return y

    out = np.zeros((B, T, H * v.shape[-1]))
    for b in range(B):
        kr = rot(kp[b, 0], pos[b])
        for h in range(H):
            Q = np.concatenate([qn[b, h], rot(qp[b, h], pos[b])], axis=1)
            K = np.concatenate([kn[b, h], kr], axis=1)
            s = Q @ K.T * float(np.float32(d["softmax_scale"]))
            s[np.triu_indices(T, 1)] = -np.inf
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h * v.shape[-1]:(h + 1) * v.shape[-1]] = p @ v[b, h]
    return out.reshape(B * T, -1)


@pytest.mark.parametrize("kind", ["arange", "offset", "random"])
def test_attention_with_rotation_matches_numpy(kind):
    d = inputs.make_inputs(2, 9, seed=11, H_=3, Dn=4, Dr=6, Dv=5, with_weight=False)
    pos = inputs.make_positions(2, 9, kind, seed=2)
    r = rope(beta_fast=32.0, rope_theta=10000.0, original_max_position_embeddings=16.0)
    got, fm = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                    None, d["softmax_scale"], pos, r)
    assert not fm.any()
    np.testing.assert_allclose(got, _numpy_attention(d, pos.numpy().astype(np.int64), r),
                               rtol=1e-11, atol=1e-12)


def test_constant_positions_leave_attention_unrotated():
    """All positions equal: every query and key turn by the same angles, so
    no score changes and the result is the unrotated attention (exactly at
    position 0, where the rotation is the identity)."""
    d = inputs.make_inputs(1, 40, seed=12, H_=2, with_weight=False)
    plain, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                d["softmax_scale"])
    zero, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                    d["softmax_scale"], torch.zeros(1, 40, dtype=torch.int32),
                                    K2)
    assert np.array_equal(zero, plain)
    c, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                 d["softmax_scale"], torch.full((1, 40), 5000, dtype=torch.int32),
                                 K2)
    np.testing.assert_allclose(c, plain, rtol=1e-10, atol=1e-12)


def test_shifted_positions_leave_attention_unchanged_and_rotation_matters():
    d = inputs.make_inputs(1, 60, seed=13, H_=2, with_weight=False)
    p0 = inputs.make_positions(1, 60)
    a, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                 d["softmax_scale"], p0, K2)
    b, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                 d["softmax_scale"], p0 + 70000, K2)
    np.testing.assert_allclose(a, b, rtol=1e-8, atol=1e-10)
    plain, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                d["softmax_scale"])
    assert np.abs(a - plain).max() > 1e-3   # the rotation does change the result


def test_rows_subset_and_default_positions():
    """Sampled rows equal the full result's rows; None positions mean 0..T-1."""
    d = inputs.make_inputs(2, 50, seed=14, H_=2, with_weight=False)
    full, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                    d["softmax_scale"], None, K2)
    rows = [(0, 0), (1, 49), (1, 7), (0, 33)]
    part, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                    d["softmax_scale"], inputs.make_positions(2, 50), K2,
                                    rows=rows)
    assert np.array_equal(part, full[[b * 50 + i for b, i in rows]])
