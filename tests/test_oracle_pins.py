"""Pins for the fp64 oracle, CPU only.

The pages ("Kimi K2 · Mix and project", code excerpts modeling_deepseek.py
799-840 and 848-852) print the definition but no worked values, so the oracle
is pinned by: hand-worked tiny cases (tests/golden/tiny_cases.json), closed
forms (T=1, equal scores, a one-hot mask, a dominant score), invariants
(probability rows sum to one, causality, shift and key-permutation
invariance, which heads a change reaches) and a library matmul for o_proj.
Each case names the mistake it is there to catch.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def small(B=1, H=2, T=9, Dn=8, Dr=4, Dv=8, seed=1, key_padding=False, q_scale=1.0):
    d = inputs.make_inputs(B, T, H_=H, Dn=Dn, Dr=Dr, Dv=Dv, D=12, seed=seed,
                           key_padding=key_padding, min_valid=1, q_scale=q_scale)
    return d


def run_attn(d, mask="default", scale=None, rows=None, want_probs=False):
    m = d["mask"] if mask == "default" else mask
    s = d["softmax_scale"] if scale is None else scale
    return oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                            m, s, rows=rows, want_probs=want_probs)


def _mask_from_json(m):
    def conv(x):
        return float("-inf") if x == "-inf" else float(x)
    return bf16(np.vectorize(conv, otypes=[np.float64])(np.array(m, dtype=object)))


# ---------------------------------------------------------------- golden cases
with open(os.path.join(HERE, "golden", "tiny_cases.json")) as f:
    GOLDEN = json.load(f)["cases"]


@pytest.mark.parametrize("case", GOLDEN, ids=[c["name"] for c in GOLDEN])
def test_golden_tiny_cases(case):
    """Hand-worked cases: catch a missing scale, a dropped rotary term, a
    per-head instead of shared rotary key, a mask that is scaled or gets an
    extra causal term, a wrong head-merge order and a transposed W_o."""
    t = {k: bf16(case[k]) for k in ("q_nope", "q_pe", "k_nope", "k_pe", "v")}
    for k in t:
        assert torch.equal(t[k].float(), torch.tensor(case[k], dtype=torch.float32)), k
    mask = _mask_from_json(case["mask"]) if case["mask"] is not None else None
    W = bf16(case["W_o"])
    attn, fm, probs = oracle.attn_rows(t["q_nope"], t["q_pe"], t["k_nope"], t["k_pe"],
                                       t["v"], mask, case["softmax_scale"],
                                       want_probs=True)
    np.testing.assert_allclose(attn, np.array(case["expected_attn"]), rtol=1e-14, atol=1e-14)
    if "expected_probs" in case:
        np.testing.assert_allclose(probs, np.array(case["expected_probs"]), rtol=1e-14,
                                   atol=1e-15)
    if "expected_fully_masked" in case:
        assert fm.tolist() == case["expected_fully_masked"]
    else:
        assert not fm.any()
    out = oracle.oproj_rows(attn, W)
    np.testing.assert_allclose(out, np.array(case["expected_out"]), rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- invariants
def test_probability_rows_sum_to_one_and_causal_zeros():
    """Softmax normalisation over the key axis; causal rows put no weight on
    later keys (catches softmax over the wrong axis, a missing max shift)."""
    d = small(B=2, H=3, T=11, q_scale=3.0)
    _, fm, probs = run_attn(d, want_probs=True)
    assert not fm.any()
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=0, atol=1e-12)
    T = 11
    rows_i = np.tile(np.arange(T), 2)
    for r, i in enumerate(rows_i):
        assert np.all(probs[r, :, i + 1:] == 0.0)
        assert np.all(probs[r, :, : i + 1] > 0.0)


def test_mask_rows_sum_to_one():
    d = small(B=3, H=2, T=13, key_padding=True)
    _, fm, probs = run_attn(d, want_probs=True)
    assert not fm.any()
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=0, atol=1e-12)
    m = d["mask"].float().numpy()[:, 0]  # [B,T,T]
    allowed = np.isfinite(m).reshape(3 * 13, 1, 13)
    assert np.all(probs[~np.broadcast_to(allowed, probs.shape)] == 0.0)


@pytest.mark.parametrize("which", ["k_nope", "k_pe", "v"])
def test_causality_later_positions_do_not_matter(which):
    """Row t is bit-identical after perturbing keys or values at positions > t
    (catches a causal mask off by one or applied to the wrong axis)."""
    d = small(B=1, H=2, T=12)
    t = 6
    base, _ = run_attn(d)
    d2 = dict(d)
    x = d[which].clone()
    g = torch.Generator().manual_seed(5)
    x[:, :, t + 1:, :] = torch.randn(x[:, :, t + 1:, :].shape, generator=g).to(torch.bfloat16) * 4
    d2[which] = x
    pert, _ = run_attn(d2)
    T = 12
    assert np.array_equal(base[: t + 1], pert[: t + 1])
    assert not np.array_equal(base[t + 1:], pert[t + 1:])
    assert T == base.shape[0]


def test_T1_closed_form_is_V0_times_Wo():
    """T = 1: one allowed key, p = 1, so out = V_0 . W_o^T for any q, k, scale
    (catches a wrong head-merge order or a transposed W_o)."""
    d = inputs.make_inputs(2, 1, seed=3, q_scale=7.0)
    attn, fm = run_attn(d, scale=3.0)
    assert not fm.any()
    v0 = oracle.bf16_to_f64(d["v"])[:, :, 0, :].reshape(2, -1)  # [B, H*Dv], column h*Dv+e
    assert np.array_equal(attn, v0)
    out = oracle.oproj_rows(attn, d["W_o"])
    W = oracle.bf16_to_f64(d["W_o"])
    np.testing.assert_allclose(out, v0 @ W.T, rtol=1e-12, atol=1e-12)
    assert out.shape == (2, inputs.D_MODEL)


@pytest.mark.parametrize("how", ["q_zero", "scale_zero"])
def test_equal_scores_give_prefix_mean(how):
    """All scores equal (q = 0, or softmax_scale = 0): attn[t] is the running
    mean of v[0..t] (closed form)."""
    d = small(B=2, H=3, T=10)
    if how == "q_zero":
        d["q_nope"] = torch.zeros_like(d["q_nope"])
        d["q_pe"] = torch.zeros_like(d["q_pe"])
        attn, _ = run_attn(d)
    else:
        attn, _ = run_attn(d, scale=0.0)
    v = oracle.bf16_to_f64(d["v"])  # [B,H,T,Dv]
    pm = np.cumsum(v, axis=2) / np.arange(1, 11).reshape(1, 1, 10, 1)
    expect = pm.transpose(0, 2, 1, 3).reshape(2 * 10, -1)
    np.testing.assert_allclose(attn, expect, rtol=1e-13, atol=1e-13)


def test_one_hot_mask_selects_one_value_row():
    """A mask with a single finite entry per row puts all weight on that key,
    so attn equals that value row exactly (catches a softmax over queries or
    a mask indexed [j, i])."""
    B, H, T = 2, 2, 7
    d = small(B=B, H=H, T=T)
    g = torch.Generator().manual_seed(9)
    pick = torch.randint(0, T, (B, T), generator=g)
    m = torch.full((B, 1, T, T), float("-inf"))
    for b in range(B):
        for i in range(T):
            m[b, 0, i, pick[b, i]] = 0.0
    attn, fm = run_attn(d, mask=m.to(torch.bfloat16))
    assert not fm.any()
    v = oracle.bf16_to_f64(d["v"])
    for b in range(B):
        for i in range(T):
            expect = v[b, :, pick[b, i], :].reshape(-1)
            assert np.array_equal(attn[b * T + i], expect)


def test_dominant_score_limit():
    """Huge q: each row's softmax collapses onto its largest allowed score,
    with no overflow (catches a missing max subtraction)."""
    d = small(B=1, H=2, T=8, q_scale=64.0)
    attn, _, probs = run_attn(d, want_probs=True)
    assert np.all(np.isfinite(attn))
    v = oracle.bf16_to_f64(d["v"])
    for i in range(8):
        for h in range(2):
            j = int(np.argmax(probs[i, h]))
            if probs[i, h, j] > 1 - 1e-12:
                np.testing.assert_allclose(attn[i, h * 8:(h + 1) * 8], v[0, h, j], atol=1e-9)


def test_mask_row_shift_invariance():
    """Adding one constant to every entry of a mask row leaves the row's
    softmax unchanged (catches a mask that is scaled with the scores)."""
    B, H, T = 1, 2, 6
    d = small(B=B, H=H, T=T)
    g = torch.Generator().manual_seed(4)
    m = (torch.randn(B, 1, T, T, generator=g)).to(torch.bfloat16)
    a1, _ = run_attn(d, mask=m)
    m2 = (m.float() + 2.0).to(torch.bfloat16)
    # the +2 shift is exact in bf16 only where no rounding happens; compare on
    # the values the mask really holds
    same = torch.equal((m2.float() - 2.0), m.float())
    a2, _ = run_attn(d, mask=m2)
    if same:
        np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-12)
    m3 = torch.zeros_like(m)
    a3, _ = run_attn(d, mask=m3)
    m4 = torch.full_like(m, 5.0)
    a4, _ = run_attn(d, mask=m4)
    np.testing.assert_allclose(a3, a4, rtol=1e-12, atol=1e-12)


def test_key_permutation_invariance_under_full_mask():
    """With an all-zero mask (every key allowed) permuting the key positions of
    k_nope, the shared k_pe and v together leaves every row unchanged
    (catches the shared rotary key read at the wrong position)."""
    B, H, T = 1, 3, 9
    d = small(B=B, H=H, T=T)
    m = torch.zeros(B, 1, T, T, dtype=torch.bfloat16)
    a1, _ = run_attn(d, mask=m)
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(2))
    d2 = dict(d)
    for k in ("k_nope", "k_pe", "v"):
        d2[k] = d[k][:, :, perm, :].contiguous()
    a2, _ = run_attn(d2, mask=m)
    np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-12)


def test_which_heads_a_change_reaches():
    """Changing k_nope of one head moves only that head's 128-column block;
    changing the shared k_pe moves every head (catches per-head rotary keys
    or a head-merge stride error)."""
    B, H, T, Dv = 1, 3, 6, 8
    d = small(B=B, H=H, T=T, Dv=Dv)
    base, _ = run_attn(d)
    d2 = dict(d)
    x = d["k_nope"].clone()
    x[:, 1] = (x[:, 1].float() * -1.5).to(torch.bfloat16)
    d2["k_nope"] = x
    a2, _ = run_attn(d2)
    diff = np.abs(a2 - base).reshape(T, H, Dv).max(axis=(0, 2))
    assert diff[0] == 0 and diff[2] == 0 and diff[1] > 0
    d3 = dict(d)
    d3["k_pe"] = (d["k_pe"].float() * -2.0).to(torch.bfloat16)
    a3, _ = run_attn(d3)
    diff = np.abs(a3 - base).reshape(T, H, Dv).max(axis=(0, 2))
    assert np.all(diff > 0)


def test_sampled_rows_equal_full_rows():
    """Evaluating a subset of rows gives exactly the rows of the full call."""
    d = small(B=2, H=2, T=10, key_padding=True)
    full, _ = run_attn(d)
    rows = [(1, 9), (0, 0), (1, 3), (0, 7)]
    part, _ = run_attn(d, rows=rows)
    for r, (b, i) in enumerate(rows):
        assert np.array_equal(part[r], full[b * 10 + i])


def test_brute_force_small_random_against_matrix_form():
    """T <= 8, random: the oracle's loops agree with the matrix form
    softmax(Q K^T * scale + M) V built from numpy matmul and exp."""
    for seed, kp in ((11, False), (12, True)):
        B, H, T, Dn, Dr, Dv = 2, 2, 8, 5, 3, 4
        d = small(B=B, H=H, T=T, Dn=Dn, Dr=Dr, Dv=Dv, seed=seed, key_padding=kp)
        attn, _ = run_attn(d)
        f = oracle.bf16_to_f64
        Q = np.concatenate([f(d["q_nope"]), f(d["q_pe"])], axis=-1)
        Kpe = np.broadcast_to(f(d["k_pe"]), (B, H, T, Dr))
        K = np.concatenate([f(d["k_nope"]), Kpe], axis=-1)
        scale = float(np.float32(d["softmax_scale"]))
        S = (Q @ K.transpose(0, 1, 3, 2)) * scale
        if d["mask"] is not None:
            S = S + f(d["mask"])
        else:
            S = S + np.where(np.tril(np.ones((T, T))) > 0, 0.0, -np.inf)
        S = S - S.max(-1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(-1, keepdims=True)
        O = P @ f(d["v"])
        expect = O.transpose(0, 2, 1, 3).reshape(B * T, H * Dv)
        np.testing.assert_allclose(attn, expect, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- o_proj
def test_oproj_matches_library_matmul_nonsquare():
    """o_proj = attn . W_o^T with W_o [N, K], N != K (catches a transposed W)."""
    g = torch.Generator().manual_seed(0)
    a = torch.randn(5, 24, generator=g, dtype=torch.float64).numpy()
    W = (torch.randn(40, 24, generator=g) * 0.02).to(torch.bfloat16)
    out = oracle.oproj_rows(a, W)
    np.testing.assert_allclose(out, a @ oracle.bf16_to_f64(W).T, rtol=1e-12, atol=1e-14)


def test_oproj_one_hot_rows_select_columns():
    K, N = 16, 7
    a = np.arange(3 * K, dtype=np.float64).reshape(3, K)
    cols = [3, 0, 15, 8, 8, 1, 2]
    W = torch.zeros(N, K)
    for n, c in enumerate(cols):
        W[n, c] = 1.0
    out = oracle.oproj_rows(a, W.to(torch.bfloat16))
    assert np.array_equal(out, a[:, cols])


def test_weight_shape_matches_printed_parameter_count():
    """The page's parameter table gives o_proj 58,720,256 weights = 8,192 x 7,168."""
    d = inputs.make_inputs(1, 1, seed=0)
    assert tuple(d["W_o"].shape) == (7168, 8192)
    assert d["W_o"].numel() == 58_720_256
    assert inputs.H * inputs.DV == 8192
    assert math.isclose(inputs.DEFAULT_SCALE, 1 / math.sqrt(192))


def test_full_path_rows():
    d = inputs.make_inputs(1, 3, seed=0)
    out, fm = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"],
                                     d["v"], None, d["softmax_scale"], d["W_o"],
                                     rows=[(0, 0), (0, 2)])
    assert out.shape == (2, 7168) and not fm.any()
    attn, _ = run_attn(d, rows=[(0, 0), (0, 2)])
    np.testing.assert_allclose(out, attn @ oracle.bf16_to_f64(d["W_o"]).T, rtol=1e-10,
                               atol=1e-12)
