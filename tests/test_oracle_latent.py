"""Pins of the oracle's latent up-projection (k_nope and v from the
compressed KV latent) and of attention fed by it, on the CPU.

What the oracle follows: config.json on page "Kimi K2 · Block input"
(kv_lora_rank 512, num_attention_heads 64, qk_nope_head_dim 128, v_head_dim
128, attention_bias false) and the per-head k_nope / value_states the excerpt
of page "Kimi K2 · Mix and project" starts from; the reading (one bias-free
linear map per token, each head's rows holding its 128 key parts then its 128
values) is in oracle/mla_oracle.c, section "latent". The pins catch a
transposed weight, the key and value halves swapped, heads in the wrong
order, and the up-projection confused across tokens or batches.
"""
import numpy as np
import torch

import oracle
from mla_causal_attention_attn_b200 import inputs


def bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def test_one_hot_weight_places_heads_and_halves():
    """W row h*(Dn+Dv) + n picks latent element (5h + n) % R: the key part of
    head h must hold elements 5h .. 5h+Dn-1 and its value part the next Dv."""
    B, T, R, H, Dn, Dv = 2, 3, 16, 3, 4, 2
    x = torch.arange(B * T * R, dtype=torch.float32).reshape(B, T, R)  # exact in bf16
    W = np.zeros((H * (Dn + Dv), R))
    for h in range(H):
        for n in range(Dn + Dv):
            W[h * (Dn + Dv) + n, (5 * h + n) % R] = 1.0
    k, v = oracle.kv_up(bf16(x), bf16(W), H, Dn, Dv)
    xs = x.numpy()
    for b in range(B):
        for h in range(H):
            for t in range(T):
                idx = [(5 * h + n) % R for n in range(Dn + Dv)]
                assert np.array_equal(k[b, h, t], xs[b, t, idx[:Dn]])
                assert np.array_equal(v[b, h, t], xs[b, t, idx[Dn:]])


def test_kv_up_matches_float64_matmul():
    """Against numpy's float64 matmul of the widened operands, re-laid out."""
    d = inputs.make_latent_inputs(2, 5, seed=3, H_=4, Dn=6, Dv=3, R=24, with_weight=False)
    k, v = oracle.kv_up(d["c_kv"], d["W_kv_b"], 4, 6, 3)
    kv = oracle.bf16_to_f64(d["c_kv"]) @ oracle.bf16_to_f64(d["W_kv_b"]).T  # [B, T, H*9]
    kv = kv.reshape(2, 5, 4, 9).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(k, kv[..., :6], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(v, kv[..., 6:], rtol=1e-13, atol=1e-13)


def test_kv_up_is_linear_in_the_latent():
    g = torch.Generator().manual_seed(4)
    x = torch.randint(-8, 8, (1, 6, 32), generator=g).float()
    y = torch.randint(-8, 8, (1, 6, 32), generator=g).float()
    W = torch.randint(-4, 4, (2 * 10, 32), generator=g).float()
    kx, vx = oracle.kv_up(bf16(x), bf16(W), 2, 6, 4)
    ky, vy = oracle.kv_up(bf16(y), bf16(W), 2, 6, 4)
    ks, vs = oracle.kv_up(bf16(3 * x + y), bf16(W), 2, 6, 4)
    assert np.array_equal(ks, 3 * kx + ky) and np.array_equal(vs, 3 * vx + vy)  # small integers


def test_attention_on_exact_kv_equals_attention_on_the_same_bf16_values():
    """When the up-projection's results are bf16 values (integer operands),
    attention fed the float64 arrays equals attention fed the same values as
    bf16 tensors, bit for bit."""
    g = torch.Generator().manual_seed(5)
    B, T, R, H = 1, 37, 8, 2
    d = inputs.make_inputs(B, T, seed=6, H_=H, with_weight=False)
    x = torch.randint(-3, 4, (B, T, R), generator=g).float()
    W = torch.randint(-2, 3, (H * 256, R), generator=g).float()
    k, v = oracle.kv_up(bf16(x), bf16(W), H, 128, 128)
    got, _ = oracle.attn_rows_kv64(d["q_nope"], d["q_pe"], k, d["k_pe"], v, None,
                                   d["softmax_scale"])
    want, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], bf16(k), d["k_pe"], bf16(v), None,
                               d["softmax_scale"])
    assert np.array_equal(got, want)


def test_latent_path_numpy_brute_force():
    """The whole latent path on tiny shapes against a numpy restatement."""
    d = inputs.make_latent_inputs(1, 6, seed=8, H_=2, Dn=4, Dr=2, Dv=3, R=5, D=7)
    f = oracle.bf16_to_f64
    kv = (f(d["c_kv"])[0] @ f(d["W_kv_b"]).T).reshape(6, 2, 7)
    qn, qp, kp, W_o = f(d["q_nope"])[0], f(d["q_pe"])[0], f(d["k_pe"])[0, 0], f(d["W_o"])
    attn = np.zeros((6, 2 * 3))
    for h in range(2):
        Q = np.concatenate([qn[h], qp[h]], axis=1)
        K = np.concatenate([kv[:, h, :4], kp], axis=1)
        s = Q @ K.T * float(np.float32(d["softmax_scale"]))
        s[np.triu_indices(6, 1)] = -np.inf
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        attn[:, 3 * h:3 * h + 3] = p @ kv[:, h, 4:]
    got, fm = oracle.attn_oproj_rows_latent(d["q_nope"], d["q_pe"], d["c_kv"], d["W_kv_b"],
                                            d["k_pe"], None, d["softmax_scale"], d["W_o"])
    assert not fm.any()
    np.testing.assert_allclose(got, attn @ W_o.T, rtol=1e-12, atol=1e-13)
