"""GPU parity of the latent up-projection (mla_kv_up_proj) and of the whole
path from the latent (mla_attn_oproj_latent) against the fp64 oracle,
through the C ABI.

The oracle computes k_nope and v exactly (fp64) from the latent and feeds
them to attention unrounded; the library rounds them once to bf16 for the
attention kernel, as the model's bf16 linear layer does (config.json on page
"Kimi K2 · Block input": kv_lora_rank 512; reading in oracle/mla_oracle.c,
section "latent").
"""
import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, sample_rows, to_f64

pytestmark = pytest.mark.gpu


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


@pytest.mark.parametrize("B,T", [(1, 1), (1, 127), (2, 129), (3, 300), (1, 1000)])
def test_kv_up_all_elements(cuda_device, B, T):
    """Every element of k_nope and v; T spans one to several 128-row tiles,
    ragged tails, and token rows that cross from one sequence to the next
    inside a tile (B > 1)."""
    d = inputs.make_latent_inputs(B, T, seed=900 + T, with_weight=False)
    g = to_dev(d, cuda_device)
    k, v = binding.kv_up_proj(g["c_kv"], g["W_kv_b"])
    torch.cuda.synchronize()
    st, word = binding.device_status()
    assert st == 0, f"status {st} {word:#x}"
    rk, rv = oracle.kv_up(d["c_kv"], d["W_kv_b"], 64, 128, 128)
    assert_parity(to_f64(k).reshape(-1, 128), rk.reshape(-1, 128), f"kv_up k_nope B={B} T={T}")
    assert_parity(to_f64(v).reshape(-1, 128), rv.reshape(-1, 128), f"kv_up v B={B} T={T}")


def test_kv_up_full_size_sampled_heads(cuda_device):
    """B=1, T=4096 (32 x 64 output tiles, several waves of the persistent
    grid): every token of four heads at both ends and the middle."""
    d = inputs.make_latent_inputs(1, 4096, seed=901, with_weight=False)
    g = to_dev(d, cuda_device)
    k, v = binding.kv_up_proj(g["c_kv"], g["W_kv_b"])
    torch.cuda.synchronize()
    heads = [0, 1, 31, 63]
    rows = np.concatenate([np.arange(h * 256, h * 256 + 256) for h in heads])
    rk, rv = oracle.kv_up(d["c_kv"], d["W_kv_b"][rows], 4, 128, 128)
    assert_parity(to_f64(k[:, heads]).reshape(-1, 128), rk.reshape(-1, 128), "kv_up 4096 k")
    assert_parity(to_f64(v[:, heads]).reshape(-1, 128), rv.reshape(-1, 128), "kv_up 4096 v")


@pytest.mark.parametrize("B,T,masked", [(1, 64, False), (2, 300, False), (2, 300, True)])
def test_latent_path_all_rows(cuda_device, B, T, masked):
    d = inputs.make_latent_inputs(B, T, seed=910 + T, key_padding=masked, min_valid=60)
    g = to_dev(d, cuda_device)
    ws = torch.empty(binding.attn_oproj_latent_workspace_bytes(B, T, masked), dtype=torch.uint8,
                     device=cuda_device)
    out = binding.attn_oproj_latent(g["q_nope"], g["q_pe"], g["c_kv"], g["k_pe"], g["W_kv_b"],
                                    g["W_o"], mask=g["mask"], softmax_scale=g["softmax_scale"],
                                    workspace=ws)
    torch.cuda.synchronize()
    st, word = binding.last_device_status(ws)
    assert st == 0, f"status {st} {word:#x}"
    ref, fm = oracle.attn_oproj_rows_latent(d["q_nope"], d["q_pe"], d["c_kv"], d["W_kv_b"],
                                            d["k_pe"], d["mask"], d["softmax_scale"], d["W_o"])
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, f"latent path B={B} T={T} mask={masked}")


def test_latent_path_is_the_composition(cuda_device):
    """The fused call equals mla_kv_up_proj followed by mla_attn_oproj, bit
    for bit (same kernels, same bf16 k_nope and v)."""
    d = inputs.make_latent_inputs(1, 700, seed=920)
    g = to_dev(d, cuda_device)
    fused = binding.attn_oproj_latent(g["q_nope"], g["q_pe"], g["c_kv"], g["k_pe"], g["W_kv_b"],
                                      g["W_o"], softmax_scale=g["softmax_scale"])
    k, v = binding.kv_up_proj(g["c_kv"], g["W_kv_b"])
    comp = binding.attn_oproj(g["q_nope"], g["q_pe"], k, g["k_pe"], v, g["W_o"],
                              softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    assert torch.equal(fused, comp)


def test_latent_path_full_size_sampled_rows(cuda_device):
    """B=1, T=4096 from the latent, sampled rows."""
    d = inputs.make_latent_inputs(1, 4096, seed=930)
    rows = sample_rows(1, 4096, 200, seed=3)
    g = to_dev(d, cuda_device)
    out = binding.attn_oproj_latent(g["q_nope"], g["q_pe"], g["c_kv"], g["k_pe"], g["W_kv_b"],
                                    g["W_o"], softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    got = to_f64(out[0, [r[1] for r in rows]])
    del g, out
    ref, fm = oracle.attn_oproj_rows_latent(d["q_nope"], d["q_pe"], d["c_kv"], d["W_kv_b"],
                                            d["k_pe"], None, d["softmax_scale"], d["W_o"],
                                            rows=rows)
    assert not fm.any()
    m = assert_parity(got, ref, f"latent b1_t4096 ({len(rows)} rows)")
    print(m)
