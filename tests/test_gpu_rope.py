"""GPU parity of the rotary calls (mla_attn_prefill_rope, mla_attn_oproj_rope)
against the fp64 oracle, through the C ABI.

The inputs' q_pe and k_pe are unrotated; the library rotates them (YaRN, the
rotary step of page "Kimi K2 · Mix and project", excerpt
modeling_deepseek.py 799-840, with config.json's rope_scaling from page
"Kimi K2 · Block input") and the oracle does the same in fp64. Positions
cover 0..T-1, per-sequence offsets and unstructured random values.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, sample_rows, to_f64

pytestmark = pytest.mark.gpu

K2 = inputs.KIMI_K2_ROPE
RAMPED = dict(K2, rope_theta=10000.0, factor=40.0, beta_fast=32.0, mscale=2.0)


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def gpu_rope(g, pos, rope, mask=None, ws=None, stream=None):
    return binding.attn_prefill_rope(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                     position_ids=pos, rope=rope, mask=mask,
                                     softmax_scale=g["softmax_scale"], workspace=ws,
                                     stream=stream)


def check_ws(ws):
    st, word = binding.last_device_status(ws)
    assert st == 0, f"status {binding.STATUS.get(st, st)} word={word:#x}"


@pytest.mark.parametrize("B,T,kind", [(1, 1, "arange"), (1, 65, "random"), (2, 129, "offset"),
                                      (1, 300, "arange"), (3, 257, "random"),
                                      (2, 512, "offset")])
def test_rope_causal_all_rows(cuda_device, B, T, kind):
    d = inputs.make_inputs(B, T, seed=700 + T + B, with_weight=False)
    pos = inputs.make_positions(B, T, kind, seed=T)
    g = to_dev(d, cuda_device)
    ws = torch.empty(binding.attn_prefill_rope_workspace_bytes(B, T, False), dtype=torch.uint8,
                     device=cuda_device)
    out = gpu_rope(g, pos.to(cuda_device), K2, ws=ws)
    torch.cuda.synchronize()
    check_ws(ws)
    ref, fm = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                    d["softmax_scale"], pos, K2)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, f"rope causal B={B} T={T} {kind}")


def test_rope_default_positions_and_ramped_parameters(cuda_device):
    """position_ids None (0..T-1), and a parameter set with a wide ramp and
    an attention factor of 1.257 (the values flow through, not the defaults)."""
    B, T = 2, 300
    d = inputs.make_inputs(B, T, seed=71, with_weight=False)
    g = to_dev(d, cuda_device)
    for r in (K2, RAMPED):
        out = gpu_rope(g, None, r)
        torch.cuda.synchronize()
        ref, _ = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                       None, d["softmax_scale"], None, r)
        assert_parity(to_f64(out).reshape(B * T, -1), ref, f"rope defaults {r['rope_theta']}")


def test_rope_with_keypad_mask_all_rows(cuda_device):
    B, T = 2, 300
    d = inputs.make_inputs(B, T, seed=72, key_padding=True, min_valid=50, with_weight=False)
    pos = inputs.make_positions(B, T, "offset")
    g = to_dev(d, cuda_device)
    out = gpu_rope(g, pos.to(cuda_device), K2, mask=g["mask"])
    torch.cuda.synchronize()
    ref, fm = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                    d["mask"], d["softmax_scale"], pos, K2)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, "rope keypad mask")


@pytest.mark.parametrize("masked", [False, True])
def test_rope_zero_positions_is_the_plain_call(cuda_device, masked):
    """At position 0 cos = 1 and sin = 0 exactly, so the rotation is the
    identity and the rotary call gives the plain call's result bit for bit."""
    B, T = 2, 300
    d = inputs.make_inputs(B, T, seed=73, key_padding=masked, min_valid=100, with_weight=False)
    g = to_dev(d, cuda_device)
    zero = torch.zeros(B, T, dtype=torch.int32, device=cuda_device)
    a = gpu_rope(g, zero, K2, mask=g["mask"])
    b = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                             mask=g["mask"], softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_rope_fused_small_all_rows(cuda_device):
    """The whole path with rotation: B=1, T=64 (small-M o_proj), every element."""
    d = inputs.make_workload(inputs.WORKLOADS["b1_t64_causal"])
    pos = inputs.make_positions(1, 64, "random", seed=9)
    g = to_dev(d, cuda_device)
    ws = torch.empty(binding.attn_oproj_rope_workspace_bytes(1, 64, False), dtype=torch.uint8,
                     device=cuda_device)
    out = binding.attn_oproj_rope(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                  g["W_o"], position_ids=pos.to(cuda_device), rope=K2,
                                  softmax_scale=g["softmax_scale"], workspace=ws)
    torch.cuda.synchronize()
    check_ws(ws)
    ref, fm = oracle.attn_oproj_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"],
                                          d["v"], None, d["softmax_scale"], pos, K2, d["W_o"])
    assert not fm.any()
    assert_parity(to_f64(out).reshape(64, -1), ref, "rope fused b1_t64")


@pytest.mark.parametrize("name", ["b1_t4096_causal", "b1_t32768_causal_qx2"])
def test_rope_fused_full_size_sampled_rows(cuda_device, name):
    """Full-size workloads with positions 0..T-1 (past the original 4096
    context at T = 32768, where the interpolated pairs matter), sampled rows."""
    w = inputs.WORKLOADS[name]
    d = inputs.make_workload(w)
    rows = sample_rows(w.B, w.T, 300, seed=2)
    g = to_dev(d, cuda_device)
    out = binding.attn_oproj_rope(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                  g["W_o"], position_ids=None, rope=K2,
                                  softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    got = to_f64(out[[r[0] for r in rows], [r[1] for r in rows]])
    del g, out
    ref, fm = oracle.attn_oproj_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"],
                                          d["v"], None, d["softmax_scale"], None, K2, d["W_o"],
                                          rows=rows)
    assert not fm.any()
    m = assert_parity(got, ref, f"rope {name} ({len(rows)} rows)")
    print(name, len(rows), m)
