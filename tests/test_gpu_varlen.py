"""GPU parity of the compact key-padding form (mla_attn_prefill_varlen,
mla_attn_oproj_varlen) against the fp64 oracle.

The oracle is given the equivalent dense additive mask (0 where key j <= query
i and j < valid_len[b], -inf elsewhere), built from the same clamped lengths;
rows with no allowed key must come back as zeros.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, assert_peaked, sample_rows, to_f64

pytestmark = pytest.mark.gpu


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def check_status():
    st, word = binding.device_status()
    assert st == 0, f"device status {binding.STATUS.get(st, st)} word={word:#x}"


def gpu_varlen(g, vl_dev):
    return binding.attn_prefill_varlen(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                       vl_dev, softmax_scale=g["softmax_scale"])


@pytest.mark.parametrize("B,T,lens", [
    (3, 300, [300, 1, 150]),        # full, one key, ragged
    (2, 256, [128, 129]),           # tile boundary and one past it
    (2, 129, [1, 129]),
    (4, 200, [0, 200, 64, 5000]),   # no key at all, full, one tile, clamped from above
    (1, 64, [-3]),                  # clamped from below: no key
])
def test_varlen_all_rows(cuda_device, B, T, lens):
    d = inputs.make_inputs(B, T, seed=B * 100 + T, with_weight=False)
    vl = torch.tensor(lens, dtype=torch.int32)
    clamped = vl.clamp(0, T).to(torch.int64)
    mask = inputs.keypad_mask(clamped, T)
    ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], mask,
                               d["softmax_scale"])
    out = gpu_varlen(to_dev(d, cuda_device), vl.to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    got = to_f64(out).reshape(B * T, -1)
    rows_fm = fm.any(axis=1)
    # rows of sequences with no valid key, and only those, are fully masked
    expect_fm = np.repeat((clamped == 0).numpy(), T)
    assert np.array_equal(rows_fm, expect_fm)
    assert np.all(got[rows_fm] == 0.0)
    if (~rows_fm).any():
        assert_parity(got[~rows_fm], ref[~rows_fm], f"varlen B={B} T={T} lens={lens}")


def test_varlen_full_length_is_the_causal_kernel(cuda_device):
    """valid_len = T everywhere is plain causal attention, bit for bit."""
    B, T = 2, 333
    d = inputs.make_inputs(B, T, seed=9, with_weight=False)
    g = to_dev(d, cuda_device)
    a = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                             softmax_scale=g["softmax_scale"])
    b = gpu_varlen(g, torch.full((B,), T, dtype=torch.int32, device=cuda_device))
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(a, b)


def test_varlen_agrees_with_dense_mask_path(cuda_device):
    """The compact and the dense form of the same padding give the same
    attention (both within the tolerance of the oracle, and of each other)."""
    B, T = 3, 400
    d = inputs.make_inputs(B, T, seed=17, key_padding=True, min_valid=1, with_weight=False)
    g = to_dev(d, cuda_device)
    dense = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                 mask=g["mask"], softmax_scale=g["softmax_scale"])
    compact = gpu_varlen(g, d["valid_len"].to(torch.int32).to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], d["mask"],
                               d["softmax_scale"])
    assert not fm.any()
    assert_parity(to_f64(compact).reshape(B * T, -1), ref, "varlen vs oracle")
    assert_parity(to_f64(compact).reshape(B * T, -1), to_f64(dense).reshape(B * T, -1),
                  "varlen vs dense mask")


def test_varlen_fused_full_size_sampled_rows(cuda_device):
    """B=8, T=4096 with key padding (lengths drawn in [512, 4096]) through
    mla_attn_oproj_varlen, as the benchmark's compact-mask workload runs it."""
    w = inputs.WORKLOADS["b8_t4096_keypad_mask"]
    d = inputs.make_workload(w)
    rows = sample_rows(w.B, w.T, 600, seed=2, valid_len=d["valid_len"])
    g = to_dev(d, cuda_device)
    out = binding.attn_oproj_varlen(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                    d["valid_len"].to(torch.int32).to(cuda_device), g["W_o"],
                                    softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    check_status()
    got = to_f64(out[[r[0] for r in rows], [r[1] for r in rows]])
    del g, out
    ref, fm = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                     d["mask"], d["softmax_scale"], d["W_o"], rows=rows)
    assert not fm.any()
    m = assert_parity(got, ref, f"varlen fused b8_t4096 ({len(rows)} rows)")
    print(m)


@pytest.mark.parametrize("B,T,lens", [
    (6, 320, [63, 64, 65, 127, 128, 129]),   # key limits on both sides of 64-key halves
    (4, 191, [191, 190, 192, 1]),            # ragged T inside a second half tile
    (3, 257, [257, 193, 2]),                 # one row past two full tiles
])
def test_varlen_half_tile_boundaries_peaked(cuda_device, B, T, lens):
    """Causal attention scores 64 keys at a time. On inputs whose query row i
    points at keys i and i+1, every row t < len(b) has the answer v_t,
    checked element by element within half a bf16 ulp, so a key limit that
    is off by one at a 64-key boundary, a ragged tail or the diagonal fails
    here. Rows t >= len(b) match the oracle under the path's tolerance."""
    d = inputs.make_peaked_inputs(B, T, seed=B * 31 + T)
    vl = torch.tensor(lens, dtype=torch.int32)
    clamped = vl.clamp(0, T).to(torch.int64)
    mask = inputs.keypad_mask(clamped, T)
    ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], mask,
                               d["softmax_scale"])
    assert not fm.any()
    g = to_dev(d, cuda_device)
    out = gpu_varlen(g, vl.to(cuda_device))
    causal = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                  softmax_scale=g["softmax_scale"])
    torch.cuda.synchronize()
    check_status()
    got = to_f64(out).reshape(B * T, -1)
    assert_parity(got, ref, f"varlen peaked B={B} T={T}")
    rows = np.array([b * T + t for b in range(B) for t in range(int(clamped[b]))])
    assert_peaked(got, ref, rows, f"varlen peaked B={B} T={T}")
    # plain causal on the same inputs: every row has one answer
    ref_c, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                d["softmax_scale"])
    got_c = to_f64(causal).reshape(B * T, -1)
    assert_peaked(got_c, ref_c, np.arange(B * T), f"causal peaked B={B} T={T}")
