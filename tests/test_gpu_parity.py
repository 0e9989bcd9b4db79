"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element on every row; they span several
128-row / 128-key tiles and ragged tails. The five full-size workloads are
compared on sampled rows (the oracle evaluates any row on its own), launched
exactly as the benchmark launches them.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, assert_peaked, metrics, sample_rows, to_f64

pytestmark = pytest.mark.gpu


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def oracle_attn(d, rows=None):
    return oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], d["mask"],
                            d["softmax_scale"], rows=rows)


def gpu_attn(g, stream=None):
    return binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                mask=g["mask"], softmax_scale=g["softmax_scale"], stream=stream)


def gpu_full(g):
    return binding.attn_oproj(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"], g["W_o"],
                              mask=g["mask"], softmax_scale=g["softmax_scale"])


def check_status():
    st, word = binding.device_status()
    assert st == 0, f"device status {binding.STATUS.get(st, st)} word={word:#x}"


# ------------------------------------------------------------------ o_proj
@pytest.mark.parametrize("M", [1, 31, 32, 33, 64, 100, 128, 129, 300, 1000])
def test_oproj_all_rows(cuda_device, M):
    """mla_o_proj on every row. M <= 128 runs the small-M kernel (token tile
    of 32, 64 or 128, K split over a two-CTA cluster); larger M the tiled
    GEMM (M = 129: 128x128 tiles, 300: 128x224, 1000: 256x224)."""
    g = torch.Generator().manual_seed(M)
    attn = torch.randn(M, inputs.K_OPROJ, generator=g).to(torch.bfloat16)
    W = (torch.randn(inputs.D_MODEL, inputs.K_OPROJ, generator=g) * 0.02).to(torch.bfloat16)
    out = binding.o_proj(attn.to(cuda_device), W.to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref = oracle.oproj_rows(oracle.bf16_to_f64(attn), W)
    assert_parity(to_f64(out), ref, f"o_proj M={M}")


@pytest.mark.parametrize("M", [4096 + 77, 8192 + 77])
def test_oproj_large_sampled(cuda_device, M):
    """Ragged large M, sampled rows: 256x224 tiles whose last tile has an empty
    second row half (M = 4173), 128x256 tiles (M = 8269)."""
    g = torch.Generator().manual_seed(5)
    attn = torch.randn(M, inputs.K_OPROJ, generator=g).to(torch.bfloat16)
    W = (torch.randn(inputs.D_MODEL, inputs.K_OPROJ, generator=g) * 0.02).to(torch.bfloat16)
    out = binding.o_proj(attn.to(cuda_device), W.to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    rows = sorted(set([0, 1, 127, 128, 129, M - 1, M - 2, M - 78, M - 77]
                      + list(np.random.default_rng(0).integers(0, M, 100))))
    ref = oracle.oproj_rows(oracle.bf16_to_f64(attn[rows]), W)
    assert_parity(to_f64(out[rows]), ref, f"o_proj M={M} sampled")


# ------------------------------------------------------------------ attention
CAUSAL_SHAPES = [(1, 1), (1, 2), (2, 63), (1, 64), (1, 65), (1, 127), (1, 128), (2, 129),
                 (1, 255), (1, 257), (3, 300), (1, 512)]


@pytest.mark.parametrize("B,T", CAUSAL_SHAPES)
def test_attn_causal_all_rows(cuda_device, B, T):
    d = inputs.make_inputs(B, T, seed=T * 10 + B, with_weight=False)
    out = gpu_attn(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle_attn(d)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, f"attn causal B={B} T={T}")


@pytest.mark.parametrize("B,T,min_valid", [(3, 300, 1), (2, 256, 100), (2, 129, 1), (1, 64, 7)])
def test_attn_keypad_mask_all_rows(cuda_device, B, T, min_valid):
    d = inputs.make_inputs(B, T, seed=B * 1000 + T, key_padding=True, min_valid=min_valid,
                           with_weight=False)
    out = gpu_attn(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle_attn(d)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, f"attn keypad B={B} T={T}")


def test_attn_general_additive_mask_and_fully_masked_rows(cuda_device):
    """Finite non-zero mask values, -inf holes, a mask row stride larger than
    T, and rows with no allowed key (written as zeros)."""
    B, T, ld = 2, 200, 208
    d = inputs.make_inputs(B, T, seed=77, with_weight=False)
    g = torch.Generator().manual_seed(3)
    m = torch.randn(B, 1, T, ld, generator=g) * 2.0
    holes = torch.rand(B, 1, T, ld, generator=g) < 0.3
    m[holes] = float("-inf")
    m[0, 0, 5, :] = float("-inf")          # fully masked rows
    m[1, 0, 150, :] = float("-inf")
    m[1, 0, 0:128, 128:] = float("-inf")   # a whole tile skipped
    m[0, 0, 128:, 128:] = 0.0              # a whole all-zero tile
    mask = m.to(torch.bfloat16)
    d["mask"] = mask[..., :T]
    ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                               d["mask"].contiguous(), d["softmax_scale"])
    gd = to_dev(d, cuda_device)
    gd["mask"] = mask.to(cuda_device)[..., :T]  # strided view, row stride ld
    out = gpu_attn(gd)
    torch.cuda.synchronize()
    check_status()
    got = to_f64(out).reshape(B * T, -1)
    rows_fm = fm.any(axis=1)
    assert rows_fm[5] and rows_fm[T + 150]
    assert np.all(got[rows_fm] == 0.0)
    assert_parity(got[~rows_fm], ref[~rows_fm], "attn general mask")


@pytest.mark.parametrize("B,T", [(1, 256), (2, 300)])
def test_attn_explicit_causal_mask_is_the_causal_call(cuda_device, B, T):
    """An explicit [B,1,T,T] causal mask (0 where key <= query, -inf above)
    classifies into all-zero, causal-diagonal and skipped tiles, which take
    the fast softmax routes. On inputs whose row i points at keys i and i+1
    both the explicit and the implicit form give v_i within half a bf16 ulp
    on every row; on random inputs both match the oracle and each other. (On
    128-key tiles the two forms agree bit for bit:
    test_gpu_attn_kernels.py.)"""
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    m = torch.zeros(T, T)
    m[j > i] = float("-inf")
    mask = m.to(torch.bfloat16).expand(B, 1, T, T).contiguous()
    for peaked in (False, True):
        d = (inputs.make_peaked_inputs(B, T, seed=31 + T) if peaked
             else inputs.make_inputs(B, T, seed=31 + T, with_weight=False))
        d["mask"] = mask
        g = to_dev(d, cuda_device)
        explicit = to_f64(gpu_attn(g)).reshape(B * T, -1)
        g["mask"] = None
        implicit = to_f64(gpu_attn(g)).reshape(B * T, -1)
        torch.cuda.synchronize()
        check_status()
        ref, fm = oracle_attn(d)
        assert not fm.any()
        for name, got in (("explicit", explicit), ("implicit", implicit)):
            assert_parity(got, ref, f"{name} causal peaked={peaked}")
            if peaked:
                assert_peaked(got, ref, np.arange(B * T), f"{name} causal peaked")
        assert_parity(explicit, implicit, "explicit vs implicit causal")


def _prefix_mask(B, T, lens, causal):
    """0 where key j < lens[b] (and j <= query i when causal), -inf elsewhere."""
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    allowed = (j.unsqueeze(0) < torch.tensor(lens).view(-1, 1, 1)).expand(B, T, T)
    if causal:
        allowed = allowed & (j <= i).unsqueeze(0)
    m = torch.full(allowed.shape, float("-inf"))
    m.masked_fill_(allowed, 0.0)
    return m.to(torch.bfloat16).unsqueeze(1).contiguous()


def test_attn_prefix_mask_tiles_all_rows(cuda_device):
    """A non-causal key-padding mask: every row of a tile allows the same key
    prefix, so the tiles cut by the padding take the prefix route (above the
    diagonal too; batch 3's in the ragged last key tile). Rows of batch 0 get
    a staircase of per-row limits instead, which is no prefix and takes the
    mixed route."""
    B, T = 4, 300
    d = inputs.make_inputs(B, T, seed=123, with_weight=False)
    m = _prefix_mask(B, T, [300, 1, 150, 290], causal=False).float()
    for i in range(T):
        m[0, 0, i, 200 + i % 50:] = float("-inf")
    d["mask"] = m.to(torch.bfloat16)
    out = gpu_attn(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle_attn(d)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, "attn prefix mask")


@pytest.mark.parametrize("B,T,lens", [(3, 700, [700, 333, 129]), (2, 4096, [4096, 1937])])
def test_attn_keypad_dense_mask_matches_varlen(cuda_device, B, T, lens):
    """Causal attention with key padding, once as a dense mask and once as
    valid_len, on inputs whose row i points at keys i and i+1: rows t < len
    give v_t within half a bf16 ulp in both forms, and every row matches the
    oracle in both. At T = 4096 both forms run half tiles with the separate
    PV issuer. (On 128-key tiles the two forms agree bit for bit outside
    the query tile holding the last valid key: test_gpu_attn_kernels.py.)"""
    d = inputs.make_peaked_inputs(B, T, seed=5)
    d["mask"] = _prefix_mask(B, T, lens, causal=True)
    g = to_dev(d, cuda_device)
    dense = to_f64(gpu_attn(g)).reshape(B * T, -1)
    compact = to_f64(binding.attn_prefill_varlen(
        g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
        torch.tensor(lens, dtype=torch.int32, device=cuda_device),
        softmax_scale=g["softmax_scale"])).reshape(B * T, -1)
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle_attn(d)
    assert not fm.any()
    rows = np.array([b * T + t for b in range(B) for t in range(lens[b])])
    for name, got in (("dense", dense), ("valid_len", compact)):
        assert_parity(got, ref, f"keypad {name}")
        assert_peaked(got, ref, rows, f"keypad {name}")


@pytest.mark.parametrize("scale_mul", [-1.0, 0.0])
@pytest.mark.parametrize("form", ["causal", "causal_mask", "keypad_mask"])
def test_attn_non_positive_scale(cuda_device, scale_mul, form):
    """A negative or zero softmax scale takes the exact route on every tile,
    where the causal cut, the causal-pattern tiles and the prefix tiles of a
    mask are applied as explicit -inf entries."""
    B, T = 2, 300
    d = inputs.make_inputs(B, T, seed=41, with_weight=False)
    d["softmax_scale"] = d["softmax_scale"] * scale_mul
    if form == "causal_mask":
        d["mask"] = _prefix_mask(B, T, [T, T], causal=True)
    elif form == "keypad_mask":
        d["mask"] = _prefix_mask(B, T, [170, 300], causal=True)
    out = gpu_attn(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle_attn(d)
    assert not fm.any()
    assert_parity(to_f64(out).reshape(B * T, -1), ref, f"attn scale*{scale_mul} {form}")


def test_attn_causal_future_invariance(cuda_device):
    """Rows <= t are bit-identical after changing keys/values at positions > t."""
    B, T, t = 1, 300, 140
    d = inputs.make_inputs(B, T, seed=9, with_weight=False)
    a = gpu_attn(to_dev(d, cuda_device)).clone()
    d2 = dict(d)
    for k in ("k_nope", "k_pe", "v"):
        x = d[k].clone()
        x[:, :, t + 1:] = (x[:, :, t + 1:].float() * -3.0 + 1.0).to(torch.bfloat16)
        d2[k] = x
    b2 = gpu_attn(to_dev(d2, cuda_device))
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(a[:, : t + 1], b2[:, : t + 1])
    assert not torch.equal(a[:, t + 1:], b2[:, t + 1:])


def test_attn_on_side_stream(cuda_device):
    d = inputs.make_inputs(1, 200, seed=4, with_weight=False)
    s = torch.cuda.Stream()
    gd = to_dev(d, cuda_device)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out = gpu_attn(gd, stream=s)
    s.synchronize()
    ref, _ = oracle_attn(d)
    assert_parity(to_f64(out).reshape(200, -1), ref, "side stream")


# ------------------------------------------------------------------ whole path
def test_fused_small_all_rows(cuda_device):
    """B=1, T=64 causal (the small workload), every output element."""
    d = inputs.make_workload(inputs.WORKLOADS["b1_t64_causal"])
    out = gpu_full(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, fm = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                     None, d["softmax_scale"], d["W_o"])
    assert not fm.any()
    m = assert_parity(to_f64(out).reshape(64, -1), ref, "fused b1_t64")
    print(m)


def test_fused_ragged_all_rows(cuda_device):
    d = inputs.make_inputs(2, 200, seed=21)
    out = gpu_full(to_dev(d, cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref, _ = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                    None, d["softmax_scale"], d["W_o"])
    assert_parity(to_f64(out).reshape(400, -1), ref, "fused B=2 T=200")


FULL = ["b1_t4096_causal", "b16_t1024_causal", "b8_t4096_keypad_mask", "b1_t32768_causal_qx2"]


@pytest.mark.parametrize("name", FULL)
def test_fused_full_size_sampled_rows(cuda_device, name):
    w = inputs.WORKLOADS[name]
    d = inputs.make_workload(w)
    n_random = 300 if w.T >= 32768 else 600
    rows = sample_rows(w.B, w.T, n_random, seed=1, valid_len=d["valid_len"])
    gd = to_dev(d, cuda_device)
    out = gpu_full(gd)
    torch.cuda.synchronize()
    check_status()
    got = to_f64(out[[r[0] for r in rows], [r[1] for r in rows]])
    del gd, out
    ref, fm = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                     d["mask"], d["softmax_scale"], d["W_o"], rows=rows)
    assert not fm.any()
    m = assert_parity(got, ref, f"{name} ({len(rows)} rows)")
    print(name, len(rows), m)
