"""GPU parity of the FP8 o_proj calls (mla_quantize_act_fp8,
mla_quantize_weight_fp8, mla_o_proj_fp8, mla_attn_oproj_fp8) against the
oracle's e4m3 quantisers and block-scaled product.

The quantisers decide integers (codes) and their scales in fp32 on both
sides, so they are compared bit for bit. The GEMM is given the oracle's codes
and scales (computed on the CPU from the same bf16 inputs) and compared with
the oracle's fp64 product under the path's tolerance, plus a tighter bound
on the relative Frobenius error (the kernel's only rounding of note is the
final bf16 store).
"""
import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, metrics, to_f64

pytestmark = pytest.mark.gpu

K, N = inputs.K_OPROJ, inputs.D_MODEL
G = binding.FP8_GROUP
TIGHT_REL = 4e-3


def check_status():
    st, word = binding.device_status()
    assert st == 0, f"device status {binding.STATUS.get(st, st)} word={word:#x}"


@pytest.fixture(scope="module")
def weight():
    """W_o (bf16, as the benchmark draws it) and the oracle's quantisation."""
    g = torch.Generator().manual_seed(11)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    qw, sw = oracle.quant_weight_fp8(W)
    return W, qw, sw


def activations(M, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-6, 4, (M, 1), generator=g))
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M", [1, 37, 300])
def test_quantize_act_bit_exact(cuda_device, M):
    x = activations(M, seed=M)
    xf = x.float()
    if M > 1:
        xf[1, G:2 * G] = 0.0                   # a group of zeros: scale 1, codes 0
        xf[1, :G] = -0.0                       # negative zeros: codes 0x80
        xf[0, 7] = 3e4                         # one large entry in a group
        x = xf.to(torch.bfloat16)
    q, s = binding.quantize_act_fp8(x.to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    rq, rs = oracle.quant_rows_fp8(x)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quantize_weight_bit_exact(cuda_device, weight):
    W, qw, sw = weight
    q, s = binding.quantize_weight_fp8(W.to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sw.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), qw)


def gpu_fp8_gemm(qa, sa, qw, sw, dev):
    out = binding.o_proj_fp8(torch.from_numpy(qa).to(dev), torch.from_numpy(sa).to(dev),
                             torch.from_numpy(qw).to(dev), torch.from_numpy(sw).to(dev))
    torch.cuda.synchronize()
    check_status()
    return out


@pytest.mark.parametrize("M", [1, 100, 128, 129, 300, 1000])
def test_oproj_fp8_all_rows(cuda_device, weight, M):
    """Every row: one tile row (M <= 128), a ragged second (129, 300), and
    eight row blocks (1000) of the persistent 128 x 128 tiles."""
    _, qw, sw = weight
    qa, sa = oracle.quant_rows_fp8(activations(M, seed=100 + M))
    out = gpu_fp8_gemm(qa, sa, qw, sw, cuda_device)
    ref = oracle.oproj_fp8_rows(qa, sa, qw, sw)
    m = assert_parity(to_f64(out), ref, f"o_proj fp8 M={M}")
    assert m["rel_frob"] <= TIGHT_REL, m


def test_oproj_fp8_large_sampled(cuda_device, weight):
    """M = 4096 + 77 (the last row block ragged), sampled rows."""
    _, qw, sw = weight
    M = 4096 + 77
    qa, sa = oracle.quant_rows_fp8(activations(M, seed=7))
    out = gpu_fp8_gemm(qa, sa, qw, sw, cuda_device)
    rows = sorted(set([0, 1, 127, 128, 129, M - 1, M - 2, M - 78, M - 77]
                      + list(np.random.default_rng(1).integers(0, M, 120))))
    ref = oracle.oproj_fp8_rows(qa, sa, qw, sw, rows=rows)
    m = assert_parity(to_f64(out[rows]), ref, "o_proj fp8 M=4173 sampled")
    assert m["rel_frob"] <= TIGHT_REL, m


def test_oproj_fp8_close_to_bf16_definition(cuda_device, weight):
    """Against the bf16 o_proj's exact value the FP8 form carries the e4m3
    rounding of both operands (3 mantissa bits): a few per cent, no more."""
    W, qw, sw = weight
    x = activations(256, seed=3)
    q, s = binding.quantize_act_fp8(x.to(cuda_device))
    out = binding.o_proj_fp8(q, s, torch.from_numpy(qw).to(cuda_device),
                             torch.from_numpy(sw).to(cuda_device))
    torch.cuda.synchronize()
    check_status()
    ref = oracle.oproj_rows(oracle.bf16_to_f64(x), W)
    m = metrics(to_f64(out), ref)
    assert 1e-3 < m["rel_frob"] < 6e-2, m


# e4m3 rounding of one operand: half a step is 2^-4 .. 2^-5 of a value, so
# its relative RMS is about 2^-5 at most.
ONE_OPERAND_FP8 = 3e-2


@pytest.mark.parametrize("B,T,masked", [(2, 300, False), (1, 200, True)])
def test_attn_oproj_fp8_all_rows(cuda_device, weight, B, T, masked):
    """The fused call on every row.

    (1) It is the composition of the three calls checked above (attention,
    activation quantiser, FP8 GEMM), bit for bit.
    (2) Against the oracle's own composition (fp64 attention rounded to bf16,
    quantised, block-scaled product) it agrees within the e4m3 rounding of
    one operand: the kernel's bf16 attention differs from the oracle's in the
    last bit of some values, which moves those groups' scales and codes by up
    to one e4m3 step, so the quantisation decisions are not the same ones.
    (3) Against the exact bf16 definition it stays within the FP8 band."""
    W, qw, sw = weight
    d = inputs.make_inputs(B, T, seed=B * 7 + T, key_padding=masked, min_valid=50,
                           with_weight=False)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    Wq, Ws = torch.from_numpy(qw).to(cuda_device), torch.from_numpy(sw).to(cuda_device)
    out = binding.attn_oproj_fp8(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"], Wq, Ws,
                                 mask=g["mask"], softmax_scale=g["softmax_scale"])
    attn = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                mask=g["mask"], softmax_scale=g["softmax_scale"])
    aq, asc = binding.quantize_act_fp8(attn)
    steps = binding.o_proj_fp8(aq, asc, Wq, Ws)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(out.reshape(B * T, -1), steps)
    ref_attn, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                    d["mask"], d["softmax_scale"])
    assert not fm.any()
    got = to_f64(out).reshape(B * T, -1)
    qa, sa = oracle.quant_rows_fp8(torch.from_numpy(ref_attn).to(torch.bfloat16))
    m = metrics(got, oracle.oproj_fp8_rows(qa, sa, qw, sw))
    assert m["finite"] and m["rel_frob"] <= ONE_OPERAND_FP8, m
    m = metrics(got, oracle.oproj_rows(ref_attn, W))
    assert 1e-3 < m["rel_frob"] < 6e-2, m
