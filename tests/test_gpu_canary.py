"""Every output element written, nothing written outside the outputs.

The stand-in for a memory sanitizer on this hardware: each output is a
prefix of a larger buffer filled with a canary (NaN for bf16 and fp32, 0xA5
for e4m3 codes). After the call no canary may remain inside the output, the
guard band after it must be untouched, and the inputs must be bit-identical
to what they were. Shapes are ragged so that the last row blocks and key
tiles are partial; both o_proj kernels and both FP8 tile widths run.
"""
import pytest
import torch

from mla_causal_attention_attn_b200 import binding, inputs

pytestmark = pytest.mark.gpu

GUARD = 4096
NAN_BF16 = 0x7FC0
NAN_F32 = 0x7FC00000
CODE_CANARY = 0xA5


def check_status():
    st, word = binding.device_status()
    assert st == 0, f"device status {binding.STATUS.get(st, st)} word={word:#x}"


def canary_buffer(n, dtype, dev):
    if dtype == torch.bfloat16:
        return torch.full((n + GUARD,), NAN_BF16, dtype=torch.int16, device=dev).view(dtype)
    if dtype == torch.float32:
        return torch.full((n + GUARD,), NAN_F32, dtype=torch.int32, device=dev).view(dtype)
    return torch.full((n + GUARD,), CODE_CANARY, dtype=torch.uint8, device=dev)


def bits(t):
    return t.view({torch.bfloat16: torch.int16, torch.float32: torch.int32}.get(t.dtype, t.dtype))


def check_written(buf, n, name):
    body, guard = buf[:n], buf[n:]
    if buf.dtype == torch.uint8:
        # a code may legitimately equal the canary: compare against a second run
        return body
    assert not torch.isnan(body.float()).any(), f"{name}: unwritten elements"
    ref = canary_buffer(0, buf.dtype, buf.device)
    assert torch.equal(bits(guard), bits(ref[:GUARD])), f"{name}: write past the end"
    return body


def snapshot(d):
    return {k: v.clone() for k, v in d.items() if isinstance(v, torch.Tensor)}


def assert_unchanged(before, d):
    for k, v in before.items():
        assert torch.equal(bits(v), bits(d[k])), f"input {k} was modified"


@pytest.mark.parametrize("B,T,masked", [(2, 300, False), (1, 200, True)])
def test_attention_writes_exactly_its_output(cuda_device, B, T, masked):
    d = inputs.make_inputs(B, T, seed=3, key_padding=masked, min_valid=50, with_weight=False)
    g = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    before = snapshot({k: g[k] for k in ("q_nope", "q_pe", "k_nope", "k_pe", "v")})
    n = B * T * inputs.K_OPROJ
    buf = canary_buffer(n, torch.bfloat16, cuda_device)
    binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"], mask=g["mask"],
                         softmax_scale=g["softmax_scale"], out=buf[:n].view(B, T, -1))
    torch.cuda.synchronize()
    check_status()
    check_written(buf, n, "attention output")
    assert_unchanged(before, g)


@pytest.mark.parametrize("M", [64, 300])
def test_oproj_writes_exactly_its_output(cuda_device, M):
    """M = 64: the small-M cluster kernel; M = 300: the tiled GEMM."""
    gen = torch.Generator().manual_seed(M)
    attn = torch.randn(M, inputs.K_OPROJ, generator=gen).to(torch.bfloat16).to(cuda_device)
    W = (torch.randn(inputs.D_MODEL, inputs.K_OPROJ, generator=gen) * 0.02).to(
        torch.bfloat16).to(cuda_device)
    before = snapshot({"attn": attn, "W": W})
    n = M * inputs.D_MODEL
    buf = canary_buffer(n, torch.bfloat16, cuda_device)
    binding.o_proj(attn, W, out=buf[:n].view(M, -1))
    torch.cuda.synchronize()
    check_status()
    check_written(buf, n, "o_proj output")
    assert_unchanged(before, {"attn": attn, "W": W})


@pytest.mark.parametrize("M", [100, 300])
def test_fp8_calls_write_exactly_their_outputs(cuda_device, M):
    """M = 100: 128-wide FP8 tiles; M = 300: 256-wide."""
    gen = torch.Generator().manual_seed(7 + M)
    x = torch.randn(M, inputs.K_OPROJ, generator=gen).to(torch.bfloat16).to(cuda_device)
    W = (torch.randn(inputs.D_MODEL, inputs.K_OPROJ, generator=gen) * 0.02).to(
        torch.bfloat16).to(cuda_device)
    before = snapshot({"x": x, "W": W})
    G = binding.FP8_K_GROUPS
    nq, ns = M * inputs.K_OPROJ, G * M
    qbuf = canary_buffer(nq, torch.uint8, cuda_device)
    sbuf = canary_buffer(ns, torch.float32, cuda_device)
    q, s = binding.quantize_act_fp8(x, q=qbuf[:nq].view(M, -1), scale=sbuf[:ns].view(G, M))
    Wq, Ws = binding.quantize_weight_fp8(W)
    n = M * inputs.D_MODEL
    obuf = canary_buffer(n, torch.bfloat16, cuda_device)
    binding.o_proj_fp8(q, s, Wq, Ws, out=obuf[:n].view(M, -1))
    torch.cuda.synchronize()
    check_status()
    check_written(sbuf, ns, "activation scales")
    assert torch.all(qbuf[nq:] == CODE_CANARY), "codes: write past the end"
    # codes equal to the canary byte are legal; a second run from another
    # canary shows every code was written
    qbuf2 = torch.zeros(nq, dtype=torch.uint8, device=cuda_device)
    binding.quantize_act_fp8(x, q=qbuf2.view(M, -1), scale=torch.empty_like(s))
    torch.cuda.synchronize()
    assert torch.equal(qbuf[:nq], qbuf2)
    check_written(obuf, n, "FP8 o_proj output")
    assert_unchanged(before, {"x": x, "W": W})
