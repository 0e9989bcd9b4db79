"""mla_attn_oproj_noalloc: the whole path for callers that cannot allocate
device memory (a host framework that owns every device allocation, a plugin
handed only its inputs and outputs). It uses the library's own fixed scratch
instead of a caller workspace.

Both calls run the same kernels on the same inputs, so the no-alloc output
must equal mla_attn_oproj's (the call with a workspace) bit for bit, on
several calls in a row: the scratch is shared by every call and keeps the
previous call's contents, so a later call must not see an earlier one's data,
and any aliasing or stale-contents mistake shows as a changed bit. This file
sorts last so that, if it fails, a run stopped at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

from mla_causal_attention_attn_b200 import binding, inputs

OK, WORKSPACE = 0, -5
A = 0x7f0000000000  # 16-byte aligned fake device address (never dereferenced)


def _noalloc(lib, g, out, stream):
    m = g["mask"]
    ld = int(m.stride(2)) if m is not None else 0
    return lib.mla_attn_oproj_noalloc(
        g["q_nope"].data_ptr(), g["q_pe"].data_ptr(), g["k_nope"].data_ptr(),
        g["k_pe"].data_ptr(), g["v"].data_ptr(), m.data_ptr() if m is not None else None, ld,
        g["q_nope"].shape[0], g["q_nope"].shape[2], ctypes.c_float(g["softmax_scale"]),
        g["W_o"].data_ptr(), out.data_ptr(), stream)


def test_rejects_problems_larger_than_its_scratch():
    """B*T above MLA_NOALLOC_MAX_TOKENS is refused before anything runs."""
    lib = binding.load()
    assert binding.NOALLOC_MAX_TOKENS == 4096
    args = [A] * 5 + [None, 0]
    assert lib.mla_attn_oproj_noalloc(*args, 1, 4097, 0.07, A, A, None) == WORKSPACE
    assert lib.mla_attn_oproj_noalloc(*args, 2, 2049, 0.07, A, A, None) == WORKSPACE
    assert lib.mla_attn_oproj_noalloc(*args, 1, 4096, 0.07, None, A, None) == -1  # W_o missing


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_twice_in_a_row(cuda_device):
    lib = binding.load()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [
        # explicit key-padding mask, row stride not a multiple of 8
        inputs.make_inputs(2, 300, seed=31, key_padding=True, min_valid=40),
        # causal, 8 query tiles
        inputs.make_inputs(1, 1024, seed=32),
        # B*T <= 128: o_proj runs the small-M cluster kernel on the scratch
        inputs.make_inputs(1, 64, seed=33),
        # the first case again, after the scratch held the others
        inputs.make_inputs(2, 300, seed=31, key_padding=True, min_valid=40),
    ]
    for k, d in enumerate(cases):
        g = {n: (t.to(cuda_device) if isinstance(t, torch.Tensor) else t) for n, t in d.items()}
        B, T = g["q_nope"].shape[0], g["q_nope"].shape[2]
        out = torch.full((B, T, inputs.D_MODEL), float("nan"), dtype=torch.bfloat16,
                         device=cuda_device)
        st = _noalloc(lib, g, out, stream)
        assert st == OK, binding.STATUS.get(st, st)
        ref = binding.attn_oproj(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                 g["W_o"], mask=g["mask"], softmax_scale=g["softmax_scale"])
        torch.cuda.synchronize()
        status, word = binding.device_status()
        assert status == OK, f"device status {status} ({word:#x})"
        assert torch.isfinite(out.float()).all(), f"call {k + 1}"
        assert torch.equal(out, ref), f"no-alloc call {k + 1} differs from mla_attn_oproj"
