"""The two attention kernels on the same causal inputs.

Causal and valid-length calls run the one-SM kernel, or, in a process started
with MLA_ATTN_KERNEL=pair, the CTA-pair kernel (one M = 256 MMA over two SMs,
double-buffered scores). Each is run in a child process with the variable set
accordingly. Both must match the fp64 oracle, and they must agree with each
other: the per-row
arithmetic (fp32 scores, the same softmax routes, P rounded to bf16, fp32
accumulation of P V) is the same, so any difference beyond a rounding flip of
a bf16 output would point at a layout or masking mistake in one of them.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import assert_parity, to_f64

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CASES = [(1, 1), (1, 130), (2, 300), (1, 1024), (3, 257)]

CHILD = r"""
import sys, torch
sys.path.insert(0, ROOT)
from mla_causal_attention_attn_b200 import binding, inputs
dev = torch.device("cuda:0")
outs = {}
for B, T in CASES:
    d = inputs.make_inputs(B, T, seed=1300 + T + B, with_weight=False)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    outs[f"{B}x{T}"] = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"],
                                            g["v"], softmax_scale=g["softmax_scale"]).cpu()
    vl = torch.tensor([max(1, T - 77 * (b + 1)) for b in range(B)], dtype=torch.int32)
    outs[f"{B}x{T}v"] = binding.attn_prefill_varlen(g["q_nope"], g["q_pe"], g["k_nope"],
                                                    g["k_pe"], g["v"], vl.to(dev),
                                                    softmax_scale=g["softmax_scale"]).cpu()
torch.cuda.synchronize()
st, word = binding.device_status()
assert st == 0, (st, word)
torch.save(outs, OUT)
"""


def run_child(kernel, out_path):
    env = dict(os.environ, MLA_ATTN_KERNEL=kernel)
    code = f"ROOT = {ROOT!r}\nOUT = {out_path!r}\nCASES = {CASES!r}\n" + CHILD
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    return torch.load(out_path)


def test_one_sm_and_pair_kernels_agree(cuda_device, tmp_path):
    pair_all = run_child("pair", str(tmp_path / "pair.pt"))
    one_sm = run_child("one_sm", str(tmp_path / "one_sm.pt"))
    report = {}
    for B, T in CASES:
        d = inputs.make_inputs(B, T, seed=1300 + T + B, with_weight=False)
        pair, pair_v = pair_all[f"{B}x{T}"], pair_all[f"{B}x{T}v"]
        ref, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                  d["softmax_scale"])
        for name, got in (("pair", pair), ("one_sm", one_sm[f"{B}x{T}"])):
            assert_parity(to_f64(got).reshape(B * T, -1), ref, f"{name} causal B={B} T={T}")
        for a, b_, tag in ((pair, one_sm[f"{B}x{T}"], ""), (pair_v, one_sm[f"{B}x{T}v"], "v")):
            diff = (a.float() - b_.float()).abs()
            ulp = (b_.float().abs().clamp_min(1e-30).log2().floor() - 7).exp2()
            report[f"{B}x{T}{tag}"] = {"equal": bool(torch.equal(a, b_)),
                                       "max_diff_ulps": float((diff / ulp).max())}
            assert float((diff / ulp).max()) <= 1.0, (B, T, tag, report)
    print(json.dumps(report))
