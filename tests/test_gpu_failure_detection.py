"""Failure detection without a GPU fault.

Every mbarrier wait in the kernels is bounded. Here one wait is made to run
out on purpose: with MLA_TEST_STALL_WAIT=1 the attention kernel's first CTA
waits on a barrier nothing ever completes, and MLA_WAIT_LIMIT_NS shortens the
limit to 0.2 s. The CTA must give up, let its in-flight copies and MMAs land,
free its tensor memory and return; mla_device_status must report
MLA_ERR_TIMEOUT with the attention kernel's code and the wait site; and the
context must stay usable (a following o_proj call is checked against the
oracle). Both variables are read once per process, so this runs in a child.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CHILD = r"""
import json, sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import metrics, to_f64
dev = torch.device("cuda:0")
d = inputs.make_inputs(1, 512, seed=5, with_weight=False)
g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
st_launch = 0
try:
    binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                         softmax_scale=g["softmax_scale"])
except binding.MLAError as e:
    st_launch = e.status
status, word = binding.device_status()
# the context must still work
gen = torch.Generator().manual_seed(1)
a = torch.randn(64, 8192, generator=gen).to(torch.bfloat16)
W = (torch.randn(7168, 8192, generator=gen) * 0.02).to(torch.bfloat16)
out = binding.o_proj(a.to(dev), W.to(dev))
torch.cuda.synchronize()
status2, word2 = binding.device_status()
m = metrics(to_f64(out), oracle.oproj_rows(oracle.bf16_to_f64(a), W))
print(json.dumps({"launch": st_launch, "status": status, "word": word, "status2": status2,
                  "rel_frob": m["rel_frob"], "max_abs": m["max_abs"]}))
"""


def test_bounded_wait_times_out_and_context_survives():
    env = dict(os.environ)
    env["MLA_TEST_STALL_WAIT"] = "1"
    env["MLA_WAIT_LIMIT_NS"] = "200000000"
    code = "ROOT = %r\n" % ROOT + CHILD
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    r = json.loads(res.stdout.strip().splitlines()[-1])
    assert r["launch"] == 0
    assert r["status"] == -7, r                       # MLA_ERR_TIMEOUT
    assert r["word"] & (1 << 16), r                   # timeout flag
    assert (r["word"] >> 8) & 0xFF == 2, r            # attention kernel
    assert r["status2"] == 0, r                       # cleared, nothing new
    assert r["rel_frob"] <= 1e-2 and r["max_abs"] <= 3e-2, r
