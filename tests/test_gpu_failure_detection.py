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


CHILD_SMALL_M = r"""
import json, sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import metrics, to_f64
dev = torch.device("cuda:0")
gen = torch.Generator().manual_seed(2)
a = torch.randn(64, 8192, generator=gen).to(torch.bfloat16)
W = (torch.randn(7168, 8192, generator=gen) * 0.02).to(torch.bfloat16)
Wd = W.to(dev)
st_launch = 0
try:
    binding.o_proj(a.to(dev), Wd)          # M = 64: the small-M kernel, one cluster stalled
except binding.MLAError as e:
    st_launch = e.status
status, word = binding.device_status()
# the context must still work: attention, then a tiled o_proj (M = 256)
d = inputs.make_inputs(1, 200, seed=4, with_weight=False)
g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
att = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                           softmax_scale=g["softmax_scale"])
a2 = torch.randn(256, 8192, generator=gen).to(torch.bfloat16)
out2 = binding.o_proj(a2.to(dev), Wd)
torch.cuda.synchronize()
status2, word2 = binding.device_status()
ref, _ = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                          d["softmax_scale"])
ma = metrics(to_f64(att).reshape(200, -1), ref)
mo = metrics(to_f64(out2), oracle.oproj_rows(oracle.bf16_to_f64(a2), W))
print(json.dumps({"launch": st_launch, "status": status, "word": word, "status2": status2,
                  "attn_rel": ma["rel_frob"], "attn_abs": ma["max_abs"],
                  "oproj_rel": mo["rel_frob"], "oproj_abs": mo["max_abs"]}))
"""


def test_cluster_handoff_wait_times_out_and_context_survives():
    """The small-M o_proj hands a partial sum between the two CTAs of a
    cluster through two bounded waits. With MLA_TEST_STALL_WAIT=2 the rank-1
    CTA of the first cluster never reports its partial: rank 0's wait for it
    and rank 1's wait for the read must both give up (neither CTA touches the
    other's shared memory), MLA_ERR_TIMEOUT must name the small-M kernel, and
    the context must stay usable for attention and the tiled o_proj."""
    env = dict(os.environ)
    env["MLA_TEST_STALL_WAIT"] = "2"
    env["MLA_WAIT_LIMIT_NS"] = "200000000"
    code = "ROOT = %r\n" % ROOT + CHILD_SMALL_M
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    r = json.loads(res.stdout.strip().splitlines()[-1])
    assert r["launch"] == 0
    assert r["status"] == -7, r                       # MLA_ERR_TIMEOUT
    assert r["word"] & (1 << 16), r                   # timeout flag
    assert (r["word"] >> 8) & 0xFF == 4, r            # small-M o_proj kernel
    assert r["word"] & 0xFF in (7, 8), r              # one of the two cluster hand-off waits
    assert r["status2"] == 0, r
    assert r["attn_rel"] <= 1e-2 and r["attn_abs"] <= 3e-2, r
    assert r["oproj_rel"] <= 1e-2 and r["oproj_abs"] <= 3e-2, r
