"""Failure detection without a GPU fault.

Every mbarrier wait in the kernels is bounded. Here one wait is made to run
out on purpose: with MLA_TEST_STALL_WAIT=1 the attention kernel's first CTA
waits on a barrier nothing ever completes, and MLA_WAIT_LIMIT_NS shortens the
limit to 0.2 s. The CTA must give up, let its in-flight copies and MMAs land,
free its tensor memory and return; mla_device_status must report
MLA_ERR_TIMEOUT with the attention kernel's code and the wait site; and the
context must stay usable (a following o_proj call is checked against the
oracle). Both variables are read once per process, so this runs in a child.
The same hooks check that a timeout lands in the status word of the call that
had it (its workspace) and nowhere else.
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


@pytest.mark.parametrize("pv_issuer", ["0", "1"])
def test_bounded_wait_times_out_and_context_survives(pv_issuer):
    """With one issuer per query tile, and with the PV products issued by a
    thread of their own (which must see the abort while it polls)."""
    env = dict(os.environ)
    env["MLA_TEST_STALL_WAIT"] = "1"
    env["MLA_WAIT_LIMIT_NS"] = "200000000"
    env["MLA_ATTN_PV_ISSUER"] = pv_issuer
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


CHILD_PER_CALL = r"""
import json, sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import oracle
from mla_causal_attention_attn_b200 import binding, inputs
from parity import metrics, to_f64
dev = torch.device("cuda:0")
d = inputs.make_inputs(1, 512, seed=6, key_padding=True, min_valid=300)
g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
ws_a = torch.empty(binding.attn_oproj_workspace_bytes(1, 512, True), dtype=torch.uint8, device=dev)
ws_b = torch.empty(binding.attn_oproj_workspace_bytes(1, 512, False), dtype=torch.uint8,
                   device=dev)
ws_a.fill_(0xff)   # a stale word from "an earlier call" must not leak into this one
torch.cuda.synchronize()
args = (g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"], g["W_o"])
# stream A: the masked call, whose first attention CTA stalls until its wait runs out
out_a = binding.attn_oproj(*args, mask=g["mask"], softmax_scale=g["softmax_scale"],
                           workspace=ws_a, stream=sa)
# stream B, meanwhile: a causal call on its own workspace
out_b = binding.attn_oproj(*args, mask=None, softmax_scale=g["softmax_scale"], workspace=ws_b,
                           stream=sb)
st_a, word_a = binding.last_device_status(ws_a, sa)
st_b, word_b = binding.last_device_status(ws_b, sb)
st_g, word_g = binding.device_status()           # the device-wide word saw nothing
# the same workspace, next call (causal, no stall): its word starts clean
out_a2 = binding.attn_oproj(*args, mask=None, softmax_scale=g["softmax_scale"], workspace=ws_a,
                            stream=sa)
st_a2, word_a2 = binding.last_device_status(ws_a, sa)
torch.cuda.synchronize()
ref, _ = oracle.attn_oproj_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], None,
                                d["softmax_scale"], d["W_o"])
mb = metrics(to_f64(out_b).reshape(512, -1), ref)
ma2 = metrics(to_f64(out_a2).reshape(512, -1), ref)
print(json.dumps({"st_a": st_a, "word_a": word_a, "st_b": st_b, "word_b": word_b, "st_g": st_g,
                  "word_g": word_g, "st_a2": st_a2, "word_a2": word_a2,
                  "b_rel": mb["rel_frob"], "b_abs": mb["max_abs"],
                  "a2_rel": ma2["rel_frob"], "a2_abs": ma2["max_abs"]}))
"""


def test_status_word_is_per_workspace():
    """Two fused calls on two streams with two workspaces. With
    MLA_TEST_STALL_WAIT=3 only the call given an explicit mask stalls: its
    workspace reports MLA_ERR_TIMEOUT (attention kernel), the other call's
    workspace and the device-wide word report MLA_OK, the unaffected call's
    output matches the oracle, and the next call on the timed-out workspace
    starts from a clean word."""
    env = dict(os.environ)
    env["MLA_TEST_STALL_WAIT"] = "3"
    env["MLA_WAIT_LIMIT_NS"] = "200000000"
    code = "ROOT = %r\n" % ROOT + CHILD_PER_CALL
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    r = json.loads(res.stdout.strip().splitlines()[-1])
    assert r["st_a"] == -7, r                        # MLA_ERR_TIMEOUT, in A's workspace
    assert r["word_a"] & (1 << 16), r
    assert (r["word_a"] >> 8) & 0xFF == 2, r         # attention kernel
    assert r["st_b"] == 0 and r["word_b"] == 0, r
    assert r["st_g"] == 0 and r["word_g"] == 0, r
    assert r["st_a2"] == 0 and r["word_a2"] == 0, r
    assert r["b_rel"] <= 1e-2 and r["b_abs"] <= 3e-2, r
    assert r["a2_rel"] <= 1e-2 and r["a2_abs"] <= 3e-2, r
