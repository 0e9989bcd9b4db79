"""The attention kernels side by side, and sharp checks of their key masks.

Causal and valid-length calls run, by MLA_ATTN_KERNEL (read once per
process), the one-SM kernel with 64-key (half-tile) score buffers (the
default; under an explicit mask a CTA whose query tiles skip a key tile
before a used one keeps 128-key tiles), the same kernel on 128-key tiles
("tile"), or the CTA-pair kernel ("pair"). The half-tile kernel issues
its PV products either from each query tile's MMA issuer ("half") or from a
thread of their own ("halfpv"; MLA_ATTN_PV_ISSUER=1, the default from
T = 4096 on). Each runs here in a child process with the variables set.
Checked:
- every kernel against the fp64 oracle, on random inputs (causal and
  valid_len) and on inputs whose query row i points at keys i and i+1
  (inputs.make_peaked_inputs). On those the causal answer of row i is v_i to
  bf16 precision, so they are compared element by element within half a bf16
  ulp: a kernel that let key i+1 in, or kept key i out, would be off by the
  size of v itself, at any row, tile boundary or ragged tail. The running
  max jumps on the diagonal there, so the rescale of O is exercised too;
- the two half-tile issue orders run the same MMAs on the same operands in
  the same order per accumulator: bit-identical outputs;
- the tile and pair kernels do the same per-row arithmetic (128-key tiles,
  the same softmax routes): equal to within one bf16 ulp;
- the half-tile kernel against the tile kernel: rows whose allowed keys all
  lie in the first 64 are bit-identical (the same maximum, sums and products);
  on the other rows the running max starts from 64 keys instead of 128, so P
  rounds differently, and their errors against the oracle are of one size;
- on 128-key tiles an explicit causal mask gives the causal call's result bit
  for bit, and a dense causal key-padding mask the valid_len call's outside
  the query tile holding the last valid key (whose diagonal mask tile is
  mixed).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from mla_causal_attention_attn_b200 import inputs
from parity import assert_parity, assert_peaked, to_f64

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CASES = [(1, 1), (1, 130), (2, 300), (1, 1024), (3, 257)]
PEAKED = [(1, 1), (2, 300), (1, 1024)]


def lens_of(B, T):
    return [max(1, T - 77 * (b + 1)) for b in range(B)]


CHILD = r"""
import sys, torch
sys.path.insert(0, ROOT)
from mla_causal_attention_attn_b200 import binding, inputs
dev = torch.device("cuda:0")
outs = {}

def run(d, tag, lens, mask=None):
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    outs[tag] = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                                     softmax_scale=g["softmax_scale"]).cpu()
    vl = torch.tensor(lens, dtype=torch.int32, device=dev)
    outs[tag + "v"] = binding.attn_prefill_varlen(g["q_nope"], g["q_pe"], g["k_nope"],
                                                  g["k_pe"], g["v"], vl,
                                                  softmax_scale=g["softmax_scale"]).cpu()
    if mask is not None:
        outs[tag + "m"] = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"],
                                               g["v"], mask=mask.to(dev),
                                               softmax_scale=g["softmax_scale"]).cpu()

for B, T in CASES:
    run(inputs.make_inputs(B, T, seed=1300 + T + B, with_weight=False), f"r{B}x{T}", LENS(B, T))
for B, T in PEAKED:
    run(inputs.make_peaked_inputs(B, T, seed=1400 + T + B), f"p{B}x{T}", LENS(B, T))
if MASK_FORMS:
    for B, T in [(1, 256), (2, 300)]:
        lens = [T] * B
        run(inputs.make_inputs(B, T, seed=31 + T, with_weight=False), f"c{B}x{T}", lens,
            inputs.keypad_mask(torch.tensor(lens), T))
    lens = [700, 333, 129]
    run(inputs.make_inputs(3, 700, seed=5, with_weight=False), "k3x700", lens,
        inputs.keypad_mask(torch.tensor(lens), 700))
if EXTRA:
    # explicit masks (a general additive one, a causal key-padding one) and
    # the rotary call, with and without a mask: these run the selected
    # kernel's masked and rotary instances
    for tag, d in EXTRA_INPUTS().items():
        g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        m = g["mask"]
        if tag.startswith("rope"):
            outs[tag] = binding.attn_prefill_rope(
                g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"], g["v"],
                position_ids=g["pos"], rope=inputs.KIMI_K2_ROPE, mask=m,
                softmax_scale=g["softmax_scale"]).cpu()
        else:
            outs[tag] = binding.attn_prefill(g["q_nope"], g["q_pe"], g["k_nope"], g["k_pe"],
                                             g["v"], mask=m,
                                             softmax_scale=g["softmax_scale"]).cpu()
torch.cuda.synchronize()
st, word = binding.device_status()
assert st == 0, (st, word)
torch.save(outs, OUT)
"""

EXTRA_SRC = r"""
def EXTRA_INPUTS():
    import torch
    from mla_causal_attention_attn_b200 import inputs
    out = {}
    d = inputs.make_inputs(2, 300, seed=901, with_weight=False)
    gm = torch.Generator().manual_seed(902)
    m = torch.randn(2, 1, 300, 300, generator=gm) * 2.0
    m.masked_fill_(torch.rand(2, 1, 300, 300, generator=gm) < 0.3, float("-inf"))
    m[..., 0] = 0.0
    d["mask"] = m.to(torch.bfloat16)
    out["gen2x300"] = d
    d = inputs.make_inputs(2, 300, seed=903, with_weight=False)
    d["mask"] = inputs.keypad_mask(torch.tensor([300, 150]), 300)
    out["kp2x300"] = d
    d = inputs.make_inputs(2, 300, seed=904, with_weight=False)
    d["pos"] = inputs.make_positions(2, 300, "offset")
    out["rope2x300"] = d
    d = dict(inputs.make_inputs(2, 300, seed=905, with_weight=False))
    d["pos"] = inputs.make_positions(2, 300, "random", seed=906)
    d["mask"] = inputs.keypad_mask(torch.tensor([300, 111]), 300)
    out["ropem2x300"] = d
    # a skipped key tile inside a query tile's range: batch 0's query tiles
    # 2 and 3 see key tiles 0, 2, 3 but not 1, so their CTA runs 128-key
    # tiles while the others take half tiles; batch 1 skips its last key
    # tile, and its query tile 1 has no allowed key at all (its rows are
    # written as zeros while query tile 0 of the same CTA runs). T = 400: the
    # last key tile's second half lies past T.
    gm = torch.Generator().manual_seed(907)
    m = torch.randn(2, 1, 400, 400, generator=gm)
    m[0, 0, 256:, 128:256] = float("-inf")
    m[1, 0, :, 384:] = float("-inf")
    m[1, 0, 128:256, :] = float("-inf")
    m = m.to(torch.bfloat16)
    d = inputs.make_inputs(2, 400, seed=908, with_weight=False)
    d["mask"] = m
    out["gap2x400"] = d
    d = dict(inputs.make_inputs(2, 400, seed=909, with_weight=False))
    d["pos"] = inputs.make_positions(2, 400, "offset")
    d["mask"] = m
    out["ropegap2x400"] = d
    # the smallest explicit masks: T = 1 (the second 64-key half of the only
    # key tile lies past T) and T = 65 (it holds one key)
    for T, seed in ((1, 910), (65, 911)):
        d = inputs.make_inputs(1, T, seed=seed, with_weight=False)
        gm = torch.Generator().manual_seed(seed + 100)
        d["mask"] = (torch.randn(1, 1, T, T, generator=gm) * 2.0).to(torch.bfloat16)
        out[f"gen1x{T}"] = d
    return out
"""
exec(EXTRA_SRC)

LENS_SRC = "def LENS(B, T):\n    return [max(1, T - 77 * (b + 1)) for b in range(B)]\n"


def run_child(kernel, out_path, mask_forms=False, extra=False, cases=None, peaked=None):
    env = dict(os.environ)
    env.pop("MLA_ATTN_KERNEL", None)
    env["MLA_ATTN_PV_ISSUER"] = "1" if kernel == "halfpv" else "0"
    if kernel not in ("half", "halfpv"):
        env["MLA_ATTN_KERNEL"] = kernel
    cases = CASES if cases is None else cases
    peaked = PEAKED if peaked is None else peaked
    code = (f"ROOT = {ROOT!r}\nOUT = {out_path!r}\nCASES = {cases!r}\nPEAKED = {peaked!r}\n"
            f"MASK_FORMS = {mask_forms!r}\nEXTRA = {extra!r}\n" + LENS_SRC + EXTRA_SRC + CHILD)
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    return torch.load(out_path)


def varlen_mask(B, T, lens):
    return inputs.keypad_mask(torch.tensor(lens), T)


def ulps(a, b):
    """|a - b| in units of b's bf16 ulp, elementwise."""
    diff = (a.float() - b.float()).abs()
    return diff / (b.float().abs().clamp_min(1e-30).log2().floor() - 7).exp2()


def oracle_case(d, mask):
    ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"], mask,
                               d["softmax_scale"])
    assert not fm.any()
    return ref


def test_kernels_against_oracle_and_each_other(cuda_device, tmp_path):
    outs = {k: run_child(k, str(tmp_path / f"{k}.pt"))
            for k in ("half", "halfpv", "tile", "pair")}
    for tag in outs["half"]:
        assert torch.equal(outs["halfpv"][tag], outs["half"][tag]), (tag, "issue orders differ")
    report = {}
    err2 = {"half": 0.0, "tile": 0.0}
    for kind, cases in (("r", CASES), ("p", PEAKED)):
        for B, T in cases:
            if kind == "r":
                d = inputs.make_inputs(B, T, seed=1300 + T + B, with_weight=False)
            else:
                d = inputs.make_peaked_inputs(B, T, seed=1400 + T + B)
            lens = lens_of(B, T)
            for form, mask in (("", None), ("v", varlen_mask(B, T, lens))):
                tag = f"{kind}{B}x{T}{form}"
                ref = oracle_case(d, mask)
                got = {k: to_f64(outs[k][tag]).reshape(B * T, -1) for k in outs}
                for k in outs:
                    assert_parity(got[k], ref, f"{k} {tag}")
                if kind == "p":
                    # rows with one answer: every row of the causal form; rows
                    # t < len of the valid-length form
                    rows = np.array([b * T + t for b in range(B) for t in range(T)
                                     if form == "" or t < lens[b]])
                    for k in outs:
                        assert_peaked(got[k], ref, rows, f"{k} {tag}")
                    continue
                u = ulps(outs["pair"][tag], outs["tile"][tag])
                report[tag] = {"pair_vs_tile_max_ulps": float(u.max())}
                assert float(u.max()) <= 1.0, (tag, report)
                # half vs tile: rows t < 64 see keys 0..63 only
                first = [b * T + t for b in range(B) for t in range(min(T, 64))]
                a = outs["half"][tag].reshape(B * T, -1)[first]
                b_ = outs["tile"][tag].reshape(B * T, -1)[first]
                assert torch.equal(a, b_), (tag, "rows t < 64 differ")
                for k in err2:
                    err2[k] += float(((got[k] - ref) ** 2).sum())
                report[tag]["half_equal_tile"] = bool(torch.equal(outs["half"][tag],
                                                                  outs["tile"][tag]))
    rms = {k: v ** 0.5 for k, v in err2.items()}
    report["err_norm"] = rms
    print(json.dumps(report))
    assert rms["half"] <= 1.25 * rms["tile"] + 1e-9, report


def test_tile_mode_mask_forms_are_bit_exact(cuda_device, tmp_path):
    """On 128-key tiles: explicit causal mask == causal call; dense causal
    key-padding mask == valid_len call outside the query tile holding the last
    valid key."""
    outs = run_child("tile", str(tmp_path / "tile.pt"), mask_forms=True)
    for B, T in [(1, 256), (2, 300)]:
        assert torch.equal(outs[f"c{B}x{T}m"], outs[f"c{B}x{T}"]), (B, T)
    dense, compact = outs["k3x700m"], outs["k3x700v"]
    T = 700
    for b, L in enumerate([700, 333, 129]):
        keep = torch.ones(T, dtype=torch.bool)
        qt = (L - 1) // 128
        if L < T:
            keep[qt * 128:(qt + 1) * 128] = False
        assert torch.equal(dense[b][keep], compact[b][keep]), f"b={b} L={L}"


def test_every_kernel_masks_and_rotary_against_oracle(cuda_device, tmp_path):
    """The explicit-mask and rotary instances of each kernel setting (the
    CTA-pair kernel runs them too when selected) against the fp64 oracle: a
    general additive mask, a causal key-padding mask, a mask that skips a
    key tile inside a query tile's range (those CTAs keep 128-key tiles in
    the half-tile settings), and the rotary call with offset positions, and
    with random positions under a mask."""
    want = {}
    for tag, d in EXTRA_INPUTS().items():
        B, _, T, _ = d["q_nope"].shape
        if tag.startswith("rope"):
            ref, fm = oracle.attn_rows_rope(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"],
                                            d["v"], d["mask"], d["softmax_scale"], d["pos"],
                                            inputs.KIMI_K2_ROPE)
        else:
            ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                       d["mask"], d["softmax_scale"])
        want[tag] = (ref, fm, B, T)
    for kernel in ("half", "halfpv", "tile", "pair"):
        outs = run_child(kernel, str(tmp_path / f"x_{kernel}.pt"), extra=True, cases=[],
                         peaked=[])
        for tag, (ref, fm, B, T) in want.items():
            got = to_f64(outs[tag]).reshape(B * T, -1)
            rows = ~fm.any(axis=1)
            assert np.all(got[~rows] == 0.0), (kernel, tag)
            assert_parity(got[rows], ref[rows], f"{kernel} {tag}")


def test_pv_issuer_bit_identical_at_full_size(cuda_device, tmp_path):
    """B=1, T=4096 (where the separate PV issuer is the default), random and
    peaked inputs, causal and valid-length forms: the two issue orders give
    the same bits, and on the peaked inputs every allowed row is v_t to half
    a bf16 ulp."""
    cases, peaked = [(1, 4096)], [(1, 4096)]
    outs = {k: run_child(k, str(tmp_path / f"full_{k}.pt"), cases=cases, peaked=peaked)
            for k in ("half", "halfpv")}
    for tag in outs["half"]:
        assert torch.equal(outs["halfpv"][tag], outs["half"][tag]), (tag, "issue orders differ")
    B, T = peaked[0]
    d = inputs.make_peaked_inputs(B, T, seed=1400 + T + B)
    lens = lens_of(B, T)
    for form, mask in (("", None), ("v", varlen_mask(B, T, lens))):
        rows = np.array([t for t in range(T) if form == "" or t < lens[0]])
        ref, fm = oracle.attn_rows(d["q_nope"], d["q_pe"], d["k_nope"], d["k_pe"], d["v"],
                                   mask, d["softmax_scale"], rows=[(0, int(t)) for t in rows])
        got = to_f64(outs["halfpv"][f"p{B}x{T}{form}"]).reshape(B * T, -1)[rows]
        assert_peaked(got, ref, np.arange(len(rows)), f"halfpv p{B}x{T}{form}")
