"""Seeded synthetic inputs for the MLA prefill + o_proj path.

This module only draws random numbers and lays them out; it holds none of the
attention or projection arithmetic. The CUDA path and the CPU oracle are both
fed from it, so they always see the same bytes.

Shapes follow the page "Kimi K2 · Mix and project" (per-head tensors are
[B, 64 heads, T, .], the shared rotary key is [B, 1, T, 64], the value width is
128, o_proj maps 64*128 = 8192 -> 7168) and the model configuration printed on
"Kimi K2 · Block input" (hidden_size 7168, num_attention_heads 64,
qk_nope_head_dim 128, qk_rope_head_dim 64, v_head_dim 128).

Recipe (one torch CPU generator, seeded, fp32 normal draws in this order, then
a round-to-nearest-even cast to bf16):
  q_nope, q_pe, k_nope, k_pe, v   ~ N(0, 1)   (q_nope, q_pe times q_scale)
  W_o                              ~ N(0, 0.02)
  valid lengths (key padding only) ~ U{min_valid .. T}
"""
from __future__ import annotations

import dataclasses
import math

import torch

H = 64          # num_attention_heads
DN = 128        # qk_nope_head_dim
DR = 64         # qk_rope_head_dim
DV = 128        # v_head_dim
D_MODEL = 7168  # hidden_size
K_OPROJ = H * DV  # 8192, o_proj input width

DEFAULT_SCALE = 1.0 / math.sqrt(DN + DR)

# The rotary parameters of the configuration printed on "Kimi K2 · Block
# input" (config.json: rope_theta and the rope_scaling block). They are
# inputs of the rotary path, handed as they are to the kernels and to the
# oracle.
KIMI_K2_ROPE = {
    "rope_theta": 50000.0,
    "factor": 32.0,
    "original_max_position_embeddings": 4096.0,
    "beta_fast": 1.0,
    "beta_slow": 1.0,
    "mscale": 1.0,
    "mscale_all_dim": 1.0,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: batch, length and how the inputs are drawn."""
    name: str
    B: int
    T: int
    q_scale: float = 1.0
    key_padding: bool = False
    min_valid: int = 512
    compact_mask: bool = False  # key padding passed as valid lengths, not the dense mask

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads the library is checked and measured on.
WORKLOADS = {
    "b1_t64_causal": Workload("b1_t64_causal", 1, 64),
    "b1_t4096_causal": Workload("b1_t4096_causal", 1, 4096),
    "b16_t1024_causal": Workload("b16_t1024_causal", 16, 1024),
    "b1_t32768_causal_qx2": Workload("b1_t32768_causal_qx2", 1, 32768, q_scale=2.0),
    "b8_t4096_keypad_mask": Workload("b8_t4096_keypad_mask", 8, 4096, key_padding=True),
    # the same inputs, the padding given as per-sequence valid lengths
    "b8_t4096_keypad_varlen": Workload("b8_t4096_keypad_varlen", 8, 4096, key_padding=True,
                                       compact_mask=True),
}


def _randn(gen: torch.Generator, shape, std: float = 1.0, mul: float = 1.0):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mul != 1.0:
        x.mul_(mul)
    return x.to(torch.bfloat16)


def keypad_mask(valid_len: torch.Tensor, T: int) -> torch.Tensor:
    """Additive [B,1,T,T] bf16 mask: 0 where key j <= query i and j < valid_len[b],
    -inf elsewhere (causal plus key padding, the 4-D mask form the model's eager
    path passes to attention)."""
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    allowed = (j <= i).unsqueeze(0) & (j.unsqueeze(0) < valid_len.view(-1, 1, 1))
    m = torch.full(allowed.shape, float("-inf"), dtype=torch.float32)
    m.masked_fill_(allowed, 0.0)
    return m.to(torch.bfloat16).unsqueeze(1).contiguous()


def make_inputs(B: int, T: int, *, q_scale: float = 1.0, key_padding: bool = False,
                min_valid: int = 512, seed: int = 0, H_: int = H, Dn: int = DN,
                Dr: int = DR, Dv: int = DV, D: int = D_MODEL, with_weight: bool = True):
    """Draw one set of inputs on the CPU. Returns a dict of contiguous tensors:
    q_nope, q_pe, k_nope, k_pe, v, W_o (bf16), mask (bf16 or None),
    valid_len (int64 or None) and softmax_scale (float)."""
    gen = torch.Generator().manual_seed(seed)
    out = {
        "q_nope": _randn(gen, (B, H_, T, Dn), mul=q_scale),
        "q_pe": _randn(gen, (B, H_, T, Dr), mul=q_scale),
        "k_nope": _randn(gen, (B, H_, T, Dn)),
        "k_pe": _randn(gen, (B, 1, T, Dr)),
        "v": _randn(gen, (B, H_, T, Dv)),
    }
    out["W_o"] = _randn(gen, (D, H_ * Dv), std=0.02) if with_weight else None
    if key_padding:
        lo = min(min_valid, T)
        valid = torch.randint(lo, T + 1, (B,), generator=gen, dtype=torch.int64)
        out["valid_len"] = valid
        out["mask"] = keypad_mask(valid, T)
    else:
        out["valid_len"] = None
        out["mask"] = None
    out["softmax_scale"] = 1.0 / math.sqrt(Dn + Dr)
    return out


def make_peaked_inputs(B: int, T: int, *, gain: float = 6.0, seed: int = 0):
    """Inputs whose query row i points at key rows i and i+1.

    Keys and values are drawn as by make_inputs. Per head, query row i is
    gain * (key row i + key row i+1) over all 192 dims, its rotary part built
    from the shared rotary key; the last row is 2 * gain * key row T-1. With
    the default softmax scale the scores of keys i and i+1 then stand tens of
    nats above the row's others, and which of the two is higher differs from
    row to row. A check on these inputs is sharp where random ones are not:
    under the causal mask row i's output is v_i to bf16 precision, while a
    kernel that let key i+1 in, or kept key i out, is off by the size of v."""
    d = make_inputs(B, T, seed=seed, with_weight=False)

    def nxt(x):
        return torch.cat([x[:, :, 1:], x[:, :, -1:]], dim=2).float()

    d["q_nope"] = (gain * (d["k_nope"].float() + nxt(d["k_nope"]))).to(torch.bfloat16)
    q_pe = gain * (d["k_pe"].float() + nxt(d["k_pe"]))
    d["q_pe"] = q_pe.expand(B, H, T, DR).contiguous().to(torch.bfloat16)
    return d


def make_positions(B: int, T: int, kind: str = "arange", seed: int = 0) -> torch.Tensor:
    """position_ids [B, T] int32 for the rotary path:
    "arange"  0..T-1 in every sequence (what a None position_ids means);
    "offset"  sequence b starts at 1000 * b + 17 (a prefill after a cached prefix);
    "random"  independent draws from U{0 .. 2^17 - 1} (no structure at all)."""
    if kind == "arange":
        p = torch.arange(T, dtype=torch.int64).repeat(B, 1)
    elif kind == "offset":
        p = torch.arange(T, dtype=torch.int64).repeat(B, 1) + \
            (1000 * torch.arange(B, dtype=torch.int64) + 17).view(B, 1)
    elif kind == "random":
        gen = torch.Generator().manual_seed(seed)
        p = torch.randint(0, 1 << 17, (B, T), generator=gen, dtype=torch.int64)
    else:
        raise ValueError(kind)
    return p.to(torch.int32).contiguous()


KV_RANK = 512  # kv_lora_rank


def make_latent_inputs(B: int, T: int, *, q_scale: float = 1.0, key_padding: bool = False,
                       min_valid: int = 512, seed: int = 0, H_: int = H, Dn: int = DN,
                       Dr: int = DR, Dv: int = DV, R: int = KV_RANK, D: int = D_MODEL,
                       with_weight: bool = True):
    """Inputs of the path that starts from the compressed KV latent: the
    make_inputs set (whose k_nope and v are then unused), followed by draws of
    c_kv [B, T, R] ~ N(0, 1) and W_kv_b [H*(Dn+Dv), R] ~ N(0, 0.02) (the
    configuration's initializer_range, as for W_o)."""
    out = make_inputs(B, T, q_scale=q_scale, key_padding=key_padding, min_valid=min_valid,
                      seed=seed, H_=H_, Dn=Dn, Dr=Dr, Dv=Dv, D=D, with_weight=with_weight)
    gen = torch.Generator().manual_seed(seed + 7919)
    out["c_kv"] = _randn(gen, (B, T, R))
    out["W_kv_b"] = _randn(gen, (H_ * (Dn + Dv), R), std=0.02)
    return out


def make_workload(w: Workload, seed: int = 0, with_weight: bool = True):
    return make_inputs(w.B, w.T, q_scale=w.q_scale, key_padding=w.key_padding,
                       min_valid=w.min_valid, seed=seed, with_weight=with_weight)
