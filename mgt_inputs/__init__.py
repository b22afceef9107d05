"""Seeded synthetic inputs for the tensor-parallel GPT layer, shared by the oracle tests,
the GPU parity tests and the benchmark.

This module holds NO arithmetic of the layer itself: it only draws random tensors, names the
workload shapes, and permutes full (unsharded) nn.Linear weights into the per-shard packed
layout that the C ABI consumes. The permutation restates the partitioning described on the
page "Megatron-LM 3D并行原理与万亿参数训练实战指南" (trdm.cn), section 2.1 (tensor
parallelism): W_q, W_k, W_v are split by output columns ("column-parallel"), each shard
keeping whole heads; W_o is split by input rows ("row-parallel"). The page
"Megatron-LM：NVIDIA大模型训练框架" (second-brain-czx), section "张量并行", shows the same
split as ColumnParallelLinear(gather_output=False) / RowParallelLinear(input_is_parallel=True).
The MLP (fc1 column-split, fc2 row-split) follows the same pattern.

Packed layouts (row-major, weights stored nn.Linear-style [out, in], y = x W^T + b):
    w_qkv  [p][3][H/p][d][h]   shard t owns heads t*H/p .. (t+1)*H/p-1 of each of Q, K, V
    b_qkv  [p][3][H/p][d]
    w_o    [p][h][h/p]         shard t owns input columns t*h/p .. (t+1)*h/p-1
    w1     [p][f/p][h]         shard t owns output rows t*f/p .. (t+1)*f/p-1
    b1     [p][f/p]
    (SwiGLU: w1 [p][2][f/p][h], b1 [p][2][f/p]: shard t's gate rows, then its up rows; the
     full matrix is [2f, h] with all gate rows first, then all up rows)
    w2     [p][h][f/p]
    b_o, b2, ln gammas/betas   replicated [h]
Activations: x, y [b, s, h]; qkv [b*s][p][3][H/p][d]; attention output [b*s][p][H/p][d]
(= head-major [b*s, h]); u, a [b*s][p][f/p] (= [b*s, f]).

Variants (the trdm.cn page, section 3.3, lists them as launch flags): swiglu=1 replaces GeLU by
SwiGLU, a = silu(gate) * up, fc1 producing gate and up (2f outputs); disable_bias_linear=1
drops the biases of all four linear layers (the LayerNorm affine parameters stay).

Sequence parallelism (sequence_parallel=1): the tensors outside the tensor-parallel regions
(x, y, dx, dy and the LayerNorm / residual activations) are split along the sequence, shard t
owning positions t*s/p .. (t+1)*s/p - 1 of every sequence, and laid out shard-major:
[p][b][s/p][h] (to_sp / from_sp convert from / to [b, s, h]).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict

import torch

__all__ = [
    "LayerConfig", "CONFIGS", "VARIANTS", "config_by_name", "make_inputs", "pack_params",
    "unpack_params", "PARAM_NAMES", "BIAS_NAMES", "to_sp", "from_sp",
]

PARAM_NAMES = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
               "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")
BIAS_NAMES = ("b_qkv", "b_o", "b1", "b2")


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    hidden: int
    heads: int
    ffn: int
    seq: int
    micro_batch: int
    tp_size: int
    dtype: str               # "f32" or "bf16"
    seed: int
    init_std: float = 0.02
    out_init_std: float = 0.02   # std of the row-parallel weights (w_o, w2)
    ln_eps: float = 1e-5
    gelu_tanh: int = 0
    causal: int = 1
    swiglu: int = 0               # 1: a = silu(gate) * up instead of GeLU(u)
    disable_bias_linear: int = 0  # 1: no biases in the QKV, out-proj, fc1, fc2 layers
    sequence_parallel: int = 0    # 1: x, y, dx, dy (and LN/residual regions) sequence-sharded

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads

    @property
    def tokens(self) -> int:
        return self.seq * self.micro_batch

    @property
    def fc1_rows(self) -> int:
        """Output width of fc1: f, or 2f (gate and up) with SwiGLU."""
        return 2 * self.ffn if self.swiglu else self.ffn

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)

    def model_flops(self) -> float:
        """fwd+bwd model FLOPs: 3 x forward, causal attention counted as half of s^2."""
        T, h, f = self.tokens, self.hidden, self.ffn
        mlp = (3 if self.swiglu else 2) * h * f  # fc1 (f or 2f outputs) + fc2
        fwd = 2.0 * T * (4 * h * h + mlp) + 2.0 * self.micro_batch * self.seq ** 2 * h
        return 3.0 * fwd


# The five workloads: a tiny fp32 correctness layer and four bf16 GPT layers.
CONFIGS = (
    LayerConfig("tiny-h64-tp2-f32", 64, 4, 256, 32, 2, 2, "f32", 1000),
    LayerConfig("gpt-h1024-bf16", 1024, 16, 4096, 2048, 4, 1, "bf16", 1001),
    LayerConfig("gpt-h4096-tp2-bf16", 4096, 32, 11008, 2048, 1, 2, "bf16", 1002),
    LayerConfig("gpt-h6144-tp4-bf16", 6144, 48, 24576, 4096, 2, 4, "bf16", 1003),
    LayerConfig("gpt-h12288-tp8-bf16", 12288, 96, 49152, 2048, 1, 8, "bf16", 1004,
                out_init_std=0.02 / math.sqrt(2 * 96)),
)


# The MLP/bias variants: a tiny fp32 SwiGLU layer and the h=4096 layer in its LLaMA form
# (SwiGLU over the same f = 11008, no linear biases).
VARIANTS = (
    LayerConfig("tiny-h64-tp2-f32-swiglu", 64, 4, 256, 32, 2, 2, "f32", 1005, swiglu=1),
    LayerConfig("llama-h4096-tp2-bf16-swiglu-nobias", 4096, 32, 11008, 2048, 1, 2, "bf16", 1006,
                swiglu=1, disable_bias_linear=1),
    # sequence-parallel layer with two sequences per micro-batch, so that the shard-major layout
    # is a real permutation of the token order
    LayerConfig("gpt-h4096-tp2-sp-b2-bf16", 4096, 32, 11008, 1024, 2, 2, "bf16", 1007,
                sequence_parallel=1),
)


def to_sp(cfg: LayerConfig, t: torch.Tensor) -> torch.Tensor:
    """[b, s, h] -> the sequence-parallel layout [p][b][s/p][h] (a permutation of rows)."""
    b, s, p = cfg.micro_batch, cfg.seq, cfg.tp_size
    return t.reshape(b, p, s // p, -1).permute(1, 0, 2, 3).contiguous()


def from_sp(cfg: LayerConfig, t: torch.Tensor) -> torch.Tensor:
    """Inverse of to_sp: [p][b][s/p][h] -> [b, s, h]."""
    b, s, p = cfg.micro_batch, cfg.seq, cfg.tp_size
    return t.reshape(p, b, s // p, -1).permute(1, 0, 2, 3).reshape(b, s, -1).contiguous()


def config_by_name(name: str) -> LayerConfig:
    for c in CONFIGS + VARIANTS:
        if c.name == name:
            return c
    raise KeyError(name)


def _randn(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def make_inputs(cfg: LayerConfig, nonzero_affine: bool = False, dy_scale: float = 1.0
                ) -> Dict[str, torch.Tensor]:
    """Draw the full (unsharded) fp32 tensors for one layer, in the fixed order
    x, W_qkv, W_o, W1, W2, dy from torch.Generator('cpu').manual_seed(cfg.seed).

    x ~ N(0,1); weights ~ N(0, init_std) except W_o, W2 ~ N(0, out_init_std); LN gamma=1,
    beta=0; biases 0; dy ~ N(0,1)*dy_scale. With nonzero_affine=True, biases and the LN
    affine parameters are drawn too (after dy, from the same generator) so that tests
    exercise every term. For bf16 configs every tensor is rounded to bf16 and returned as
    the fp32 value of that bf16 number, so both sides see identical inputs.

    Full-layout tensors: x, dy [b, s, h]; w_qkv [3h, h] with rows [Q heads | K heads | V heads]
    (head n of Q = rows n*d..(n+1)*d-1); w_o [h, h]; w1 [f, h]; w2 [h, f]; b_qkv [3h]; b1 [f].
    SwiGLU: w1 [2f, h], b1 [2f] (gate rows, then up rows). disable_bias_linear: no b_* keys.
    """
    h, f, b, s = cfg.hidden, cfg.ffn, cfg.micro_batch, cfg.seq
    g = torch.Generator("cpu").manual_seed(cfg.seed)
    t = {}
    t["x"] = _randn(g, (b, s, h), 1.0)
    t["w_qkv"] = _randn(g, (3 * h, h), cfg.init_std)
    t["w_o"] = _randn(g, (h, h), cfg.out_init_std)
    t["w1"] = _randn(g, (cfg.fc1_rows, h), cfg.init_std)
    t["w2"] = _randn(g, (h, f), cfg.out_init_std)
    t["dy"] = _randn(g, (b, s, h), dy_scale)
    if nonzero_affine:
        t["ln1_g"] = 1.0 + _randn(g, (h,), 0.1)
        t["ln1_b"] = _randn(g, (h,), 0.1)
        t["b_qkv"] = _randn(g, (3 * h,), 0.05)
        t["b_o"] = _randn(g, (h,), 0.05)
        t["ln2_g"] = 1.0 + _randn(g, (h,), 0.1)
        t["ln2_b"] = _randn(g, (h,), 0.1)
        t["b1"] = _randn(g, (cfg.fc1_rows,), 0.05)
        t["b2"] = _randn(g, (h,), 0.05)
    else:
        t["ln1_g"] = torch.ones(h)
        t["ln1_b"] = torch.zeros(h)
        t["b_qkv"] = torch.zeros(3 * h)
        t["b_o"] = torch.zeros(h)
        t["ln2_g"] = torch.ones(h)
        t["ln2_b"] = torch.zeros(h)
        t["b1"] = torch.zeros(cfg.fc1_rows)
        t["b2"] = torch.zeros(h)
    if cfg.dtype == "bf16":
        # LN parameters stay fp32 on the device; everything else is a bf16 tensor there.
        for k in ("x", "dy", "w_qkv", "w_o", "w1", "w2", "b_qkv", "b_o", "b1", "b2"):
            t[k] = t[k].to(torch.bfloat16).to(torch.float32)
    if cfg.disable_bias_linear:  # drawn above all the same, so the other tensors do not move
        for k in BIAS_NAMES:
            del t[k]
    return t


def pack_params(cfg: LayerConfig, full: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Permute full-layout weights into the per-shard packed layout (pure index shuffling)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    d = h // H
    out = {}
    # [3][H][d][h] -> [3][p][H/p][d][h] -> [p][3][H/p][d][h]
    out["w_qkv"] = (full["w_qkv"].reshape(3, p, H // p, d, h).permute(1, 0, 2, 3, 4)
                    .contiguous())
    if "b_qkv" in full:
        out["b_qkv"] = full["b_qkv"].reshape(3, p, H // p, d).permute(1, 0, 2, 3).contiguous()
    # [h][p][h/p] -> [p][h][h/p]
    out["w_o"] = full["w_o"].reshape(h, p, h // p).permute(1, 0, 2).contiguous()
    if cfg.swiglu:  # [2][p][f/p][h] (gate rows, then up rows) -> [p][2][f/p][h]
        out["w1"] = full["w1"].reshape(2, p, f // p, h).permute(1, 0, 2, 3).contiguous()
        if "b1" in full:
            out["b1"] = full["b1"].reshape(2, p, f // p).permute(1, 0, 2).contiguous()
    else:
        out["w1"] = full["w1"].reshape(p, f // p, h).contiguous()
        if "b1" in full:
            out["b1"] = full["b1"].reshape(p, f // p).contiguous()
    out["w2"] = full["w2"].reshape(h, p, f // p).permute(1, 0, 2).contiguous()
    for k in ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b2"):
        if k in full:
            out[k] = full[k].clone()
    return out


def unpack_params(cfg: LayerConfig, packed: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Inverse of pack_params (also used to gather packed gradients)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    d = h // H
    out = {}
    out["w_qkv"] = (packed["w_qkv"].reshape(p, 3, H // p, d, h).permute(1, 0, 2, 3, 4)
                    .reshape(3 * h, h).contiguous())
    if "b_qkv" in packed:
        out["b_qkv"] = (packed["b_qkv"].reshape(p, 3, H // p, d).permute(1, 0, 2, 3)
                        .reshape(3 * h))
    out["w_o"] = packed["w_o"].reshape(p, h, h // p).permute(1, 0, 2).reshape(h, h).contiguous()
    if cfg.swiglu:
        out["w1"] = (packed["w1"].reshape(p, 2, f // p, h).permute(1, 0, 2, 3)
                     .reshape(2 * f, h).contiguous())
        if "b1" in packed:
            out["b1"] = packed["b1"].reshape(p, 2, f // p).permute(1, 0, 2).reshape(2 * f)
    else:
        out["w1"] = packed["w1"].reshape(f, h).contiguous()
        if "b1" in packed:
            out["b1"] = packed["b1"].reshape(f).contiguous()
    out["w2"] = packed["w2"].reshape(p, h, f // p).permute(1, 0, 2).reshape(h, f).contiguous()
    for k in ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b2"):
        if k in packed:
            out[k] = packed[k].clone()
    return out
