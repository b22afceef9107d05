"""fp64 oracle of the layer split across real tensor-parallel ranks: rank t holds only shard t
of the packed parameters (plus the replicated LayerNorm parameters and row-parallel biases)
and computes only its shard. Every place where the single-process oracle sums over shards
becomes an all-reduce (sum) across the ranks:
  forward:  the out-proj partials O_t W_o,t^T and the fc2 partials a_t W2,t^T
            (the AllReduce after the row-parallel layer);
  backward: the dln2 contributions du_t W1,t and the dln1 contributions dqkv_t W_qkv,t
            (the input of a column-parallel layer is replicated, so its gradient is the sum
            of the shards' contributions).
LayerNorm, the residuals and the replicated parameters' gradients are computed redundantly
on every rank from all-reduced data, so they agree across ranks without further exchange.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "Megatron-LM 3D并行原理与万亿参数训练实战指南" (trdm.cn), section 2.1 (tensor
parallelism): Q/K/V split by output columns with x broadcast to every rank and no
communication; W_o split by input rows with the ranks' partial outputs summed by an
AllReduce. The page names the forward reduction. The backward's two are its adjoint (the
reading the single-process oracle states: a broadcast input's gradient is the sum of the
shards' contributions).

all_reduce: a function taking a float64 numpy array and returning the elementwise sum of that
array over all ranks (every rank calls it with the same shape, in the same order).
"""
from __future__ import annotations

import numpy as np

from .layer import (_flags, _np, attention_bwd, attention_fwd, gelu, gelu_grad, layer_norm,
                    layer_norm_grad, swiglu, swiglu_grad)

REPLICATED = ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b2")
SHARDED = ("w_qkv", "b_qkv", "w_o", "w1", "b1", "w2")


def rank_shard(packed, rank):
    """The parameters rank `rank` holds: its slice [rank] of every packed sharded tensor and
    the replicated ones whole."""
    out = {}
    for k, v in packed.items():
        v = _np(v)
        out[k] = v[rank] if k in SHARDED else v
    return out


def layer_fwd_rank(cfg, shard, x, all_reduce):
    """Forward on one rank. x: [b, s, h] (replicated). Returns (y [b, s, h], saved)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp = b * s, h // H, H // p
    sw, nb = _flags(cfg)
    x2 = _np(x).reshape(T, h)
    ln1, _, rstd1, xhat1 = layer_norm(x2, shard["ln1_g"], shard["ln1_b"], cfg.ln_eps)
    # column-parallel QKV: this rank's heads only
    qkv = ln1 @ shard["w_qkv"].reshape(3 * hp * d, h).T
    if not nb:
        qkv = qkv + shard["b_qkv"].reshape(-1)
    qkv = qkv.reshape(T, 1, 3, hp, d)
    O, lse = attention_fwd(qkv, b, s, hp, 1)
    # row-parallel out-proj: partial sum of this rank, all-reduced, then b_o and x once
    h1 = x2 + all_reduce(O.reshape(T, h // p) @ shard["w_o"].T)
    if not nb:
        h1 = h1 + shard["b_o"]
    ln2, _, rstd2, xhat2 = layer_norm(h1, shard["ln2_g"], shard["ln2_b"], cfg.ln_eps)
    if sw:  # this rank's gate and up halves
        u = np.stack([ln2 @ shard["w1"][c].T + (0.0 if nb else shard["b1"][c])
                      for c in range(2)], axis=1)  # [T][2][f/p]
        a = swiglu(u[:, 0], u[:, 1])
    else:
        u = ln2 @ shard["w1"].T + (0.0 if nb else shard["b1"])
        a = gelu(u, cfg.gelu_tanh)
    y = h1 + all_reduce(a @ shard["w2"].T)
    if not nb:
        y = y + shard["b2"]
    saved = dict(ln1=ln1, rstd1=rstd1, xhat1=xhat1, qkv=qkv, O=O, lse=lse, h1=h1, ln2=ln2,
                 rstd2=rstd2, xhat2=xhat2, u=u, a=a)
    return y.reshape(b, s, h), saved


def layer_bwd_rank(cfg, shard, saved, dy, all_reduce):
    """Backward on one rank. dy: [b, s, h] (replicated). Returns (dx [b, s, h], grads of this
    rank's parameters: its shard of every sharded tensor, the replicated ones whole)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp = b * s, h // H, H // p
    sw, nb = _flags(cfg)
    dy2 = _np(dy).reshape(T, h)
    g = {}
    # fc2 (row-parallel)
    if not nb:
        g["b2"] = dy2.sum(axis=0)
    g["w2"] = dy2.T @ saved["a"]
    da = dy2 @ shard["w2"]
    u = saved["u"]
    du = np.stack(swiglu_grad(u[:, 0], u[:, 1], da), axis=1) if sw else \
        da * gelu_grad(u, cfg.gelu_tanh)
    # fc1 (column-parallel): ln2's gradient sums the ranks' contributions
    rows = (2 if sw else 1) * (f // p)
    du2 = du.reshape(T, rows)
    if not nb:
        g["b1"] = du.sum(axis=0)
    g["w1"] = (du2.T @ saved["ln2"]).reshape(shard["w1"].shape)
    dln2 = all_reduce(du2 @ shard["w1"].reshape(rows, h))
    d_ln, g["ln2_g"], g["ln2_b"] = layer_norm_grad(dln2, saved["xhat2"], saved["rstd2"],
                                                   shard["ln2_g"])
    dh1 = dy2 + d_ln
    # out-proj (row-parallel)
    if not nb:
        g["b_o"] = dh1.sum(axis=0)
    g["w_o"] = dh1.T @ saved["O"].reshape(T, h // p)
    dO = (dh1 @ shard["w_o"]).reshape(T, 1, hp, d)
    dqkv = attention_bwd(saved["qkv"], dO, b, s, hp, 1).reshape(T, 3 * hp * d)
    # QKV (column-parallel): ln1's gradient sums the ranks' contributions
    if not nb:
        g["b_qkv"] = dqkv.sum(axis=0).reshape(3, hp, d)
    g["w_qkv"] = (dqkv.T @ saved["ln1"]).reshape(3, hp, d, h)
    dln1 = all_reduce(dqkv @ shard["w_qkv"].reshape(3 * hp * d, h))
    d_ln1, g["ln1_g"], g["ln1_b"] = layer_norm_grad(dln1, saved["xhat1"], saved["rstd1"],
                                                    shard["ln1_g"])
    dx = dh1 + d_ln1
    return dx.reshape(b, s, h), g
