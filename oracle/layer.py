"""fp64 oracle: the plain definition of one pre-LayerNorm GPT layer with Megatron-style
tensor-parallel partitioning, forward and hand-written reverse-mode backward.

TEST INFRASTRUCTURE ONLY (see the package docstring). Float64 numpy throughout; the only
library primitives are matmul, exp, log, tanh and scipy's erf.

Sources (web pages about Megatron-LM; they print no formulas, so each reading is stated):
  [TP]   "Megatron-LM 3D并行原理与万亿参数训练实战指南" (trdm.cn), section 2.1 (tensor
         parallelism): W_q/W_k/W_v column-split, x broadcast to every shard, each shard
         computes its own heads without communication; W_o row-split, each shard's partial
         output summed by AllReduce; the softmax needs whole heads, hence column-then-row.
  [API]  "Megatron-LM：NVIDIA大模型训练框架" (second-brain-czx), section "张量并行":
         ColumnParallelLinear(h, 3h, gather_output=False) then RowParallelLinear(h, h,
         input_is_parallel=True) around the attention.
  [MD]   the trdm.cn page, section 3.2 (model definition): LayerNorm statistics global over the
         hidden dimension; hidden and head counts divisible by tp_size; softmax in fp32
         (attention_softmax_in_fp32); apply_query_key_layer_scaling flag.
  [ACT]  the trdm.cn page, section 3.3 (launch flags): GeLU is the default MLP activation.
  [RC]   the trdm.cn page, section 4.1 (checkpointing / recompute): only the layer input is
         kept and intermediates are recomputed in backward -- mathematically the identity.
  [VAR]  the trdm.cn page, section 3.3 (launch flags): --swiglu replaces GeLU by SwiGLU, and
         --disable-bias-linear removes the biases of the linear layers.
  [SP]   "Megatron-LM：NVIDIA大模型训练框架" (second-brain-czx), sequence-parallel section: the
         LayerNorm / dropout / residual regions are split along the sequence across the tensor-
         parallel ranks, an all-gather precedes the column-parallel layer and a reduce-scatter
         replaces the all-reduce after the row-parallel one.

Readings where the pages are silent (each also listed in the design notes):
  * LayerNorm: biased variance (divide by h), eps inside the square root, affine gamma/beta.
  * Pre-LN block with two LayerNorms and two residuals: y = h1 + MLP(LN2(h1)),
    h1 = x + Attn(LN1(x)).
  * Softmax scale 1/sqrt(d); query-key layer scaling is an identity under an fp32 softmax.
  * Causal mask: key j visible to query i iff j <= i; masked probabilities are exactly 0.
  * Row-parallel biases (b_o, b2) are added once, after the shard sum.
  * GeLU exact: u * Phi(u); the tanh form is selected by gelu_tanh=1.
  * QKV packing: shard-major, then [Q|K|V], then head, then head_dim.
  * No dropout.
  * SwiGLU: fc1 gives two halves per shard, gate then up (each f/p wide); a = silu(gate)*up
    with silu(z) = z*sigmoid(z); fc2 is unchanged (input width f).
  * disable_bias_linear: b_qkv, b_o, b1, b2 are absent (not zero) and get no gradient; the
    LayerNorm affine parameters stay.
  * sequence_parallel: shard t owns positions t*s/p .. (t+1)*s/p - 1 of every sequence of x, y,
    dx, dy and of the LN/residual activations, held shard-major as [p][b][s/p][h]; in the
    backward the all-gather's adjoint is a reduce-scatter and the reduce-scatter's an
    all-gather, and the replicated LayerNorm parameters' gradients are summed over shards.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

f64 = np.float64


# ----------------------------------------------------------------------------- LayerNorm
def layer_norm(x, gamma, beta, eps):
    """LN over the last axis of x [rows, h]: mean, biased variance, xhat=(x-mean)*rstd,
    y = gamma*xhat + beta. Statistics are over the full hidden dimension on every shard
    ([MD]: the normalisation statistics must agree across the TP group; under the column/row
    split the LN input is replicated, so each shard sees the whole row).
    Returns (y, mean, rstd, xhat)."""
    x = np.asarray(x, f64)
    mean = x.mean(axis=-1)
    var = ((x - mean[:, None]) ** 2).mean(axis=-1)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mean[:, None]) * rstd[:, None]
    return xhat * gamma + beta, mean, rstd, xhat


def layer_norm_grad(dy, xhat, rstd, gamma):
    """Reverse of layer_norm given the upstream grad dy [rows, h].
    With g = dy*gamma: dx = rstd * (g - mean(g) - xhat * mean(g*xhat)),
    dgamma = sum_rows dy*xhat, dbeta = sum_rows dy."""
    g = dy * gamma
    dx = rstd[:, None] * (g - g.mean(axis=-1, keepdims=True)
                          - xhat * (g * xhat).mean(axis=-1, keepdims=True))
    return dx, (dy * xhat).sum(axis=0), dy.sum(axis=0)


# ----------------------------------------------------------------------------- GeLU ([ACT])
_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
_TANH_C = 0.044715


def gelu(u, tanh_approx=0):
    """Exact GeLU u*Phi(u) = u/2 * (1 + erf(u/sqrt 2)); tanh form if tanh_approx."""
    if tanh_approx:
        return 0.5 * u * (1.0 + np.tanh(_SQRT_2_OVER_PI * (u + _TANH_C * u ** 3)))
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def gelu_grad(u, tanh_approx=0):
    """d GeLU / du: exact form Phi(u) + u*phi(u)."""
    if tanh_approx:
        z = _SQRT_2_OVER_PI * (u + _TANH_C * u ** 3)
        t = np.tanh(z)
        return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * _SQRT_2_OVER_PI * (
            1.0 + 3.0 * _TANH_C * u * u)
    cdf = 0.5 * (1.0 + erf(u / math.sqrt(2.0)))
    pdf = np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    return cdf + u * pdf


# ----------------------------------------------------------------------------- attention
def causal_softmax(S):
    """Row-wise softmax of S [s, s] over the visible keys j <= i; masked entries are 0.
    Returns (P, lse) with lse_i = log sum_{j<=i} exp(S_ij)."""
    s = S.shape[0]
    mask = np.tril(np.ones((s, s), dtype=bool))
    Sm = np.where(mask, S, -np.inf)
    m = Sm.max(axis=1)
    e = np.where(mask, np.exp(Sm - m[:, None]), 0.0)
    z = e.sum(axis=1)
    return e / z[:, None], m + np.log(z)


def attention_head_fwd(q, k, v):
    """One head of causal attention on q, k, v [s, d]: S = q k^T / sqrt(d) (scale reading),
    P = causal softmax (kept in full precision, [MD]), o = P v. Returns (o, lse, P)."""
    d = q.shape[1]
    P, lse = causal_softmax((q @ k.T) / math.sqrt(d))
    return P @ v, lse, P


def attention_head_bwd(q, k, v, P, do):
    """Reverse of attention_head_fwd: dv = P^T do; dP = do v^T; dS = P*(dP - rowsum(P*dP));
    dq = dS k / sqrt(d); dk = dS^T q / sqrt(d)."""
    d = q.shape[1]
    dv = P.T @ do
    dP = do @ v.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    return dS @ k / math.sqrt(d), dS.T @ q / math.sqrt(d), dv


def attention_fwd(qkv, b, s, heads, tp):
    """Causal attention over a packed qkv [b*s, p, 3, H/p, d]: each shard owns whole heads
    ([TP]: column-split Q/K/V let each shard run its heads' softmax locally).
    Returns O [b*s, p, H/p, d] and lse [b, H, s]."""
    T = b * s
    hp = heads // tp
    d = qkv.shape[-1]
    O = np.empty((T, tp, hp, d))
    lse = np.empty((b, heads, s))
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for t in range(tp):
            for j in range(hp):
                o, l, _ = attention_head_fwd(qkv[rows, t, 0, j], qkv[rows, t, 1, j],
                                             qkv[rows, t, 2, j])
                O[rows, t, j] = o
                lse[bi, t * hp + j] = l
    return O, lse


def attention_bwd(qkv, dO, b, s, heads, tp):
    """Backward of attention_fwd; P is recomputed from q and k ([RC]). Returns dqkv in the
    packed layout of qkv."""
    hp = heads // tp
    dqkv = np.empty_like(qkv)
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for t in range(tp):
            for j in range(hp):
                q, k, v = qkv[rows, t, 0, j], qkv[rows, t, 1, j], qkv[rows, t, 2, j]
                _, _, P = attention_head_fwd(q, k, v)
                dq, dk, dv = attention_head_bwd(q, k, v, P, dO[rows, t, j])
                dqkv[rows, t, 0, j] = dq
                dqkv[rows, t, 1, j] = dk
                dqkv[rows, t, 2, j] = dv
    return dqkv


# ----------------------------------------------------------------------------- SwiGLU ([VAR])
def sigmoid(z):
    """Logistic function 1/(1+exp(-z)), written as (1 + tanh(z/2))/2 (the same function,
    without overflow for large |z|)."""
    return 0.5 * (1.0 + np.tanh(0.5 * z))


def silu(z):
    """SiLU (swish): z * sigmoid(z)."""
    return z * sigmoid(z)


def silu_grad(z):
    """d/dz [z*sigmoid(z)] = sigmoid(z) * (1 + z*(1 - sigmoid(z)))."""
    sg = sigmoid(z)
    return sg * (1.0 + z * (1.0 - sg))


def swiglu(gate, up):
    """SwiGLU activation: silu(gate) * up, elementwise."""
    return silu(gate) * up


def swiglu_grad(gate, up, da):
    """Reverse of swiglu for the upstream grad da: (d gate, d up)."""
    return da * up * silu_grad(gate), da * silu(gate)


# ----------------------------------------------------------------------------- the layer
def _flags(cfg):
    return bool(getattr(cfg, "swiglu", 0)), bool(getattr(cfg, "disable_bias_linear", 0))


def _np(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().to(dtype=__import__("torch").float64).numpy()
    return np.asarray(a, f64)


def layer_fwd(cfg, params, x):
    """Forward of the layer on packed per-shard parameters (the TP path); with
    cfg.sequence_parallel, x and y are in the sequence-parallel layout (layer_fwd_sp).

    cfg: object with hidden, heads, ffn, seq, micro_batch, tp_size, ln_eps, gelu_tanh and
    optionally swiglu, disable_bias_linear.
    params: dict of packed arrays (layouts in the mgt_inputs docstring). x: [b, s, h].
    Returns (y [b, s, h], saved dict of every intermediate)."""
    if getattr(cfg, "sequence_parallel", 0):
        return layer_fwd_sp(cfg, params, x)
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp = b * s, h // H, H // p
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    bias = (lambda key: 0.0) if nb else (lambda key: P[key])  # noqa: E731
    x2 = _np(x).reshape(T, h)

    ln1, mu1, rstd1, xhat1 = layer_norm(x2, P["ln1_g"], P["ln1_b"], cfg.ln_eps)
    # Column-parallel QKV ([TP], [API]): every shard multiplies the replicated ln1 by its own
    # row block of W_qkv; no reduction.
    qkv = np.empty((T, p, 3, hp, d))
    for t in range(p):
        w_t = P["w_qkv"][t].reshape(3 * hp * d, h)
        b_t = 0.0 if nb else P["b_qkv"][t].reshape(-1)
        qkv[:, t] = (ln1 @ w_t.T + b_t).reshape(T, 3, hp, d)
    O, lse = attention_fwd(qkv, b, s, H, p)
    # Row-parallel out-proj ([TP]): shard t multiplies its slice of the attention output by
    # its input-column block of W_o; the partials are summed (the AllReduce), then b_o is
    # added once and the residual x.
    acc = np.zeros((T, h))
    for t in range(p):
        acc += O[:, t].reshape(T, h // p) @ P["w_o"][t].T
    h1 = x2 + bias("b_o") + acc
    ln2, mu2, rstd2, xhat2 = layer_norm(h1, P["ln2_g"], P["ln2_b"], cfg.ln_eps)
    # Column-parallel fc1 + activation, row-parallel fc2 with shard sum, bias once, residual.
    if sw:  # u [T][p][2][f/p]: each shard's gate half, then its up half
        u = np.empty((T, p, 2, f // p))
        for t in range(p):
            for c in range(2):
                u[:, t, c] = ln2 @ P["w1"][t, c].T + (0.0 if nb else P["b1"][t, c])
        a = swiglu(u[:, :, 0], u[:, :, 1])
    else:
        u = np.empty((T, p, f // p))
        for t in range(p):
            u[:, t] = ln2 @ P["w1"][t].T + (0.0 if nb else P["b1"][t])
        a = gelu(u, cfg.gelu_tanh)
    acc2 = np.zeros((T, h))
    for t in range(p):
        acc2 += a[:, t] @ P["w2"][t].T
    y = h1 + bias("b2") + acc2
    saved = dict(x=x2, ln1=ln1, mu1=mu1, rstd1=rstd1, xhat1=xhat1, qkv=qkv, O=O, lse=lse,
                 h1=h1, ln2=ln2, mu2=mu2, rstd2=rstd2, xhat2=xhat2, u=u, a=a)
    return y.reshape(b, s, h), saved


def layer_bwd(cfg, params, saved, dy):
    """Hand-written reverse of layer_fwd (packed TP path). Returns (dx [b,s,h], grads in the
    packed parameter layout, intermediate grads); with cfg.sequence_parallel, dy and dx are in
    the sequence-parallel layout (layer_bwd_sp)."""
    if getattr(cfg, "sequence_parallel", 0):
        return layer_bwd_sp(cfg, params, saved, dy)
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp = b * s, h // H, H // p
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    dy2 = _np(dy).reshape(T, h)
    g = {}
    # fc2 (row-parallel): y = h1 + b2 + sum_t a_t W2_t^T
    if not nb:
        g["b2"] = dy2.sum(axis=0)
    g["w2"] = np.empty((p, h, f // p))
    da = np.empty((T, p, f // p))
    for t in range(p):
        g["w2"][t] = dy2.T @ saved["a"][:, t]
        da[:, t] = dy2 @ P["w2"][t]
    u = saved["u"]
    if sw:
        du = np.stack(swiglu_grad(u[:, :, 0], u[:, :, 1], da), axis=2)  # [T][p][2][f/p]
    else:
        du = da * gelu_grad(u, cfg.gelu_tanh)
    # fc1 (column-parallel): the input ln2 was broadcast to every shard, so its gradient is
    # the sum of the shards' contributions.
    if not nb:
        g["b1"] = du.sum(axis=0)
    rows = (2 if sw else 1) * (f // p)  # fc1 output rows per shard
    g["w1"] = np.empty((p,) + P["w1"].shape[1:])
    dln2 = np.zeros((T, h))
    for t in range(p):
        du_t = du[:, t].reshape(T, rows)
        g["w1"][t] = (du_t.T @ saved["ln2"]).reshape(P["w1"].shape[1:])
        dln2 += du_t @ P["w1"][t].reshape(rows, h)
    d_ln, g["ln2_g"], g["ln2_b"] = layer_norm_grad(dln2, saved["xhat2"], saved["rstd2"],
                                                   P["ln2_g"])
    dh1 = dy2 + d_ln
    # out-proj (row-parallel)
    if not nb:
        g["b_o"] = dh1.sum(axis=0)
    g["w_o"] = np.empty((p, h, h // p))
    dO = np.empty((T, p, hp, d))
    for t in range(p):
        g["w_o"][t] = dh1.T @ saved["O"][:, t].reshape(T, h // p)
        dO[:, t] = (dh1 @ P["w_o"][t]).reshape(T, hp, d)
    dqkv = attention_bwd(saved["qkv"], dO, b, s, H, p)
    # QKV (column-parallel)
    if not nb:
        g["b_qkv"] = np.empty((p, 3, hp, d))
    g["w_qkv"] = np.empty((p, 3, hp, d, h))
    dln1 = np.zeros((T, h))
    for t in range(p):
        dq_t = dqkv[:, t].reshape(T, 3 * hp * d)
        if not nb:
            g["b_qkv"][t] = dq_t.sum(axis=0).reshape(3, hp, d)
        g["w_qkv"][t] = (dq_t.T @ saved["ln1"]).reshape(3, hp, d, h)
        dln1 += dq_t @ P["w_qkv"][t].reshape(3 * hp * d, h)
    d_ln1, g["ln1_g"], g["ln1_b"] = layer_norm_grad(dln1, saved["xhat1"], saved["rstd1"],
                                                    P["ln1_g"])
    dx = dh1 + d_ln1
    inter = dict(du=du, dln2=dln2, dh1=dh1, dO=dO, dqkv=dqkv, dln1=dln1)
    return dx.reshape(b, s, h), g, inter


# ----------------------------------------------------------------------------- sequence parallel
def all_gather_seq(xs, b, s, p):
    """Sequence all-gather: the shards' pieces [p][b][s/p][n] -> the whole [b*s, n] in token
    order, shard t's piece at positions t*s/p .. (t+1)*s/p - 1 of every sequence ([SP])."""
    sp = s // p
    full = np.empty((b, s, xs.shape[-1]))
    for t in range(p):
        full[:, t * sp:(t + 1) * sp] = xs[t]
    return full.reshape(b * s, -1)


def reduce_scatter_seq(parts, b, s, p):
    """Sequence reduce-scatter: the p shards' partial sums over all tokens ([b*s, n] each) are
    added, and shard t keeps its positions: -> [p][b][s/p][n] ([SP])."""
    sp = s // p
    total = np.zeros_like(parts[0])
    for q in parts:
        total = total + q
    full = total.reshape(b, s, -1)
    return np.stack([full[:, t * sp:(t + 1) * sp] for t in range(p)])


def layer_fwd_sp(cfg, params, x_sp):
    """The layer with sequence parallelism ([SP]): x_sp [p][b][s/p][h]. Each shard normalises
    its own positions; the column-parallel layers run on the all-gathered LayerNorm output;
    the row-parallel partial sums are reduce-scattered back to the sequence shards before the
    bias and the residual. Returns (y [p][b][s/p][h], saved)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp, sp = b * s, h // H, H // p, s // p
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    bias = (lambda key: 0.0) if nb else (lambda key: P[key])  # noqa: E731
    xs = _np(x_sp).reshape(p, b, sp, h)

    def shard_ln(src, g, be):
        out = np.empty_like(src)
        xhat = np.empty_like(src)
        rstd = np.empty((p, b * sp))
        for t in range(p):
            y_, _, r_, xh_ = layer_norm(src[t].reshape(b * sp, h), g, be, cfg.ln_eps)
            out[t] = y_.reshape(b, sp, h)
            xhat[t] = xh_.reshape(b, sp, h)
            rstd[t] = r_
        return out, xhat, rstd

    ln1_s, xhat1, rstd1 = shard_ln(xs, P["ln1_g"], P["ln1_b"])
    ln1 = all_gather_seq(ln1_s, b, s, p)
    qkv = np.empty((T, p, 3, hp, d))
    for t in range(p):
        w_t = P["w_qkv"][t].reshape(3 * hp * d, h)
        b_t = 0.0 if nb else P["b_qkv"][t].reshape(-1)
        qkv[:, t] = (ln1 @ w_t.T + b_t).reshape(T, 3, hp, d)
    O, lse = attention_fwd(qkv, b, s, H, p)
    z = reduce_scatter_seq([O[:, t].reshape(T, h // p) @ P["w_o"][t].T for t in range(p)],
                           b, s, p)
    h1_s = xs + bias("b_o") + z
    ln2_s, xhat2, rstd2 = shard_ln(h1_s, P["ln2_g"], P["ln2_b"])
    ln2 = all_gather_seq(ln2_s, b, s, p)
    if sw:
        u = np.empty((T, p, 2, f // p))
        for t in range(p):
            for c in range(2):
                u[:, t, c] = ln2 @ P["w1"][t, c].T + (0.0 if nb else P["b1"][t, c])
        a = swiglu(u[:, :, 0], u[:, :, 1])
    else:
        u = np.empty((T, p, f // p))
        for t in range(p):
            u[:, t] = ln2 @ P["w1"][t].T + (0.0 if nb else P["b1"][t])
        a = gelu(u, cfg.gelu_tanh)
    z2 = reduce_scatter_seq([a[:, t] @ P["w2"][t].T for t in range(p)], b, s, p)
    y_s = h1_s + bias("b2") + z2
    # the layout-held activations in the shard-major row order ([p][b][s/p] flattened)
    saved = dict(x=xs, ln1=ln1_s.reshape(T, h), ln1_full=ln1, xhat1=xhat1, rstd1=rstd1,
                 qkv=qkv, O=O, lse=lse, h1=h1_s.reshape(T, h), ln2=ln2_s.reshape(T, h),
                 ln2_full=ln2, xhat2=xhat2, rstd2=rstd2, u=u, a=a)
    return y_s, saved


def layer_bwd_sp(cfg, params, saved, dy_sp):
    """Reverse of layer_fwd_sp: the all-gathers' adjoints are reduce-scatters and vice versa;
    LayerNorm parameter gradients are summed over the shards. Returns (dx [p][b][s/p][h],
    grads, intermediate grads with the sequence-parallel ones in the shard-major row order)."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s = cfg.micro_batch, cfg.seq
    T, d, hp, sp = b * s, h // H, H // p, s // p
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    dys = _np(dy_sp).reshape(p, b, sp, h)
    g = {}
    dy = all_gather_seq(dys, b, s, p)  # adjoint of the reduce-scatter after fc2
    if not nb:
        g["b2"] = dy.sum(axis=0)
    g["w2"] = np.empty((p, h, f // p))
    da = np.empty((T, p, f // p))
    for t in range(p):
        g["w2"][t] = dy.T @ saved["a"][:, t]
        da[:, t] = dy @ P["w2"][t]
    u = saved["u"]
    if sw:
        du = np.stack(swiglu_grad(u[:, :, 0], u[:, :, 1], da), axis=2)
    else:
        du = da * gelu_grad(u, cfg.gelu_tanh)
    if not nb:
        g["b1"] = du.sum(axis=0)
    rows = (2 if sw else 1) * (f // p)
    g["w1"] = np.empty((p,) + P["w1"].shape[1:])
    parts = []
    for t in range(p):
        du_t = du[:, t].reshape(T, rows)
        g["w1"][t] = (du_t.T @ saved["ln2_full"]).reshape(P["w1"].shape[1:])
        parts.append(du_t @ P["w1"][t].reshape(rows, h))
    dln2_s = reduce_scatter_seq(parts, b, s, p)  # adjoint of the all-gather before fc1

    def shard_ln_grad(dsrc, xhat, rstd, gam):
        dx_ = np.empty_like(dsrc)
        dg, dbe = np.zeros(h), np.zeros(h)
        for t in range(p):
            a_, g_, b_ = layer_norm_grad(dsrc[t].reshape(b * sp, h),
                                         xhat[t].reshape(b * sp, h), rstd[t], gam)
            dx_[t] = a_.reshape(b, sp, h)
            dg += g_
            dbe += b_
        return dx_, dg, dbe

    d_ln, g["ln2_g"], g["ln2_b"] = shard_ln_grad(dln2_s, saved["xhat2"], saved["rstd2"],
                                                 P["ln2_g"])
    dh1_s = dys + d_ln
    if not nb:
        g["b_o"] = dh1_s.reshape(T, h).sum(axis=0)
    dh1 = all_gather_seq(dh1_s, b, s, p)  # adjoint of the reduce-scatter after out-proj
    g["w_o"] = np.empty((p, h, h // p))
    dO = np.empty((T, p, hp, d))
    for t in range(p):
        g["w_o"][t] = dh1.T @ saved["O"][:, t].reshape(T, h // p)
        dO[:, t] = (dh1 @ P["w_o"][t]).reshape(T, hp, d)
    dqkv = attention_bwd(saved["qkv"], dO, b, s, H, p)
    if not nb:
        g["b_qkv"] = np.empty((p, 3, hp, d))
    g["w_qkv"] = np.empty((p, 3, hp, d, h))
    parts = []
    for t in range(p):
        dq_t = dqkv[:, t].reshape(T, 3 * hp * d)
        if not nb:
            g["b_qkv"][t] = dq_t.sum(axis=0).reshape(3, hp, d)
        g["w_qkv"][t] = (dq_t.T @ saved["ln1_full"]).reshape(3, hp, d, h)
        parts.append(dq_t @ P["w_qkv"][t].reshape(3 * hp * d, h))
    dln1_s = reduce_scatter_seq(parts, b, s, p)  # adjoint of the all-gather before QKV
    d_ln1, g["ln1_g"], g["ln1_b"] = shard_ln_grad(dln1_s, saved["xhat1"], saved["rstd1"],
                                                  P["ln1_g"])
    dx_s = dh1_s + d_ln1
    inter = dict(du=du, dln2=dln2_s.reshape(T, h), dh1=dh1_s.reshape(T, h), dO=dO, dqkv=dqkv,
                 dln1=dln1_s.reshape(T, h))
    return dx_s, g, inter


def layer_fwd_full(cfg, params, x):
    """The same layer on full, unsharded matrices (no tensor parallelism): w_qkv [3h, h] with
    rows [Q | K | V], head n of each at rows n*d..(n+1)*d-1; w_o [h, h]; w1 [f, h] (SwiGLU:
    [2f, h], gate rows then up rows); w2 [h, f].
    Used to check that the sharded computation equals the unsharded one."""
    h, H, f = cfg.hidden, cfg.heads, cfg.ffn
    b, s = cfg.micro_batch, cfg.seq
    T, d = b * s, h // H
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    bias = (lambda key: 0.0) if nb else (lambda key: P[key])  # noqa: E731
    x2 = _np(x).reshape(T, h)
    ln1, mu1, rstd1, xhat1 = layer_norm(x2, P["ln1_g"], P["ln1_b"], cfg.ln_eps)
    qkv = ln1 @ P["w_qkv"].T + bias("b_qkv")
    O = np.empty((T, h))
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for n in range(H):
            c = slice(n * d, (n + 1) * d)
            o, _, _ = attention_head_fwd(qkv[rows, c], qkv[rows, h:][:, c],
                                         qkv[rows, 2 * h:][:, c])
            O[rows, c] = o
    h1 = x2 + O @ P["w_o"].T + bias("b_o")
    ln2, mu2, rstd2, xhat2 = layer_norm(h1, P["ln2_g"], P["ln2_b"], cfg.ln_eps)
    u = ln2 @ P["w1"].T + bias("b1")
    a = swiglu(u[:, :f], u[:, f:]) if sw else gelu(u, cfg.gelu_tanh)
    y = h1 + a @ P["w2"].T + bias("b2")
    saved = dict(x=x2, ln1=ln1, xhat1=xhat1, rstd1=rstd1, qkv=qkv, O=O, h1=h1, ln2=ln2,
                 xhat2=xhat2, rstd2=rstd2, u=u, a=a)
    return y.reshape(b, s, h), saved


def layer_bwd_full(cfg, params, saved, dy):
    """Reverse of layer_fwd_full. Returns (dx, grads in the full layout)."""
    h, H, f = cfg.hidden, cfg.heads, cfg.ffn
    b, s = cfg.micro_batch, cfg.seq
    T, d = b * s, h // H
    sw, nb = _flags(cfg)
    P = {k: _np(v) for k, v in params.items()}
    dy2 = _np(dy).reshape(T, h)
    g = {}
    if not nb:
        g["b2"] = dy2.sum(axis=0)
    g["w2"] = dy2.T @ saved["a"]
    da = dy2 @ P["w2"]
    u = saved["u"]
    if sw:
        du = np.concatenate(swiglu_grad(u[:, :f], u[:, f:], da), axis=1)
    else:
        du = da * gelu_grad(u, cfg.gelu_tanh)
    if not nb:
        g["b1"] = du.sum(axis=0)
    g["w1"] = du.T @ saved["ln2"]
    d_ln, g["ln2_g"], g["ln2_b"] = layer_norm_grad(du @ P["w1"], saved["xhat2"],
                                                   saved["rstd2"], P["ln2_g"])
    dh1 = dy2 + d_ln
    if not nb:
        g["b_o"] = dh1.sum(axis=0)
    g["w_o"] = dh1.T @ saved["O"]
    dO = dh1 @ P["w_o"]
    qkv = saved["qkv"]
    dqkv = np.empty_like(qkv)
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for n in range(H):
            c = slice(n * d, (n + 1) * d)
            q, k, v = qkv[rows, c], qkv[rows, h:][:, c], qkv[rows, 2 * h:][:, c]
            _, _, Pm = attention_head_fwd(q, k, v)
            dq, dk, dv = attention_head_bwd(q, k, v, Pm, dO[rows, c])
            dqkv[rows, n * d:(n + 1) * d] = dq
            dqkv[rows, h + n * d:h + (n + 1) * d] = dk
            dqkv[rows, 2 * h + n * d:2 * h + (n + 1) * d] = dv
    if not nb:
        g["b_qkv"] = dqkv.sum(axis=0)
    g["w_qkv"] = dqkv.T @ saved["ln1"]
    d_ln1, g["ln1_g"], g["ln1_b"] = layer_norm_grad(dqkv @ P["w_qkv"], saved["xhat1"],
                                                    saved["rstd1"], P["ln1_g"])
    dx = dh1 + d_ln1
    return dx.reshape(b, s, h), g


def gather_grads(cfg, g):
    """Packed per-shard gradients -> full layout (index permutation, the inverse of the
    packing), so sharded results can be compared with layer_bwd_full."""
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    d, hp = h // H, H // p
    sw, _ = _flags(cfg)
    out = dict(g)
    out["w_qkv"] = np.asarray(g["w_qkv"]).reshape(p, 3, hp, d, h).transpose(1, 0, 2, 3, 4) \
        .reshape(3 * h, h)
    if "b_qkv" in g:
        out["b_qkv"] = np.asarray(g["b_qkv"]).reshape(p, 3, hp, d).transpose(1, 0, 2, 3) \
            .reshape(3 * h)
    out["w_o"] = np.asarray(g["w_o"]).reshape(p, h, h // p).transpose(1, 0, 2).reshape(h, h)
    if sw:  # [p][2][f/p] -> [2][p][f/p]: all gate rows, then all up rows
        out["w1"] = np.asarray(g["w1"]).reshape(p, 2, f // p, h).transpose(1, 0, 2, 3) \
            .reshape(2 * f, h)
        if "b1" in g:
            out["b1"] = np.asarray(g["b1"]).reshape(p, 2, f // p).transpose(1, 0, 2) \
                .reshape(2 * f)
    else:
        out["w1"] = np.asarray(g["w1"]).reshape(f, h)
        if "b1" in g:
            out["b1"] = np.asarray(g["b1"]).reshape(f)
    out["w2"] = np.asarray(g["w2"]).reshape(p, h, f // p).transpose(1, 0, 2).reshape(h, f)
    return out
