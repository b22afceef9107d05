"""Pins for the fp64 oracle: each test checks it against something other than itself --
torch float64 library routines (independent implementations), autograd, central finite
differences, closed forms and invariants, and the sharded == unsharded identity that the
tensor-parallel partitioning guarantees. Runs on CPU only."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mgt_inputs import LayerConfig, make_inputs, pack_params, unpack_params



def tiny(p=2, **kw):
    base = dict(name="pin", hidden=16, heads=4, ffn=32, seq=7, micro_batch=2, tp_size=p,
                dtype="f32", seed=7)
    base.update(kw)
    return LayerConfig(**base)


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ------------------------------------------------------------------ LayerNorm
def test_layer_norm_moments():
    rng = np.random.default_rng(0)
    x = rng.normal(3.0, 2.5, size=(64, 96))
    eps = 1e-5
    y, mean, rstd, xhat = oracle.layer_norm(x, np.ones(96), np.zeros(96), eps)
    assert np.max(np.abs(y.mean(axis=1))) < 1e-12
    var = x.var(axis=1)
    np.testing.assert_allclose(y.var(axis=1), var / (var + eps), rtol=1e-12)
    np.testing.assert_allclose(mean, x.mean(axis=1), rtol=1e-13)


def test_layer_norm_vs_torch():
    rng = np.random.default_rng(1)
    x, g, b = rng.normal(size=(10, 40)), rng.normal(size=40), rng.normal(size=40)
    y, *_ = oracle.layer_norm(x, g, b, 1e-5)
    yt = F.layer_norm(torch.tensor(x), (40,), torch.tensor(g), torch.tensor(b), 1e-5)
    assert rel(y, yt.numpy()) < 1e-13


def test_layer_norm_grad_vs_autograd():
    rng = np.random.default_rng(2)
    x, g, b, dy = (rng.normal(size=(9, 24)), rng.normal(size=24), rng.normal(size=24),
                   rng.normal(size=(9, 24)))
    y, mean, rstd, xhat = oracle.layer_norm(x, g, b, 1e-5)
    dx, dg, db = oracle.layer_norm_grad(dy, xhat, rstd, g)
    xt, gt, bt = (torch.tensor(v, requires_grad=True) for v in (x, g, b))
    F.layer_norm(xt, (24,), gt, bt, 1e-5).backward(torch.tensor(dy))
    assert rel(dx, xt.grad.numpy()) < 1e-12
    assert rel(dg, gt.grad.numpy()) < 1e-12
    assert rel(db, bt.grad.numpy()) < 1e-12


# ------------------------------------------------------------------ GeLU
@pytest.mark.parametrize("tanh", [0, 1])
def test_gelu_vs_torch(tanh):
    u = np.linspace(-8, 8, 2001)
    ut = torch.tensor(u, requires_grad=True)
    yt = F.gelu(ut, approximate="tanh" if tanh else "none")
    yt.sum().backward()
    assert np.max(np.abs(oracle.gelu(u, tanh) - yt.detach().numpy())) < 1e-14
    assert np.max(np.abs(oracle.gelu_grad(u, tanh) - ut.grad.numpy())) < 1e-13


def test_gelu_closed_forms():
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.gelu_grad(np.array([0.0]))[0] - 0.5) < 1e-15
    big = np.array([12.0, -12.0])
    np.testing.assert_allclose(oracle.gelu(big), [12.0, 0.0], atol=1e-25)
    np.testing.assert_allclose(oracle.gelu_grad(big), [1.0, 0.0], atol=1e-25)
    # exact vs tanh differ by ~1e-3 somewhere: the choice matters at the fp32 tolerance
    u = np.linspace(-4, 4, 4001)
    assert np.max(np.abs(oracle.gelu(u, 0) - oracle.gelu(u, 1))) > 1e-4


# ------------------------------------------------------------------ attention
def test_causal_softmax_invariants():
    rng = np.random.default_rng(3)
    S = rng.normal(size=(33, 33)) * 4
    P, lse = oracle.causal_softmax(S)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(P[np.triu_indices(33, 1)] == 0.0)
    assert P[0, 0] == 1.0
    ref = torch.logsumexp(torch.tensor(S).masked_fill(
        ~torch.tril(torch.ones(33, 33, dtype=torch.bool)), -math.inf), dim=1)
    assert rel(lse, ref.numpy()) < 1e-14


def test_attention_head_vs_sdpa():
    rng = np.random.default_rng(4)
    q, k, v, do = (rng.normal(size=(21, 8)) for _ in range(4))
    o, lse, P = oracle.attention_head_fwd(q, k, v)
    np.testing.assert_allclose(o[0], v[0], rtol=1e-14)      # token 0 sees only itself
    qt, kt, vt = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    ot = F.scaled_dot_product_attention(qt[None], kt[None], vt[None], is_causal=True)[0]
    assert rel(o, ot.detach().numpy()) < 1e-13
    ot.backward(torch.tensor(do))
    dq, dk, dv = oracle.attention_head_bwd(q, k, v, P, do)
    assert rel(dq, qt.grad.numpy()) < 1e-12
    assert rel(dk, kt.grad.numpy()) < 1e-12
    assert rel(dv, vt.grad.numpy()) < 1e-12


# ------------------------------------------------------------------ the layer
def torch_layer(cfg, full, x):
    """An independent float64 composition from torch library routines (pre-LN GPT block)."""
    h, H = cfg.hidden, cfg.heads
    d = h // H
    b, s = cfg.micro_batch, cfg.seq
    bias = lambda k: full.get(k)  # noqa: E731  (absent under disable_bias_linear)
    ln1 = F.layer_norm(x, (h,), full["ln1_g"], full["ln1_b"], cfg.ln_eps)
    qkv = F.linear(ln1, full["w_qkv"], bias("b_qkv"))
    q, k, v = qkv.split(h, dim=-1)
    heads = lambda t: t.reshape(b, s, H, d).transpose(1, 2)  # noqa: E731
    o = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    o = o.transpose(1, 2).reshape(b, s, h)
    h1 = x + F.linear(o, full["w_o"], bias("b_o"))
    ln2 = F.layer_norm(h1, (h,), full["ln2_g"], full["ln2_b"], cfg.ln_eps)
    u = F.linear(ln2, full["w1"], bias("b1"))
    if cfg.swiglu:
        gate, up = u.chunk(2, dim=-1)
        a = F.silu(gate) * up
    else:
        a = F.gelu(u, approximate="tanh" if cfg.gelu_tanh else "none")
    return h1 + F.linear(a, full["w2"], bias("b2"))


VARIANT_KW = {"gelu": {}, "gelu_tanh": {"gelu_tanh": 1}, "swiglu": {"swiglu": 1},
              "nobias": {"disable_bias_linear": 1},
              "swiglu_nobias": {"swiglu": 1, "disable_bias_linear": 1}}


@pytest.mark.parametrize("variant", list(VARIANT_KW))
def test_layer_vs_torch_composition(variant):
    cfg = tiny(p=2, **VARIANT_KW[variant])
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    y, saved = oracle.layer_fwd(cfg, pack_params(cfg, full), full["x"])
    dx, g, _ = oracle.layer_bwd(cfg, pack_params(cfg, full), saved, full["dy"])
    g = oracle.gather_grads(cfg, g)
    leaves = {k: full[k].clone().requires_grad_(True) for k in
              ("x", "ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o", "ln2_g", "ln2_b", "w1",
               "b1", "w2", "b2") if k in full}
    assert set(g) == set(leaves) - {"x"}
    yt = torch_layer(cfg, leaves, leaves["x"])
    assert rel(y, yt.detach().numpy()) < 1e-13
    yt.backward(full["dy"])
    assert rel(dx, leaves["x"].grad.numpy()) < 1e-12
    for k in g:
        assert rel(g[k], leaves[k].grad.numpy()) < 1e-11, k


@pytest.mark.parametrize("p,variant", [(2, "gelu"), (4, "gelu"), (2, "swiglu"),
                                       (4, "swiglu_nobias")])
def test_sharded_equals_unsharded(p, variant):
    """Column-split QKV/fc1 and row-split out-proj/fc2 with summed partials give the result of
    the unsplit layer (the partitioning claim of the trdm.cn page, section 2.1). With SwiGLU
    each shard holds matching gate and up rows, so the activation stays shard-local."""
    cfg = tiny(p=p, hidden=32, heads=4, ffn=64, **VARIANT_KW[variant])
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    y_s, sv_s = oracle.layer_fwd(cfg, pack_params(cfg, full), full["x"])
    dx_s, g_s, _ = oracle.layer_bwd(cfg, pack_params(cfg, full), sv_s, full["dy"])
    y_f, sv_f = oracle.layer_fwd_full(cfg, full, full["x"])
    dx_f, g_f = oracle.layer_bwd_full(cfg, full, sv_f, full["dy"])
    assert rel(y_s, y_f) < 1e-12
    assert rel(dx_s, dx_f) < 1e-12
    g_s = oracle.gather_grads(cfg, g_s)
    for k in g_f:
        assert rel(g_s[k], g_f[k]) < 1e-12, k
    # the packed tp=1 layout is the full layout
    cfg1 = cfg.replace(tp_size=1)
    y_1, _ = oracle.layer_fwd(cfg1, pack_params(cfg1, full), full["x"])
    assert rel(y_1, y_f) < 1e-12


def test_seq1_attention_is_v_projection():
    """With one token the causal softmax is [1], so the attention output is v and the block's
    first residual branch equals v W_o^T + b_o with v = ln1 W_v^T + b_v."""
    cfg = tiny(p=2, seq=1, micro_batch=3)
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double().numpy() for k, v in t.items()}
    _, saved = oracle.layer_fwd(cfg, pack_params(cfg, {k: torch.tensor(v) for k, v in
                                                      full.items()}), full["x"])
    h = cfg.hidden
    x = full["x"].reshape(-1, h)
    mu = x.mean(1, keepdims=True)
    xhat = (x - mu) / np.sqrt(((x - mu) ** 2).mean(1, keepdims=True) + cfg.ln_eps)
    ln1 = xhat * full["ln1_g"] + full["ln1_b"]
    v = ln1 @ full["w_qkv"][2 * h:].T + full["b_qkv"][2 * h:]
    expect = x + v @ full["w_o"].T + full["b_o"]
    assert rel(saved["h1"], expect) < 1e-13


@pytest.mark.parametrize("variant", ["gelu", "swiglu", "swiglu_nobias"])
def test_backward_central_finite_differences(variant):
    """Central differences of L = <y, dy> along random directions, for x and every
    parameter: relative error <= 1e-6. The step 1e-5 balances truncation (O(eps^2)) against
    rounding (1e-16*|L|/eps); both stay near 1e-10 here."""
    cfg = tiny(p=2, hidden=8, heads=2, ffn=16, seq=5, **VARIANT_KW[variant])
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    packed = {k: v.numpy() for k, v in pack_params(cfg, full).items()}
    x, dy = full["x"].numpy(), full["dy"].numpy()
    _, saved = oracle.layer_fwd(cfg, packed, x)
    dx, g, _ = oracle.layer_bwd(cfg, packed, saved, dy)

    def loss(pk, xx):
        y, _ = oracle.layer_fwd(cfg, pk, xx)
        return float(np.sum(y * dy))

    rng = np.random.default_rng(11)
    eps = 1e-5
    for name in ["x"] + list(packed):
        for _ in range(2):
            if name == "x":
                vdir = rng.normal(size=x.shape)
                lp, lm = loss(packed, x + eps * vdir), loss(packed, x - eps * vdir)
                an = float(np.sum(dx * vdir))
            else:
                vdir = rng.normal(size=packed[name].shape)
                pp = dict(packed); pp[name] = packed[name] + eps * vdir
                pm = dict(packed); pm[name] = packed[name] - eps * vdir
                lp, lm = loss(pp, x), loss(pm, x)
                an = float(np.sum(g[name] * vdir))
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), (name, fd, an)


def test_pack_unpack_roundtrip():
    cfg = tiny(p=4, hidden=32, heads=8, ffn=64)
    t = make_inputs(cfg, nonzero_affine=True)
    back = unpack_params(cfg, pack_params(cfg, t))
    for k in back:
        assert torch.equal(back[k], t[k]), k
    # head n of Q lands in shard n // (H/p), local head n % (H/p)
    pk = pack_params(cfg, t)
    d, hp = cfg.head_dim, cfg.heads // cfg.tp_size
    for n in range(cfg.heads):
        assert torch.equal(pk["w_qkv"][n // hp, 0, n % hp], t["w_qkv"][n * d:(n + 1) * d])
        assert torch.equal(pk["w_qkv"][n // hp, 2, n % hp],
                           t["w_qkv"][2 * cfg.hidden + n * d:2 * cfg.hidden + (n + 1) * d])


# ------------------------------------------------------------------ SwiGLU and no-bias
def test_silu_and_sigmoid_vs_torch():
    z = torch.linspace(-60.0, 60.0, 4001, dtype=torch.float64)
    zn = z.numpy()
    assert rel(oracle.sigmoid(zn), torch.sigmoid(z).numpy()) < 1e-15
    assert rel(oracle.silu(zn), F.silu(z).numpy()) < 1e-15
    zz = z.clone().requires_grad_(True)
    F.silu(zz).sum().backward()
    assert rel(oracle.silu_grad(zn), zz.grad.numpy()) < 1e-14


def test_swiglu_closed_forms_and_grad():
    rng = np.random.default_rng(3)
    gate, up, da = rng.normal(size=(3, 50, 20)) * 3.0
    # silu(0) = 0, so a zero gate gives a = 0 and no gradient to up; large gates pass through
    assert np.all(oracle.swiglu(np.zeros(5), np.arange(5.0)) == 0.0)
    assert rel(oracle.swiglu(np.full(3, 40.0), up[0, :3]), 40.0 * up[0, :3]) < 1e-15
    assert np.max(np.abs(oracle.swiglu(np.full(3, -40.0), up[0, :3]))) < 1e-15
    tg = torch.tensor(gate, requires_grad=True)
    tu = torch.tensor(up, requires_grad=True)
    (F.silu(tg) * tu).backward(torch.tensor(da))
    dg, du = oracle.swiglu_grad(gate, up, da)
    assert rel(dg, tg.grad.numpy()) < 1e-14
    assert rel(du, tu.grad.numpy()) < 1e-14


@pytest.mark.parametrize("swiglu", [0, 1])
def test_no_bias_equals_zero_bias(swiglu):
    """Dropping the linear biases is the layer with those biases fixed at zero: identical y,
    dx and weight/LN gradients, and no bias gradients at all."""
    cfg = tiny(p=2, swiglu=swiglu)
    cfg_nb = cfg.replace(disable_bias_linear=1)
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    for k in ("b_qkv", "b_o", "b1", "b2"):
        full[k] = torch.zeros_like(full[k])
    full_nb = {k: v for k, v in full.items() if k not in ("b_qkv", "b_o", "b1", "b2")}
    y0, s0 = oracle.layer_fwd(cfg, pack_params(cfg, full), full["x"])
    y1, s1 = oracle.layer_fwd(cfg_nb, pack_params(cfg_nb, full_nb), full["x"])
    assert np.array_equal(y0, y1)
    dx0, g0, _ = oracle.layer_bwd(cfg, pack_params(cfg, full), s0, full["dy"])
    dx1, g1, _ = oracle.layer_bwd(cfg_nb, pack_params(cfg_nb, full_nb), s1, full["dy"])
    assert np.array_equal(dx0, dx1)
    assert set(g1) == set(g0) - {"b_qkv", "b_o", "b1", "b2"}
    for k in g1:
        assert np.array_equal(g0[k], g1[k]), k


def test_swiglu_packing_pairs_gate_and_up():
    """Shard t of the packed SwiGLU fc1 holds gate rows t*f/p.. and the up rows with the same
    indices, so gate j and up j meet on one shard."""
    cfg = tiny(p=4, hidden=32, heads=8, ffn=64, swiglu=1)
    t = make_inputs(cfg, nonzero_affine=True)
    pk = pack_params(cfg, t)
    f, fp = cfg.ffn, cfg.ffn // cfg.tp_size
    for j in range(f):
        assert torch.equal(pk["w1"][j // fp, 0, j % fp], t["w1"][j])
        assert torch.equal(pk["w1"][j // fp, 1, j % fp], t["w1"][f + j])
        assert pk["b1"][j // fp, 1, j % fp] == t["b1"][f + j]
    back = unpack_params(cfg, pk)
    for k in back:
        assert torch.equal(back[k], t[k]), k


# ------------------------------------------------------------------ sequence parallelism
def test_sequence_collectives_are_adjoint():
    """<reduce_scatter(u_0..u_p-1), v> = sum_t <u_t, all_gather(v)>: the reduce-scatter after a
    row-parallel layer and the all-gather before a column-parallel one are each other's
    adjoints, which is what the backward relies on; and gather(scatter-of-one) is the identity
    on the shard layout."""
    rng = np.random.default_rng(5)
    b, s, p, n = 3, 12, 4, 5
    parts = [rng.normal(size=(b * s, n)) for _ in range(p)]
    v = rng.normal(size=(p, b, s // p, n))
    lhs = float(np.sum(oracle.reduce_scatter_seq(parts, b, s, p) * v))
    g = oracle.all_gather_seq(v, b, s, p)
    rhs = float(sum(np.sum(u * g) for u in parts))
    assert abs(lhs - rhs) <= 1e-12 * abs(rhs)
    one = [g] + [np.zeros_like(g)] * (p - 1)
    assert np.array_equal(oracle.reduce_scatter_seq(one, b, s, p), v)
    # token (bb, pos) of the gathered tensor is shard pos // (s/p), row (bb, pos % (s/p))
    for bb in range(b):
        for pos in range(s):
            assert np.array_equal(g[bb * s + pos], v[pos // (s // p), bb, pos % (s // p)])


@pytest.mark.parametrize("variant", ["gelu", "swiglu_nobias"])
def test_sequence_parallel_equals_plain_layer(variant):
    """Sharding the LayerNorm/residual regions along the sequence (all-gather before QKV and
    fc1, reduce-scatter after out-proj and fc2) computes the same layer: y and dx equal the
    plain layer's in the shard-major layout, every gradient is equal."""
    from mgt_inputs import to_sp
    cfg = tiny(p=2, hidden=16, heads=4, ffn=32, seq=8, micro_batch=3, **VARIANT_KW[variant])
    cfg_sp = cfg.replace(sequence_parallel=1)
    t = make_inputs(cfg, nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    pk = pack_params(cfg, full)
    y, sv = oracle.layer_fwd(cfg, pk, full["x"])
    dx, g, inter = oracle.layer_bwd(cfg, pk, sv, full["dy"])
    y_sp, sv_sp = oracle.layer_fwd(cfg_sp, pk, to_sp(cfg, full["x"]))
    dx_sp, g_sp, inter_sp = oracle.layer_bwd(cfg_sp, pk, sv_sp, to_sp(cfg, full["dy"]))
    assert rel(y_sp, to_sp(cfg, torch.tensor(y)).numpy()) < 1e-12
    assert rel(dx_sp, to_sp(cfg, torch.tensor(dx)).numpy()) < 1e-12
    assert set(g) == set(g_sp)
    for k in g:
        assert rel(g_sp[k], g[k]) < 1e-12, k
    # token-parallel intermediates are unchanged; sequence-parallel ones are permuted
    assert rel(inter_sp["dqkv"], inter["dqkv"]) < 1e-12
    sp_rows = lambda a: to_sp(cfg, torch.tensor(a).reshape(cfg.micro_batch, cfg.seq, -1))  # noqa
    assert rel(inter_sp["dh1"], sp_rows(inter["dh1"]).reshape(-1, cfg.hidden).numpy()) < 1e-12


def test_sequence_parallel_finite_differences():
    """The sequence-parallel backward against central differences on x (given in the
    shard-major layout) and two parameters."""
    from mgt_inputs import to_sp
    cfg = tiny(p=2, hidden=8, heads=2, ffn=16, seq=6, micro_batch=2, sequence_parallel=1)
    t = make_inputs(cfg.replace(sequence_parallel=0), nonzero_affine=True)
    full = {k: v.double() for k, v in t.items()}
    packed = {k: v.numpy() for k, v in pack_params(cfg, full).items()}
    x = to_sp(cfg, full["x"]).numpy()
    dy = to_sp(cfg, full["dy"]).numpy()
    _, saved = oracle.layer_fwd(cfg, packed, x)
    dx, g, _ = oracle.layer_bwd(cfg, packed, saved, dy)

    def loss(pk, xx):
        y, _ = oracle.layer_fwd(cfg, pk, xx)
        return float(np.sum(y * dy))

    rng = np.random.default_rng(13)
    eps = 1e-5
    for name in ("x", "ln1_g", "w1"):
        vdir = rng.normal(size=(x if name == "x" else packed[name]).shape)
        if name == "x":
            lp, lm, an = loss(packed, x + eps * vdir), loss(packed, x - eps * vdir), np.sum(dx * vdir)
        else:
            pp = dict(packed); pp[name] = packed[name] + eps * vdir
            pm = dict(packed); pm[name] = packed[name] - eps * vdir
            lp, lm, an = loss(pp, x), loss(pm, x), np.sum(g[name] * vdir)
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), (name, fd, an)
