"""Shared helpers of the GPU parity tests: run the CUDA layer through the C ABI and compare it
tensor by tensor with the fp64 oracle on the same seeded inputs.

Metric (per tensor): max|gpu - ref| / max|ref|. Bars: 1e-4 for the fp32 layer, 2e-2 for the
bf16 layer (bf16 storage of activations, fp32 accumulation)."""
import numpy as np
import torch

import oracle
import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import make_inputs, pack_params, to_sp
from tensor_transformer_layer_megatron_b200.runner import LayerRun

GRAD_NAMES = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o", "ln2_g", "ln2_b", "w1", "b1",
              "w2", "b2")


def tol(cfg):
    return 1e-4 if cfg.dtype == "f32" else 2e-2


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got))
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def to_np(t):
    return t.detach().float().cpu().double().numpy()


def layer_io(cfg, t):
    """x and dy as the layer takes them: [b, s, h], or the shard-major sequence-parallel
    layout [p][b][s/p][h]."""
    if getattr(cfg, "sequence_parallel", 0):
        return to_sp(cfg, t["x"]), to_sp(cfg, t["dy"])
    return t["x"], t["dy"]


def run_gpu(cfg, t):
    packed = pack_params(cfg, t)
    layer = mgt.Layer.from_config(cfg)
    x, dy = layer_io(cfg, t)
    run = LayerRun(layer, packed, x, dy)
    run.step()
    run.check()
    torch.cuda.synchronize()
    return packed, layer, run


def gpu_intermediates(cfg, layer, run):
    """Every saved / workspace intermediate of the GPU layer, as zero-argument fetchers (each
    copies one tensor to the host only when called, so the largest layers compare one tensor
    at a time)."""
    T, h, f, p, H = cfg.tokens, cfg.hidden, cfg.ffn, cfg.tp_size, cfg.heads
    d = h // H
    act = run.act

    def v(buf, n, dt, shp):
        return lambda: to_np(layer.view(buf, n, dt, shp))

    out = dict(
        ln1=v(run.saved, "ln1", act, (T, h)),
        qkv=v(run.saved, "qkv", act, (T, p, 3, H // p, d)),
        O=v(run.saved, "attn_o", act, (T, p, H // p, d)),
        lse=v(run.saved, "attn_lse", torch.float32, (cfg.micro_batch, H, cfg.seq)),
        h1=v(run.saved, "h1", act, (T, h)),
        ln2=v(run.saved, "ln2", act, (T, h)),
        a=v(run.saved, "fc1_a", act, (T, p, f // p)),
        dln2=v(run.ws, "dln2", act, (T, h)),
        dh1=v(run.ws, "dh1", act, (T, h)),
        dO=v(run.ws, "dO", act, (T, p, H // p, d)),
        dqkv=v(run.ws, "dqkv", act, (T, p, 3, H // p, d)),
        dln1=v(run.ws, "dln1", act, (T, h)),
    )
    # the fc1 pre-activations u (SwiGLU: [gate | up]) and their gradient
    u_shape = (T, p, 2, f // p) if getattr(cfg, "swiglu", 0) else (T, p, f // p)
    out["u"] = v(run.saved, "fc1_u", act, u_shape)
    out["du"] = v(run.ws, "du", act, u_shape)
    return out


def full_parity(cfg, nonzero_affine=True, intermediates=True):
    """Whole-layer parity: y, dx, all 12 parameter gradients (and, optionally, every saved
    intermediate). Returns the dict of relative errors."""
    t = make_inputs(cfg, nonzero_affine=nonzero_affine)
    packed, layer, run = run_gpu(cfg, t)
    x, dy = layer_io(cfg, t)
    y_ref, saved = oracle.layer_fwd(cfg, packed, x)
    dx_ref, g_ref, inter = oracle.layer_bwd(cfg, packed, saved, dy)
    del t, x, dy
    errs = {"y": rel_err(to_np(run.y), y_ref), "dx": rel_err(to_np(run.dx), dx_ref)}
    del y_ref, dx_ref
    # a layer without linear biases has no bias gradients on either side
    assert set(run.grads) == set(g_ref), (sorted(run.grads), sorted(g_ref))
    for k in GRAD_NAMES:
        if k in g_ref:
            errs["d_" + k] = rel_err(to_np(run.grads[k]), g_ref.pop(k))
    if intermediates:
        gi = gpu_intermediates(cfg, layer, run)
        ref = dict(ln1=saved["ln1"], qkv=saved["qkv"], O=saved["O"], lse=saved["lse"],
                   h1=saved["h1"], ln2=saved["ln2"], a=saved["a"], u=saved["u"], **inter)
        del inter
        for k, fetch in gi.items():
            r = ref.pop(k)
            errs[k] = rel_err(fetch(), r() if callable(r) else r)
            del r
    return errs


def stage_parity(cfg, nonzero_affine=True):
    """Every intermediate of the GPU layer against the oracle's primitives applied to the GPU's
    own inputs of that stage (the bf16 values the kernel actually consumed), so each kernel's
    own error is measured apart from the bf16 rounding of the activations upstream of it.
    Stages: LN1, QKV GEMM, attention (O, lse), out-proj (h1), LN2, fc1 (u, a), fc2 (y), fc2
    dgrad with the activation backward (du), fc1 dgrad (dln2), LN2 backward (dh1), out-proj
    dgrad (dO), attention backward (dqkv), QKV dgrad (dln1), LN1 backward (dx). Plain layer
    only (no sequence parallelism). Returns the dict of relative errors."""
    assert not getattr(cfg, "sequence_parallel", 0)
    t = make_inputs(cfg, nonzero_affine=nonzero_affine)
    packed, layer, run = run_gpu(cfg, t)
    h, H, f, p = cfg.hidden, cfg.heads, cfg.ffn, cfg.tp_size
    b, s, T, d, hp = cfg.micro_batch, cfg.seq, cfg.tokens, cfg.hidden // cfg.heads, \
        cfg.heads // cfg.tp_size
    sw, nb = bool(getattr(cfg, "swiglu", 0)), bool(getattr(cfg, "disable_bias_linear", 0))
    Pm = {k: np.asarray(v.double().numpy() if hasattr(v, "double") else v, np.float64)
          for k, v in packed.items()}
    bias = (lambda k: 0.0) if nb else (lambda k: Pm[k])  # noqa: E731
    gi = gpu_intermediates(cfg, layer, run)
    x = to_np(run.x).reshape(T, h)
    dy = to_np(run.dy).reshape(T, h)
    errs = {}
    # forward
    errs["ln1"] = rel_err(gi["ln1"](), oracle.layer_norm(x, Pm["ln1_g"], Pm["ln1_b"],
                                                         cfg.ln_eps)[0])
    ln1 = gi["ln1"]()
    qkv = np.empty((T, p, 3, hp, d))
    for tt in range(p):
        qkv[:, tt] = (ln1 @ Pm["w_qkv"][tt].reshape(3 * hp * d, h).T +
                      (0.0 if nb else Pm["b_qkv"][tt].reshape(-1))).reshape(T, 3, hp, d)
    errs["qkv"] = rel_err(gi["qkv"](), qkv)
    del ln1, qkv
    qkv = gi["qkv"]()
    O, lse = oracle.attention_fwd(qkv, b, s, H, p)
    errs["O"] = rel_err(gi["O"](), O)
    errs["lse"] = rel_err(gi["lse"](), lse)
    del O, lse
    Og = gi["O"]()
    acc = np.zeros((T, h))
    for tt in range(p):
        acc += Og[:, tt].reshape(T, h // p) @ Pm["w_o"][tt].T
    errs["h1"] = rel_err(gi["h1"](), x + bias("b_o") + acc)
    del Og, acc
    h1 = gi["h1"]()
    errs["ln2"] = rel_err(gi["ln2"](), oracle.layer_norm(h1, Pm["ln2_g"], Pm["ln2_b"],
                                                         cfg.ln_eps)[0])
    ln2 = gi["ln2"]()
    if sw:
        u = np.empty((T, p, 2, f // p))
        for tt in range(p):
            for c in range(2):
                u[:, tt, c] = ln2 @ Pm["w1"][tt, c].T + (0.0 if nb else Pm["b1"][tt, c])
        a = oracle.swiglu(u[:, :, 0], u[:, :, 1])
    else:
        u = np.empty((T, p, f // p))
        for tt in range(p):
            u[:, tt] = ln2 @ Pm["w1"][tt].T + (0.0 if nb else Pm["b1"][tt])
        a = oracle.gelu(u, cfg.gelu_tanh)
    errs["u"] = rel_err(gi["u"](), u)
    errs["a"] = rel_err(gi["a"](), a)
    del ln2, u, a
    ag = gi["a"]()
    acc = np.zeros((T, h))
    for tt in range(p):
        acc += ag[:, tt] @ Pm["w2"][tt].T
    errs["y"] = rel_err(to_np(run.y).reshape(T, h), h1 + bias("b2") + acc)
    del ag, acc
    # backward
    ug = gi["u"]()
    da = np.empty((T, p, f // p))
    for tt in range(p):
        da[:, tt] = dy @ Pm["w2"][tt]
    if sw:
        du = np.stack(oracle.swiglu_grad(ug[:, :, 0], ug[:, :, 1], da), axis=2)
    else:
        du = da * oracle.gelu_grad(ug, cfg.gelu_tanh)
    errs["du"] = rel_err(gi["du"](), du)
    del ug, da, du
    dug = gi["du"]()
    rows = (2 if sw else 1) * (f // p)
    dln2 = np.zeros((T, h))
    for tt in range(p):
        dln2 += dug[:, tt].reshape(T, rows) @ Pm["w1"][tt].reshape(rows, h)
    errs["dln2"] = rel_err(gi["dln2"](), dln2)
    del dug, dln2
    _, _, rstd2, xhat2 = oracle.layer_norm(h1, Pm["ln2_g"], Pm["ln2_b"], cfg.ln_eps)
    dl, _, _ = oracle.layer_norm_grad(gi["dln2"](), xhat2, rstd2, Pm["ln2_g"])
    errs["dh1"] = rel_err(gi["dh1"](), dy + dl)
    del h1, xhat2, rstd2, dl
    dh1 = gi["dh1"]()
    dO = np.empty((T, p, hp, d))
    for tt in range(p):
        dO[:, tt] = (dh1 @ Pm["w_o"][tt]).reshape(T, hp, d)
    errs["dO"] = rel_err(gi["dO"](), dO)
    del dO
    errs["dqkv"] = rel_err(gi["dqkv"](), oracle.attention_bwd(qkv, gi["dO"](), b, s, H, p))
    del qkv
    dqg = gi["dqkv"]()
    dln1 = np.zeros((T, h))
    for tt in range(p):
        dln1 += dqg[:, tt].reshape(T, 3 * hp * d) @ Pm["w_qkv"][tt].reshape(3 * hp * d, h)
    errs["dln1"] = rel_err(gi["dln1"](), dln1)
    del dqg, dln1
    _, _, rstd1, xhat1 = oracle.layer_norm(x, Pm["ln1_g"], Pm["ln1_b"], cfg.ln_eps)
    dl, _, _ = oracle.layer_norm_grad(gi["dln1"](), xhat1, rstd1, Pm["ln1_g"])
    errs["dx"] = rel_err(to_np(run.dx).reshape(T, h), dh1 + dl)
    return errs
