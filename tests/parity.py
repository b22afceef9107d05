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
