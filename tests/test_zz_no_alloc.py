"""The allocation-free LayerNorm backward (mgt_layernorm_bwd_noalloc), for callers that cannot
call cudaMalloc where they run the backward (frameworks that own all device memory through
their own pool allocator; hot loops where an allocation would synchronise the device).

It must reproduce what mgt_layer_bwd computes for the first LayerNorm: given the layer's own
dL/d ln1, residual gradient dL/dh1, input x and saved statistics, its dx, dgamma and dbeta must
match the layer's dx and ln1 gradients, on two calls in a row. At the widths where the
kernels change (h = 4096: the one-pass kernel for 512-vector rows; h = 16384: the separate dx
and parameter kernels at the array's limit) it is checked against the fp64 oracle, after a
call on other inputs with more rows has filled more of the shared array than the checked call
reads, so a read of a stale partial row would show. This file is collected last so that a
stop-at-first-failure run has already run every other test."""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import LayerConfig, make_inputs, pack_params
from oracle.layer import layer_norm_grad
from tensor_transformer_layer_megatron_b200.runner import LayerRun

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}
TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def rel(a, b):
    a = np.asarray(a.detach().double().cpu().numpy() if torch.is_tensor(a) else a, np.float64)
    b = np.asarray(b.detach().double().cpu().numpy() if torch.is_tensor(b) else b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layernorm_bwd_noalloc_matches_layer(dtype):
    if dtype == "bf16":
        cfg = LayerConfig("noalloc-bf16", hidden=512, heads=4, ffn=1024, seq=96, micro_batch=3,
                          tp_size=2, dtype="bf16", seed=4242)
    else:
        cfg = LayerConfig("noalloc-f32", hidden=64, heads=4, ffn=256, seq=32, micro_batch=2,
                          tp_size=2, dtype="f32", seed=4243)
    t = make_inputs(cfg, nonzero_affine=True)
    layer = mgt.Layer.from_config(cfg)
    run = LayerRun(layer, pack_params(cfg, t), t["x"], t["dy"])
    run.step()
    run.check()
    torch.cuda.synchronize()
    T, h = cfg.tokens, cfg.hidden
    dln1 = layer.view(run.ws, "dln1", run.act, (T, h))
    dh1 = layer.view(run.ws, "dh1", run.act, (T, h))
    mean = layer.view(run.saved, "ln1_mean", torch.float32, (T,))
    rstd = layer.view(run.saved, "ln1_rstd", torch.float32, (T,))
    for call in range(2):
        dx = torch.full_like(run.dx, float("nan"))
        dg = torch.full((h,), float("nan"), dtype=torch.float32, device="cuda")
        db = torch.full((h,), float("nan"), dtype=torch.float32, device="cuda")
        mgt.layernorm_bwd_noalloc(dtype, T, h, dln1, dh1, run.x, run.params["ln1_g"], mean, rstd,
                                  dx, dg, db)
        torch.cuda.synchronize()
        for name, got, ref in (("dx", dx, run.dx), ("dgamma", dg, run.grads["ln1_g"]),
                               ("dbeta", db, run.grads["ln1_b"])):
            err = rel(got, ref)
            assert err <= TOL[dtype], (call, name, err)


def _ln_case(dtype, rows, h, seed, with_dres=True):
    """Seeded LayerNorm-backward inputs: x with its own fp32 statistics, dy, dres, gamma."""
    g = torch.Generator("cpu").manual_seed(seed)
    x = (torch.randn(rows, h, generator=g) * 1.5 + 0.3).to(TORCH_DT[dtype])
    dy = torch.randn(rows, h, generator=g).to(TORCH_DT[dtype])
    dres = torch.randn(rows, h, generator=g).to(TORCH_DT[dtype]) if with_dres else None
    gamma = (1.0 + 0.1 * torch.randn(h, generator=g)).float()
    x64 = x.double()
    mean = x64.mean(dim=1).float()
    rstd = torch.rsqrt(x64.var(dim=1, unbiased=False) + 1e-5).float()
    return dict(x=x, dy=dy, dres=dres, gamma=gamma, mean=mean, rstd=rstd)


def _call(dtype, case):
    dev = {k: (v.cuda() if v is not None else None) for k, v in case.items()}
    rows, h = case["x"].shape
    dx = torch.full((rows, h), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    dg = torch.full((h,), float("nan"), dtype=torch.float32, device="cuda")
    db = torch.full((h,), float("nan"), dtype=torch.float32, device="cuda")
    mgt.layernorm_bwd_noalloc(dtype, rows, h, dev["dy"], dev["dres"], dev["x"], dev["gamma"],
                              dev["mean"], dev["rstd"], dx, dg, db)
    torch.cuda.synchronize()
    return dx.cpu(), dg.cpu(), db.cpu()


def _oracle(case):
    """fp64 oracle LayerNorm backward on exactly the values the kernel reads."""
    x = case["x"].double().numpy()
    mean = case["mean"].double().numpy()
    rstd = case["rstd"].double().numpy()
    xhat = (x - mean[:, None]) * rstd[:, None]
    dx, dg, db = layer_norm_grad(case["dy"].double().numpy(), xhat, rstd,
                                 case["gamma"].double().numpy())
    if case["dres"] is not None:
        dx = dx + case["dres"].double().numpy()
    return dx, dg, db


@pytest.mark.parametrize("dtype,h", [("bf16", 4096), ("bf16", 16384), ("f32", 8192)])
def test_layernorm_bwd_noalloc_matches_oracle_after_larger_call(dtype, h):
    # A call on other inputs with many rows leaves more partial rows in the shared array than
    # the checked calls (fewer rows, hence fewer partial slices) write and read.
    _call(dtype, _ln_case(dtype, 2048, h, seed=7000 + h))
    for rows, with_dres, seed in ((100, True, 7100 + h), (37, False, 7200 + h)):
        case = _ln_case(dtype, rows, h, seed, with_dres)
        ref = _oracle(case)
        for call in range(2):
            got = _call(dtype, case)
            for name, gv, rv in zip(("dx", "dgamma", "dbeta"), got, ref):
                err = rel(gv, rv)
                assert err <= TOL[dtype], (rows, call, name, err)


def test_layernorm_bwd_noalloc_rejects_oversize():
    a = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(mgt.MgtError) as ei:
        mgt.layernorm_bwd_noalloc("bf16", 4, 16384 + 8, a, None, a, z, z, z, a, z, z)
    assert ei.value.code == 2
