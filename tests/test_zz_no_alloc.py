"""The allocation-free LayerNorm backward (mgt_layernorm_bwd_noalloc), for callers that cannot
call cudaMalloc where they run the backward (frameworks that own all device memory through
their own pool allocator; hot loops where an allocation would synchronise the device).

It must reproduce what mgt_layer_bwd computes for the first LayerNorm: given the layer's own
dL/d ln1, residual gradient dL/dh1, input x and saved statistics, its dx, dgamma and dbeta must
match the layer's dx and ln1 gradients. Two calls in a row check that the shared scratch array
left over from a previous call does not leak into the next result. This file is collected last
so that a stop-at-first-failure run has already run every other test."""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import LayerConfig, make_inputs, pack_params
from tensor_transformer_layer_megatron_b200.runner import LayerRun

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


def rel(a, b):
    a = a.detach().double().cpu().numpy()
    b = b.detach().double().cpu().numpy()
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


def test_layernorm_bwd_noalloc_rejects_oversize():
    a = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(mgt.MgtError) as ei:
        mgt.layernorm_bwd_noalloc("bf16", 4, 16384 + 8, a, None, a, z, z, z, a, z, z)
    assert ei.value.code == 2
