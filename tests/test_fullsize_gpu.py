"""Parity at the full workload sizes, in the launch configuration the benchmark times.

h=1024 and h=4096 layers (and the h=4096 layer in its SwiGLU, no-bias form and with sequence
parallelism over two sequences): the whole layer
(y, dx, every parameter gradient and every saved or workspace intermediate) against the fp64
oracle on the benchmark's own seeded inputs.

h=6144 and h=12288 layers (too large for a whole-layer fp64 run in a test): the GPU runs the full
layer with the benchmark's inputs except that the upstream gradient dy is zero beyond the first m
positions of every sequence. By causality y at positions < m depends only on x at positions < m,
and with dy zero elsewhere every parameter gradient and dx[:, :m] equal those of the m-token
prefix problem, which the oracle computes exactly; dx[:, m:] must be exactly zero."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from mgt_inputs import config_by_name, make_inputs
from parity import GRAD_NAMES, full_parity, rel_err, run_gpu, to_np, tol

pytestmark = pytest.mark.gpu


def _log(name, errs):
    path = os.environ.get("MGT_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"config": name, "errors": errs}) + "\n")


@pytest.mark.parametrize("name", ["gpt-h1024-bf16", "gpt-h4096-tp2-bf16",
                                  "llama-h4096-tp2-bf16-swiglu-nobias",
                                  "gpt-h4096-tp2-sp-b2-bf16"])
def test_full_layer_parity_at_full_size(name):
    cfg = config_by_name(name)
    errs = full_parity(cfg, nonzero_affine=False, intermediates=True)
    _log(name, errs)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("name,m", [("gpt-h6144-tp4-bf16", 64), ("gpt-h12288-tp8-bf16", 32)])
def test_causal_prefix_parity_at_full_size(name, m):
    cfg = config_by_name(name)
    t = make_inputs(cfg)
    t["dy"][:, m:] = 0.0
    packed, layer, run = run_gpu(cfg, t)
    y_gpu, dx_gpu = to_np(run.y), to_np(run.dx)
    grads = {k: to_np(run.grads[k]) for k in GRAD_NAMES}
    del run
    torch.cuda.empty_cache()
    sub = cfg.replace(seq=m)
    y_ref, saved = oracle.layer_fwd(sub, packed, t["x"][:, :m])
    dx_ref, g_ref, _ = oracle.layer_bwd(sub, packed, saved, t["dy"][:, :m])
    errs = {"y_prefix": rel_err(y_gpu[:, :m], y_ref), "dx_prefix": rel_err(dx_gpu[:, :m], dx_ref)}
    for k in GRAD_NAMES:
        errs["d_" + k] = rel_err(grads[k], g_ref[k])
    _log(name, errs)
    assert np.all(dx_gpu[:, m:] == 0.0)
    assert np.all(np.isfinite(y_gpu))
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)
