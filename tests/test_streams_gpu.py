"""The backward's second stream (weight gradients and bias column sums, forked from the
caller's stream and joined back) against the single-stream order that profiling uses: the same
kernels on the same inputs must give the same dx and parameter gradients, bit for bit: every
reduction, the bias column sums included, adds its partial sums in a fixed order, so the
result does not depend on scheduling. Results are read on the caller's stream right after the call,
so a missing join would show as stale gradients. A second backward overwrites everything."""
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import LayerConfig, make_inputs, pack_params
from tensor_transformer_layer_megatron_b200.runner import LayerRun

pytestmark = pytest.mark.gpu

def _snapshot(run):
    out = {"dx": run.dx.float().cpu()}
    out.update({k: v.cpu() for k, v in run.grads.items()})
    return out


@pytest.mark.parametrize("swiglu", [0, 1])
def test_two_stream_backward_matches_single_stream(swiglu):
    cfg = LayerConfig("streams-h512-p2-s256-b2", hidden=512, heads=4, ffn=1536, seq=256,
                      micro_batch=2, tp_size=2, dtype="bf16", seed=4501, swiglu=swiglu)
    t = make_inputs(cfg, nonzero_affine=True)
    layer = mgt.Layer.from_config(cfg)
    run = LayerRun(layer, pack_params(cfg, t), t["x"], t["dy"])
    run.fwd()
    layer.profile(True)  # one stream: every launch on the caller's stream
    run.bwd()
    run.check()
    one = _snapshot(run)
    layer.profile(False)
    for g in run.grads.values():  # stale values would survive a missing join
        g.fill_(float("nan"))
    run.dx.fill_(float("nan"))
    run.bwd()  # two streams
    two = _snapshot(run)
    run.check()
    for k, ref in one.items():
        got = two[k]
        assert torch.isfinite(got).all(), k
        assert torch.equal(got, ref), k


@pytest.mark.parametrize("swiglu", [0, 1])
def test_graph_replay_matches_eager_step(swiglu):
    """The step captured into a CUDA graph (two streams, and programmatic-launch edges between
    dependent kernels, each of which waits for its predecessor before touching memory) gives
    the eager step's y, dx and gradients bit for bit, replay after replay. Outputs are poisoned
    before each replay, so a kernel that read before its predecessor finished writing, or a
    write that went missing, would show."""
    cfg = LayerConfig("graph-h512-p2-s256-b2", hidden=512, heads=4, ffn=1536, seq=256,
                      micro_batch=2, tp_size=2, dtype="bf16", seed=4502, swiglu=swiglu)
    t = make_inputs(cfg, nonzero_affine=True)
    layer = mgt.Layer.from_config(cfg)
    run = LayerRun(layer, pack_params(cfg, t), t["x"], t["dy"])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run.step(s)
        run.check(s)
        ref = _snapshot(run)
        ref["y"] = run.y.float().cpu()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            run.step(s)
        for _ in range(3):
            for v in run.grads.values():
                v.fill_(float("nan"))
            run.dx.fill_(float("nan"))
            run.y.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            got = _snapshot(run)
            got["y"] = run.y.float().cpu()
            for k, r in ref.items():
                assert torch.isfinite(got[k]).all(), k
                assert torch.equal(got[k], r), k
        run.check(s)
        del g
