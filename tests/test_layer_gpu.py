"""Layer parity of the CUDA path against the fp64 oracle, through the C ABI, on seeded inputs:
small layers spanning several tiles with ragged tails (tokens, sequence, ffn per shard),
tp_size 1/2/4, head_dim 64/128, both GeLU forms, the SwiGLU and no-bias variants, and the
fp32 correctness layer."""
import pytest

from mgt_inputs import LayerConfig, config_by_name
from parity import full_parity, tol

pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(name=name, dtype="bf16", seed=hash(name) % 10000)
    base.update(kw)
    return LayerConfig(**base)


SMALL = [
    small("h128-d64-p2-s80-b2", hidden=128, heads=2, ffn=256, seq=80, micro_batch=2, tp_size=2),
    small("h256-d128-p2-s200", hidden=256, heads=2, ffn=512, seq=200, micro_batch=1, tp_size=2),
    small("h512-d128-p4-s130-b3", hidden=512, heads=4, ffn=1536, seq=130, micro_batch=3,
          tp_size=4),
    small("h256-d64-p1-s64", hidden=256, heads=4, ffn=768, seq=64, micro_batch=1, tp_size=1),
    small("h256-d128-p2-f640", hidden=256, heads=2, ffn=640, seq=96, micro_batch=2, tp_size=2),
    small("h256-d64-p2-tanh", hidden=256, heads=4, ffn=512, seq=33, micro_batch=2, tp_size=2,
          gelu_tanh=1),
    small("h128-d64-p1-s1", hidden=128, heads=2, ffn=256, seq=1, micro_batch=4, tp_size=1),
    # rows of 256 and 384 16-byte vectors: the LayerNorm kernels' shared-memory row ring (one
    # and two vectors per thread, the second only for some threads)
    small("h2048-d128-p2-s72-b2", hidden=2048, heads=16, ffn=2048, seq=72, micro_batch=2,
          tp_size=2),
    small("h3072-d128-p4-s40-b3", hidden=3072, heads=24, ffn=3072, seq=40, micro_batch=3,
          tp_size=4),
]

# SwiGLU (fc1 tiles pair a shard's gate and up rows) and no-bias layers. f/p = 128 sends the
# fc2 dgrad (SwiGLU backward epilogue) to the one-CTA kernel, wider f/p to the CTA pairs.
VARIANTS = [
    small("h128-d64-p2-swiglu-s80-b2", hidden=128, heads=2, ffn=256, seq=80, micro_batch=2,
          tp_size=2, swiglu=1),
    small("h256-d128-p2-swiglu-s200", hidden=256, heads=2, ffn=512, seq=200, micro_batch=1,
          tp_size=2, swiglu=1),
    small("h512-d64-p4-swiglu-nobias-s130-b3", hidden=512, heads=8, ffn=1536, seq=130,
          micro_batch=3, tp_size=4, swiglu=1, disable_bias_linear=1),
    small("h256-d64-p1-nobias-s64", hidden=256, heads=4, ffn=768, seq=64, micro_batch=1,
          tp_size=1, disable_bias_linear=1),
    # sequence parallelism: shard-major [p][b][s/p][h] LN/residual regions (a real permutation
    # of the tokens with b > 1)
    small("h256-d128-p2-sp-s256-b2", hidden=256, heads=2, ffn=512, seq=256, micro_batch=2,
          tp_size=2, sequence_parallel=1),
    small("h512-d64-p4-sp-swiglu-s512-b3", hidden=512, heads=8, ffn=1536, seq=512,
          micro_batch=3, tp_size=4, sequence_parallel=1, swiglu=1),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_layer_bf16_small(cfg):
    errs = full_parity(cfg)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("affine", [False, True])
def test_layer_f32_tiny(affine):
    cfg = config_by_name("tiny-h64-tp2-f32")
    errs = full_parity(cfg, nonzero_affine=affine)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("affine", [False, True])
def test_layer_f32_ring_rows(affine):
    """fp32 layer with h = 1024: LayerNorm rows of 256 vectors take the row-ring kernels."""
    cfg = LayerConfig("h1024-f32-p2-s24-b2", hidden=1024, heads=16, ffn=1024, seq=24,
                      micro_batch=2, tp_size=2, dtype="f32", seed=4401)
    errs = full_parity(cfg, nonzero_affine=affine)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("cfg", VARIANTS, ids=lambda c: c.name)
def test_layer_bf16_variants(cfg):
    errs = full_parity(cfg)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("nobias", [0, 1])
@pytest.mark.parametrize("affine", [False, True])
def test_layer_f32_tiny_swiglu(affine, nobias):
    cfg = config_by_name("tiny-h64-tp2-f32-swiglu").replace(disable_bias_linear=nobias)
    errs = full_parity(cfg, nonzero_affine=affine)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("affine", [False, True])
def test_layer_f32_tiny_sequence_parallel(affine):
    cfg = config_by_name("tiny-h64-tp2-f32").replace(sequence_parallel=1)
    errs = full_parity(cfg, nonzero_affine=affine)
    bad = {k: v for k, v in errs.items() if v > tol(cfg)}
    assert not bad, (bad, errs)
