"""The exponential of the attention softmax. Both attention kernels evaluate part of their
2^x on the FMA pipe with a degree-3 polynomial (range reduction to [-1/2, 1/2], exponent
added back in the integer domain) so that the special-function unit does not bound the
softmax. Checked here through mgt_debug_exp2 against the exact 2^x (fp64) and against the
hardware exponential on the same inputs: relative error within the fitted bound of 7.5e-5
(plus fp32 rounding) over the whole range the softmax feeds it, exact powers of two at
integers, and the documented clamp below -125."""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt

pytestmark = pytest.mark.gpu

POLY_BOUND = 7.5e-5 + 2.0 ** -22


def _run(x, path):
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    mgt.debug_exp2(xd, y, path)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_poly_exp2_relative_error_over_softmax_range():
    g = np.random.default_rng(11)
    x = np.concatenate([np.linspace(-125.0, 127.0, 1_000_003),
                        g.uniform(-30.0, 8.0, 1_000_000),
                        np.arange(-125, 128, dtype=np.float64),          # integers: exact
                        np.arange(-125, 127) + 0.5]).astype(np.float32)  # rounding ties
    ref = np.exp2(x.astype(np.float64))
    poly = _run(x, 1)
    rel = np.abs(poly - ref) / ref
    assert rel.max() <= POLY_BOUND, (rel.max(), x[np.argmax(rel)])
    # at the integers the reduced argument is 0, so the result is the polynomial's constant
    # term times 2^j: within the bound of the exact power of two
    ints = np.arange(-125, 128, dtype=np.float32)
    pi = _run(ints, 1)
    assert np.all(np.abs(pi / np.exp2(ints.astype(np.float64)) - 1.0) <= POLY_BOUND)
    # the hardware path on the same inputs agrees with the exact value far more closely
    hw = _run(x, 0)
    assert (np.abs(hw - ref) / ref).max() <= 1e-6


def test_poly_exp2_clamp_and_hardware_zero():
    x = np.array([-126.0, -200.0, -1e30, -np.inf, -125.0, 0.0], dtype=np.float32)
    poly = _run(x, 1)
    # everything at or below -125 evaluates as 2^-125 (to the polynomial's accuracy), all
    # bit-identical since the clamped input is the same
    assert np.all(np.abs(poly[:5] / 2.0 ** -125 - 1.0) <= POLY_BOUND)
    assert np.all(poly[:5] == poly[4])
    assert poly[5] == pytest.approx(1.0, rel=POLY_BOUND)
    hw = _run(np.array([-np.inf, 0.0], dtype=np.float32), 0)
    assert hw[0] == 0.0 and hw[1] == 1.0
