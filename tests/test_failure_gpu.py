"""Failure detection without a GPU fault: a device-side wait that runs out ends in a status the
host reads, and the context stays usable. The probe waits, with a 20 ms limit, on a barrier
nothing arrives on, through the same bounded wait every pipelined kernel uses; it writes into a
layer's status word, so mgt_layer_get_error must report MGT_ETIMEOUT once and then clear, and
the same layer must still produce correct results afterwards."""
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import LayerConfig
from parity import full_parity, tol

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    cfg = LayerConfig("probe", hidden=256, heads=2, ffn=512, seq=64, micro_batch=1, tp_size=2,
                      dtype="bf16", seed=9)
    layer = mgt.Layer.from_config(cfg)
    saved, ws = layer.alloc_buffers()
    word = layer.status_word_ptr(ws)
    assert layer.get_error(ws) == 0
    mgt.debug_bounded_wait(20_000_000, word)
    assert layer.get_error(ws) == 4  # MGT_ETIMEOUT, and the word is cleared
    assert layer.get_error(ws) == 0
    errs = full_parity(cfg, intermediates=False)  # kernels still run correctly afterwards
    assert max(errs.values()) <= tol(cfg), errs


def test_probe_rejects_bad_limits():
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, -5, 2_000_000_000):
        with pytest.raises(mgt.MgtError):
            mgt.debug_bounded_wait(bad, z.data_ptr())
