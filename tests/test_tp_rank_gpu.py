"""Real tensor-parallel ranks (mgt_tp_rank_*) on one GPU against the fp64 oracle.

The p ranks run in p host threads, each on its own CUDA stream, over their own shards of the
packed parameters. The all-reduce callback orders the exchange on the host side: each rank
synchronises its stream (its partial is written), the ranks meet at a barrier, one thread adds
the partials on the device, and each rank copies the sum back into its buffer. No kernel ever
waits on another (the GPU runs the ranks' kernels independently; only the host threads
wait), and a failing rank breaks the barrier (60 s timeout) instead of hanging. Expected
values: the single-process oracle (y and dx whole on every rank, each rank's slice of the
packed gradients, the replicated gradients whole). The oracle's own rank decomposition
(oracle/tp_dist.py) is pinned against it in test_tp_dist_oracle.py. Bar: 2e-2 per tensor,
max|gpu - ref| / max|ref| (bf16 activations, fp32 accumulation)."""
import threading

import numpy as np
import pytest
import torch

import oracle
import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import LayerConfig, make_inputs, pack_params
from parity import rel_err

pytestmark = pytest.mark.gpu

SHARDED = ("w_qkv", "b_qkv", "w_o", "w1", "b1", "w2")
LN = ("ln1_g", "ln1_b", "ln2_g", "ln2_b")


def _band_sizes(T, bands):
    """Rows of each band: an even split rounded up to whole 128-row tiles."""
    per = ((T + bands - 1) // bands + 127) // 128 * 128
    return [min(per, T - r0) for r0 in range(0, T, per)]


def _run_ranks(cfg, t, bands=1):
    p = cfg.tp_size
    packed = pack_params(cfg, t)
    dev = torch.device("cuda", 0)
    ranks, bufs = [], []
    for r in range(p):
        rk = mgt.TPRank(cfg.hidden, cfg.heads, cfg.ffn, cfg.seq, cfg.micro_batch, p, r,
                        cfg.ln_eps, cfg.gelu_tanh, swiglu=cfg.swiglu,
                        disable_bias_linear=cfg.disable_bias_linear)
        if bands > 1:
            rk.set_bands(bands)
        shard = {k: (v[r] if k in SHARDED else v)
                 .to(device=dev, dtype=torch.float32 if k in LN else torch.bfloat16)
                 .contiguous() for k, v in packed.items()}
        saved, ws = rk.alloc_buffers(dev)
        bufs.append(dict(
            params=shard,
            grads={k: torch.full(v.shape, float("nan"), dtype=torch.float32, device=dev)
                   for k, v in shard.items()},
            x=t["x"].to(device=dev, dtype=torch.bfloat16).contiguous(),
            dy=t["dy"].to(device=dev, dtype=torch.bfloat16).contiguous(),
            saved=saved, ws=ws))
        bufs[r]["y"] = torch.empty_like(bufs[r]["x"])
        bufs[r]["dx"] = torch.empty_like(bufs[r]["x"])
        ranks.append(rk)
    streams = [torch.cuda.Stream(dev) for _ in range(p)]
    off, nbytes = ranks[0].partial_region()
    barrier = threading.Barrier(p, timeout=60)
    views = [None] * p
    shared = {}
    calls = [0] * p

    sizes = _band_sizes(cfg.tokens, bands)
    row_bytes = 4 * cfg.hidden

    def make_allreduce(r):
        def allreduce(ptr, count, stream):
            # the reductions arrive band by band, in row order, inside the partial buffer; one
            # band comes on the caller's stream, several on the rank's communication stream
            ws = bufs[r]["ws"]
            band = calls[r] % len(sizes)
            start = off + row_bytes * sum(sizes[:band])
            assert ptr == ws.data_ptr() + start and count * 4 == row_bytes * sizes[band]
            assert (stream == streams[r].cuda_stream) == (bands == 1)
            calls[r] += 1
            view = ws[start:start + 4 * count].view(torch.float32)
            torch.cuda.ExternalStream(stream, device=dev).synchronize()
            views[r] = view
            barrier.wait()
            if r == 0:
                total = views[0].clone()
                for q in range(1, p):
                    total += views[q]
                streams[0].synchronize()
                shared["total"] = total
            barrier.wait()
            view.copy_(shared["total"])
            torch.cuda.synchronize(dev)
            barrier.wait()  # every rank holds the sum before the next reduction reuses it
        return allreduce

    errors = []

    def work(r):
        b = bufs[r]
        try:
            with torch.cuda.stream(streams[r]):
                ar = make_allreduce(r)
                ranks[r].fwd(b["params"], b["x"], b["y"], b["saved"], b["ws"], ar, streams[r])
                ranks[r].bwd(b["params"], b["x"], b["saved"], b["dy"], b["dx"], b["grads"],
                             b["ws"], ar, streams[r])
            streams[r].synchronize()
        except Exception as e:  # noqa: BLE001
            errors.append((r, repr(e)))
            barrier.abort()

    threads = [threading.Thread(target=work, args=(r,)) for r in range(p)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    torch.cuda.synchronize()
    assert not errors, errors
    assert calls == [4 * len(sizes)] * p, calls
    for b in bufs:  # device status word: no bounded wait gave up
        assert int(b["ws"][:4].view(torch.int32).item()) == 0
    return packed, bufs


CASES = [
    LayerConfig("tp2-h256-d64-s128-b2", hidden=256, heads=4, ffn=512, seq=128, micro_batch=2,
                tp_size=2, dtype="bf16", seed=4701),
    LayerConfig("tp2-h512-d128-swiglu-nobias-s96", hidden=512, heads=4, ffn=1024, seq=96,
                micro_batch=1, tp_size=2, dtype="bf16", seed=4702, swiglu=1,
                disable_bias_linear=1),
    LayerConfig("tp4-h512-d64-s80-tanh", hidden=512, heads=8, ffn=1024, seq=80, micro_batch=2,
                tp_size=4, dtype="bf16", seed=4703, gelu_tanh=1),
]


@pytest.mark.parametrize("bands", [1, 2])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_tp_ranks_match_oracle(cfg, bands):
    t = make_inputs(cfg, nonzero_affine=True)
    packed, bufs = _run_ranks(cfg, t, bands)
    y_ref, saved = oracle.layer_fwd(cfg, packed, t["x"])
    dx_ref, g_ref, _ = oracle.layer_bwd(cfg, packed, saved, t["dy"])
    for r, b in enumerate(bufs):
        errs = {"y": rel_err(b["y"].double().cpu().numpy(), y_ref),
                "dx": rel_err(b["dx"].double().cpu().numpy(), dx_ref)}
        for k, ref in g_ref.items():
            want = ref[r] if k in SHARDED else ref
            errs["d_" + k] = rel_err(b["grads"][k].double().cpu().numpy(), np.asarray(want))
        bad = {k: v for k, v in errs.items() if v > 2e-2}
        assert not bad, (r, bad, errs)


def test_tp_rank_reports_a_failed_allreduce():
    """A collective that fails (here: the callback raises) ends the rank's call with an error
    status instead of a hang, and leaves the context usable."""
    cfg = CASES[0]
    t = make_inputs(cfg)
    packed = pack_params(cfg, t)
    dev = torch.device("cuda", 0)
    rk = mgt.TPRank(cfg.hidden, cfg.heads, cfg.ffn, cfg.seq, cfg.micro_batch, cfg.tp_size, 0)
    shard = {k: (v[0] if k in SHARDED else v)
             .to(device=dev, dtype=torch.float32 if k in LN else torch.bfloat16).contiguous()
             for k, v in packed.items()}
    x = t["x"].to(device=dev, dtype=torch.bfloat16).contiguous()
    y = torch.empty_like(x)
    saved, ws = rk.alloc_buffers(dev)

    def failing(ptr, count, stream):
        raise RuntimeError("collective failed")

    with pytest.raises(mgt.MgtError) as ei:
        rk.fwd(shard, x, y, saved, ws, failing)
    assert ei.value.code == 3
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
