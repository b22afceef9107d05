"""Pins for the rank-decomposed oracle (oracle/tp_dist.py): the layer split across real
tensor-parallel ranks, run as gloo processes on the CPU with torch.distributed.all_reduce as
the collective, must reproduce the single-process oracle. y and dx match on every rank, each
rank's sharded gradients match its slice of the packed gradients, and the replicated
gradients match on every rank. A dropped or misplaced reduction (either forward all-reduce or
either backward one) leaves a shard's contribution out and fails these comparisons for
p >= 2. fp64 throughout."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, kw, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from mgt_inputs import LayerConfig, make_inputs, pack_params
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = LayerConfig(**kw)
        t = make_inputs(cfg, nonzero_affine=True)
        packed = pack_params(cfg, t)

        def all_reduce(a):
            buf = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
            dist.all_reduce(buf)
            return buf.numpy()

        shard = oracle.rank_shard(packed, rank)
        y_r, saved_r = oracle.layer_fwd_rank(cfg, shard, t["x"], all_reduce)
        dx_r, g_r = oracle.layer_bwd_rank(cfg, shard, saved_r, t["dy"], all_reduce)
        y, saved = oracle.layer_fwd(cfg, packed, t["x"])
        dx, g, _ = oracle.layer_bwd(cfg, packed, saved, t["dy"])

        def rel(a, b):
            a, b = np.asarray(a), np.asarray(b)
            return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))

        errs = {"y": rel(y_r, y), "dx": rel(dx_r, dx)}
        assert set(g_r) == set(g), (sorted(g_r), sorted(g))
        for k in g:
            ref = g[k][rank] if k in oracle.tp_dist.SHARDED else g[k]
            errs["d_" + k] = rel(g_r[k], ref)
        out.put((rank, errs))
    finally:
        dist.destroy_process_group()


CASES = [
    dict(name="dist-gelu-p2", hidden=64, heads=4, ffn=128, seq=16, micro_batch=2, tp_size=2,
         dtype="f32", seed=4601),
    dict(name="dist-swiglu-nobias-p2", hidden=64, heads=4, ffn=128, seq=12, micro_batch=2,
         tp_size=2, dtype="f32", seed=4602, swiglu=1, disable_bias_linear=1),
    dict(name="dist-gelu-tanh-p4", hidden=64, heads=4, ffn=192, seq=10, micro_batch=1,
         tp_size=4, dtype="f32", seed=4603, gelu_tanh=1),
]


@pytest.mark.parametrize("kw", CASES, ids=lambda k: k["name"])
def test_rank_decomposed_oracle_matches_single_process(kw):
    world = kw["tp_size"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, kw, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, errs in res:
        bad = {k: v for k, v in errs.items() if v > 1e-12}
        assert not bad, (rank, bad)
