"""The process-group all-reduce that tensor-parallel ranks get from the binding
(process_group_allreduce), on two gloo ranks with CPU workspaces: the callback must locate
the partial buffer inside the rank's workspace from the pointer the layer passes -- the whole
buffer, or one row band of it when the shard sums are banded (mgt_tp_rank_set_bands) -- sum it
over the ranks in place, leave the rest of the workspace alone, and reject a pointer outside
the partial buffer."""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import tensor_transformer_layer_megatron_b200 as mgt
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        off, count = 256, 1000
        ws = torch.zeros(off + 4 * count + 512, dtype=torch.uint8)
        ws[:off] = 7
        part = ws[off:off + 4 * count].view(torch.float32)
        part.copy_(torch.arange(count, dtype=torch.float32) * (rank + 1))
        ar = mgt.process_group_allreduce(ws, off, 4 * count)
        ar(ws.data_ptr() + off, count, 0)
        total = sum(r + 1 for r in range(world))
        want = torch.arange(count, dtype=torch.float32) * total
        ok = torch.equal(part, want) and bool((ws[:off] == 7).all()) and \
            bool((ws[off + 4 * count:] == 0).all())
        # banded: three row bands in order, each summed on its own
        part.copy_(torch.arange(count, dtype=torch.float32) * (rank + 1))
        for b0, b1 in ((0, 400), (400, 800), (800, 1000)):
            ar(ws.data_ptr() + off + 4 * b0, b1 - b0, 0)
        ok = ok and torch.equal(part, want) and bool((ws[off + 4 * count:] == 0).all())
        rejected = True
        for ptr, n in ((ws.data_ptr(), count), (ws.data_ptr() + off + 4, count),
                       (ws.data_ptr() + off + 2, 10), (ws.data_ptr() + off + 4 * 990, 20)):
            try:
                ar(ptr, n, 0)
                rejected = False
            except ValueError:
                pass
        out.put((rank, ok, rejected))
    finally:
        dist.destroy_process_group()


def test_process_group_allreduce_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True, True), (1, True, True)], res
