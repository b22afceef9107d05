"""The process-group all-reduce that tensor-parallel ranks get from the binding
(process_group_allreduce), on two gloo ranks with CPU workspaces: the callback must locate
the partial buffer inside the rank's workspace from the pointer the layer passes, sum it over
the ranks in place, leave the rest of the workspace alone, and reject a pointer outside the
workspace."""
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
        ar = mgt.process_group_allreduce(ws, off)
        ar(ws.data_ptr() + off, count, 0)
        want = torch.arange(count, dtype=torch.float32) * sum(r + 1 for r in range(world))
        ok = torch.equal(part, want) and bool((ws[:off] == 7).all()) and \
            bool((ws[off + 4 * count:] == 0).all())
        try:
            ar(ws.data_ptr(), count, 0)
            rejected = False
        except ValueError:
            rejected = True
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
