"""Device-side bookkeeping for one layer: moves packed parameters and a batch to the GPU in the
dtypes the C ABI expects, owns the output/gradient/saved/workspace buffers, and calls the
binding. Memory and marshalling only -- no arithmetic of the layer happens here."""
from __future__ import annotations

from typing import Dict

import torch

from . import PARAM_ORDER, Layer, MgtError

LN_PARAMS = ("ln1_g", "ln1_b", "ln2_g", "ln2_b")


class LayerRun:
    def __init__(self, layer: Layer, packed: Dict[str, torch.Tensor], x: torch.Tensor,
                 dy: torch.Tensor, device="cuda"):
        self.layer = layer
        act = torch.bfloat16 if layer.dtype == "bf16" else torch.float32
        self.act = act
        # Biases are absent from `packed` for a layer without linear biases.
        names = [k for k in PARAM_ORDER if k in packed]
        self.params = {k: packed[k].to(device=device,
                                       dtype=torch.float32 if k in LN_PARAMS else act)
                       .contiguous() for k in names}
        self.grads = {k: torch.empty(packed[k].shape, dtype=torch.float32, device=device)
                      for k in names}
        self.x = x.to(device=device, dtype=act).contiguous()
        self.dy = dy.to(device=device, dtype=act).contiguous()
        self.y = torch.empty_like(self.x)
        self.dx = torch.empty_like(self.x)
        self.saved, self.ws = layer.alloc_buffers(device)

    def fwd(self, stream=None):
        self.layer.fwd(self.params, self.x, self.y, self.saved, self.ws, stream)

    def bwd(self, stream=None):
        self.layer.bwd(self.params, self.x, self.saved, self.dy, self.dx, self.grads, self.ws,
                       stream)

    def step(self, stream=None):
        self.fwd(stream)
        self.bwd(stream)

    def check(self, stream=None):
        code = self.layer.get_error(self.ws, stream)
        if code != 0:
            raise MgtError(code, "device status")
