"""fp64 CPU oracle for the tensor-parallel GPT layer (forward and backward).

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package: only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg may use it. It shares no code with the
CUDA path (no kernels, headers, helpers or constants); the only thing both sides share is the
seeded input generator in mgt_inputs, which holds none of the layer's arithmetic.

It is the plain definition of the layer, written in numpy float64 with library matmuls as the
only primitive. No blocking, fusion or reordering beyond what the definition states.
"""
from .layer import (  # noqa: F401
    layer_norm, layer_norm_grad, gelu, gelu_grad, causal_softmax, attention_head_fwd,
    attention_head_bwd, attention_fwd, attention_bwd, layer_fwd, layer_bwd, layer_fwd_full,
    layer_bwd_full, gather_grads, sigmoid, silu, silu_grad, swiglu, swiglu_grad,
    all_gather_seq, reduce_scatter_seq, layer_fwd_sp, layer_bwd_sp,
)
from .fp8 import E4M3_MAX, e4m3_round, quantize_e4m3, gemm_fp8  # noqa: F401
from .tp_dist import rank_shard, layer_fwd_rank, layer_bwd_rank  # noqa: F401
