"""Python binding of libmgt.so, the B200 (sm_100a) tensor-parallel GPT layer.

Argument marshalling only: every step of the layer runs in the CUDA kernels behind the C ABI
declared in include/mgt_layer.h. PyTorch is used for device memory and streams. There is no
fallback: if the shared library is missing or fails to load, importing the binding's Layer raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

__all__ = ["Layer", "MgtError", "load_library", "gemm_bf16", "layernorm_bwd_noalloc", "REGIONS",
           "PARAM_ORDER", "lib_path"]

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libmgt.so")

PARAM_ORDER = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
               "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")

REGIONS = {
    "ln1": 0, "ln1_mean": 1, "ln1_rstd": 2, "qkv": 3, "attn_o": 4, "attn_lse": 5, "h1": 6,
    "ln2": 7, "ln2_mean": 8, "ln2_rstd": 9, "fc1_u": 10, "fc1_a": 11,
    "status": 64, "du": 65, "dln2": 66, "dh1": 67, "dO": 68, "dqkv": 69, "dln1": 70,
    "attn_D": 71, "dq_acc": 72, "ln_partial": 73,
}

STATUS = {0: "MGT_OK", 1: "MGT_EINVAL", 2: "MGT_EUNSUPPORTED", 3: "MGT_ECUDA",
          4: "MGT_ETIMEOUT", 5: "MGT_ENOMEM"}


class MgtError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(code, "?"), code))
        self.code = code


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("heads", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("seq", ctypes.c_int32), ("micro_batch", ctypes.c_int32),
                ("tp_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("recompute_attn", ctypes.c_int32), ("gelu_tanh", ctypes.c_int32),
                ("swiglu", ctypes.c_int32), ("disable_bias_linear", ctypes.c_int32),
                ("sequence_parallel", ctypes.c_int32)]


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in PARAM_ORDER]


# mgt_allreduce_fn: (float* buf, int64 count, void* user, void* stream) -> mgt_status
ALLREDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                ctypes.c_void_p)


class _KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("ms", ctypes.c_double), ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_LIB = None


def load_library():
    """Load libmgt.so (raises OSError if it is missing: there is no fallback)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(lib_path):
        raise OSError("libmgt.so is not built (%s); run python -m "
                      "tensor_transformer_layer_megatron_b200.build" % lib_path)
    lib = ctypes.CDLL(lib_path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.mgt_layer_init.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(vp)]
    lib.mgt_layer_sizes.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.mgt_layer_region.argtypes = [vp, ctypes.c_int, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.mgt_layer_fwd.argtypes = [vp, ctypes.POINTER(_Params), vp, vp, vp, vp, vp]
    lib.mgt_layer_bwd.argtypes = [vp, ctypes.POINTER(_Params), vp, vp, vp, vp,
                                  ctypes.POINTER(_Params), vp, vp]
    lib.mgt_layer_get_error.argtypes = [vp, vp, vp]
    lib.mgt_layer_profile.argtypes = [vp, ctypes.c_int]
    lib.mgt_layer_profile_read.argtypes = [vp, ctypes.POINTER(_KernelStat), ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int)]
    lib.mgt_layer_destroy.argtypes = [vp]
    lib.mgt_layer_destroy.restype = None
    lib.mgt_status_string.argtypes = [ctypes.c_int]
    lib.mgt_status_string.restype = ctypes.c_char_p
    lib.mgt_gemm_bf16.argtypes = [i32, i32, i32, i32, i32, vp, ctypes.c_int64, vp,
                                  ctypes.c_int64, vp, ctypes.c_int64, vp, vp]
    lib.mgt_layernorm_bwd_noalloc.argtypes = [i32, ctypes.c_int64, i32, vp, vp, vp, vp, vp, vp,
                                              vp, vp, vp, vp]
    lib.mgt_fp8_quantize.argtypes = [i32, ctypes.c_int64, vp, vp, vp, vp]
    lib.mgt_gemm_fp8.argtypes = [i32, i32, i32, vp, ctypes.c_int64, vp, ctypes.c_int64, vp, vp,
                                 vp, i32, ctypes.c_int64, vp, vp]
    lib.mgt_tp_rank_init.argtypes = [ctypes.POINTER(_Config), i32, ctypes.POINTER(vp)]
    lib.mgt_tp_rank_sizes.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.mgt_tp_rank_partial.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.mgt_tp_rank_fwd.argtypes = [vp, ctypes.POINTER(_Params), vp, vp, vp, vp, ALLREDUCE_FN,
                                    vp, vp]
    lib.mgt_tp_rank_bwd.argtypes = [vp, ctypes.POINTER(_Params), vp, vp, vp, vp,
                                    ctypes.POINTER(_Params), vp, ALLREDUCE_FN, vp, vp]
    lib.mgt_tp_rank_set_bands.argtypes = [vp, i32]
    lib.mgt_tp_rank_destroy.argtypes = [vp]
    lib.mgt_tp_rank_destroy.restype = None
    lib.mgt_debug_bounded_wait.argtypes = [ctypes.c_int64, vp, vp]
    lib.mgt_debug_exp2.argtypes = [i32, ctypes.c_int64, vp, vp, vp]
    lib.mgt_debug_exp2.restype = ctypes.c_int
    lib.mgt_layer_status_word.argtypes = [vp, vp, ctypes.POINTER(vp)]
    lib.mgt_debug_bounded_wait.restype = ctypes.c_int
    lib.mgt_layer_status_word.restype = ctypes.c_int
    for name in ("mgt_layer_init", "mgt_layer_sizes", "mgt_layer_region", "mgt_layer_fwd",
                 "mgt_layer_bwd", "mgt_layer_get_error", "mgt_layer_profile",
                 "mgt_layer_profile_read", "mgt_gemm_bf16", "mgt_layernorm_bwd_noalloc",
                 "mgt_fp8_quantize", "mgt_gemm_fp8", "mgt_tp_rank_init", "mgt_tp_rank_sizes",
                 "mgt_tp_rank_partial", "mgt_tp_rank_fwd", "mgt_tp_rank_bwd",
                 "mgt_tp_rank_set_bands"):
        getattr(lib, name).restype = ctypes.c_int
    _LIB = lib
    return lib


def _check(code: int, what: str):
    if code != 0:
        raise MgtError(code, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class Layer:
    """One tensor-parallel GPT layer (logical tp_size shards on one GPU).

    dtype: "bf16" or "f32". Parameters are passed as a dict of device tensors in the packed
    per-shard layouts of include/mgt_layer.h (see PARAM_ORDER)."""

    def __init__(self, hidden, heads, ffn, seq, micro_batch, tp_size=1, dtype="bf16",
                 ln_eps=1e-5, gelu_tanh=0, causal=1, swiglu=0, disable_bias_linear=0,
                 sequence_parallel=0):
        self.lib = load_library()
        self.cfg = _Config(hidden, heads, ffn, seq, micro_batch, tp_size,
                           1 if dtype == "bf16" else 0, causal, ln_eps, 1, gelu_tanh, swiglu,
                           disable_bias_linear, sequence_parallel)
        self.dtype = dtype
        self.has_bias = not disable_bias_linear
        h = ctypes.c_void_p()
        _check(self.lib.mgt_layer_init(ctypes.byref(self.cfg), ctypes.byref(h)), "mgt_layer_init")
        self.handle = h

    @classmethod
    def from_config(cls, cfg):
        """Build from any object with hidden, heads, ffn, seq, micro_batch, tp_size, dtype,
        ln_eps, gelu_tanh (and optionally swiglu, disable_bias_linear, sequence_parallel)
        attributes."""
        return cls(cfg.hidden, cfg.heads, cfg.ffn, cfg.seq, cfg.micro_batch, cfg.tp_size,
                   cfg.dtype, cfg.ln_eps, cfg.gelu_tanh, swiglu=getattr(cfg, "swiglu", 0),
                   disable_bias_linear=getattr(cfg, "disable_bias_linear", 0),
                   sequence_parallel=getattr(cfg, "sequence_parallel", 0))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self.lib.mgt_layer_destroy(h)
            self.handle = None

    # ------------------------------------------------------------------ sizes / regions
    def sizes(self):
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self.lib.mgt_layer_sizes(self.handle, ctypes.byref(a), ctypes.byref(b)),
               "mgt_layer_sizes")
        return a.value, b.value

    def region(self, name):
        o, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self.lib.mgt_layer_region(self.handle, REGIONS[name], ctypes.byref(o),
                                         ctypes.byref(n)), "mgt_layer_region")
        return o.value, n.value

    def alloc_buffers(self, device="cuda"):
        """Caller-owned `saved` and (zeroed) `workspace` byte buffers."""
        import torch
        s, w = self.sizes()
        return (torch.empty(max(s, 256), dtype=torch.uint8, device=device),
                torch.zeros(max(w, 256), dtype=torch.uint8, device=device))

    def view(self, buf, name, dtype, shape):
        """Typed view of one region of a saved/workspace buffer (for inspection and tests)."""
        import math
        o, n = self.region(name)
        esz = buf.new_empty(0, dtype=dtype).element_size()
        cnt = math.prod(shape)
        assert cnt * esz == n, (name, cnt * esz, n)
        return buf[o:o + n].view(dtype).view(*shape)

    # ------------------------------------------------------------------ compute
    @staticmethod
    def _params(p: Dict) -> _Params:
        """Pointers in PARAM_ORDER; an absent entry (a bias of a layer built with
        disable_bias_linear) is passed as NULL."""
        return _Params(*[_ptr(p.get(n)) for n in PARAM_ORDER])

    def _check_types(self, params, acts, grads=None):
        import torch
        act = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        for n in PARAM_ORDER:
            if n not in params and not self.has_bias and n.startswith("b"):
                continue
            want = torch.float32 if n.startswith("ln") else act
            if params[n].dtype != want:
                raise TypeError("parameter %s must be %s" % (n, want))
            if grads is not None and grads[n].dtype != torch.float32:
                raise TypeError("gradient %s must be float32" % n)
        for t in acts:
            if t.dtype != act:
                raise TypeError("activations must be %s" % act)

    def fwd(self, params, x, y, saved, workspace, stream=None):
        self._check_types(params, (x, y))
        _check(self.lib.mgt_layer_fwd(self.handle, ctypes.byref(self._params(params)),
                                      _ptr(x), _ptr(y), _ptr(saved), _ptr(workspace),
                                      _stream_handle(stream)), "mgt_layer_fwd")

    def bwd(self, params, x, saved, dy, dx, grads, workspace, stream=None):
        self._check_types(params, (x, dy, dx), grads)
        _check(self.lib.mgt_layer_bwd(self.handle, ctypes.byref(self._params(params)),
                                      _ptr(x), _ptr(saved), _ptr(dy), _ptr(dx),
                                      ctypes.byref(self._params(grads)), _ptr(workspace),
                                      _stream_handle(stream)), "mgt_layer_bwd")

    def get_error(self, workspace, stream=None) -> int:
        return self.lib.mgt_layer_get_error(self.handle, _ptr(workspace), _stream_handle(stream))

    def status_word_ptr(self, workspace) -> int:
        """Device address of the status word inside `workspace`."""
        w = ctypes.c_void_p()
        _check(self.lib.mgt_layer_status_word(self.handle, _ptr(workspace), ctypes.byref(w)),
               "mgt_layer_status_word")
        return w.value

    def profile(self, enable=True):
        _check(self.lib.mgt_layer_profile(self.handle, 1 if enable else 0), "mgt_layer_profile")

    def profile_read(self):
        arr = (_KernelStat * 64)()
        n = ctypes.c_int()
        _check(self.lib.mgt_layer_profile_read(self.handle, arr, 64, ctypes.byref(n)),
               "mgt_layer_profile_read")
        return {arr[i].name.decode(): dict(launches=arr[i].launches, ms=arr[i].ms,
                                           flops=arr[i].flops, bytes=arr[i].bytes)
                for i in range(n.value)}


class TPRank:
    """One rank of a real tensor-parallel group (see mgt_tp_rank_* in include/mgt_layer.h):
    the rank's shard of the packed parameters, whole x / dy / y / dx, and a caller-provided
    all-reduce.

    allreduce(ptr, count, stream_handle) -> None must replace the `count` fp32 values at device
    address `ptr` by their sum over all ranks, ordered on the CUDA stream `stream_handle`
    (an int, 0 for the default stream). It is called 2 times per fwd and 2 per bwd (times the
    number of row bands, set_bands), always inside the workspace region `partial_region()`
    names; banded calls come on the rank's communication stream. bf16 only."""

    def __init__(self, hidden, heads, ffn, seq, micro_batch, tp_size, rank, ln_eps=1e-5,
                 gelu_tanh=0, swiglu=0, disable_bias_linear=0):
        self.lib = load_library()
        self.cfg = _Config(hidden, heads, ffn, seq, micro_batch, tp_size, 1, 1, ln_eps, 1,
                           gelu_tanh, swiglu, disable_bias_linear, 0)
        self.dtype = "bf16"
        self.has_bias = not disable_bias_linear
        h = ctypes.c_void_p()
        _check(self.lib.mgt_tp_rank_init(ctypes.byref(self.cfg), rank, ctypes.byref(h)),
               "mgt_tp_rank_init")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self.lib.mgt_tp_rank_destroy(h)
            self.handle = None

    def sizes(self):
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self.lib.mgt_tp_rank_sizes(self.handle, ctypes.byref(a), ctypes.byref(b)),
               "mgt_tp_rank_sizes")
        return a.value, b.value

    def set_bands(self, bands):
        """Split every shard sum into `bands` row bands whose exchanges overlap the next band's
        GEMM (see mgt_tp_rank_set_bands)."""
        _check(self.lib.mgt_tp_rank_set_bands(self.handle, int(bands)), "mgt_tp_rank_set_bands")

    def partial_region(self):
        o, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self.lib.mgt_tp_rank_partial(self.handle, ctypes.byref(o), ctypes.byref(n)),
               "mgt_tp_rank_partial")
        return o.value, n.value

    def alloc_buffers(self, device="cuda"):
        import torch
        s, w = self.sizes()
        return (torch.empty(max(s, 256), dtype=torch.uint8, device=device),
                torch.zeros(max(w, 256), dtype=torch.uint8, device=device))

    @staticmethod
    def _callback(allreduce):
        def cb(ptr, count, user, stream):
            try:
                allreduce(ptr, count, stream or 0)
                return 0
            except Exception:  # noqa: BLE001 - reported to the C side as a CUDA-class error
                import traceback
                traceback.print_exc()
                return 3
        return ALLREDUCE_FN(cb)

    def fwd(self, params, x, y, saved, workspace, allreduce, stream=None):
        Layer._check_types(self, params, (x, y))
        cb = self._callback(allreduce)
        _check(self.lib.mgt_tp_rank_fwd(self.handle, ctypes.byref(Layer._params(params)),
                                        _ptr(x), _ptr(y), _ptr(saved), _ptr(workspace), cb,
                                        None, _stream_handle(stream)), "mgt_tp_rank_fwd")

    def bwd(self, params, x, saved, dy, dx, grads, workspace, allreduce, stream=None):
        Layer._check_types(self, params, (x, dy, dx), grads)
        cb = self._callback(allreduce)
        _check(self.lib.mgt_tp_rank_bwd(self.handle, ctypes.byref(Layer._params(params)),
                                        _ptr(x), _ptr(saved), _ptr(dy), _ptr(dx),
                                        ctypes.byref(Layer._params(grads)), _ptr(workspace),
                                        cb, None, _stream_handle(stream)), "mgt_tp_rank_bwd")


def process_group_allreduce(workspace, offset, nbytes=None, group=None):
    """The all-reduce a TPRank needs, over a torch.distributed process group (NCCL for device
    workspaces): the callback views the `count` fp32 values at the address the layer passes,
    which must lie inside the rank's partial buffer (`nbytes` bytes at `offset` of
    `workspace`, TPRank.partial_region(); the rest of the workspace by default) -- the whole
    buffer, or one row band of it -- and sums them over the group in place, on the stream the
    layer passes (torch.distributed enqueues the collective there). Every rank of the group
    must make the same TPRank calls in the same order."""
    import torch
    import torch.distributed as dist
    base = workspace.data_ptr()
    end = workspace.numel() if nbytes is None else offset + nbytes

    def allreduce(ptr, count, stream):
        start = ptr - base
        if start < offset or (start - offset) % 4 or start + 4 * count > end or count < 1:
            raise ValueError("all-reduce buffer outside the rank's partial buffer")
        view = workspace[start:start + 4 * count].view(torch.float32)
        if workspace.is_cuda:
            with torch.cuda.stream(torch.cuda.ExternalStream(stream, device=workspace.device)):
                dist.all_reduce(view, group=group)
        else:
            dist.all_reduce(view, group=group)
    return allreduce


def gemm_bf16(A, B, C, M, N, K, a_mn, b_mn, lda, ldb, ldc, status, stream=None):
    """C[m, n] = sum_k A(m, k) B(n, k) on the tcgen05 path (see mgt_gemm_bf16)."""
    import torch
    if A.dtype != torch.bfloat16 or B.dtype != torch.bfloat16 or C.dtype != torch.float32:
        raise TypeError("gemm_bf16 takes bf16 A, B and an fp32 C")
    lib = load_library()
    _check(lib.mgt_gemm_bf16(M, N, K, a_mn, b_mn, _ptr(A), lda, _ptr(B), ldb, _ptr(C), ldc,
                             _ptr(status), _stream_handle(stream)), "mgt_gemm_bf16")


def fp8_quantize(x, q, scales, stream=None):
    """Per-tensor e4m3 quantisation (see mgt_fp8_quantize): x fp32 or bf16, q uint8 with
    x.numel() bytes, scales a 2-float device tensor receiving {amax, amax / 448}."""
    import torch
    if x.dtype not in (torch.float32, torch.bfloat16) or q.dtype != torch.uint8 or \
            scales.dtype != torch.float32 or scales.numel() < 2 or q.numel() < x.numel():
        raise TypeError("fp8_quantize takes fp32/bf16 x, uint8 q, 2 fp32 scales")
    lib = load_library()
    _check(lib.mgt_fp8_quantize(1 if x.dtype == torch.bfloat16 else 0, x.numel(), _ptr(x),
                                _ptr(q), _ptr(scales), _stream_handle(stream)),
           "mgt_fp8_quantize")


def gemm_fp8(A, B, a_scales, b_scales, C, M, N, K, lda, ldb, ldc, status, stream=None):
    """C = (A B^T) * a_scales[1] * b_scales[1] with e4m3 bytes A [M][K], B [N][K] (see
    mgt_gemm_fp8); C fp32 or bf16."""
    import torch
    if A.dtype != torch.uint8 or B.dtype != torch.uint8 or \
            C.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("gemm_fp8 takes uint8 A, B and an fp32/bf16 C")
    lib = load_library()
    _check(lib.mgt_gemm_fp8(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(a_scales),
                            _ptr(b_scales), _ptr(C), 0 if C.dtype == torch.float32 else 1, ldc,
                            _ptr(status), _stream_handle(stream)), "mgt_gemm_fp8")


def layernorm_bwd_noalloc(dtype, rows, h, dy, dres, x, gamma, mean, rstd, dx, dgamma, dbeta,
                          stream=None):
    """LayerNorm backward with library-owned scratch (see mgt_layernorm_bwd_noalloc): for
    callers that cannot allocate device memory. dtype: "bf16" or "f32"."""
    import torch
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    for t in (dy, dres, x, dx):
        if t is not None and t.dtype != act:
            raise TypeError("dy, dres, x, dx must be %s" % act)
    for t in (gamma, mean, rstd, dgamma, dbeta):
        if t.dtype != torch.float32:
            raise TypeError("gamma, mean, rstd, dgamma, dbeta must be float32")
    lib = load_library()
    _check(lib.mgt_layernorm_bwd_noalloc(1 if dtype == "bf16" else 0, rows, h, _ptr(dy),
                                         _ptr(dres), _ptr(x), _ptr(gamma), _ptr(mean),
                                         _ptr(rstd), _ptr(dx), _ptr(dgamma), _ptr(dbeta),
                                         _stream_handle(stream)), "mgt_layernorm_bwd_noalloc")


def debug_exp2(x, y, path, stream=None):
    """y = 2^x through the attention kernels' exponential (see mgt_debug_exp2): path 0 the
    hardware approximation, 1 the FMA-pipe polynomial. x, y fp32 device tensors."""
    import torch
    if x.dtype != torch.float32 or y.dtype != torch.float32 or y.numel() < x.numel():
        raise TypeError("debug_exp2 takes fp32 x and y")
    lib = load_library()
    _check(lib.mgt_debug_exp2(int(path), x.numel(), _ptr(x), _ptr(y), _stream_handle(stream)),
           "mgt_debug_exp2")


def debug_bounded_wait(limit_ns, status_ptr, stream=None):
    """Run the bounded-wait failure probe (see mgt_debug_bounded_wait); status_ptr is a device
    address of an int32 status word."""
    lib = load_library()
    _check(lib.mgt_debug_bounded_wait(int(limit_ns), ctypes.c_void_p(status_ptr),
                                      _stream_handle(stream)), "mgt_debug_bounded_wait")
