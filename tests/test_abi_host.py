"""Host-only checks of the C ABI (no GPU): the library loads, exports every function that
include/mgt_layer.h declares, validates configurations synchronously, and lays out its buffers
consistently."""
import ctypes
import os
import re

import pytest

import tensor_transformer_layer_megatron_b200 as mgt
from mgt_inputs import CONFIGS, VARIANTS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mgt_layer.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"typedef[^;]*;", "", src)  # type declarations (a function-pointer type too)
    return sorted(set(re.findall(r"\b(mgt_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = mgt.load_library()
    names = declared_functions()
    assert "mgt_layer_fwd" in names and "mgt_layer_bwd" in names and "mgt_layer_init" in names
    for n in names:
        assert hasattr(lib, n), n


def _init(**kw):
    base = dict(hidden=64, heads=4, ffn=256, seq=32, micro_batch=2, tp_size=2, dtype=0,
                causal=1, ln_eps=1e-5, recompute_attn=1, gelu_tanh=0, swiglu=0,
                disable_bias_linear=0, sequence_parallel=0)
    base.update(kw)
    lib = mgt.load_library()
    cfg = mgt._Config(*[base[f] for f, _ in mgt._Config._fields_])
    h = ctypes.c_void_p()
    st = lib.mgt_layer_init(ctypes.byref(cfg), ctypes.byref(h))
    if st == 0:
        lib.mgt_layer_destroy(h)
    else:
        assert not h.value
    return st


def test_golden_tp_divisibility():
    path = os.path.join(ROOT, "tests", "golden", "tp_divisibility.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows
    for hidden, heads, tp, expect, per_shard in rows:
        st = _init(hidden=int(hidden), heads=int(heads), ffn=4 * int(hidden), seq=16,
                   micro_batch=1, tp_size=int(tp), dtype=1)
        assert mgt.STATUS[st] == "MGT_" + expect, (hidden, tp)
        if expect == "OK":
            assert int(hidden) // int(tp) == int(per_shard)


@pytest.mark.parametrize("kw,code", [
    (dict(hidden=0), 1), (dict(seq=-1), 1), (dict(heads=3), 1),       # h % H
    (dict(tp_size=3), 1),                                              # h % p
    (dict(heads=8, tp_size=16, hidden=128), 1),                        # H % p
    (dict(ffn=255), 1),                                                # f % p
    (dict(causal=0), 2), (dict(dtype=7), 2),
    (dict(dtype=1), 2),                   # bf16 needs head_dim 64/128 (here 16)
    (dict(dtype=1, hidden=128, heads=2, tp_size=2, ffn=200), 2),      # f/p = 100, not a multiple of 64
    (dict(hidden=512, heads=4), 2),       # fp32 head_dim 128 > 64
    (dict(swiglu=2), 1), (dict(disable_bias_linear=-1), 1),           # flags are 0 or 1
    (dict(sequence_parallel=3), 1),
    (dict(sequence_parallel=1, seq=33), 1),                           # s % p
    (dict(sequence_parallel=1, dtype=1, hidden=256, heads=2, ffn=512, seq=192), 2),  # s/p % 128
])
def test_init_rejects(kw, code):
    assert _init(**kw) == code


def test_init_accepts_every_workload():
    for c in CONFIGS:
        assert _init(hidden=c.hidden, heads=c.heads, ffn=c.ffn, seq=c.seq,
                     micro_batch=c.micro_batch, tp_size=c.tp_size,
                     dtype=1 if c.dtype == "bf16" else 0) == 0, c.name


def test_null_handle_and_status_strings():
    lib = mgt.load_library()
    assert lib.mgt_layer_sizes(None, None, None) == 1
    assert lib.mgt_layer_fwd(None, None, None, None, None, None, None) == 1
    assert lib.mgt_status_string(4) == b"device wait timed out"


@pytest.mark.parametrize("cfg", CONFIGS + VARIANTS, ids=lambda c: c.name)
def test_region_layout(cfg):
    L = mgt.Layer.from_config(cfg)
    saved, ws = L.sizes()
    T, h, f, e = cfg.tokens, cfg.hidden, cfg.ffn, 2 if cfg.dtype == "bf16" else 4
    f1 = cfg.fc1_rows  # SwiGLU keeps [gate | up] and its gradient: 2f columns
    expect = {"ln1": T * h * e, "qkv": 3 * T * h * e, "attn_o": T * h * e,
              "attn_lse": cfg.micro_batch * cfg.heads * cfg.seq * 4, "fc1_u": T * f1 * e,
              "fc1_a": T * f * e, "du": T * f1 * e, "dqkv": 3 * T * h * e}
    spans = []
    for name, rid in mgt.REGIONS.items():
        o, n = L.region(name)
        assert o % 256 == 0
        if name in expect:
            assert n == expect[name], name
        spans.append((rid >= 64, o, o + n))
        assert o + n <= (ws if rid >= 64 else saved)
    for buf in (False, True):
        s = sorted((a, b) for k, a, b in spans if k == buf)
        for (a0, b0), (a1, b1) in zip(s, s[1:]):
            assert b0 <= a1  # regions never overlap


# FP8 entry points: argument checks run before any CUDA call, so they are testable on the
# host. Fake, never-dereferenced addresses stand in for device pointers.
P16 = 0x10000  # 16-byte aligned
P_ODD = 0x10001


def test_fp8_quantize_rejects():
    lib = mgt.load_library()
    assert lib.mgt_fp8_quantize(1, 0, P16, P16, P16, None) == 1       # n < 1
    assert lib.mgt_fp8_quantize(1, 8, None, P16, P16, None) == 1      # null x
    assert lib.mgt_fp8_quantize(1, 8, P16, None, P16, None) == 1      # null q
    assert lib.mgt_fp8_quantize(1, 8, P16, P16, None, None) == 1      # null scales
    assert lib.mgt_fp8_quantize(7, 8, P16, P16, P16, None) == 2       # unknown dtype
    assert lib.mgt_fp8_quantize(0, 8, P16, P_ODD, P16, None) == 2     # q not 2-byte aligned


@pytest.mark.parametrize("M,N,K,lda,ldb,ldc,cd,code", [
    (0, 8, 16, 16, 16, 8, 0, 1),      # empty M
    (8, 0, 16, 16, 16, 8, 0, 1),      # empty N
    (8, 8, 0, 16, 16, 8, 0, 1),       # empty K
    (8, 8, 16, 8, 16, 8, 0, 1),       # lda < K
    (8, 8, 16, 16, 8, 8, 0, 1),       # ldb < K
    (8, 8, 16, 16, 16, 4, 0, 1),      # ldc < N
    (8, 8, 16, 16, 16, 8, 5, 2),      # unknown output dtype
    (8, 8, 24, 24, 32, 8, 0, 2),      # K not a multiple of 16 (TMA K steps of 16 bytes)
    (8, 8, 16, 24, 16, 8, 0, 2),      # lda not a multiple of 16 bytes
    (8, 10, 16, 16, 16, 10, 0, 2),    # fp32 rows not 16-byte multiples
    (8, 12, 16, 16, 16, 12, 1, 2),    # bf16 rows not 16-byte multiples
])
def test_gemm_fp8_rejects(M, N, K, lda, ldb, ldc, cd, code):
    lib = mgt.load_library()
    assert lib.mgt_gemm_fp8(M, N, K, P16, lda, P16, ldb, P16, P16, P16, cd, ldc, P16,
                            None) == code


def test_gemm_fp8_rejects_null_and_misaligned_pointers():
    lib = mgt.load_library()
    assert lib.mgt_gemm_fp8(8, 8, 16, None, 16, P16, 16, P16, P16, P16, 0, 8, P16, None) == 1
    assert lib.mgt_gemm_fp8(8, 8, 16, P16, 16, P16, 16, P16, P16, P16, 0, 8, None, None) == 1
    assert lib.mgt_gemm_fp8(8, 8, 16, P_ODD, 16, P16, 16, P16, P16, P16, 0, 8, P16, None) == 2
    assert lib.mgt_gemm_fp8(8, 8, 16, P16, 16, P16, 16, P16, P16, P_ODD, 0, 8, P16, None) == 2


def test_tp_rank_init_validates():
    lib = mgt.load_library()
    base = dict(hidden=256, heads=4, ffn=512, seq=128, micro_batch=2, tp_size=2)

    def init(rank, **kw):
        c = dict(base, **kw)
        cfg = mgt._Config(c["hidden"], c["heads"], c["ffn"], c["seq"], c["micro_batch"],
                          c["tp_size"], c.get("dtype", 1), 1, 1e-5, 1, 0, 0, 0,
                          c.get("sp", 0))
        h = ctypes.c_void_p()
        st = lib.mgt_tp_rank_init(ctypes.byref(cfg), rank, ctypes.byref(h))
        if st == 0:
            lib.mgt_tp_rank_destroy(h)
        return st

    assert init(0) == 0 and init(1) == 0
    assert init(2) == 1 and init(-1) == 1                    # rank outside the group
    assert init(0, dtype=0) == 2                              # bf16 only
    assert init(0, sp=1) == 2                                 # no sequence parallelism here
    assert init(0, heads=3) == 1                              # the layer itself is invalid
    r = mgt.TPRank(256, 4, 512, 128, 2, 2, 1)
    saved, ws = r.sizes()
    off, n = r.partial_region()
    assert n == 256 * 256 * 4 and off % 256 == 0 and off + n <= ws
    # null pointers and a missing all-reduce are rejected before any CUDA call
    null = mgt._Params(*([None] * 12))
    assert lib.mgt_tp_rank_fwd(r.handle, ctypes.byref(null), None, None, None, None,
                               mgt.ALLREDUCE_FN(0), None, None) == 1


@pytest.mark.parametrize("bad", ["dy", "dres", "x", "gamma", "mean", "rstd", "dx", "dgamma",
                                 "dbeta"])
def test_layernorm_bwd_noalloc_rejects_misaligned_pointers(bad):
    # The pointers are never dereferenced: validation must reject a misaligned view before any
    # CUDA call (this host has no GPU, so reaching the device lookup would return MGT_ECUDA).
    lib = mgt.load_library()
    ptr = {k: 0x10000 + 0x1000 * i for i, k in enumerate(
        ("dy", "dres", "x", "gamma", "mean", "rstd", "dx", "dgamma", "dbeta"))}
    ptr[bad] += 2 if bad in ("mean", "rstd", "dgamma", "dbeta") else 4
    vp = ctypes.c_void_p
    st = lib.mgt_layernorm_bwd_noalloc(1, 16, 512, vp(ptr["dy"]), vp(ptr["dres"]), vp(ptr["x"]),
                                       vp(ptr["gamma"]), vp(ptr["mean"]), vp(ptr["rstd"]),
                                       vp(ptr["dx"]), vp(ptr["dgamma"]), vp(ptr["dbeta"]), None)
    assert st == 2, (bad, st)


def test_debug_exp2_rejects_bad_arguments():
    lib = mgt.load_library()
    vp = ctypes.c_void_p
    assert lib.mgt_debug_exp2(2, 4, vp(P16), vp(P16), None) == 1   # unknown path
    assert lib.mgt_debug_exp2(1, -1, vp(P16), vp(P16), None) == 1  # negative count
    assert lib.mgt_debug_exp2(1, 4, None, vp(P16), None) == 1      # null input
    assert lib.mgt_debug_exp2(0, 0, None, None, None) == 0         # nothing to do
