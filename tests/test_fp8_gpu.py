"""FP8 (e4m3) path on the GPU against the oracle: the per-tensor quantiser element by element
(same fp32 scaling, same round-to-nearest-even decision, saturation), and the tcgen05
kind::f8f6f4 GEMM on oracle-quantised operands over ragged and full-size shapes."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import tensor_transformer_layer_megatron_b200 as mgt

pytestmark = pytest.mark.gpu


def _encode(qvals):
    """e4m3 values (exactly representable) -> their bytes."""
    return torch.tensor(np.asarray(qvals, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)


def _decode(qbytes):
    return qbytes.cpu().view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [1, 7, 1000, (1 << 20) + 3])
def test_fp8_quantize_matches_oracle(dtype, n):
    g = torch.Generator("cpu").manual_seed(2000 + n)
    x = torch.randn(n, generator=g) * 2.5
    x[0] = 37.0 if n > 1 else x[0]  # a clear amax
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    xd = x.cuda()
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(2, dtype=torch.float32, device="cuda")
    mgt.fp8_quantize(xd, q, scales)
    torch.cuda.synchronize()
    ref_q, amax, d = oracle.quantize_e4m3(x.float().numpy())
    assert float(scales[0]) == amax
    assert float(scales[1]) == d
    got = _decode(q)
    assert np.array_equal(got, ref_q), np.flatnonzero(got != ref_q)[:10]


SHAPES = [(256, 512, 128), (200, 300, 256), (1, 8, 16), (129, 129, 144), (1000, 520, 4096),
          (2048, 12288, 4096)]


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fp8_gemm_matches_oracle(M, N, K, out):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    qa, amax_a, da = oracle.quantize_e4m3(rng.normal(size=(M, K)))
    qb, amax_b, db = oracle.quantize_e4m3(rng.normal(size=(N, K)) * 0.5)
    A = _encode(qa).cuda()
    B = _encode(qb).cuda()
    sa = torch.tensor([amax_a, da], dtype=torch.float32, device="cuda")
    sb = torch.tensor([amax_b, db], dtype=torch.float32, device="cuda")
    al = 4 if out == "f32" else 8  # 16-byte output rows
    ldc = (N + al - 1) // al * al
    C = torch.full((M, ldc), float("nan"), device="cuda",
                   dtype=torch.float32 if out == "f32" else torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mgt.gemm_fp8(A, B, sa, sb, C, M, N, K, K, K, ldc, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = C[:, :N].double().cpu().numpy()
    ref = oracle.gemm_fp8(qa, np.float32(da), qb, np.float32(db))
    err = float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
    path = os.environ.get("MGT_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"fp8_gemm": [M, N, K, out], "err": err}) + "\n")
    assert np.all(np.isfinite(got))
    # products of e4m3 codes are exact in fp32; what remains is fp32 accumulation over K and
    # the scale multiply (the layer's fp32 bound), plus the bf16 output rounding (2^-9)
    assert err <= (1e-4 if out == "f32" else 1e-4 + 2.0 ** -8), err
    if ldc > N:  # padding columns are never written
        assert torch.isnan(C[:, N:].float()).all()
