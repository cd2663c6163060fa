"""Arenas training linear on the CUDA path vs the oracle (needs a B200).

"Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
Sparsification", digest paragraph on Arenas: Y = X T alpha + lambda_t X W with
lambda_t cosine-decayed to 0.  One tensor-core kernel computes both products;
Y must meet the method's gate and the fp32 accumulation bound of both terms."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, gate, packed_to_host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sw():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_ternary_weight_b200.build import build
    build()
    import sparse_ternary_weight_b200 as sw
    return sw


CASES = [
    # (M, N, K, gran, group)
    (1, 128, 64, "group", 64),
    (17, 130, 256, "tensor", 0),
    (128, 256, 1024, "group", 128),
    (300, 384, 3072, "group", 128),
    (513, 129, 1024, "channel", 0),
    (64, 1000, 2048, "group", 256),
    (200, 512, 8192, "channel", 0),
]


@pytest.mark.parametrize("lam", [0.0, 0.37])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_arenas_vs_oracle(sw, orc_omp, case, lam):
    import torch
    M, N, K, gname, group = case
    g = GRAN[gname]
    grp = group if gname == "group" else 128
    W = synth.weights_student_t(N, K, 50000 + N + K)
    Wd = synth.f32_to_bf16_bits(W)
    Xb = synth.activations_bf16(M, K, 50500 + M)
    P = sw.quantize_pack(to_dev(W), g, grp)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    Wdt = to_dev(Wd.view(np.int16)).view(torch.bfloat16)
    y32 = sw.arenas_linear(X, P, Wdt, lam, torch.float32)
    yb = sw.arenas_linear(X, P, Wdt, lam, torch.bfloat16)
    assert sw.device_status() == 0
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc_omp.arenas_linear(Xb, idx, sgn, sc, Wd, np.float32(lam), N, K, g, grp)
    y = y32.cpu().numpy().astype(np.float64)
    assert gate(y, y_ref) <= 1e-3
    Xf = np.abs(synth.bf16_bits_to_f32(Xb)).astype(np.float64)
    Wq = np.abs(orc_omp.unpack_f32(idx, sgn, sc, N, K, g, grp)).astype(np.float64)
    Wl = np.abs(synth.bf16_bits_to_f32(Wd)).astype(np.float64)
    bound = 2.0 ** -16 * (Xf @ Wq.T + abs(lam) * (Xf @ Wl.T)) + 1e-30
    assert np.all(np.abs(y - y_ref) <= bound), float((np.abs(y - y_ref) / bound).max())
    assert gate(yb.float().cpu().numpy(), y_ref) <= 1e-3 + 2.0 ** -8
    assert torch.equal(yb, y32.to(torch.bfloat16))
    if lam == 0.0:
        # no residual: the plain prefill kernel (M > 32 goes there), bit for bit
        assert M <= 32 or torch.equal(y32, sw.linear(X, P, torch.float32))


def test_arenas_lambda_schedule(sw, orc):
    for step, total in ((0, 1000), (250, 1000), (500, 1000), (999, 1000), (1000, 1000), (5, 0)):
        assert abs(sw.arenas_lambda(step, total, 0.8) - np.float32(orc.arenas_lambda(step, total, 0.8))) <= 1e-7
