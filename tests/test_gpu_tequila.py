"""The Tequila-style dead-weight term on the CUDA path vs the oracle (needs a B200).

"Sherry, Tequila and Fairies in Python", sections 1.2 and 2.1: the weights the
quantiser zeroes are kept as B = eps * w (here Sherry's zeroed weight of every
block of 4, rounded to bf16) and add F.linear(ones, B) -- a per-row bias -- or
F.linear(sign(x), B) to the layer.  The dead-weight plane and its row sums
must equal the oracle's bit for bit; Y must meet the method's gate and the
fp32 accumulation bound widened by the term's own fp32 sum."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, elementwise_bound, gate, packed_to_host, to_dev

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


def _u16(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("case", [(64, 256, "group", 128, "f32"), (3072, 3072, "group", 128, "f32"),
                                  (1024, 8192, "channel", 0, "f32"), (33, 96, "group", 32, "bf16"),
                                  (300, 3072, "tensor", 0, "bf16"), (1, 32, "group", 32, "f32")],
                         ids=lambda c: f"{c[0]}x{c[1]}-{c[2]}{c[3]}-{c[4]}")
def test_dead_plane_bit_exact(sw, orc, case):
    import torch
    N, K, gname, group, dt = case
    g = GRAN[gname]
    grp = group if gname == "group" else 128
    eps = 1e-2
    W = synth.weights_student_t(N, K, 40000 + N + K)
    Wh = synth.f32_to_bf16_bits(W) if dt == "bf16" else W
    Wd = to_dev(Wh.view(np.int16)).view(torch.bfloat16) if dt == "bf16" else to_dev(W)
    P, D, bias = sw.quantize_pack_tequila(Wd, g, grp, eps)
    D_ref, b_ref = orc.tequila_dead(Wh, np.float32(eps))
    assert np.array_equal(_u16(D), D_ref)
    assert np.array_equal(bias.cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
    ref = orc.quantize_pack(Wh, g, grp)
    got = packed_to_host(P)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    assert np.array_equal(got[2].view(np.uint32), ref[2].view(np.uint32))


@pytest.mark.parametrize("ydt", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["ones", "sign"])
@pytest.mark.parametrize("case", [(1, 3000, 3072, "group", 128), (2, 513, 1024, "channel", 0),
                                  (5, 300, 1024, "tensor", 0), (13, 129, 3072, "group", 128),
                                  (40, 200, 512, "group", 64), (300, 77, 2080, "group", 32)],
                         ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_linear_tequila_vs_oracle(sw, orc, case, mode, ydt):
    import torch
    M, N, K, gname, group = case
    g = GRAN[gname]
    grp = group if gname == "group" else 128
    W = synth.weights_student_t(N, K, 41000 + N + K)
    Xb = synth.activations_bf16(M, K, 41500 + M)
    Xb[:, ::7] = 0  # exact zeros: sign(0) = 0
    P, D, bias = sw.quantize_pack_tequila(to_dev(W), g, grp, 1e-2)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    dt = torch.float32 if ydt == "f32" else torch.bfloat16
    Y = sw.linear_tequila(X, P, D, bias, mode, dt)
    torch.cuda.synchronize()
    idx, sgn, sc = packed_to_host(P)
    Dh = _u16(D)
    T = orc.tequila_term(Xb, idx, Dh, bias.cpu().numpy(), N, K, 0 if mode == "ones" else 1)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, g, grp) + T
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, g, grp)
    y = Y.float().cpu().numpy()
    if ydt == "bf16":
        assert gate(y, y_ref) <= 1e-3 + 2.0 ** -8
        # bf16 Y is the rounding of the fp32 result
        assert torch.equal(Y, sw.linear_tequila(X, P, D, bias, mode, torch.float32).to(torch.bfloat16))
        return
    assert gate(y, y_ref) <= 1e-3
    dabs = np.abs(synth.bf16_bits_to_f32(Dh)).astype(np.float64).sum(1)
    bound = elementwise_bound(synth.bf16_bits_to_f32(Xb), Wq) + 2.0 ** -20 * dabs + 2.0 ** -24 * np.abs(y_ref)
    assert np.all(np.abs(y.astype(np.float64) - y_ref) <= bound)
