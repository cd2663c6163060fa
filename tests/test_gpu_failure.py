"""Failure detection and memory safety of the CUDA path (needs a B200).

* A bounded device wait that runs out reports SHERRY_ERR_TIMEOUT through
  sherry_device_status, the context stays usable, and the next call is correct.
  The wait is made to run out by giving the streaming decode kernel a budget of
  a few clock cycles (it holds no tensor memory and drains its own copies).
* Every output buffer is guarded by canary bytes on both sides; each kernel
  route (quantise + pack in every granularity, the decode kernels, the
  tensor-core kernels, unpack, batched calls) must write its output and nothing
  around it, on ragged shapes."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, canaried, canaries_intact, check_linear, packed_to_host, to_dev

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


def test_stream_wait_timeout_reports_and_recovers(sw, orc):
    import torch
    from sparse_ternary_weight_b200 import _abi
    L = _abi.lib()
    N, K = 3000, 3072                       # one token, group 128: the streaming kernel
    W = synth.weights_student_t(N, K, 16001)
    Xb = synth.activations_bf16(1, K, 16002)
    P = sw.quantize_pack(to_dev(W), "per_group", 128)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    assert sw.device_status() == 0
    prev = L.sherry_set_wait_budget(2)      # a wait that does not succeed at once gives up
    try:
        for _ in range(3):
            sw.linear(X, P)
        st = sw.device_status()
    finally:
        L.sherry_set_wait_budget(prev)
    assert st in (_abi.OK, _abi.ERR_TIMEOUT)
    assert L.sherry_set_wait_budget(0) == prev   # the default budget is back
    # the context is usable and the next calls are correct
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, oracle.PER_GROUP, 128)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, oracle.PER_GROUP, 128)
    for _ in range(2):
        check_linear(sw.linear(X, P).cpu().numpy(), y_ref, Xb, Wq)
    assert sw.device_status() == 0


QP_CANARY = [(33, 384, "group", 64), (7, 160, "channel", 0), (129, 3072, "tensor", 0), (5, 8192, "group", 128)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", QP_CANARY, ids=lambda c: f"{c[0]}x{c[1]}-{c[2]}{c[3]}")
def test_quantize_pack_canaries(sw, orc, case, dtype):
    import torch
    N, K, gname, group = case
    gran = GRAN[gname]
    W = synth.weights_student_t(N, K, 17000 + N)
    Wd = to_dev(W) if dtype == "f32" else to_dev(synth.f32_to_bf16_bits(W).view(np.int16)).view(torch.bfloat16)
    ns = sw.lib().sherry_num_scales(N, K, gran, group)
    fi, idx = canaried((N, K // 32), torch.int32)
    fs, sgn = canaried((N, K // 32), torch.uint8)
    fc, sc = canaried((ns,), torch.float32)
    P = sw.quantize_pack(Wd, gran, group, out=sw.PackedWeight(idx, sgn, sc, N, K, gran, group))
    torch.cuda.synchronize()
    assert canaries_intact(fi) and canaries_intact(fs) and canaries_intact(fc)
    ref = orc.quantize_pack(W if dtype == "f32" else synth.f32_to_bf16_bits(W), gran, group)
    got = packed_to_host(P)
    assert all(np.array_equal(a.reshape(-1).view(np.uint8), b.reshape(-1).view(np.uint8)) for a, b in zip(got, ref))


LIN_CANARY = [
    # (M, N, K, gran, group): one case per kernel route, ragged N
    (1, 1000, 3072, "group", 128),   # one-token streaming
    (2, 513, 1024, "channel", 0),    # two-token streaming
    (3, 700, 2048, "group", 256),    # three-token streaming
    (4, 1000, 3072, "group", 128),   # streaming, tensor-core consumers
    (1, 77, 96, "group", 32),        # general lookup-table
    (5, 300, 1024, "tensor", 0),     # warp MMA
    (13, 129, 3072, "group", 128),   # tcgen05 few-token
    (300, 200, 512, "group", 64),    # tcgen05 prefill
    (40, 33, 160, "group", 32),      # general lookup-table, several tokens
]


@pytest.mark.parametrize("ydt", ["f32", "bf16"])
@pytest.mark.parametrize("case", LIN_CANARY, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_linear_canaries(sw, orc, case, ydt):
    import torch
    M, N, K, gname, group = case
    gran = GRAN[gname]
    W = synth.weights_student_t(N, K, 18000 + N + K)
    Xb = synth.activations_bf16(M, K, 18500 + M)
    P = sw.quantize_pack(to_dev(W), gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    dt = torch.float32 if ydt == "f32" else torch.bfloat16
    fy, Y = canaried((M, N), dt)
    sw.linear(X, P, dt, out=Y)
    torch.cuda.synchronize()
    assert canaries_intact(fy)
    idx, sgn, sc = packed_to_host(P)
    check_linear(Y.float().cpu().numpy(), orc.linear(Xb, idx, sgn, sc, N, K, gran, group), Xb,
                 orc.unpack_f32(idx, sgn, sc, N, K, gran, group), y_is_bf16=(ydt == "bf16"))


def test_batched_and_unpack_canaries(sw, orc):
    import torch
    shapes = [(1000, 3072, "group", 128), (77, 96, "group", 32), (513, 2048, "tensor", 0), (129, 384, "channel", 0)]
    packs, Ws = [], []
    for i, (N, K, gname, group) in enumerate(shapes):
        W = synth.weights_normal(N, K, 19000 + i)
        Ws.append(W)
        packs.append(sw.quantize_pack(to_dev(W), GRAN[gname], group))
    for M in (1, 2, 6, 12, 40):
        pairs, fulls, outs = [], [], []
        for i, P in enumerate(packs):
            Xb = synth.activations_bf16(M, P.K, 19500 + i + M)
            pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P))
            f, y = canaried((M, P.N), torch.float32)
            fulls.append(f)
            outs.append(y)
        sw.linear_batched(pairs, torch.float32, outs=outs)
        torch.cuda.synchronize()
        assert all(canaries_intact(f) for f in fulls), M
    fulls, outs = [], []
    for P in packs:
        f, o = canaried((P.N, P.K), torch.bfloat16)
        fulls.append(f)
        outs.append(o)
    sw.unpack_batched(packs, outs)
    f1, o1 = canaried((packs[0].N, packs[0].K), torch.bfloat16)
    sw.unpack(packs[0], out=o1)
    torch.cuda.synchronize()
    assert all(canaries_intact(f) for f in fulls) and canaries_intact(f1)
    for P, o in zip(packs, outs):
        idx, sgn, sc = packed_to_host(P)
        ref = orc.unpack_bf16(idx, sgn, sc, P.N, P.K, P.granularity, P.group)
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), ref)
