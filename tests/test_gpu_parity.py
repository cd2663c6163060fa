"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Packed idx/sgn planes and scales must be bit-exact; unpacked bf16 weights must
be bit-exact; Y must satisfy max|y - y_ref| / max|y_ref| <= 1e-3 against the
fp64 oracle and, for fp32 Y, every element must lie within 2^-16 * sum|x||w|
of it (the fp32 accumulation bound, far tighter than the gate)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, check_linear, packed_to_host, to_dev

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


def _weights(kind, N, K, seed):
    if kind == "normal":
        return synth.weights_normal(N, K, seed, outlier_frac=0.01)
    if kind == "t4":
        return synth.weights_student_t(N, K, seed)
    if kind == "ties":   # coarse grid: many ties and exact zeros, signed zeros
        W = np.round(synth.weights_normal(N, K, seed) * 64) / np.float32(64)
        W[:, ::7] = -0.0
        return W.astype(np.float32)
    raise ValueError(kind)


QP_CASES = [
    # (N, K, gran, group, kind)
    (64, 256, "group", 128, "normal"),
    (1, 32, "group", 32, "normal"),
    (3, 96, "group", 96, "ties"),
    (7, 160, "group", 32, "t4"),
    (33, 384, "group", 128, "ties"),
    (33, 384, "group", 64, "t4"),
    (5, 3072, "group", 128, "t4"),
    (17, 8192, "group", 256, "normal"),
    (9, 3072, "group", 3072, "t4"),
    (2, 65536, "group", 128, "t4"),
    (64, 256, "channel", 0, "normal"),
    (3, 96, "channel", 0, "ties"),
    (5, 3072, "channel", 0, "t4"),
    (11, 8192, "channel", 0, "ties"),
    (64, 256, "tensor", 0, "normal"),
    (7, 96, "tensor", 0, "ties"),
    (129, 3072, "tensor", 0, "t4"),
    (300, 160, "tensor", 0, "t4"),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", QP_CASES, ids=lambda c: f"{c[0]}x{c[1]}-{c[2]}{c[3]}-{c[4]}")
def test_quantize_pack_bit_exact(sw, orc, case, dtype):
    import torch
    N, K, gname, group, kind = case
    W = _weights(kind, N, K, seed=N * 7 + K)
    gran = GRAN[gname]
    if dtype == "bf16":
        Wb = synth.f32_to_bf16_bits(W)
        Wd = to_dev(Wb.view(np.int16)).view(torch.bfloat16)
        ref = orc.quantize_pack(Wb, gran, group)
    else:
        Wd = to_dev(W)
        ref = orc.quantize_pack(W, gran, group)
    P = sw.quantize_pack(Wd, gran, group)
    got = packed_to_host(P)
    for g, r, name in zip(got, ref, ("idx", "sgn", "scales")):
        assert np.array_equal(g.reshape(-1).view(np.uint8), r.reshape(-1).view(np.uint8)), name


def test_quantize_pack_empty_and_degenerate(sw, orc):
    import torch
    # N = 0: per-tensor scale = 0 / max(0, 1) = 0
    W = torch.zeros((0, 64), dtype=torch.float32, device="cuda")
    P = sw.quantize_pack(W, "per_tensor")
    assert P.scales.cpu().tolist() == [0.0]
    P = sw.quantize_pack(W, "per_group", 32)
    assert P.idx.numel() == 0
    # all-zero weights: every scale 0, every block zeroes position 0, kept signs +
    W = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    P = sw.quantize_pack(W, "per_channel")
    idx, sgn, sc = packed_to_host(P)
    assert np.all(idx == 0) and np.all(sgn == 0) and np.all(sc == 0)
    # all weights -0.0: same code as +0.0
    Wn = torch.full((4, 64), -0.0, dtype=torch.float32, device="cuda")
    idx2, sgn2, _ = packed_to_host(sw.quantize_pack(Wn, "per_channel"))
    assert np.array_equal(idx, idx2) and np.array_equal(sgn, sgn2)


@pytest.mark.parametrize("case", [(64, 256, "group", 128), (33, 384, "group", 96), (5, 3072, "channel", 0),
                                  (129, 160, "tensor", 0), (16, 8192, "group", 32)],
                         ids=lambda c: f"{c[0]}x{c[1]}-{c[2]}{c[3]}")
def test_unpack_bit_exact(sw, orc, case):
    N, K, gname, group = case
    gran = GRAN[gname]
    W = _weights("t4", N, K, seed=31 + N)
    P = sw.quantize_pack(to_dev(W), gran, group)
    idx, sgn, sc = packed_to_host(P)
    ref = orc.unpack_bf16(idx, sgn, sc, N, K, gran, group)
    got = sw.unpack(P).cpu().view(__import__("torch").int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


LIN_CASES = [
    # (M, N, K, gran, group)
    (1, 64, 256, "group", 128),     # the tiny single-linear workload
    (1, 1, 32, "group", 32),
    (1, 100, 96, "group", 96),      # K % 128 != 0 path
    (1, 257, 384, "group", 64),
    (1, 300, 3072, "group", 128),
    (1, 1024, 3072, "group", 128),
    (1, 3072, 8192, "group", 128),
    (1, 70, 8192, "channel", 0),
    (1, 513, 160, "tensor", 0),
    (1, 200, 1024, "group", 256),
    (1, 130, 512, "group", 256),    # one-token kernel, one 512-weight unit, two groups of 256
    (1, 64, 2048, "group", 32),
    (2, 129, 512, "group", 128),    # two tokens: streaming kernel from here on
    (2, 300, 3072, "group", 128),
    (2, 513, 1024, "channel", 0),
    (2, 77, 1536, "group", 256),
    (2, 1000, 8192, "tensor", 0),
    (3, 64, 3072, "channel", 0),    # three tokens: streaming lookup kernel; four: its tensor-core consumers
    (3, 1000, 2048, "group", 256),
    (4, 500, 1024, "group", 128),
    (4, 77, 768, "tensor", 0),
    (4, 100, 96, "group", 32),      # K % 256 != 0: general kernel
    (5, 33, 256, "tensor", 0),
    (8, 1024, 3072, "group", 128),
    (16, 512, 2048, "group", 128),
    (16, 77, 96, "group", 32),
    (17, 256, 1024, "group", 128),
    (33, 130, 512, "channel", 0),
]


@pytest.mark.parametrize("ydt", ["f32", "bf16"])
@pytest.mark.parametrize("case", LIN_CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_linear_vs_oracle(sw, orc, case, ydt):
    import torch
    M, N, K, gname, group = case
    gran = GRAN[gname]
    W = _weights("t4", N, K, seed=1000 + N + K)
    Xb = synth.activations_bf16(M, K, seed=2000 + M + K)
    P = sw.quantize_pack(to_dev(W), gran, group)
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y32 = sw.linear(X, P, torch.float32)
    check_linear(y32.cpu().numpy(), y_ref, Xb, Wq)
    if ydt == "bf16":
        yb = sw.linear(X, P, torch.bfloat16)
        check_linear(yb.float().cpu().numpy(), y_ref, Xb, Wq, y_is_bf16=True)
        # bf16 Y is the round-to-nearest-even of the fp32 accumulator
        assert torch.equal(yb, y32.to(torch.bfloat16))
    # deterministic
    assert torch.equal(sw.linear(X, P, torch.float32), y32)


def test_linear_hand_worked_row(sw):
    """The hand-worked 32-weight row (tests/golden/hand_worked.json): y = 15.25."""
    import json
    import os
    import torch
    hw = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))["row"]
    W = torch.tensor([hw["w"]], dtype=torch.float32, device="cuda")
    for g, grp in (("per_channel", 0), ("per_group", 32), ("per_tensor", 0)):
        P = sw.quantize_pack(W, g, grp)
        assert P.idx.cpu().numpy().view(np.uint32)[0, 0] == int(hw["idx_word"], 16)
        assert P.sgn.cpu().tolist() == [[int(hw["sgn_byte"], 16)]]
        assert P.scales.cpu().tolist() == [hw["alpha"]]
        X = torch.ones((1, 32), dtype=torch.bfloat16, device="cuda")
        assert sw.linear(X, P).item() == hw["y_all_ones"]
        assert sw.unpack(P).float().cpu().numpy().tolist() == [[t * hw["alpha"] for t in hw["t"]]]


def test_linear_batched_matches_oracle(sw, orc):
    import torch
    shapes = [(1024, 3072, "group", 128), (300, 3072, "channel", 0), (64, 96, "group", 32),
              (513, 8192, "group", 128), (77, 160, "tensor", 0), (2048, 2048, "group", 64)]
    for M in (1, 2, 4, 7, 16):
        pairs, refs = [], []
        for i, (N, K, gname, group) in enumerate(shapes):
            gran = GRAN[gname]
            W = _weights("normal", N, K, seed=3000 + i)
            Xb = synth.activations_bf16(M, K, seed=4000 + i + 10 * M)
            P = sw.quantize_pack(to_dev(W), gran, group)
            idx, sgn, sc = packed_to_host(P)
            refs.append((orc.linear(Xb, idx, sgn, sc, N, K, gran, group),
                         orc.unpack_f32(idx, sgn, sc, N, K, gran, group), Xb))
            pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P))
        outs = sw.linear_batched(pairs, torch.float32)
        for y, (y_ref, Wq, Xb) in zip(outs, refs):
            check_linear(y.cpu().numpy(), y_ref, Xb, Wq)
        outs2 = sw.linear_batched(pairs, torch.float32)
        assert all(torch.equal(a, b) for a, b in zip(outs, outs2))


def test_split_k_tickets_left_zero(sw):
    """A split-K call leaves its ticket counters at zero, so back-to-back calls
    on one workspace stay correct."""
    import torch
    W = torch.randn(64, 8192, device="cuda") * 0.02
    P = sw.quantize_pack(W)
    X = torch.randn(1, 8192, device="cuda").to(torch.bfloat16)
    from sparse_ternary_weight_b200 import _abi
    L = _abi.lib()
    wsb = L.sherry_workspace_bytes(_abi.OP_LINEAR, 1, 64, 8192, _abi.PER_GROUP, 128)
    assert wsb > 0   # this shape splits K across CTAs
    ys = [sw.linear(X, P) for _ in range(5)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    ws = sw._ws_cache[(str(X.device), "linear")]
    ticket_bytes = 256 * 1024  # the ticket region at the front of every linear workspace
    assert int(ws[:ticket_bytes].view(torch.int32).abs().sum()) == 0


STREAM_SHAPES = [(1024, 3072, "group", 128), (300, 3072, "channel", 0), (3072, 8192, "group", 128),
                 (77, 1024, "group", 256), (513, 2048, "tensor", 0), (8192, 3072, "group", 128),
                 (1, 512, "group", 128), (257, 3072, "group", 256), (96, 1536, "group", 256)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 12, 16])
def test_stream_batch_many_problems_vs_oracle(sw, orc, M):
    """Batches of 1 to 16 tokens over many eligible linears (the streaming kernel,
    lookup tables up to three tokens, tensor-core consumers from four: units split
    evenly over CTAs, tiles straddling CTAs finished through the ticket)."""
    import torch
    pairs, refs = [], []
    for i in range(24):
        N, K, gname, group = STREAM_SHAPES[i % len(STREAM_SHAPES)]
        gran = GRAN[gname]
        W = _weights("t4" if i % 2 else "normal", N, K, seed=5000 + i)
        Xb = synth.activations_bf16(M, K, seed=6000 + i + 100 * M)
        P = sw.quantize_pack(to_dev(W), gran, group)
        idx, sgn, sc = packed_to_host(P)
        refs.append((orc.linear(Xb, idx, sgn, sc, N, K, gran, group), orc.unpack_f32(idx, sgn, sc, N, K, gran, group),
                     Xb))
        pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P))
    for ydt in (torch.float32, torch.bfloat16):
        outs = sw.linear_batched(pairs, ydt)
        for y, (y_ref, Wq, Xb) in zip(outs, refs):
            check_linear(y.float().cpu().numpy(), y_ref, Xb, Wq, y_is_bf16=(ydt == torch.bfloat16))
        again = sw.linear_batched(pairs, ydt)
        assert all(torch.equal(a, b) for a, b in zip(outs, again))
    # single calls agree with the oracle as well
    for (X, P), (y_ref, Wq, Xb) in zip(pairs[:8], refs[:8]):
        check_linear(sw.linear(X, P).cpu().numpy(), y_ref, Xb, Wq)


PREFILL_CASES = [
    # (M, N, K, gran, group): M >= 17 runs the tcgen05 kernel
    (17, 128, 64, "tensor", 0),
    (128, 128, 128, "group", 128),
    (129, 200, 256, "group", 64),
    (300, 384, 3072, "group", 128),
    (513, 129, 1024, "group", 256),
    (64, 256, 2048, "channel", 0),
    (40, 1000, 512, "group", 512),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_prefill_tensor_core_vs_oracle(sw, orc, case):
    import torch
    from sparse_ternary_weight_b200 import _abi
    M, N, K, gname, group = case
    gran = GRAN[gname]
    W = _weights("t4", N, K, seed=7000 + N + K)
    Xb = synth.activations_bf16(M, K, seed=8000 + M + K)
    P = sw.quantize_pack(to_dev(W), gran, group)
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y32 = sw.linear(X, P, torch.float32)
    yb = sw.linear(X, P, torch.bfloat16)
    assert _abi.lib().sherry_device_status(None) == 0
    check_linear(y32.cpu().numpy(), y_ref, Xb, Wq)
    check_linear(yb.float().cpu().numpy(), y_ref, Xb, Wq, y_is_bf16=True)
    assert torch.equal(yb, y32.to(torch.bfloat16))
    assert torch.equal(sw.linear(X, P, torch.float32), y32)


SKINNY_CASES = [
    # (M, N, K, gran, group): 9 <= M <= 32 runs the tcgen05 few-token kernel
    (9, 128, 256, "group", 128),
    (10, 300, 1024, "channel", 0),
    (11, 1024, 3072, "group", 128),
    (12, 77, 512, "tensor", 0),
    (16, 2048, 2048, "group", 64),
    (17, 200, 768, "group", 256),
    (24, 129, 3072, "group", 128),
    (32, 512, 8192, "channel", 0),
]


@pytest.mark.parametrize("case", SKINNY_CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_skinny_tensor_core_vs_oracle(sw, orc, case):
    import torch
    from sparse_ternary_weight_b200 import _abi
    M, N, K, gname, group = case
    gran = GRAN[gname]
    W = _weights("normal", N, K, seed=9000 + N + K)
    Xb = synth.activations_bf16(M, K, seed=9500 + M + K)
    P = sw.quantize_pack(to_dev(W), gran, group)
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y32 = sw.linear(X, P, torch.float32)
    yb = sw.linear(X, P, torch.bfloat16)
    assert _abi.lib().sherry_device_status(None) == 0
    check_linear(y32.cpu().numpy(), y_ref, Xb, Wq)
    check_linear(yb.float().cpu().numpy(), y_ref, Xb, Wq, y_is_bf16=True)
    assert torch.equal(yb, y32.to(torch.bfloat16))


def test_skinny_batch_vs_oracle(sw, orc):
    """Several linears with 9..16 tokens in one launch of the tcgen05 few-token kernel."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    shapes = [(1024, 3072, "group", 128), (300, 3072, "channel", 0), (3072, 8192, "group", 128),
              (77, 1024, "group", 256), (513, 2048, "tensor", 0)]
    for M in (9, 13, 16):
        pairs, refs = [], []
        for i, (N, K, gname, group) in enumerate(shapes):
            gran = GRAN[gname]
            W = _weights("t4", N, K, seed=9900 + i)
            Xb = synth.activations_bf16(M, K, seed=9950 + i + 10 * M)
            P = sw.quantize_pack(to_dev(W), gran, group)
            idx, sgn, sc = packed_to_host(P)
            refs.append((orc.linear(Xb, idx, sgn, sc, N, K, gran, group), orc.unpack_f32(idx, sgn, sc, N, K, gran, group), Xb))
            pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P))
        outs = sw.linear_batched(pairs, torch.float32)
        assert _abi.lib().sherry_device_status(None) == 0
        for y, (y_ref, Wq, Xb) in zip(outs, refs):
            check_linear(y.cpu().numpy(), y_ref, Xb, Wq)


SKINNY_MIN_M = 9   # fewest tokens routed to the tcgen05 few-token kernel
MIXED_SHAPES = [(1024, 3072, "group", 128), (300, 768, "channel", 0), (200, 96, "group", 32),
                (129, 3072, "group", 128), (96, 320, "group", 64), (513, 1024, "tensor", 0)]


@pytest.mark.parametrize("M", [1, 2, 9, 20, 33, 300])
def test_batched_mixed_routes_vs_oracle(sw, orc, M):
    """A batch whose problems take different kernels (few-token tensor-core
    kernel, one prefill launch each, lookup-table kernel) agrees with the oracle;
    problems on the tensor-core kernels equal their single calls bit for bit."""
    import torch
    pairs, refs = [], []
    for i, (N, K, gname, group) in enumerate(MIXED_SHAPES):
        gran = GRAN[gname]
        W = _weights("t4", N, K, seed=12000 + i)
        Xb = synth.activations_bf16(M, K, seed=12500 + i + 7 * M)
        P = sw.quantize_pack(to_dev(W), gran, group)
        idx, sgn, sc = packed_to_host(P)
        refs.append((orc.linear(Xb, idx, sgn, sc, N, K, gran, group), orc.unpack_f32(idx, sgn, sc, N, K, gran, group), Xb))
        pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P))
    outs = sw.linear_batched(pairs, torch.float32)
    from sparse_ternary_weight_b200 import _abi
    assert _abi.lib().sherry_device_status(None) == 0
    for y, (y_ref, Wq, Xb) in zip(outs, refs):
        check_linear(y.cpu().numpy(), y_ref, Xb, Wq)
    for (X, P), y, (N, K, gname, group) in zip(pairs, outs, MIXED_SHAPES):
        mstream = 5 <= M <= 16 and K % 512 == 0 and (gname != "group" or group in (128, 256))
        tc = (not mstream and SKINNY_MIN_M <= M <= 32 and K % 256 == 0 and (gname != "group" or group % 64 == 0)) or \
             (M >= 17 and K % 64 == 0 and (gname != "group" or group % 64 == 0))
        if tc:
            assert torch.equal(sw.linear(X, P), y)


HMMA_CASES = [
    # (M, N, K, gran, group): 2 <= M <= 8 with K % 128 == 0 runs the warp-MMA kernel (larger M the
    # tcgen05 few-token kernel)
    (2, 64, 128, "group", 32),
    (2, 129, 384, "channel", 0),
    (4, 33, 640, "group", 128),
    (9, 500, 1152, "group", 96),
    (8, 1000, 8192, "tensor", 0),
    (7, 17, 2048, "group", 256),
    (8, 3072, 3072, "group", 128),
    (12, 1000, 8192, "tensor", 0),
]


@pytest.mark.parametrize("case", HMMA_CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-{c[3]}{c[4]}")
def test_warp_mma_vs_oracle(sw, orc, case):
    import torch
    from sparse_ternary_weight_b200 import _abi
    M, N, K, gname, group = case
    gran = GRAN[gname]
    W = _weights("t4", N, K, seed=13000 + N + K)
    Xb = synth.activations_bf16(M, K, seed=13500 + M + K)
    P = sw.quantize_pack(to_dev(W), gran, group)
    idx, sgn, sc = packed_to_host(P)
    y_ref = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y32 = sw.linear(X, P, torch.float32)
    yb = sw.linear(X, P, torch.bfloat16)
    assert _abi.lib().sherry_device_status(None) == 0
    check_linear(y32.cpu().numpy(), y_ref, Xb, Wq)
    check_linear(yb.float().cpu().numpy(), y_ref, Xb, Wq, y_is_bf16=True)
    assert torch.equal(yb, y32.to(torch.bfloat16))
    assert torch.equal(sw.linear(X, P, torch.float32), y32)


def test_unpack_batched_matches_single_and_oracle(sw, orc):
    """Several weights of different shapes and granularities in one unpack launch:
    bit-identical to the single calls and to the oracle."""
    import torch
    shapes = [(64, 256, "group", 128), (3, 96, "channel", 0), (33, 384, "group", 64), (7, 160, "tensor", 0),
              (300, 3072, "group", 128), (1, 32, "group", 32)]
    packs, refs = [], []
    for i, (N, K, gname, group) in enumerate(shapes):
        gran = GRAN[gname]
        W = _weights("ties" if i % 2 else "t4", N, K, seed=14000 + i)
        P = sw.quantize_pack(to_dev(W), gran, group)
        packs.append(P)
        idx, sgn, sc = packed_to_host(P)
        refs.append(orc.unpack_bf16(idx, sgn, sc, N, K, gran, group))
    outs = sw.unpack_batched(packs)
    for P, o, ref in zip(packs, outs, refs):
        got = o.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, ref)
        assert torch.equal(o, sw.unpack(P))


MAXK_CASES = [
    # (M, N, gran, group) at K = SHERRY_MAX_K: one case per linear kernel route
    (1, 5, "group", 128),   # one-token streaming kernel
    (2, 5, "group", 128),   # two-token streaming kernel
    (3, 5, "channel", 0),   # three-token streaming kernel
    (4, 5, "group", 256),   # streaming kernel, tensor-core consumers
    (1, 3, "group", 32),    # general lookup-table kernel
    (5, 5, "group", 128),   # streaming kernel, tensor-core consumers (8 token columns)
    (16, 5, "channel", 0),  # streaming kernel, tensor-core consumers (16 token columns)
    (6, 5, "group", 32),    # warp-MMA kernel
    (16, 3, "group", 64),   # tcgen05 few-token kernel (group 64: not a streaming shape)
    (64, 3, "group", 256),  # tcgen05 prefill kernel
]


@pytest.mark.parametrize("case", MAXK_CASES, ids=lambda c: f"M{c[0]}-N{c[1]}-{c[2]}{c[3]}")
def test_linear_at_max_k(sw, orc, case):
    import torch
    from sparse_ternary_weight_b200 import _abi
    M, N, gname, group = case
    K = _abi.MAX_K
    gran = GRAN[gname]
    W = _weights("t4", N, K, seed=15000 + M + N)
    Xb = synth.activations_bf16(M, K, seed=15500 + M)
    P = sw.quantize_pack(to_dev(W), gran, group)
    ref = orc.quantize_pack(W, gran, group)
    got = packed_to_host(P)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    assert np.array_equal(got[2].view(np.uint32), ref[2].view(np.uint32))
    y_ref = orc.linear(Xb, *ref, N, K, gran, group)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y = sw.linear(X, P, torch.float32)
    assert _abi.lib().sherry_device_status(None) == 0
    check_linear(y.cpu().numpy(), y_ref, Xb, orc.unpack_f32(*ref, N, K, gran, group))


def test_batched_prefill_side_streams_and_graph_capture(sw, orc):
    """A batched call with several prefill problems forks them over the library's
    side streams and joins them into the caller's stream: results equal the single
    calls bit for bit, eagerly and when the call is captured in a CUDA graph."""
    import torch
    shapes = [(384, 512, "group", 128), (130, 1024, "channel", 0), (256, 256, "group", 64),
              (1000, 512, "tensor", 0), (64, 768, "group", 256)]
    M = 300
    pairs = []
    for i, (N, K, gname, group) in enumerate(shapes):
        W = _weights("t4", N, K, seed=52000 + i)
        Xb = synth.activations_bf16(M, K, seed=52500 + i)
        pairs.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), sw.quantize_pack(to_dev(W), GRAN[gname], group)))
    singles = [sw.linear(X, P) for X, P in pairs]
    outs = sw.linear_batched(pairs, torch.float32)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(singles, outs))
    outs_g = [torch.full_like(o, float("nan")) for o in outs]
    sw.linear_batched(pairs, torch.float32, outs=outs_g)  # warm-up outside the capture
    for o in outs_g:
        o.fill_(float("nan"))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sw.linear_batched(pairs, torch.float32, outs=outs_g)
    g.replay()
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(singles, outs_g))
