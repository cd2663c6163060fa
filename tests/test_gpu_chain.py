"""Chained linears (dependent phases) and the fused per-layer packed layout on
the CUDA path vs the oracle (needs a B200).

A decoder layer for one or two tokens is four dependent steps: q/k/v, o,
gate/up, down ("Sherry, Tequila and Fairies in Python", section 1.1: every
linear of the model is F.linear with the quantised weight).  Here each step's
input is the previous step's bf16 output read in place: the o projection reads
the first M*K values of the q/k/v output and the down projection the first M*K
values of the gate/up output (stand-ins for attention and the gated activation,
which are not part of this library), and the next layer's q/k/v read the down
output.  The oracle runs the same chain itself from the same first input,
rounding every step's fp64 output to bf16 as the kernel rounds its fp32
accumulator; inputs of later steps therefore differ from the kernel's only
where an output sits within the fp32 accumulation error of a bf16 rounding
boundary, so each step's Y is held to the method's gate (1e-3 of max|y|) plus
the bf16 output allowance (2^-8)."""
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


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _layer_weights(d, f, nkv, seed):
    """q, k, v, o, gate, up, down of one layer: model width d, ffn width f, kv width nkv"""
    W = {}
    for i, (p, (N, K)) in enumerate((("q", (d, d)), ("k", (nkv, d)), ("v", (nkv, d)), ("o", (d, d)),
                                     ("gate", (f, d)), ("up", (f, d)), ("down", (d, f)))):
        W[p] = synth.weights_student_t(N, K, seed + i)
    return W


def _build(sw, layers, d, f, nkv, gran, group, M):
    import torch
    g = GRAN[gran]
    packs = []
    for l in range(layers):
        W = _layer_weights(d, f, nkv, 30000 + 16 * l)
        qkv = sw.quantize_pack_fused([to_dev(W["q"]), to_dev(W["k"]), to_dev(W["v"])], g, group)
        o = sw.quantize_pack(to_dev(W["o"]), g, group)
        gu = sw.quantize_pack_fused([to_dev(W["gate"]), to_dev(W["up"])], g, group)
        dn = sw.quantize_pack(to_dev(W["down"]), g, group)
        packs.append((qkv, o, gu, dn))
    X0 = to_dev(synth.activations_bf16(M, d, 31000).view(np.int16)).view(torch.bfloat16)
    # outputs and the inputs that view them in place
    phases, outs = [], []
    x = X0
    for (qkv, o, gu, dn) in packs:
        y_qkv = torch.empty((M, qkv.N), dtype=torch.bfloat16, device="cuda")
        y_o = torch.empty((M, o.N), dtype=torch.bfloat16, device="cuda")
        y_gu = torch.empty((M, gu.N), dtype=torch.bfloat16, device="cuda")
        y_dn = torch.empty((M, dn.N), dtype=torch.bfloat16, device="cuda")
        phases += [[(x, qkv, y_qkv)], [(y_qkv.view(-1)[: M * d].view(M, d), o, y_o)],
                   [(y_o, gu, y_gu)], [(y_gu.view(-1)[: M * f].view(M, f), dn, y_dn)]]
        x = y_dn
    return packs, X0, phases


def _oracle_chain(orc, packs, X0, M, d, f, gran, group):
    """every step's fp64 output and its bf16 rounding, computed from the first input only"""
    g = GRAN[gran]
    x = _bits(X0)
    refs = []
    for (qkv, o, gu, dn) in packs:
        for P, take in ((qkv, d), (o, None), (gu, f), (dn, None)):
            idx, sgn, sc = packed_to_host(P)
            y = orc.linear(x, idx, sgn, sc, P.N, P.K, g, group)
            yb = synth.f32_to_bf16_bits(y.astype(np.float32))
            refs.append(y)
            x = yb.reshape(-1)[: M * take].reshape(M, take) if take else yb
    return refs


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("gran,group", [("group", 128), ("channel", 128), ("group", 256)])
def test_chain_vs_oracle_chain(sw, orc_omp, M, gran, group):
    import torch
    from sparse_ternary_weight_b200 import _abi
    layers, d, f, nkv = 3, 1024, 2560, 256
    packs, X0, phases = _build(sw, layers, d, f, nkv, gran, group, M)
    sw.linear_chain(phases, torch.bfloat16)
    torch.cuda.synchronize()
    assert sw.device_status() == 0
    refs = _oracle_chain(orc_omp, packs, X0, M, d, f, gran, group)
    for i, (ph, y_ref) in enumerate(zip(phases, refs)):
        y = ph[0][2].float().cpu().numpy()
        assert gate(y, y_ref) <= 1e-3 + 2.0 ** -8, (i, gate(y, y_ref))
    # repeated calls reuse the zeroed counters and give the same bits
    first = [ph[0][2].clone() for ph in phases]
    for _ in range(3):
        sw.linear_chain(phases, torch.bfloat16)
        torch.cuda.synchronize()
        assert sw.device_status() == 0
        assert all(torch.equal(a, ph[0][2]) for a, ph in zip(first, phases))
    ws = sw._ws_cache[(str(X0.device), "linear")]
    assert int(ws[: 256 * 1024].view(torch.int32).abs().sum()) == 0   # tickets and phase counters left zero


@pytest.mark.parametrize("M", [1, 2])
def test_chain_single_phase_matches_oracle_fp32(sw, orc, M):
    """One phase of independent linears through the chained kernel: fp32 Y within the
    gate and the fp32 accumulation bound of every element.  Ragged row counts (N not
    a multiple of the 32-row blocks), K of one to several 2048-weight chunks with a
    partial last chunk, every scale granularity; guard bytes around every Y stay
    untouched."""
    import torch
    from tests.gpu_common import canaried, canaries_intact, check_linear
    shapes = [(1000, 3072, "group", 128), (513, 2048, "channel", 0), (77, 1024, "group", 256), (2048, 512, "tensor", 0),
              (40, 5120, "group", 256)]
    ph, refs, fulls = [], [], []
    for i, (N, K, gname, group) in enumerate(shapes):
        g = GRAN[gname]
        W = synth.weights_normal(N, K, 32000 + i)
        Xb = synth.activations_bf16(M, K, 32500 + i)
        P = sw.quantize_pack(to_dev(W), g, group)
        idx, sgn, sc = packed_to_host(P)
        refs.append((orc.linear(Xb, idx, sgn, sc, N, K, g, group), orc.unpack_f32(idx, sgn, sc, N, K, g, group), Xb))
        full, Y = canaried((M, N), torch.float32)
        fulls.append(full)
        ph.append((to_dev(Xb.view(np.int16)).view(torch.bfloat16), P, Y))
    sw.linear_chain([ph], torch.float32)
    torch.cuda.synchronize()
    assert sw.device_status() == 0
    for (X, P, Y), (y_ref, Wq, Xb), full in zip(ph, refs, fulls):
        check_linear(Y.cpu().numpy(), y_ref, Xb, Wq)
        assert canaries_intact(full)


@pytest.mark.parametrize("M", [1, 2])
def test_chain_many_row_blocks_per_cta(sw, orc, M):
    """Phases with more 32-row blocks than four per CTA (so a CTA walks several
    segments of one linear, rebuilding its tables) and a linear boundary inside CTA
    ranges; the second phase reads the first one's bf16 output.  Every output row
    is compared (fp32 output of the last phase against the oracle's chain)."""
    import torch
    g = oracle.PER_GROUP
    N1, K1 = 24576, 512            # 768 row blocks over the CTAs
    N2a, N2b = 9000, 700           # the second phase: two linears reading Y1 (K = N1)
    W1 = synth.weights_student_t(N1, K1, 35000)
    W2a = synth.weights_student_t(N2a, N1 // 2, 35001)
    W2b = synth.weights_student_t(N2b, N1 // 2, 35002)
    P1 = sw.quantize_pack(to_dev(W1), g, 128)
    P2a = sw.quantize_pack(to_dev(W2a), g, 128)
    P2b = sw.quantize_pack(to_dev(W2b), g, 128)
    Xb = synth.activations_bf16(M, K1, 35003)
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    Y1 = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
    Y2a = torch.empty((M, N2a), dtype=torch.float32, device="cuda")
    Y2b = torch.empty((M, N2b), dtype=torch.float32, device="cuda")
    x2 = Y1.view(-1)[: M * (N1 // 2)].view(M, N1 // 2)
    # one chain call needs one output dtype: bf16 for the first phase, fp32 written by a second call
    sw.linear_chain([[(X, P1, Y1)]], torch.bfloat16)
    sw.linear_chain([[(x2, P2a, Y2a), (x2, P2b, Y2b)]], torch.float32)
    torch.cuda.synchronize()
    assert sw.device_status() == 0
    r1 = orc.linear(Xb, *packed_to_host(P1), N1, K1, g, 128)
    assert gate(Y1.float().cpu().numpy(), r1) <= 1e-3 + 2.0 ** -8
    x2b = _bits(Y1).reshape(-1)[: M * (N1 // 2)].reshape(M, N1 // 2)
    for P, Y, N in ((P2a, Y2a, N2a), (P2b, Y2b, N2b)):
        r = orc.linear(x2b, *packed_to_host(P), N, N1 // 2, g, 128)
        assert gate(Y.cpu().numpy(), r) <= 1e-3


def test_chain_fallback_routes(sw, orc):
    """Phases the chained kernel does not take (K % 256 != 0, five tokens) run as
    ordered batched launches; results still follow the chain."""
    import torch
    for M, K1 in ((1, 96), (5, 512)):
        g = oracle.PER_GROUP
        W1 = synth.weights_student_t(K1 * 2, K1, 33000)
        W2 = synth.weights_student_t(300, K1 * 2, 33001)
        P1 = sw.quantize_pack(to_dev(W1), g, 32)
        P2 = sw.quantize_pack(to_dev(W2), g, 32)
        Xb = synth.activations_bf16(M, K1, 33002)
        X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
        Y1 = torch.empty((M, P1.N), dtype=torch.bfloat16, device="cuda")
        Y2 = torch.empty((M, P2.N), dtype=torch.bfloat16, device="cuda")
        sw.linear_chain([[(X, P1, Y1)], [(Y1, P2, Y2)]], torch.bfloat16)
        torch.cuda.synchronize()
        r1 = orc.linear(Xb, *packed_to_host(P1), P1.N, P1.K, g, 32)
        x2 = synth.f32_to_bf16_bits(r1.astype(np.float32))
        r2 = orc.linear(x2, *packed_to_host(P2), P2.N, P2.K, g, 32)
        assert gate(Y1.float().cpu().numpy(), r1) <= 1e-3 + 2.0 ** -8
        assert gate(Y2.float().cpu().numpy(), r2) <= 1e-3 + 2.0 ** -8


@pytest.mark.parametrize("gran", ["group", "channel"])
def test_fused_layout_is_the_concatenation(sw, gran):
    """q/k/v (and gate/up) packed as one weight: bit-identical to packing each part
    and stacking the planes and scales."""
    import torch
    g = GRAN[gran]
    parts = [synth.weights_student_t(N, 3072, 34000 + N) for N in (3072, 1024, 1024)]
    fused = sw.quantize_pack_fused([to_dev(W) for W in parts], g, 128)
    singles = [packed_to_host(sw.quantize_pack(to_dev(W), g, 128)) for W in parts]
    got = packed_to_host(fused)
    for i in range(3):
        assert np.array_equal(got[i].reshape(-1).view(np.uint8),
                              np.concatenate([s[i].reshape(-1) for s in singles]).view(np.uint8))


@pytest.mark.parametrize("M", [1, 2])
def test_chain_wait_timeout_reports_and_recovers(sw, orc_omp, M):
    """A chained launch whose bounded waits (stage copies, the consumers' barriers,
    the grid barrier between phases) are given a budget of a few clock cycles gives
    up instead of hanging: the status is OK or SHERRY_ERR_TIMEOUT, the context stays
    usable, and once the budget is back the same chain is correct again (the
    binding drops the workspace whose phase counters an aborted launch left)."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    L = _abi.lib()
    layers, d, f, nkv = 2, 1024, 2560, 256
    packs, X0, phases = _build(sw, layers, d, f, nkv, "group", 128, M)
    assert sw.device_status() == 0
    prev = L.sherry_set_wait_budget(2)
    try:
        for _ in range(3):
            sw.linear_chain(phases, torch.bfloat16)
        torch.cuda.synchronize()
        st = sw.device_status()
    finally:
        L.sherry_set_wait_budget(prev)
    assert st in (_abi.OK, _abi.ERR_TIMEOUT)
    sw.linear_chain(phases, torch.bfloat16)
    torch.cuda.synchronize()
    assert sw.device_status() == 0
    refs = _oracle_chain(orc_omp, packs, X0, M, d, f, "group", 128)
    for i, (ph, y_ref) in enumerate(zip(phases, refs)):
        assert gate(ph[0][2].float().cpu().numpy(), y_ref) <= 1e-3 + 2.0 ** -8, i
