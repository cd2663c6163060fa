"""Fake quantisation (the quantiser's forward output for QAT) and batched
quantise + pack on the CUDA path vs the oracle (needs a B200).

"Sherry, Tequila and Fairies in Python", section 1.1: SherryNMQuant.forward
returns sign * mask * scale; its backward passes the gradient through."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, packed_to_host, to_dev

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
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


# every distinct weight shape of the five workloads, plus ragged and edge shapes
FQ_SHAPES = [(64, 256), (2048, 2048), (512, 2048), (8192, 2048), (2048, 8192), (3072, 3072), (1024, 3072),
             (8192, 3072), (3072, 8192), (1, 32), (7, 96), (33, 384)]


@pytest.mark.parametrize("gran", ["group", "channel", "tensor"])
@pytest.mark.parametrize("shape", FQ_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_fake_quant_bit_exact(sw, orc_omp, shape, gran):
    import torch
    N, K = shape
    g = GRAN[gran]
    group = 128 if K % 128 == 0 else 32
    W = synth.weights_student_t(N, K, 20000 + N + K) if K % 3 else synth.weights_normal(N, K, 20000 + N, 0.02, 0.01)
    Wq_ref, Wb_ref = orc_omp.fake_quant(W, g, group)
    idx_r, sgn_r, sc_r = orc_omp.quantize_pack(W, g, group)
    assert np.array_equal(Wq_ref.view(np.uint32), orc_omp.unpack_f32(idx_r, sgn_r, sc_r, N, K, g, group).view(np.uint32))
    Wd = to_dev(W)
    for odt, ref in ((torch.float32, Wq_ref.view(np.uint32)), (torch.bfloat16, Wb_ref)):
        Wq, P = sw.fake_quant(Wd, g, group, out_dtype=odt)
        assert np.array_equal(_bits(Wq), ref), (shape, gran, odt)
        got = packed_to_host(P)
        assert np.array_equal(got[0], idx_r) and np.array_equal(got[1], sgn_r)
        assert np.array_equal(got[2].view(np.uint32), sc_r.view(np.uint32))


@pytest.mark.parametrize("gran", ["group", "channel", "tensor"])
def test_fake_quant_bf16_input(sw, orc, gran):
    import torch
    N, K = 129, 1024
    Wb = synth.f32_to_bf16_bits(synth.weights_student_t(N, K, 21000))
    Wq_ref, Wb_ref = orc.fake_quant(Wb, GRAN[gran], 128)
    Wd = to_dev(Wb.view(np.int16)).view(torch.bfloat16)
    Wq, _ = sw.fake_quant(Wd, GRAN[gran], 128)          # output dtype follows W: bf16
    assert Wq.dtype == torch.bfloat16 and np.array_equal(_bits(Wq), Wb_ref)
    Wq32, _ = sw.fake_quant(Wd, GRAN[gran], 128, out_dtype=torch.float32)
    assert np.array_equal(_bits(Wq32), Wq_ref.view(np.uint32))


def test_fake_quant_ste_gradient(sw):
    """Straight-through estimator: d loss / d W = d loss / d W_q, unchanged."""
    import torch
    W = (torch.randn(300, 1024, device="cuda") * 0.02).requires_grad_(True)
    X = torch.randn(5, 1024, device="cuda")
    Wq = sw.fake_quant_ste(W, "per_group", 128)
    Y = X @ Wq.t()
    G = torch.randn_like(Y)
    Y.backward(G)
    assert torch.equal(W.grad, G.t() @ X)
    assert torch.equal(Wq.detach(), sw.fake_quant(W.detach(), "per_group", 128)[0])


def test_quantize_batched_matches_single_and_oracle(sw, orc):
    import torch
    cases = [(64, 256, "group", 128, "f32"), (300, 3072, "tensor", 0, "f32"), (7, 96, "channel", 0, "bf16"),
             (129, 3072, "group", 128, "bf16"), (33, 384, "tensor", 0, "bf16"), (1, 32, "group", 32, "f32"),
             (0, 64, "tensor", 0, "f32"), (2048, 8192, "channel", 0, "f32")]
    # one binding call per granularity (group 32 for the per-group weights): equal to the
    # single calls and to the oracle
    for gname in ("group", "channel", "tensor"):
        sel = [c for c in cases if c[2] == gname]
        Ws, Wh = [], []
        for i, (N, K, _, _, dt) in enumerate(sel):
            W = synth.weights_student_t(N, K, 22000 + i) if N else np.zeros((0, K), np.float32)
            Wh.append(synth.f32_to_bf16_bits(W) if dt == "bf16" else W)
            Ws.append(to_dev(Wh[-1].view(np.int16)).view(torch.bfloat16) if dt == "bf16" else to_dev(W))
        packs = sw.quantize_pack_batched(Ws, GRAN[gname], 32)
        for P, Wd, W in zip(packs, Ws, Wh):
            ref = orc.quantize_pack(W, GRAN[gname], 32)
            single = packed_to_host(sw.quantize_pack(Wd, GRAN[gname], 32))
            got = packed_to_host(P)
            for a, b, r in zip(got, single, ref):
                assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
                assert np.array_equal(a.reshape(-1)[: r.size].view(np.uint8), r.reshape(-1).view(np.uint8))
    # mixed granularities, dtypes and fake-quant outputs in one launch through the C ABI
    from sparse_ternary_weight_b200 import _abi
    L = _abi.lib()
    D = _abi.QuantizeDesc
    arr = (D * len(cases))()
    keep, outs = [], []
    for i, (N, K, gname, group, dt) in enumerate(cases):
        W = synth.weights_student_t(N, K, 23000 + i) if N else np.zeros((0, K), np.float32)
        Wh = synth.f32_to_bf16_bits(W) if dt == "bf16" else W
        Wd = to_dev(Wh.view(np.int16)).view(torch.bfloat16) if dt == "bf16" else to_dev(W)
        g = GRAN[gname]
        grp = group if gname == "group" else 128
        ns = max(1, orc.num_scales(N, K, g, grp))
        P = sw.PackedWeight(torch.empty((N, K // 32), dtype=torch.int32, device="cuda"),
                            torch.empty((N, K // 32), dtype=torch.uint8, device="cuda"),
                            torch.empty((ns,), dtype=torch.float32, device="cuda"), N, K, g, grp)
        wq = torch.empty((N, K), dtype=torch.float32 if i % 2 else torch.bfloat16, device="cuda") if i % 3 else None
        arr[i] = D(Wd.data_ptr(), P.idx.data_ptr(), P.sgn.data_ptr(), P.scales.data_ptr(),
                   None if wq is None else wq.data_ptr(), N, K, _abi.BF16 if dt == "bf16" else _abi.F32, g, grp,
                   _abi.F32 if i % 2 else _abi.BF16)
        keep.append((Wd, Wh, P, wq, g, grp))
    wsb = L.sherry_quantize_pack_batched_workspace_bytes(arr, len(cases))
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    assert L.sherry_quantize_pack_batched(arr, len(cases), ws.data_ptr(), wsb, None) == 0
    torch.cuda.synchronize()
    for (Wd, Wh, P, wq, g, grp) in keep:
        ref = orc.quantize_pack(Wh, g, grp)
        got = packed_to_host(P)
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
        assert np.array_equal(got[2][: max(1, ref[2].size)].view(np.uint32)[: ref[2].size], ref[2].view(np.uint32))
        if P.N == 0 and g == oracle.PER_TENSOR:
            assert P.scales.cpu().tolist() == [0.0]
        if wq is not None and P.N > 0:
            fq, fb = orc.fake_quant(Wh, g, grp)
            assert np.array_equal(_bits(wq), fq.view(np.uint32) if wq.dtype == torch.float32 else fb)
