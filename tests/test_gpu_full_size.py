"""CUDA path vs the oracle at the full workload sizes, in the launch
configurations that bench.py times (needs a B200).

Workloads: the single small linear (M=1, K=256, N=64, group 128, seed 0); the
LLaMA-3.2-1B-shaped decode stack (16 layers, M=1); the LLaMA-3.2-3B-shaped
decode stack (28 layers, M = 1, 2, 4, 8, 16); the 3B-shaped prefill (M = 512,
2048, 4096 tokens, group-128 and per-channel scales); quantize + pack of the
full 3B weight set (per-tensor, per-channel, group-128).

The oracle cannot recompute every output of these workloads in seconds, so
each linear is checked on sampled weight rows (the first, the last and random
ones; for prefill also sampled token rows): the oracle quantises the same
weight rows itself (group and channel scales depend on one row only), its
packed bytes and scales must equal the library's bit for bit, and its Y for
those rows must satisfy the method's gate max|y - y_ref| / max|y_ref| <= 1e-3
and the fp32 accumulation bound.  Per-tensor scales depend on the whole tensor:
those linears are checked whole on the first and the last layer.  The inputs
are the benchmark's own seeded device-side draws, copied to the host."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import GRAN, check_linear, packed_to_host, to_dev

pytestmark = pytest.mark.gpu

ROWS_PER_LINEAR = 4
TOKENS_PER_PREFILL = 48


@pytest.fixture(scope="module")
def sw():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_ternary_weight_b200.build import build
    build()
    import sparse_ternary_weight_b200 as sw
    return sw


def _sample(n, rng, k):
    """first, last and k - 2 random indices of range(n), sorted, unique"""
    pick = {0, n - 1} | set(rng.integers(0, n, size=max(0, k - 2)).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def _gpu_rows(P, rows):
    """the library's packed rows (idx, sgn, row scales) of a per-group or per-channel weight"""
    import torch
    r = torch.from_numpy(rows).to(P.idx.device)
    idx = P.idx.index_select(0, r).cpu().numpy().view(np.uint32)
    sgn = P.sgn.index_select(0, r).cpu().numpy()
    if P.granularity == oracle.PER_GROUP:
        sc = P.scales.view(P.N, P.K // P.group).index_select(0, r).cpu().numpy().reshape(-1)
    else:
        sc = P.scales.index_select(0, r).cpu().numpy()
    return idx, sgn, sc


def _check_packed_rows(orc, W_rows, P, rows):
    """oracle quantisation of the sampled rows == the library's rows, bit for bit"""
    ref = orc.quantize_pack(W_rows, P.granularity, P.group)
    got = _gpu_rows(P, rows)
    assert np.array_equal(got[0], ref[0]), "idx plane differs"
    assert np.array_equal(got[1], ref[1]), "sgn plane differs"
    assert np.array_equal(got[2].view(np.uint32), ref[2].view(np.uint32)), "scales differ"
    return ref


def _check_y_rows(orc, ref, rows, X_host, Y_rows, K, gran, group, y_is_bf16=False):
    idx, sgn, sc = ref
    y_ref = orc.linear(X_host, idx, sgn, sc, len(rows), K, gran, group)
    Wq = orc.unpack_f32(idx, sgn, sc, len(rows), K, gran, group)
    check_linear(Y_rows, y_ref, X_host, Wq, y_is_bf16=y_is_bf16)


def _bf16_bits(t):
    return t.contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def test_single_linear_seed0(sw, orc):
    """M=1, K=256, N=64, group 128, W ~ N(0, 0.02^2) and X ~ N(0, 1) from seed 0: every output."""
    import torch
    W, Xb = synth.tiny()
    P = sw.quantize_pack(to_dev(W), "per_group", 128)
    ref = orc.quantize_pack(W, oracle.PER_GROUP, 128)
    got = packed_to_host(P)
    assert all(np.array_equal(a.view(np.uint32) if a.dtype == np.float32 else a,
                              b.view(np.uint32) if b.dtype == np.float32 else b) for a, b in zip(got, ref))
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y = sw.linear(X, P, torch.float32).cpu().numpy()
    y_ref = orc.linear(Xb, *ref, 64, 256, oracle.PER_GROUP, 128)
    check_linear(y, y_ref, Xb, orc.unpack_f32(*ref, 64, 256, oracle.PER_GROUP, 128))


def _build_stack(sw, stack, rng, gran="per_group", group=128):
    """quantise every linear of the stack on the device (as the benchmark does) and
    keep, per linear, the sampled rows and the host copy of those weight rows"""
    import torch
    cfg, layers, shp = synth.STACKS[stack]
    out = []
    for l in range(layers):
        for p in synth.PROJ:
            N, K = shp[p]
            W = synth.torch_stack_weight(stack, l, p, device="cuda")
            P = sw.quantize_pack(W, gran, group)
            rows = _sample(N, rng, ROWS_PER_LINEAR)
            W_rows = W.index_select(0, torch.from_numpy(rows).cuda()).cpu().numpy()
            del W
            out.append((l, p, P, rows, W_rows))
    torch.cuda.synchronize()
    return cfg, out


@pytest.mark.parametrize("stack,Ms", [("1b", (1,)), ("3b", (1, 2, 4, 8, 16))], ids=["1b", "3b"])
def test_decode_stack_sampled(sw, orc, stack, Ms):
    """The whole decode stack in one batched call per M (the benchmark's launch)."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    rng = np.random.default_rng(11)
    cfg, lin = _build_stack(sw, stack, rng)
    refs = [_check_packed_rows(orc, W_rows, P, rows) for (_, _, P, rows, W_rows) in lin]
    for M in Ms:
        pairs = [(synth.torch_activations_bf16(M, P.K, synth.act_seed(cfg, l, p), device="cuda"), P)
                 for (l, p, P, _, _) in lin]
        outs = sw.linear_batched(pairs, torch.float32)
        torch.cuda.synchronize()
        assert _abi.lib().sherry_device_status(None) == 0
        for (X, P), Y, (_, _, _, rows, _), ref in zip(pairs, outs, lin, refs):
            Y_rows = Y.index_select(1, torch.from_numpy(rows).cuda()).cpu().numpy()
            _check_y_rows(orc, ref, rows, _bf16_bits(X), Y_rows, P.K, P.granularity, P.group)
        del pairs, outs


@pytest.mark.parametrize("gran", ["per_group", "per_channel"])
def test_prefill_stack_sampled(sw, orc, gran):
    """The 3B stack at M = 512, 2048, 4096 tokens, one call per linear, bf16 Y
    (the benchmark's prefill launches); sampled weight rows x sampled tokens."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    rng = np.random.default_rng(12)
    cfg, lin = _build_stack(sw, "3b", rng, gran, 128)
    refs = [_check_packed_rows(orc, W_rows, P, rows) for (_, _, P, rows, W_rows) in lin]
    for M in (512, 2048, 4096):
        Xk = {K: synth.torch_activations_bf16(M, K, 900000 + K, device="cuda") for K in {P.K for (_, _, P, _, _) in lin}}
        toks = _sample(M, rng, TOKENS_PER_PREFILL)
        tt = torch.from_numpy(toks).cuda()
        Xh = {K: _bf16_bits(X.index_select(0, tt)) for K, X in Xk.items()}
        for (_, _, P, rows, _), ref in zip(lin, refs):
            Y = sw.linear(Xk[P.K], P, torch.bfloat16)
            Y_rows = Y.index_select(0, tt).index_select(1, torch.from_numpy(rows).cuda()).float().cpu().numpy()
            _check_y_rows(orc, ref, rows, Xh[P.K], Y_rows, P.K, P.granularity, P.group, y_is_bf16=True)
        torch.cuda.synchronize()
        assert _abi.lib().sherry_device_status(None) == 0
        del Xk


@pytest.mark.parametrize("gran", ["per_group", "per_channel", "per_tensor"])
def test_quantize_full_3b(sw, orc, gran):
    """Quantise + pack of every linear of the 3B set from fp32: sampled rows bit for
    bit (idx and sgn do not depend on the scale); per-tensor weights whole on the
    first and the last layer (the scale is a mean over the whole tensor).  With
    group scales also the dense bf16 unpack of every linear, sampled rows bit for bit."""
    import torch
    rng = np.random.default_rng(13)
    cfg, layers, shp = synth.STACKS["3b"]
    g = {"per_group": oracle.PER_GROUP, "per_channel": oracle.PER_CHANNEL, "per_tensor": oracle.PER_TENSOR}[gran]
    for l in range(layers):
        for p in synth.PROJ:
            N, K = shp[p]
            W = synth.torch_stack_weight("3b", l, p, device="cuda")
            P = sw.quantize_pack(W, gran, 128)
            if g == oracle.PER_TENSOR and l in (0, layers - 1):
                Wh = W.cpu().numpy()
                ref = orc.quantize_pack(Wh, g, 128)
                got = packed_to_host(P)
                assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]), (l, p)
                assert np.array_equal(got[2].view(np.uint32), ref[2].view(np.uint32)), (l, p)
                del Wh
            else:
                rows = _sample(N, rng, ROWS_PER_LINEAR)
                W_rows = W.index_select(0, torch.from_numpy(rows).cuda()).cpu().numpy()
                if g == oracle.PER_TENSOR:
                    # the row planes do not depend on the (whole-tensor) scale
                    ref = orc.quantize_pack(W_rows, g, 128)
                    r = torch.from_numpy(rows).cuda()
                    assert np.array_equal(P.idx.index_select(0, r).cpu().numpy().view(np.uint32), ref[0]), (l, p)
                    assert np.array_equal(P.sgn.index_select(0, r).cpu().numpy(), ref[1]), (l, p)
                else:
                    ref = _check_packed_rows(orc, W_rows, P, rows)
                    if g == oracle.PER_GROUP:
                        # dense bf16 unpack of the whole linear, sampled rows bit for bit
                        Wd = sw.unpack(P).index_select(0, torch.from_numpy(rows).cuda())
                        got = Wd.view(torch.int16).cpu().numpy().view(np.uint16)
                        assert np.array_equal(got, orc.unpack_bf16(*ref, len(rows), K, g, 128)), (l, p)
            del W, P
    torch.cuda.synchronize()
