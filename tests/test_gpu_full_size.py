"""CUDA path vs the oracle at the full workload sizes, in the launch
configurations that bench.py times (needs a B200).

Workloads: the single small linear (M=1, K=256, N=64, group 128, seed 0); the
LLaMA-3.2-1B-shaped decode stack (16 layers, M=1); the LLaMA-3.2-3B-shaped
decode stack (28 layers, M = 1, 2, 4, 8, 16); the 3B-shaped prefill (M = 512,
2048, 4096 tokens, group-128 and per-channel scales); quantize + pack of the
full 3B weight set (per-tensor, per-channel, group-128).

What is compared:
  * quantize + pack: every packed byte and every scale of every linear, for all
    three granularities, bit for bit (the oracle quantises each whole weight);
  * unpack: every dense bf16 weight of every group-128 linear, bit for bit;
  * decode: every output element of every linear of both stacks at every M,
    within the method's gate max|y - y_ref| / max|y_ref| <= 1e-3 and the fp32
    accumulation bound 2^-16 * sum_k |x_k| |w_k| per element;
  * prefill: all N outputs of every linear at sampled token rows (the first,
    the last and random ones), same bounds (bf16 Y: gate + 2^-8).
The oracle (C, fp64 accumulation, OpenMP over rows) takes a few seconds per
pass over the 2.8 B weights; prefill would take minutes per pass over all
tokens, hence the token sample there.  Inputs are the benchmark's own seeded
device-side draws, copied to the host; no oracle input comes from the CUDA path."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from sparse_ternary_weight_b200 import synth
from tests.gpu_common import check_linear, packed_to_host, to_dev

pytestmark = pytest.mark.gpu

TOKENS_PER_PREFILL = 32
DECODE_MS = {"1b": (1,), "3b": (1, 2, 4, 8, 16)}
GRANS = (("per_group", oracle.PER_GROUP, 128), ("per_channel", oracle.PER_CHANNEL, 128),
         ("per_tensor", oracle.PER_TENSOR, 128))


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


def _bf16_bits(t):
    return t.contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def _same(got, ref):
    """bit-for-bit equality of two arrays (floats compared as their bits)"""
    g = np.ascontiguousarray(got).reshape(-1)
    r = np.ascontiguousarray(ref).reshape(-1)
    return g.size == r.size and np.array_equal(g.view(np.uint8), r.view(np.uint8))


def test_single_linear_seed0(sw, orc):
    """M=1, K=256, N=64, group 128, W ~ N(0, 0.02^2) and X ~ N(0, 1) from seed 0: every output."""
    import torch
    W, Xb = synth.tiny()
    P = sw.quantize_pack(to_dev(W), "per_group", 128)
    ref = orc.quantize_pack(W, oracle.PER_GROUP, 128)
    got = packed_to_host(P)
    assert all(_same(a, b) for a, b in zip(got, ref))
    X = to_dev(Xb.view(np.int16)).view(torch.bfloat16)
    y = sw.linear(X, P, torch.float32).cpu().numpy()
    y_ref = orc.linear(Xb, *ref, 64, 256, oracle.PER_GROUP, 128)
    check_linear(y, y_ref, Xb, orc.unpack_f32(*ref, 64, 256, oracle.PER_GROUP, 128))


class Stack:
    """One decode stack quantised on the device as the benchmark does, with the
    oracle's own quantisation of every whole weight beside it.  Built once per
    module: each weight is drawn on the device, copied to the host, quantised by
    both sides in every requested granularity and compared, then dropped."""

    def __init__(self, sw, orc, stack, grans, keep, check_unpack=False):
        import torch
        self.cfg, layers, shp = synth.STACKS[stack]
        self.lin = []          # (layer, proj, N, K)
        self.dev = {g: [] for g in keep}    # granularity name -> device PackedWeight per linear
        self.ref = {g: [] for g in keep}    # granularity name -> oracle (idx, sgn, scales) per linear
        self.mismatch = {g: [] for g, _, _ in grans}
        self.unpack_mismatch = []
        for l in range(layers):
            for p in synth.PROJ:
                N, K = shp[p]
                self.lin.append((l, p, N, K))
                W = synth.torch_stack_weight(stack, l, p, device="cuda")
                Wh = W.cpu().numpy()
                for gname, g, grp in grans:
                    P = sw.quantize_pack(W, gname, grp)
                    ref = orc.quantize_pack(Wh, g, grp)
                    got = packed_to_host(P)
                    for name, a, b in zip(("idx", "sgn", "scales"), got, ref):
                        if not _same(a, b):
                            self.mismatch[gname].append((l, p, name))
                    if gname == "per_group" and check_unpack:
                        Wd = _bf16_bits(sw.unpack(P))
                        if not _same(Wd, orc.unpack_bf16(*ref, N, K, g, grp)):
                            self.unpack_mismatch.append((l, p))
                    if gname in self.dev:
                        self.dev[gname].append(P)
                        self.ref[gname].append(ref)
                    else:
                        del P
                del W, Wh
        torch.cuda.synchronize()


@pytest.fixture(scope="module")
def stack3b(sw, orc_omp):
    return Stack(sw, orc_omp, "3b", GRANS, keep=("per_group", "per_channel"), check_unpack=True)


@pytest.fixture(scope="module")
def stack1b(sw, orc_omp):
    return Stack(sw, orc_omp, "1b", GRANS[:1], keep=("per_group",))


@pytest.mark.parametrize("gran", [g for g, _, _ in GRANS])
def test_quantize_full_3b(stack3b, gran):
    """Quantise + pack of every linear of the 3B set (2.82 B fp32 weights): every
    idx word, sign byte and scale equals the oracle's bit for bit."""
    assert stack3b.mismatch[gran] == [], stack3b.mismatch[gran][:10]


def test_unpack_full_3b(stack3b):
    """Dense bf16 unpack of every group-128 linear of the 3B set, every weight bit for bit."""
    assert stack3b.unpack_mismatch == [], stack3b.unpack_mismatch[:10]


def test_quantize_full_1b(stack1b):
    assert stack1b.mismatch["per_group"] == [], stack1b.mismatch["per_group"][:10]


@pytest.mark.parametrize("which", ["1b", "3b"])
def test_decode_stack_every_output(sw, orc_omp, stack1b, stack3b, which):
    """The whole decode stack in one batched call per M (the benchmark's launch);
    every Y element of every linear against the oracle."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    st = stack1b if which == "1b" else stack3b
    Ms = DECODE_MS[which]
    Xs = {M: [synth.torch_activations_bf16(M, K, synth.act_seed(st.cfg, l, p), device="cuda")
              for (l, p, N, K) in st.lin] for M in Ms}
    Ys = {}
    for M in Ms:
        pairs = list(zip(Xs[M], st.dev["per_group"]))
        outs = sw.linear_batched(pairs, torch.float32)
        torch.cuda.synchronize()
        assert _abi.lib().sherry_device_status(None) == 0
        Ys[M] = [y.cpu().numpy() for y in outs]
        del outs
    for i, (l, p, N, K) in enumerate(st.lin):
        # one oracle pass per linear over the tokens of every M (stacked rows)
        Xh = np.concatenate([_bf16_bits(Xs[M][i]) for M in Ms], axis=0)
        ref = st.ref["per_group"][i]
        y_ref = orc_omp.linear(Xh, *ref, N, K, oracle.PER_GROUP, 128)
        Wq = orc_omp.unpack_f32(*ref, N, K, oracle.PER_GROUP, 128)
        r0 = 0
        for M in Ms:
            check_linear(Ys[M][i], y_ref[r0:r0 + M], Xh[r0:r0 + M], Wq)
            r0 += M
        del Wq


@pytest.mark.parametrize("gran", ["per_group", "per_channel"])
def test_prefill_stack_sampled_tokens(sw, orc_omp, stack3b, gran):
    """The 3B stack at M = 512, 2048, 4096 tokens, one call per linear, bf16 Y
    (the benchmark's prefill launches); all N outputs at sampled token rows."""
    import torch
    from sparse_ternary_weight_b200 import _abi
    rng = np.random.default_rng(12)
    g = oracle.PER_GROUP if gran == "per_group" else oracle.PER_CHANNEL
    for M in (512, 2048, 4096):
        Xk = {K: synth.torch_activations_bf16(M, K, 900000 + K, device="cuda") for (_, _, _, K) in stack3b.lin}
        toks = _sample(M, rng, TOKENS_PER_PREFILL)
        tt = torch.from_numpy(toks).cuda()
        Xh = {K: _bf16_bits(X.index_select(0, tt)) for K, X in Xk.items()}
        for (l, p, N, K), P, ref in zip(stack3b.lin, stack3b.dev[gran], stack3b.ref[gran]):
            Y = sw.linear(Xk[K], P, torch.bfloat16)
            Yt = Y.index_select(0, tt).float().cpu().numpy()
            y_ref = orc_omp.linear(Xh[K], *ref, N, K, g, 128)
            check_linear(Yt, y_ref, Xh[K], orc_omp.unpack_f32(*ref, N, K, g, 128), y_is_bf16=True)
            del Y
        torch.cuda.synchronize()
        assert _abi.lib().sherry_device_status(None) == 0
        del Xk
