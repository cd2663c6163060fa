"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Each ``pin_*`` takes an :class:`oracle.Oracle` and raises ``AssertionError`` on
a mismatch.  ``test_oracle_pins.py`` runs them on the oracle as built;
``test_oracle_mutants.py`` runs them on deliberately broken copies of the C
file to show that a plausible mistake anywhere in the oracle fails a pin.

What pins what (pages: "Sherry: Hardware-Efficient 1.25-Bit Ternary
Quantization via Fine-grained Sparsification" digest = D; "Sherry, Tequila and
Fairies in Python" section 1.1 = P):
* the 32-state code is a bijection (D: C(4,3) * 2^3 = 32 states, 5 bits);
* the zeroed weight is the smallest |w| (D: greedy Sparse-AbsMean) with the
  lowest index on ties -- brute force over 6^4 blocks against a stable sort;
* exactly one zero per block of 4 (P: 3 of every 4 nonzero; 25% sparsity);
* scale = mean |kept| (D), denominator max(L*3/4, 1) (P): exact for powers of
  two, within the pairwise-summation bound of an fp64 mean otherwise;
* hand-worked blocks and a hand-worked row (tests/golden/hand_worked.json);
* the linear y = X Wq^T (D: Y = X T alpha; P: F.linear): one-hot and all-ones
  activations, and NumPy's float64 matmul;
* bf16 unpack = round-to-nearest-even of t*alpha (torch's bf16 cast);
* argument errors (P: non-2D, K not a multiple of the block, bad group size,
  unknown granularity).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from oracle import sherry_np
from sparse_ternary_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f(v):
    return float(v) if not isinstance(v, str) else float(v)


def decode_ternary(idx, sgn, K):
    """Independent decode of the planes (written here, not shared)."""
    N = idx.shape[0]
    t = np.zeros((N, K), np.int8)
    for n in range(N):
        for b in range(K // 4):
            nib = (int(idx[n, b // 8]) >> (4 * (b % 8))) & 15
            g = (int(sgn[n, b // 8]) >> (b % 8)) & 1
            z, d1, d2 = nib >> 2, (nib >> 1) & 1, nib & 1
            kept = [i for i in range(4) if i != z]
            s0 = -1 if g else 1
            t[n, 4 * b + kept[0]] = s0
            t[n, 4 * b + kept[1]] = -s0 if d1 else s0
            t[n, 4 * b + kept[2]] = -s0 if d2 else s0
    return t


def expected_ternary(W):
    """Stable sort by |w|, first element zeroed; signs w >= 0 -> +1."""
    W = np.asarray(W, np.float32)
    N, K = W.shape
    t = np.zeros((N, K), np.int8)
    for n in range(N):
        for b in range(K // 4):
            v = [float(W[n, 4 * b + i]) for i in range(4)]
            order = sorted(range(4), key=lambda i: abs(v[i]))
            for i in range(4):
                t[n, 4 * b + i] = 0 if i == order[0] else (1 if v[i] >= 0 else -1)
    return t


# ---------------------------------------------------------------- code / argmin

def pin_code_bijection(orc: oracle.Oracle):
    facts = _load("pages_facts.json")
    states = []
    W = np.zeros((1, 128), np.float32)
    for z in range(4):
        for d1 in range(2):
            for d2 in range(2):
                for G in range(2):
                    states.append((z, d1, d2, G))
    assert len(states) == facts["states"] == math.comb(4, 3) * 2 ** 3
    for b, (z, d1, d2, G) in enumerate(states):
        kept = [i for i in range(4) if i != z]
        s0 = -1.0 if G else 1.0
        W[0, 4 * b + kept[0]] = s0
        W[0, 4 * b + kept[1]] = -s0 if d1 else s0
        W[0, 4 * b + kept[2]] = -s0 if d2 else s0
        W[0, 4 * b + z] = 0.5 if (b % 3) else -0.25
    idx, sgn, sc = orc.quantize_pack(W, oracle.PER_GROUP, 32)
    codes = set()
    for b, (z, d1, d2, G) in enumerate(states):
        nib = (int(idx[0, b // 8]) >> (4 * (b % 8))) & 15
        g = (int(sgn[0, b // 8]) >> (b % 8)) & 1
        assert nib == 4 * z + 2 * d1 + d2, (b, nib)
        assert g == G, (b, g)
        codes.add((nib, g))
    assert len(codes) == 32
    assert np.all(sc == 1.0), sc
    Wq = orc.unpack_f32(idx, sgn, sc, 1, 128, oracle.PER_GROUP, 32)
    expect = np.where(np.abs(W) == 1.0, W, 0.0)
    assert np.array_equal(Wq, expect)


def pin_argmin_bruteforce(orc: oracle.Oracle):
    vals = [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0]
    blocks = [(a, b, c, d) for a in vals for b in vals for c in vals for d in vals]
    W = np.array(blocks, np.float32).reshape(-1, 32)        # 1296 blocks -> 162 rows
    N, K = W.shape
    idx, sgn, sc = orc.quantize_pack(W, oracle.PER_CHANNEL)
    t_exp = expected_ternary(W)
    t_got = decode_ternary(idx, sgn, K)
    assert np.array_equal(t_got, t_exp)
    ones = np.ones(N, np.float32)
    Wq = orc.unpack_f32(idx, sgn, ones, N, K, oracle.PER_CHANNEL, 0)
    assert np.array_equal(Wq, t_exp.astype(np.float32))


def pin_hand_worked(orc: oracle.Oracle):
    hw = _load("hand_worked.json")
    blocks = hw["blocks"]
    W = np.zeros((1, 4 * 8 * 2), np.float32)      # 10 blocks padded to 16
    for b, e in enumerate(blocks):
        W[0, 4 * b:4 * b + 4] = [_f(v) for v in e["w"]]
    for b in range(len(blocks), 16):
        W[0, 4 * b:4 * b + 4] = [1.0, 2.0, 3.0, 4.0]
    idx, sgn, _ = orc.quantize_pack(W, oracle.PER_CHANNEL)
    for b, e in enumerate(blocks):
        nib = (int(idx[0, b // 8]) >> (4 * (b % 8))) & 15
        g = (int(sgn[0, b // 8]) >> (b % 8)) & 1
        assert (nib, g) == (e["nibble"], e["G"]), (b, nib, g, e)
        assert e["nibble"] == 4 * e["z"] + 2 * e["d1"] + e["d2"]
    t = orc.unpack_f32(idx, sgn, np.ones(1, np.float32), 1, W.shape[1], oracle.PER_CHANNEL, 0)
    for b, e in enumerate(blocks):
        assert list(t[0, 4 * b:4 * b + 4]) == [float(x) for x in e["t"]], (b, t[0, 4 * b:4 * b + 4])
    row = hw["row"]
    Wr = np.array([row["w"]], np.float32)
    for gran, group in ((oracle.PER_CHANNEL, 0), (oracle.PER_GROUP, 32), (oracle.PER_TENSOR, 0)):
        idx, sgn, sc = orc.quantize_pack(Wr, gran, group)
        assert int(idx[0, 0]) == int(row["idx_word"], 16), hex(int(idx[0, 0]))
        assert int(sgn[0, 0]) == int(row["sgn_byte"], 16)
        assert sc.tolist() == [row["alpha"]], sc
        Wq = orc.unpack_f32(idx, sgn, sc, 1, 32, gran, group)
        assert np.array_equal(Wq[0], np.array(row["t"], np.float32) * np.float32(row["alpha"]))
        X = synth.f32_to_bf16_bits(np.ones((1, 32), np.float32))
        Y = orc.linear(X, idx, sgn, sc, 1, 32, gran, group)
        assert Y[0, 0] == row["y_all_ones"], Y


def pin_sparsity(orc: oracle.Oracle):
    facts = _load("pages_facts.json")
    for seed, (N, K) in enumerate([(7, 96), (33, 256), (5, 1024)]):
        W = synth.weights_normal(N, K, seed=100 + seed)
        idx, sgn, _ = orc.quantize_pack(W, oracle.PER_CHANNEL)
        t = decode_ternary(idx, sgn, K).reshape(N, K // 4, 4)
        assert np.all((t == 0).sum(-1) == facts["block"] - facts["nonzero_per_block"])
        assert (t == 0).mean() == facts["sparsity"]
        # the zeroed weight is a smallest |w| of its block
        a = np.abs(W.reshape(N, K // 4, 4))
        zpos = np.argmax(t == 0, axis=-1)
        assert np.all(np.take_along_axis(a, zpos[..., None], -1)[..., 0] == a.min(-1))
        # kept weights keep their sign
        s = np.where(W >= 0, 1, -1).reshape(N, K // 4, 4)
        assert np.all((t == 0) | (t == s))
        # packed size: 1 uint32 + 1 byte per 32 weights = 1.25 bit/weight
        assert (idx.nbytes + sgn.nbytes) * 8 / (N * K) == facts["bits_per_weight"]


# ---------------------------------------------------------------- scales

def pin_scale_power_of_two(orc: oracle.Oracle):
    g = synth.rng(7)
    N, K = 6, 384
    signs = np.where(g.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    # per group of 128: one exponent per group
    e = g.integers(-12, 6, size=(N, K // 128))
    W = signs * np.repeat(np.exp2(e), 128, axis=1).astype(np.float32)
    _, _, sc = orc.quantize_pack(W, oracle.PER_GROUP, 128)
    assert np.array_equal(sc, np.exp2(e).astype(np.float32).reshape(-1))
    # per channel: one exponent per row
    e = g.integers(-12, 6, size=(N, 1))
    W = signs * np.exp2(e).astype(np.float32)
    _, _, sc = orc.quantize_pack(W, oracle.PER_CHANNEL)
    assert np.array_equal(sc, np.exp2(e).astype(np.float32).reshape(-1))
    # per tensor
    W = signs * np.float32(2.0 ** -5)
    _, _, sc = orc.quantize_pack(W, oracle.PER_TENSOR)
    assert sc.tolist() == [2.0 ** -5]


def _fp64_means(W, gran, group):
    """mean of kept |w| per scale domain, in fp64, zero position from a stable sort."""
    t = expected_ternary(W)
    kept = np.where(t != 0, np.abs(W).astype(np.float64), 0.0)
    N, K = W.shape
    if gran == oracle.PER_TENSOR:
        return np.array([kept.sum() / (N * K * 0.75)]), N * K
    if gran == oracle.PER_CHANNEL:
        return kept.sum(1) / (K * 0.75), K
    return kept.reshape(N, K // group, group).sum(-1).reshape(-1) / (group * 0.75), group


def pin_scale_closed_form(orc: oracle.Oracle):
    for seed, (N, K, gran, group) in enumerate([
            (9, 256, oracle.PER_GROUP, 128), (4, 384, oracle.PER_GROUP, 96),
            (5, 96, oracle.PER_CHANNEL, 0), (3, 3072, oracle.PER_CHANNEL, 0),
            (6, 160, oracle.PER_TENSOR, 0), (8, 64, oracle.PER_GROUP, 32)]):
        W = synth.weights_student_t(N, K, seed=200 + seed)
        _, _, sc = orc.quantize_pack(W, gran, group)
        ref, L = _fp64_means(W, gran, group)
        bound = (math.ceil(math.log2(L)) + 1) * 2.0 ** -24
        rel = np.abs(sc.astype(np.float64) - ref) / ref
        assert np.all(rel <= bound), (gran, group, rel.max(), bound)


def pin_c_vs_numpy(orc: oracle.Oracle):
    cases = [(16, 256, oracle.PER_GROUP, 128), (8, 384, oracle.PER_GROUP, 96),
             (4, 512, oracle.PER_GROUP, 256), (12, 64, oracle.PER_GROUP, 32),
             (5, 96, oracle.PER_CHANNEL, 0), (3, 3072, oracle.PER_CHANNEL, 0),
             (7, 224, oracle.PER_TENSOR, 0), (64, 256, oracle.PER_TENSOR, 0)]
    for seed, (N, K, gran, group) in enumerate(cases):
        W = synth.weights_normal(N, K, seed=300 + seed, outlier_frac=0.05)
        if seed % 2:   # ties and signed zeros
            W = np.round(W * 100) / np.float32(100)
            W[0, :8] = [-0.0, 0.0, -0.0, 0.0, 0.01, -0.01, 0.01, -0.0]
        a = orc.quantize_pack(W, gran, group)
        b = sherry_np.quantize_pack(W, gran, group if gran == oracle.PER_GROUP else 128)
        for x, y, name in zip(a, b, ("idx", "sgn", "scales")):
            assert x.dtype == y.dtype and np.array_equal(x.reshape(-1), y.reshape(-1)), (name, N, K, gran, group)


def pin_bf16_input(orc: oracle.Oracle):
    W = synth.weights_normal(16, 256, seed=401)
    Wb = synth.f32_to_bf16_bits(W)
    a = orc.quantize_pack(Wb, oracle.PER_GROUP, 128)
    b = orc.quantize_pack(synth.bf16_bits_to_f32(Wb), oracle.PER_GROUP, 128)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------- unpack / linear

def pin_unpack_bf16(orc: oracle.Oracle):
    import torch
    W = synth.weights_student_t(16, 256, seed=501)
    for gran, group in ((oracle.PER_GROUP, 128), (oracle.PER_CHANNEL, 0), (oracle.PER_TENSOR, 0)):
        idx, sgn, sc = orc.quantize_pack(W, gran, group)
        f = orc.unpack_f32(idx, sgn, sc, 16, 256, gran, group)
        b = orc.unpack_bf16(idx, sgn, sc, 16, 256, gran, group)
        ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(b, ref)
        # Wq = t * alpha
        t = decode_ternary(idx, sgn, 256).astype(np.float32)
        assert np.array_equal(f, t * sherry_np.scale_map(16, 256, sc, gran, group if group else 128))
    # scales that sit exactly half-way between two bf16 values round to even
    W = np.ones((2, 64), np.float32)
    W[0, :] *= np.float32(1 + 2.0 ** -8)      # -> 1.0 (even)
    W[1, :] *= np.float32(1 + 3 * 2.0 ** -8)  # -> 1 + 2^-6 (even)
    W[:, 1::2] *= -1
    idx, sgn, sc = orc.quantize_pack(W, oracle.PER_CHANNEL)
    assert sc.tolist() == [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]
    b = synth.bf16_bits_to_f32(orc.unpack_bf16(idx, sgn, sc, 2, 64, oracle.PER_CHANNEL, 0))
    t = decode_ternary(idx, sgn, 64).astype(np.float32)
    assert np.array_equal(b[0], t[0] * 1.0) and np.array_equal(b[1], t[1] * np.float32(1 + 2.0 ** -6))


def pin_linear(orc: oracle.Oracle):
    N, K = 24, 256
    W = synth.weights_student_t(N, K, seed=601)
    for gran, group in ((oracle.PER_GROUP, 128), (oracle.PER_CHANNEL, 0), (oracle.PER_TENSOR, 0),
                        (oracle.PER_GROUP, 64)):
        idx, sgn, sc = orc.quantize_pack(W, gran, group)
        Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group).astype(np.float64)
        # one-hot rows pick out one column of Wq exactly
        ks = [0, 1, 5, 127, 128, 255]
        X = np.zeros((len(ks), K), np.float32)
        for r, k in enumerate(ks):
            X[r, k] = 1.0
        Y = orc.linear(synth.f32_to_bf16_bits(X), idx, sgn, sc, N, K, gran, group)
        for r, k in enumerate(ks):
            assert np.array_equal(Y[r], Wq[:, k]), (gran, k)
        # all-ones activations give the row sums
        Y1 = orc.linear(synth.f32_to_bf16_bits(np.ones((1, K), np.float32)), idx, sgn, sc, N, K, gran, group)
        sums = np.array([math.fsum(Wq[n]) for n in range(N)])
        assert np.allclose(Y1[0], sums, rtol=1e-13, atol=1e-16)
        # general activations vs NumPy float64 matmul; row selection
        Xb = synth.activations_bf16(5, K, seed=602)
        Y = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
        ref = synth.bf16_bits_to_f32(Xb).astype(np.float64) @ Wq.T
        assert np.allclose(Y, ref, rtol=1e-12, atol=1e-14)
        Ys = orc.linear(Xb, idx, sgn, sc, N, K, gran, group, rows=[4, 0, 2])
        assert np.array_equal(Ys, Y[[4, 0, 2]])


def pin_errors(orc: oracle.Oracle):
    L = orc.L
    W = np.zeros((4, 64), np.float32)
    idx = np.zeros((4, 2), np.uint32)
    sgn = np.zeros((4, 2), np.uint8)
    sc = np.zeros(64, np.float32)   # room for a broken oracle that accepts a bad group
    p = lambda a: a.ctypes.data_as(oracle.ctypes.c_void_p)
    q = L.sherry_ref_quantize_pack
    assert q(p(W), 0, 4, 64, 2, 32, p(idx), p(sgn), p(sc)) == oracle.OK
    assert q(p(W), 0, 4, 48, 2, 16, p(idx), p(sgn), p(sc)) == oracle.ERR_SHAPE      # K % 32
    assert q(p(W), 0, 4, 0, 1, 0, p(idx), p(sgn), p(sc)) == oracle.ERR_SHAPE        # K = 0
    assert q(p(W), 0, -1, 64, 1, 0, p(idx), p(sgn), p(sc)) == oracle.ERR_SHAPE      # N < 0
    assert q(p(W), 0, 4, 64, 2, 0, p(idx), p(sgn), p(sc)) == oracle.ERR_GROUP       # group 0
    assert q(p(W), 0, 4, 64, 2, -32, p(idx), p(sgn), p(sc)) == oracle.ERR_GROUP
    assert q(p(W), 0, 4, 64, 2, 48, p(idx), p(sgn), p(sc)) == oracle.ERR_GROUP      # not x32
    assert q(p(W), 0, 4, 64, 2, 16, p(idx), p(sgn), p(sc)) == oracle.ERR_GROUP      # divides K, not x32
    assert q(p(W), 0, 4, 64, 2, 128, p(idx), p(sgn), p(sc)) == oracle.ERR_GROUP     # K % g
    assert q(p(W), 0, 4, 64, 3, 32, p(idx), p(sgn), p(sc)) == oracle.ERR_GRANULARITY
    assert q(p(W), 0, 4, 64, -1, 32, p(idx), p(sgn), p(sc)) == oracle.ERR_GRANULARITY
    assert q(p(W), 7, 4, 64, 1, 0, p(idx), p(sgn), p(sc)) == oracle.ERR_DTYPE
    assert q(None, 0, 4, 64, 1, 0, p(idx), p(sgn), p(sc)) == oracle.ERR_NULL
    assert q(p(W), 0, 4, 64, 1, 0, p(idx), p(sgn), None) == oracle.ERR_NULL
    # empty tensor: per-tensor scale = 0 / max(0, 1) = 0
    sc[:] = 7.0
    assert q(None, 0, 0, 64, 0, 0, None, None, p(sc)) == oracle.OK
    assert sc[0] == 0.0
    assert orc.num_scales(4, 64, oracle.PER_GROUP, 32) == 8
    assert orc.num_scales(4, 64, oracle.PER_CHANNEL, 0) == 4
    assert orc.num_scales(4, 64, oracle.PER_TENSOR, 0) == 1
    assert orc.num_scales(4, 64, oracle.PER_GROUP, 48) == -1


def pin_pairsum_tree(orc: oracle.Oracle):
    """The tree's order on values where it shows: 1 + 2^-24 + 2^-24 ... ."""
    u = 2.0 ** -24
    # adjacent pairs first: (1 + u) + (u + u) = 1 + 2u... in fp32: 1+u rounds to 1, u+u = 2u, 1 + 2u exact
    v = np.array([1.0, u, u, u], np.float32)
    assert orc.pairsum(v) == np.float32(1.0 + 2 * u)
    # a sequential sum would give 1.0: ((1+u)+u)+u with each step rounding to even 1.0
    # padded to 8: ((1+u) + (u+u)) + ((u+0) + (0+0)) = (1+2u) + u -> tie, even -> 1+4u;
    # a sequential sum stays at 1.0
    v = np.array([1.0, u, u, u, u], np.float32)
    assert orc.pairsum(v) == np.float32(1.0 + 4 * u)
    assert orc.pairsum(np.array([3.0], np.float32)) == 3.0
    assert orc.pairsum(np.zeros(0, np.float32)) == 0.0
    # randomized: pairsum == fp64 sum within the tree bound
    g = synth.rng(11)
    for L in (1, 2, 3, 31, 96, 1000, 4097):
        v = g.random(L, dtype=np.float32)
        ref = math.fsum(v.astype(np.float64))
        assert abs(float(orc.pairsum(v)) - ref) <= (math.ceil(math.log2(max(L, 2)))) * 2.0 ** -24 * ref


def pin_topk_reading(orc: oracle.Oracle):
    """The pages' tensor formulation (top-3 magnitudes kept per block, sign, sum of
    |kept| over the domain divided by the kept count), evaluated with torch on
    continuous inputs where ties and zeros have probability 0: same kept pattern
    and signs, scales within the summation-order bound."""
    import torch
    N, K = 32, 512
    W = synth.weights_student_t(N, K, seed=701)
    w = torch.from_numpy(W)
    blocks = w.reshape(N, K // 4, 4)
    top3 = torch.topk(blocks.abs(), 3, dim=-1).indices
    kept = torch.zeros(blocks.shape, dtype=torch.bool).scatter_(-1, top3, True)
    sparse = torch.where(kept, blocks, torch.zeros(())).reshape(N, K)
    for gran, group, view in ((oracle.PER_GROUP, 128, (N, K // 128, 128)), (oracle.PER_CHANNEL, 0, (N, K)),
                              (oracle.PER_TENSOR, 0, (1, N * K))):
        x = sparse.reshape(view)
        L = x.shape[-1]
        scale = x.abs().sum(-1, keepdim=True) / max(L * 3.0 / 4.0, 1.0)
        deq = (torch.sign(x) * scale).reshape(N, K).numpy()
        idx, sgn, sc = orc.quantize_pack(W, gran, group)
        Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group)
        assert np.array_equal(Wq == 0, deq == 0)
        assert np.array_equal(np.sign(Wq), np.sign(deq))
        bound = (math.ceil(math.log2(L)) + 2) * 2.0 ** -24
        assert np.all(np.abs(Wq - deq) <= bound * np.abs(deq) + 1e-30), gran


# ---------------------------------------------------------------- forward output (fake quantisation)

def pin_fake_quant(orc: oracle.Oracle):
    """The quantiser's forward output W_q ("Sherry, Tequila and Fairies in
    Python" section 1.1: sign of the masked weight times the domain's scale):
    * the pages' torch formulation on continuous inputs: same zero pattern and
      signs, values within the summation-order bound;
    * |w| = 2^e everywhere: W_q = t * 2^e exactly, t from a stable sort by |w|;
    * exactly one +0.0 per block; kept entries carry sign(w) and one magnitude
      per scale domain;
    * the bf16 output is torch's round-to-nearest-even cast of the fp32 one;
    * the C oracle equals the NumPy restatement and the pack -> unpack
      round trip, bit for bit."""
    import torch
    N, K = 24, 384
    W = synth.weights_student_t(N, K, seed=801)
    w = torch.from_numpy(W)
    blocks = w.reshape(N, K // 4, 4)
    top3 = torch.topk(blocks.abs(), 3, dim=-1).indices
    kept = torch.zeros(blocks.shape, dtype=torch.bool).scatter_(-1, top3, True)
    sparse = torch.where(kept, blocks, torch.zeros(())).reshape(N, K)
    t_ref = expected_ternary(W)
    for gran, group, view in ((oracle.PER_GROUP, 128, (N, K // 128, 128)), (oracle.PER_GROUP, 32, (N, K // 32, 32)),
                              (oracle.PER_CHANNEL, 0, (N, K)), (oracle.PER_TENSOR, 0, (1, N * K))):
        Wq, Wb = orc.fake_quant(W, gran, group if group else 128)
        x = sparse.reshape(view)
        L = x.shape[-1]
        deq = (torch.sign(x) * (x.abs().sum(-1, keepdim=True) / max(L * 3.0 / 4.0, 1.0))).reshape(N, K).numpy()
        assert np.array_equal(Wq == 0, deq == 0) and np.array_equal(np.sign(Wq), np.sign(deq))
        bound = (math.ceil(math.log2(L)) + 2) * 2.0 ** -24
        assert np.all(np.abs(Wq - deq) <= bound * np.abs(deq) + 1e-30), (gran, group)
        # one +0.0 per block, kept signs, one magnitude per domain
        assert np.array_equal(Wq.view(np.uint32) == 0, t_ref == 0)
        assert np.array_equal(np.sign(Wq).astype(np.int8), t_ref)
        mags = np.abs(Wq).reshape(view)
        dom_max = mags.max(axis=-1, keepdims=True)
        assert np.all((mags == 0) | (mags == dom_max)), (gran, group)
        ref_b = torch.from_numpy(Wq).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(Wb, ref_b)
        g = group if group else 128
        assert np.array_equal(Wq.view(np.uint32), sherry_np.fake_quant(W, gran, g).view(np.uint32))
        idx, sgn, sc = orc.quantize_pack(W, gran, g)
        assert np.array_equal(Wq.view(np.uint32), orc.unpack_f32(idx, sgn, sc, N, K, gran, g).view(np.uint32))
    # powers of two: exact, with ties resolved to the lowest index
    rng = synth.rng(802)
    e = rng.integers(-10, 4, size=(N, K // 128))
    signs = np.where(rng.random((N, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    W2 = (signs * np.repeat(np.exp2(e), 128, axis=1)).astype(np.float32)
    Wq, _ = orc.fake_quant(W2, oracle.PER_GROUP, 128)
    assert np.array_equal(Wq, expected_ternary(W2).astype(np.float32) * np.repeat(np.exp2(e), 128, axis=1))


# ---------------------------------------------------------------- Tequila-style dead-weight term

def pin_tequila(orc: oracle.Oracle):
    """The dead-weight term ("Sherry, Tequila and Fairies in Python", sections 1.2,
    2.1: B = eps * w where the quantiser zeroes w, then F.linear(ones, B) or
    F.linear(sign(x), B)), with Sherry's zeroed weight (smallest |w| per block):
    * D = torch's bf16 cast of eps * w at the zero position found by a stable
      sort (ties to the lowest index);
    * bias = F.linear(ones, B) and the sign term = F.linear(sign(X), B), both in
      float64 torch, within the summation-order bound;
    * one-hot activations pick single D entries; an activation of 0 at the zeroed
      position contributes nothing (torch.sign(0) = 0);
    * exact sums for equal powers of two."""
    import torch
    N, K, M = 16, 256, 3
    eps = np.float32(1e-2)
    W = synth.weights_student_t(N, K, seed=901)
    D, bias = orc.tequila_dead(W, eps)
    t = expected_ternary(W)
    dead = np.where(t == 0, W * eps, np.float32(0)).astype(np.float32)            # B before the cast
    Bb = torch.from_numpy(dead).to(torch.bfloat16)
    d_ref = Bb.float().numpy().reshape(N, K // 4, 4).sum(-1)                      # one nonzero per block
    assert np.array_equal(D, torch.from_numpy(d_ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    ones = torch.ones((1, K), dtype=torch.float64)
    b_ref = torch.nn.functional.linear(ones, Bb.double()).numpy()[0]
    L = K // 4
    assert np.all(np.abs(bias - b_ref) <= (math.ceil(math.log2(L)) + 1) * 2.0 ** -24 * Bb.double().abs().sum(1).numpy())
    idx, sgn, sc = orc.quantize_pack(W, oracle.PER_GROUP, 128)
    Xb = synth.activations_bf16(M, K, seed=902)
    Xb[0, ::5] = 0                                                                 # some exact zeros
    X = torch.from_numpy(synth.bf16_bits_to_f32(Xb)).double()
    T1 = orc.tequila_term(Xb, idx, D, bias, N, K, 1)
    ref1 = torch.nn.functional.linear(torch.sign(X), Bb.double()).numpy()
    assert np.all(np.abs(T1 - ref1) <= 1e-12 * (Bb.double().abs().sum(1).numpy() + 1e-30))
    T0 = orc.tequila_term(Xb, idx, D, bias, N, K, 0)
    assert np.array_equal(T0, np.broadcast_to(bias.astype(np.float64), (M, N)))
    # one-hot activations: k at the zeroed position of row n picks D[n][k/4]
    for k in (0, 5, 130, 255):
        Xo = np.zeros((1, K), np.uint16)
        Xo[0, k] = synth.f32_to_bf16_bits(np.array([-3.0], np.float32))[0]
        To = orc.tequila_term(Xo, idx, D, bias, N, K, 1)[0]
        want = np.where(t[:, k] == 0, -synth.bf16_bits_to_f32(D[:, k // 4]).astype(np.float64), 0.0)
        assert np.array_equal(To, want), k
    # a zero activation at every zeroed position: no term at all
    Xz = np.tile(synth.f32_to_bf16_bits(np.ones((1, K), np.float32)), (N, 1))
    Xz[t == 0] = 0
    for n in range(N):
        assert orc.tequila_term(Xz[n:n + 1], idx, D, bias, N, K, 1)[0, n] == 0.0
    # equal powers of two: D exact and the sums exact
    W2 = np.where(synth.rng(903).random((4, 128)) < 0.5, -1.0, 1.0).astype(np.float32) * np.float32(2.0 ** -3)
    D2, b2 = orc.tequila_dead(W2, np.float32(2.0 ** -7))
    t2 = expected_ternary(W2)
    z_sign = np.where(np.sign(W2)[t2 == 0] >= 0, 1.0, -1.0).reshape(4, 32)
    assert np.array_equal(synth.bf16_bits_to_f32(D2), (z_sign * 2.0 ** -10).astype(np.float32))
    assert np.array_equal(b2, (z_sign.sum(1) * 2.0 ** -10).astype(np.float32))


# ---------------------------------------------------------------- Arenas

def pin_arenas(orc: oracle.Oracle):
    """Arenas ("Sherry: ..." digest: Y = X T alpha + lambda_t X W, lambda_t
    cosine-decayed to 0):
    * lambda = 0 gives the plain linear exactly;
    * one-hot activations give column k of T alpha + lambda W;
    * a latent weight equal to the dequantised weight gives (1 + lambda) times
      the plain linear (within fp64 rounding);
    * float64 torch of X (T alpha + lambda W)^T within fp64 rounding;
    * the schedule: lambda0 at step 0, 0 at the last step, lambda0/2 half-way,
      (2 + sqrt 2)/4 lambda0 at a quarter, non-increasing."""
    import torch
    N, K, M = 24, 256, 3
    W = synth.weights_student_t(N, K, seed=1001)
    Wd = synth.f32_to_bf16_bits(W)
    for gran, group in ((oracle.PER_GROUP, 128), (oracle.PER_CHANNEL, 128), (oracle.PER_TENSOR, 128)):
        idx, sgn, sc = orc.quantize_pack(W, gran, group)
        Xb = synth.activations_bf16(M, K, seed=1002)
        plain = orc.linear(Xb, idx, sgn, sc, N, K, gran, group)
        assert np.array_equal(orc.arenas_linear(Xb, idx, sgn, sc, Wd, 0.0, N, K, gran, group), plain)
        lam = np.float32(0.3)
        Wq = orc.unpack_f32(idx, sgn, sc, N, K, gran, group).astype(np.float64)
        Wl = synth.bf16_bits_to_f32(Wd).astype(np.float64)
        ref = torch.from_numpy(synth.bf16_bits_to_f32(Xb)).double() @ torch.from_numpy(Wq + float(lam) * Wl).t()
        y = orc.arenas_linear(Xb, idx, sgn, sc, Wd, lam, N, K, gran, group)
        assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)
        for k in (0, 77, 255):
            Xo = np.zeros((1, K), np.uint16)
            Xo[0, k] = synth.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
            yo = orc.arenas_linear(Xo, idx, sgn, sc, Wd, lam, N, K, gran, group)[0]
            assert np.array_equal(yo, Wq[:, k] + float(lam) * Wl[:, k]), k
        # latent weight = the dequantised weight (exact in bf16 for a power-of-two scale)
    Wp = (np.where(synth.rng(1003).random((N, K)) < 0.5, -1.0, 1.0) * 2.0 ** -5).astype(np.float32)
    idx, sgn, sc = orc.quantize_pack(Wp, oracle.PER_GROUP, 128)
    Wq = orc.unpack_f32(idx, sgn, sc, N, K, oracle.PER_GROUP, 128)
    Xb = synth.activations_bf16(M, K, seed=1004)
    plain = orc.linear(Xb, idx, sgn, sc, N, K, oracle.PER_GROUP, 128)
    y = orc.arenas_linear(Xb, idx, sgn, sc, synth.f32_to_bf16_bits(Wq), 0.5, N, K, oracle.PER_GROUP, 128)
    assert np.allclose(y, 1.5 * plain, rtol=1e-13, atol=1e-13)
    # the schedule
    lam0 = 0.8
    assert orc.arenas_lambda(0, 1000, lam0) == lam0
    assert orc.arenas_lambda(1000, 1000, lam0) == 0.0 or abs(orc.arenas_lambda(1000, 1000, lam0)) < 1e-16
    assert abs(orc.arenas_lambda(500, 1000, lam0) - lam0 / 2) < 1e-15
    assert abs(orc.arenas_lambda(250, 1000, lam0) - lam0 * (2 + math.sqrt(2)) / 4) < 1e-15
    assert orc.arenas_lambda(2000, 1000, lam0) == orc.arenas_lambda(1000, 1000, lam0)
    seq = [orc.arenas_lambda(s, 1000, lam0) for s in range(0, 1001, 50)]
    assert all(a >= b for a, b in zip(seq, seq[1:]))


ALL_PINS = [pin_arenas, pin_tequila, pin_fake_quant, pin_topk_reading, pin_code_bijection, pin_argmin_bruteforce, pin_hand_worked, pin_sparsity,
            pin_scale_power_of_two, pin_scale_closed_form, pin_c_vs_numpy, pin_bf16_input,
            pin_unpack_bf16, pin_linear, pin_errors, pin_pairsum_tree]
