"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare (packed bytes/scales bit for bit, Y within bounds)."""
from __future__ import annotations

import numpy as np

import oracle
from sparse_ternary_weight_b200 import synth

GRAN = {"tensor": oracle.PER_TENSOR, "channel": oracle.PER_CHANNEL, "group": oracle.PER_GROUP}


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def packed_to_host(P):
    idx = P.idx.cpu().numpy().view(np.uint32)
    sgn = P.sgn.cpu().numpy()
    sc = P.scales.cpu().numpy()[: max(1, P.scales.numel())]
    return idx, sgn, sc


def gate(y, y_ref):
    """max|y - y_ref| / max|y_ref| (the method's parity metric)."""
    d = np.abs(np.asarray(y, np.float64) - y_ref).max()
    m = np.abs(y_ref).max()
    return d / m if m > 0 else d


def elementwise_bound(Xf, Wq):
    """fp32 accumulation bound per output: 2^-16 * sum_k |x_k| |w_k|."""
    return 2.0 ** -16 * (np.abs(Xf).astype(np.float64) @ np.abs(Wq).astype(np.float64).T) + 1e-30


def check_linear(y, y_ref, Xb, Wq, y_is_bf16=False):
    g = gate(y, y_ref)
    if y_is_bf16:
        assert g <= 1e-3 + 2.0 ** -8, g
        return g
    assert g <= 1e-3, g
    bound = elementwise_bound(synth.bf16_bits_to_f32(Xb), Wq)
    err = np.abs(np.asarray(y, np.float64) - y_ref)
    assert np.all(err <= bound), (err / bound).max()
    return g


CANARY_BYTE = 0xA5
CANARY_PAD = 256   # guard bytes before and after an output (keeps the view 256-byte aligned)


def canaried(shape, dtype):
    """A device output buffer guarded by CANARY_PAD bytes of a fixed pattern on
    each side: returns (whole allocation, the output view of `shape`)."""
    import torch
    n = int(np.prod(shape)) if len(shape) else 1
    item = torch.empty((), dtype=dtype).element_size()
    pad = CANARY_PAD // item
    full = torch.empty(n + 2 * pad, dtype=dtype, device="cuda")
    full.view(torch.uint8).fill_(CANARY_BYTE)
    return full, full[pad:pad + n].view(*shape)


def canaries_intact(full) -> bool:
    """True if no byte of either guard region of a `canaried` buffer changed."""
    b = full.view(__import__("torch").uint8)
    return bool((b[:CANARY_PAD] == CANARY_BYTE).all()) and bool((b[-CANARY_PAD:] == CANARY_BYTE).all())
