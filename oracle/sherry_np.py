"""NumPy restatement of Sherry's quantiser, following the pages' tensor path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Written independently of
``sherry_ref.c`` so that the two cross-check each other bit for bit.

"Sherry, Tequila and Fairies in Python", section 1.1 (the N:M quantiser): the
weight [N,K] is viewed as blocks [N, K/m, m]; the n largest magnitudes of each
block are kept (mask), the masked weight is reshaped by granularity
(per-tensor [1, N*K], per-channel [N, K], per-group [N, K/g, g]); the result is
sign(x) * sum|x| / max(len * n / m, 1) over the last axis.  Here n = 3, m = 4.

Readings that the page's code leaves open (same as the C oracle):
* ``topk`` ties: the zeroed weight is the first of the smallest magnitudes
  (``np.argmin`` returns the first occurrence);
* sign(0) = +1 for every kept weight, -0.0 included;
* the sum over the last axis is the adjacent-pairwise tree in float32 over the
  axis padded with +0.0 to a power of two;
* packing: nibble = 4*z + 2*d1 + d2 and G = sign of the first kept weight,
  8 nibbles per uint32 word and 8 G bits per byte.
"""
from __future__ import annotations

import numpy as np

PER_TENSOR, PER_CHANNEL, PER_GROUP = 0, 1, 2


def tree_sum_lastaxis(x: np.ndarray) -> np.ndarray:
    """Adjacent-pairwise float32 sum over the last axis, zero-padded to 2^k."""
    x = np.asarray(x, np.float32)
    L = x.shape[-1]
    P = 1
    while P < L:
        P *= 2
    if P != L:
        pad = np.zeros(x.shape[:-1] + (P - L,), np.float32)
        x = np.concatenate([x, pad], axis=-1)
    while x.shape[-1] > 1:
        x = (x[..., 0::2] + x[..., 1::2]).astype(np.float32)
    return x[..., 0]


def _by_granularity(a: np.ndarray, gran: int, group: int) -> np.ndarray:
    N, K = a.shape
    if gran == PER_TENSOR:
        return a.reshape(1, N * K)
    if gran == PER_CHANNEL:
        return a.reshape(N, K)
    if gran == PER_GROUP:
        if group <= 0 or K % group:
            raise ValueError("per_group quantization requires a valid group_size")
        return a.reshape(N, K // group, group)
    raise ValueError(f"unsupported granularity {gran}")


def quantize(W: np.ndarray, gran: int = PER_GROUP, group: int = 128):
    """Returns (t int8 [N,K], scales float32 [num_scales], zero_pos int [N,K/4])."""
    W = np.asarray(W, np.float32)
    if W.ndim != 2:
        raise ValueError("expects a 2D weight")
    N, K = W.shape
    if K % 4:
        raise ValueError("K is not divisible by the block size 4")
    blocks = W.reshape(N, K // 4, 4)
    z = np.argmin(np.abs(blocks), axis=-1)                     # zeroed position
    mask = np.ones(blocks.shape, bool)
    np.put_along_axis(mask, z[..., None], False, axis=-1)      # keep the top 3
    sparse = np.where(mask, blocks, np.float32(0)).reshape(N, K)
    sign = np.where(W >= 0, 1, -1).astype(np.int8)             # sign(0) = +1
    t = np.where(mask.reshape(N, K), sign, 0).astype(np.int8)
    mags = _by_granularity(np.abs(sparse).astype(np.float32), gran, group)
    L = mags.shape[-1]
    denom = max(float(L) / 4.0 * 3.0, 1.0)
    scales = (tree_sum_lastaxis(mags) / np.float32(denom)).astype(np.float32)
    return t, scales.reshape(-1), z


def pack(t: np.ndarray):
    """Ternary [N,K] with exactly one zero per block -> (idx u32 [N,K/32], sgn u8 [N,K/32])."""
    N, K = t.shape
    blk = t.reshape(N, K // 4, 4).astype(np.int64)
    z = np.argmax(blk == 0, axis=-1)
    assert np.all((blk == 0).sum(-1) == 1), "3:4 pattern violated"
    order = np.argsort(np.where(blk == 0, 99, np.arange(4)), axis=-1, kind="stable")[..., :3]
    kept = np.take_along_axis(blk, order, axis=-1)               # kept signs in position order
    G = (kept[..., 0] < 0).astype(np.uint32)
    d1 = (kept[..., 1] != kept[..., 0]).astype(np.uint32)
    d2 = (kept[..., 2] != kept[..., 0]).astype(np.uint32)
    nib = (4 * z.astype(np.uint32) + 2 * d1 + d2).reshape(N, K // 32, 8)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    idx = np.bitwise_or.reduce(nib << shifts, axis=-1).astype(np.uint32)
    gb = G.reshape(N, K // 32, 8) << np.arange(8, dtype=np.uint32)
    sgn = np.bitwise_or.reduce(gb, axis=-1).astype(np.uint8)
    return idx, sgn


def unpack_ternary(idx: np.ndarray, sgn: np.ndarray, K: int) -> np.ndarray:
    """(idx, sgn) -> ternary int8 [N,K]."""
    N = idx.shape[0]
    nib = (idx[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF     # [N, K/32, 8]
    G = (sgn[..., None].astype(np.uint32) >> np.arange(8, dtype=np.uint32)) & 1
    nib = nib.reshape(N, K // 4)
    G = G.reshape(N, K // 4)
    z = nib >> 2
    d = [(nib >> 1) & 1, nib & 1]
    first = np.where(G == 1, -1, 1)
    out = np.zeros((N, K // 4, 4), np.int8)
    for zpos in range(4):
        kept = [i for i in range(4) if i != zpos]
        sel = z == zpos
        out[..., kept[0]] = np.where(sel, first, out[..., kept[0]])
        out[..., kept[1]] = np.where(sel, np.where(d[0] == 1, -first, first), out[..., kept[1]])
        out[..., kept[2]] = np.where(sel, np.where(d[1] == 1, -first, first), out[..., kept[2]])
    return out.reshape(N, K)


def quantize_pack(W: np.ndarray, gran: int = PER_GROUP, group: int = 128):
    t, scales, _ = quantize(W, gran, group)
    idx, sgn = pack(t)
    return idx, sgn, scales


def scale_map(N: int, K: int, scales: np.ndarray, gran: int, group: int) -> np.ndarray:
    """Scale of every weight position, float32 [N,K]."""
    if gran == PER_TENSOR:
        return np.full((N, K), scales[0], np.float32)
    if gran == PER_CHANNEL:
        return np.repeat(scales.reshape(N, 1), K, axis=1).astype(np.float32)
    return np.repeat(scales.reshape(N, K // group), group, axis=1).astype(np.float32)


def fake_quant(W: np.ndarray, gran: int = PER_GROUP, group: int = 128) -> np.ndarray:
    """The quantiser's forward output in the pages' order: sign of the masked
    weight (kept weights +-1, the zeroed one 0) times the scale of its domain,
    float32 [N,K] (the zeroed positions are +0.0)."""
    t, scales, _ = quantize(W, gran, group)
    N, K = t.shape
    out = t.astype(np.float32) * scale_map(N, K, scales, gran, group)
    return np.where(t == 0, np.float32(0.0), out).astype(np.float32)
