"""Sherry 3:4-sparse ternary (1.25-bit) weights on B200: quantise+pack, packed
linear and unpack, every step in the CUDA library ``libsherry.so``.

This module only marshals arguments: torch supplies device memory and the
current stream, and each call goes straight to one C-ABI entry point
(include/sherry.h).  There is no CPU or PyTorch fallback: if the library is
missing or the tensors are not on a CUDA device, the calls raise.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

from . import _abi
from ._abi import (BF16, F32, PER_CHANNEL, PER_GROUP, PER_TENSOR, SherryError,  # noqa: F401
                   check, lib)

GRANULARITY = {"per_tensor": PER_TENSOR, "per_channel": PER_CHANNEL, "per_group": PER_GROUP}


def _gran(g) -> int:
    if isinstance(g, str):
        if g not in GRANULARITY:
            raise ValueError(f"unsupported granularity {g!r}")
        return GRANULARITY[g]
    return int(g)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device=None) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (no CPU fallback)")


@dataclass
class PackedWeight:
    """Packed planes of one [N,K] weight: idx uint32 [N,K/32] (stored as int32),
    sgn uint8 [N,K/32], scales float32, plus the scale granularity."""
    idx: "object"
    sgn: "object"
    scales: "object"
    N: int
    K: int
    granularity: int
    group: int

    def nbytes(self) -> int:
        return self.idx.numel() * 4 + self.sgn.numel() + self.scales.numel() * 4


_ws_cache: dict = {}
_ws_timeouts = [0]  # the library's timeout count when the cached buffers were last known clean


def workspace(nbytes: int, device, kind: str = "linear") -> "object":
    """A device scratch buffer of at least ``nbytes``, cached per (device, kind).
    ``kind="linear"`` buffers are zero-filled when allocated and used by the
    linear calls only: their split-K ticket counters must start at zero, and
    every successful call leaves them at zero.  Other kinds hold scratch that
    the next call overwrites.  Once any bounded device wait has been reported
    as given up (sherry_device_status, by whichever caller), every cached
    buffer is dropped: a timed-out kernel may have left tickets nonzero."""
    import torch
    if nbytes <= 0:
        return None
    seen = lib().sherry_timeout_count()
    if seen != _ws_timeouts[0]:
        _ws_cache.clear()
        _ws_timeouts[0] = seen
    key = (str(device), kind)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def device_status(device=None) -> int:
    """Synchronise the current stream of ``device`` and return the library's
    device status (0, or ERR_TIMEOUT when a bounded wait of a kernel gave up
    since the last query).  After a timeout the cached workspaces may hold
    nonzero split-K tickets; the next workspace request drops them (the
    library counts every nonzero status it reports)."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return lib().sherry_device_status(_stream(dev))


def quantize_pack(W, granularity="per_group", group: int = 128, out: PackedWeight | None = None) -> PackedWeight:
    """Greedy Sparse-AbsMean 3:4 quantise + 5-bit pack of W [N,K] (fp32 or bf16)."""
    import torch
    _require_cuda(W)
    if W.dim() != 2:
        raise ValueError("expects a 2D weight")
    W = W.contiguous()
    N, K = W.shape
    g = _gran(granularity)
    L = lib()
    ns = L.sherry_num_scales(N, K, g, group)
    if ns < 0:
        raise SherryError(_abi.ERR_SHAPE if K % 32 or K < 32 else _abi.ERR_GROUP, "quantize_pack")
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(W.dtype)
    if dt is None:
        raise SherryError(_abi.ERR_DTYPE, "quantize_pack")
    if out is None:
        out = _new_packed(N, K, g, group, ns, W.device)
    wsb = L.sherry_workspace_bytes(_abi.OP_QUANTIZE_PACK, 0, N, K, g, group)
    ws = workspace(wsb, W.device, "quantize")
    check(L.sherry_quantize_pack(_ptr(W), dt, N, K, g, group, _ptr(out.idx), _ptr(out.sgn), _ptr(out.scales),
                                 _ptr(ws), wsb, _stream(W.device)), "quantize_pack")
    return out


def _new_packed(N, K, g, group, ns, dev) -> PackedWeight:
    import torch
    return PackedWeight(torch.empty((N, K // 32), dtype=torch.int32, device=dev),
                        torch.empty((N, K // 32), dtype=torch.uint8, device=dev),
                        torch.empty((max(ns, 1),), dtype=torch.float32, device=dev), N, K, g, group)


def fake_quant(W, granularity="per_group", group: int = 128, out_dtype=None, out=None,
               packed: PackedWeight | None = None):
    """The quantiser's forward output W_q = t * alpha [N,K] (fp32 or bf16, default
    W's dtype) in one pass over W, plus the packed weight.  Returns (W_q, packed)."""
    import torch
    _require_cuda(W)
    if W.dim() != 2:
        raise ValueError("expects a 2D weight")
    W = W.contiguous()
    N, K = W.shape
    g = _gran(granularity)
    L = lib()
    ns = L.sherry_num_scales(N, K, g, group)
    if ns < 0:
        raise SherryError(_abi.ERR_SHAPE if K % 32 or K < 32 else _abi.ERR_GROUP, "fake_quant")
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(W.dtype)
    if dt is None:
        raise SherryError(_abi.ERR_DTYPE, "fake_quant")
    out_dtype = out_dtype or W.dtype
    qd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    if out is None:
        out = torch.empty((N, K), dtype=out_dtype, device=W.device)
    if packed is None:
        packed = _new_packed(N, K, g, group, ns, W.device)
    wsb = L.sherry_workspace_bytes(_abi.OP_QUANTIZE_PACK, 0, N, K, g, group)
    ws = workspace(wsb, W.device, "quantize")
    check(L.sherry_fake_quant(_ptr(W), dt, N, K, g, group, _ptr(out), qd, _ptr(packed.idx), _ptr(packed.sgn),
                              _ptr(packed.scales), _ptr(ws), wsb, _stream(W.device)), "fake_quant")
    return out, packed


def _ste_function():
    import torch

    class SherryFakeQuant(torch.autograd.Function):
        """Fake quantisation with the straight-through estimator: the forward is
        :func:`fake_quant` (one kernel), the backward passes the incoming gradient
        to W unchanged ("Sherry, Tequila and Fairies in Python", section 1.1:
        SherryNMQuant.backward returns grad_output) -- no kernel and no copy."""

        @staticmethod
        def forward(ctx, W, granularity, group):
            return fake_quant(W, granularity, group)[0]

        @staticmethod
        def backward(ctx, grad):
            return grad, None, None

    return SherryFakeQuant


_STE = None


def fake_quant_ste(W, granularity="per_group", group: int = 128):
    """Differentiable fake quantisation for QAT: W_q from the CUDA kernel, identity gradient."""
    global _STE
    if _STE is None:
        _STE = _ste_function()
    return _STE.apply(W, granularity, group)


def quantize_pack_batched(weights, granularity="per_group", group: int = 128, outs=None, wq_outs=None):
    """Quantise + pack several weights in one launch (plus one scale-finalise launch
    when any scale is per-tensor).  ``weights`` is a list of 2D fp32/bf16 tensors;
    ``wq_outs`` (optional) a list of fake-quantised outputs (or None entries)."""
    import torch
    if not weights:
        return []
    g = _gran(granularity)
    L = lib()
    dev = weights[0].device
    arr = (_abi.QuantizeDesc * len(weights))()
    packs = []
    for i, W in enumerate(weights):
        _require_cuda(W)
        if W.dim() != 2 or not W.is_contiguous():
            raise ValueError("each weight must be a contiguous 2D tensor")
        N, K = W.shape
        ns = L.sherry_num_scales(N, K, g, group)
        if ns < 0:
            raise SherryError(_abi.ERR_SHAPE if K % 32 or K < 32 else _abi.ERR_GROUP, "quantize_pack_batched")
        P = outs[i] if outs is not None else _new_packed(N, K, g, group, ns, W.device)
        packs.append(P)
        wq = wq_outs[i] if wq_outs is not None else None
        arr[i] = _abi.QuantizeDesc(_ptr(W), _ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), _ptr(wq), N, K,
                                   {torch.float32: F32, torch.bfloat16: BF16}[W.dtype], g, group,
                                   BF16 if (wq is not None and wq.dtype == torch.bfloat16) else F32)
    wsb = L.sherry_quantize_pack_batched_workspace_bytes(arr, len(weights))
    ws = workspace(wsb, dev, "quantize")
    check(L.sherry_quantize_pack_batched(arr, len(weights), _ptr(ws), wsb, _stream(dev)), "quantize_pack_batched")
    return packs


def linear(X, P: PackedWeight, out_dtype=None, out=None):
    """Y [M,N] = X [M,K] (bf16) times the packed weight transposed; fp32 or bf16 Y."""
    import torch
    _require_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2D bf16 tensor")
    X = X.contiguous()
    M, K = X.shape
    if K != P.K:
        raise ValueError("inner dimensions differ")
    out_dtype = out_dtype or torch.float32
    yd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    if out is None:
        out = torch.empty((M, P.N), dtype=out_dtype, device=X.device)
    L = lib()
    wsb = L.sherry_workspace_bytes(_abi.OP_LINEAR, M, P.N, K, P.granularity, P.group)
    ws = workspace(wsb, X.device)
    check(L.sherry_linear(_ptr(X), M, P.N, K, _ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), P.granularity, P.group,
                          _ptr(out), yd, _ptr(ws), wsb, _stream(X.device)), "linear")
    return out


def make_batch(pairs, outs) -> "ctypes.Array":
    """Descriptor array for :func:`linear_batched` from (X, PackedWeight) pairs."""
    arr = (_abi.LinearDesc * len(pairs))()
    for i, ((X, P), Y) in enumerate(zip(pairs, outs)):
        arr[i] = _abi.LinearDesc(_ptr(X), _ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), _ptr(Y), P.N, P.K,
                                 P.granularity, P.group)
    return arr


def linear_batched(pairs, out_dtype=None, outs=None, descs=None):
    """Independent linears with the same M in one call (one launch per kernel used)."""
    import torch
    out_dtype = out_dtype or torch.float32
    yd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    if not pairs:
        return []
    M = pairs[0][0].shape[0]
    for X, P in pairs:
        _require_cuda(X)
        if X.dtype != torch.bfloat16 or X.shape[0] != M or X.shape[1] != P.K or not X.is_contiguous():
            raise ValueError("each X must be contiguous bf16 [M,K] with the same M")
    if outs is None:
        outs = [torch.empty((M, P.N), dtype=out_dtype, device=X.device) for X, P in pairs]
    if descs is None:
        descs = make_batch(pairs, outs)
    L = lib()
    wsb = L.sherry_linear_batched_workspace_bytes(descs, len(pairs), M)
    ws = workspace(wsb, pairs[0][0].device)
    check(L.sherry_linear_batched(descs, len(pairs), M, yd, _ptr(ws), wsb, _stream(pairs[0][0].device)),
          "linear_batched")
    return outs


def quantize_pack_tequila(W, granularity="per_group", group: int = 128, eps: float = 1e-5):
    """Quantise + pack as :func:`quantize_pack` and, in the same pass over W, the
    Tequila-style dead-weight plane D (bf16 [N, K/4]: eps * the zeroed weight of
    each block) and its row sums (fp32 [N]).  Returns (packed, D, bias)."""
    import torch
    _require_cuda(W)
    if W.dim() != 2:
        raise ValueError("expects a 2D weight")
    W = W.contiguous()
    N, K = W.shape
    g = _gran(granularity)
    L = lib()
    ns = L.sherry_num_scales(N, K, g, group)
    if ns < 0:
        raise SherryError(_abi.ERR_SHAPE if K % 32 or K < 32 else _abi.ERR_GROUP, "quantize_pack_tequila")
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(W.dtype)
    if dt is None:
        raise SherryError(_abi.ERR_DTYPE, "quantize_pack_tequila")
    P = _new_packed(N, K, g, group, ns, W.device)
    D = torch.empty((N, K // 4), dtype=torch.bfloat16, device=W.device)
    bias = torch.empty((N,), dtype=torch.float32, device=W.device)
    wsb = L.sherry_workspace_bytes(_abi.OP_QUANTIZE_PACK, 0, N, K, g, group)
    ws = workspace(wsb, W.device, "quantize")
    check(L.sherry_quantize_pack_tequila(_ptr(W), dt, N, K, g, group, float(eps), _ptr(P.idx), _ptr(P.sgn),
                                         _ptr(P.scales), _ptr(D), _ptr(bias), _ptr(ws), wsb, _stream(W.device)),
          "quantize_pack_tequila")
    return P, D, bias


def linear_tequila(X, P: PackedWeight, D, bias, mode="sign", out_dtype=None, out=None):
    """Y = X (T alpha)^T + the dead-weight term: ``mode="ones"`` adds bias[n],
    ``mode="sign"`` adds sign(X) D^T."""
    import torch
    _require_cuda(X)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != P.K:
        raise ValueError("X must be a 2D bf16 tensor [M, K]")
    X = X.contiguous()
    M, K = X.shape
    md = {"ones": _abi.TEQUILA_ONES, "sign": _abi.TEQUILA_SIGN}[mode]
    out_dtype = out_dtype or torch.float32
    yd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    if out is None:
        out = torch.empty((M, P.N), dtype=out_dtype, device=X.device)
    L = lib()
    wsb = L.sherry_linear_tequila_workspace_bytes(M, P.N, K, P.granularity, P.group, yd)
    ws = workspace(wsb, X.device)
    check(L.sherry_linear_tequila(_ptr(X), M, P.N, K, _ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), P.granularity,
                                  P.group, _ptr(D), _ptr(bias), md, _ptr(out), yd, _ptr(ws), wsb, _stream(X.device)),
          "linear_tequila")
    return out


def arenas_lambda(step: int, total: int, lambda0: float) -> float:
    """Cosine-decayed weight of the Arenas residual: lambda0 (1 + cos(pi t / T)) / 2."""
    return float(lib().sherry_arenas_lambda(int(step), int(total), float(lambda0)))


def arenas_linear(X, P: PackedWeight, Wd, lam: float, out_dtype=None, out=None):
    """Arenas training linear Y = X (T alpha)^T + lam X Wd^T in one tensor-core
    kernel (Wd: the latent weight, bf16 [N, K])."""
    import torch
    _require_cuda(X, Wd)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != P.K:
        raise ValueError("X must be a 2D bf16 tensor [M, K]")
    if Wd.dtype != torch.bfloat16 or tuple(Wd.shape) != (P.N, P.K):
        raise ValueError("Wd must be bf16 [N, K]")
    X = X.contiguous()
    Wd = Wd.contiguous()
    M = X.shape[0]
    out_dtype = out_dtype or torch.float32
    yd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    if out is None:
        out = torch.empty((M, P.N), dtype=out_dtype, device=X.device)
    check(lib().sherry_arenas_linear(_ptr(X), M, P.N, P.K, _ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), P.granularity,
                                     P.group, _ptr(Wd), float(lam), _ptr(out), yd, _stream(X.device)), "arenas_linear")
    return out


def linear_chain(phases, out_dtype=None, descs=None):
    """Chained linears: ``phases`` is a list of phases, each a list of (X, P, Y)
    triples (X bf16 [M,K], Y [M,N] preallocated).  Every linear of a phase starts
    after every linear of the previous phase has written its Y, so an X may be
    (a view of) an earlier phase's Y.  Returns the list of Y per phase."""
    import torch
    out_dtype = out_dtype or torch.float32
    yd = {torch.float32: F32, torch.bfloat16: BF16}[out_dtype]
    flat = [t for ph in phases for t in ph]
    if not flat:
        return []
    M = flat[0][0].shape[0]
    for X, P, Y in flat:
        _require_cuda(X, Y)
        if X.dtype != torch.bfloat16 or X.shape != (M, P.K) or not X.is_contiguous():
            raise ValueError("each X must be contiguous bf16 [M,K] with the same M")
        if Y.dtype != out_dtype or Y.shape != (M, P.N) or not Y.is_contiguous():
            raise ValueError("each Y must be contiguous [M,N] of out_dtype")
    if descs is None:
        descs = make_batch([(X, P) for X, P, _ in flat], [Y for _, _, Y in flat])
    begin = [0]
    for ph in phases:
        begin.append(begin[-1] + len(ph))
    pb = (ctypes.c_int * len(begin))(*begin)
    L = lib()
    wsb = L.sherry_linear_chain_workspace_bytes(descs, len(flat), pb, len(phases), M)
    ws = workspace(wsb, flat[0][0].device)
    check(L.sherry_linear_chain(descs, len(flat), pb, len(phases), M, yd, _ptr(ws), wsb, _stream(flat[0][0].device)),
          "linear_chain")
    return [[Y for _, _, Y in ph] for ph in phases]


def quantize_pack_fused(weights, granularity="per_group", group: int = 128) -> PackedWeight:
    """One packed weight whose rows are the rows of ``weights`` in order (e.g. the
    q, k and v projections, or gate and up, of a decoder layer), so that one
    linear call computes all of them.  The planes and the group or row scales of
    each part are exactly those of packing it alone (they depend on its own rows
    only); per-tensor scales are per part and cannot share one packed weight."""
    import torch
    g = _gran(granularity)
    if g == PER_TENSOR:
        raise ValueError("per-tensor scales are one per weight: pack the parts separately")
    K = weights[0].shape[1]
    if any(W.dim() != 2 or W.shape[1] != K for W in weights):
        raise ValueError("every part must be 2D with the same K")
    N = sum(W.shape[0] for W in weights)
    L = lib()
    ns = L.sherry_num_scales(N, K, g, group)
    if ns < 0:
        raise SherryError(_abi.ERR_SHAPE if K % 32 or K < 32 else _abi.ERR_GROUP, "quantize_pack_fused")
    fused = _new_packed(N, K, g, group, ns, weights[0].device)
    spr = ns // N  # scales per row
    r0 = 0
    parts = []
    for W in weights:
        n = W.shape[0]
        parts.append(PackedWeight(fused.idx[r0:r0 + n], fused.sgn[r0:r0 + n], fused.scales[r0 * spr:(r0 + n) * spr],
                                  n, K, g, group))
        r0 += n
    quantize_pack_batched([W.contiguous() for W in weights], g, group, outs=parts)
    return fused


def unpack_batched(packs, outs=None):
    """Dense bf16 of several packed weights in one launch (each as by :func:`unpack`)."""
    import torch
    if not packs:
        return []
    if outs is None:
        outs = [torch.empty((P.N, P.K), dtype=torch.bfloat16, device=P.idx.device) for P in packs]
    arr = (_abi.UnpackDesc * len(packs))()
    for i, (P, o) in enumerate(zip(packs, outs)):
        _require_cuda(P.idx, o)
        arr[i] = _abi.UnpackDesc(_ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), P.N, P.K, P.granularity, P.group,
                                 _ptr(o))
    check(lib().sherry_unpack_batched(arr, len(packs), _stream(packs[0].idx.device)), "unpack_batched")
    return outs


def unpack(P: PackedWeight, out=None):
    """Dense bf16 [N,K] = RNE(t * alpha)."""
    import torch
    if out is None:
        out = torch.empty((P.N, P.K), dtype=torch.bfloat16, device=P.idx.device)
    check(lib().sherry_unpack(_ptr(P.idx), _ptr(P.sgn), _ptr(P.scales), P.N, P.K, P.granularity, P.group,
                              _ptr(out), _stream(P.idx.device)), "unpack")
    return out
