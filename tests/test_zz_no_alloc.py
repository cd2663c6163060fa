"""sherry_linear_noalloc: the packed linear for callers that cannot allocate
device memory (frameworks that plan all memory ahead and pass a kernel only its
inputs and outputs, plugin interfaces without a scratch argument).  It keeps its
scratch in a fixed array inside the library; here its output is checked against
the ordinary sherry_linear (which takes a caller workspace) on two calls in a
row, within the linear's parity tolerance.  This file is collected last so that
a failure here stops a -x run only after every other test has run."""
import numpy as np
import pytest

from sparse_ternary_weight_b200 import _abi

pytestmark = pytest.mark.gpu

CASES = [
    # (M, N, K, granularity, group): the streaming kernel (one and two tokens)
    # with tiles split over CTAs, the same over a wide linear, its tensor-core form
    # at 16 tokens on a full grid (the largest scratch plan), the general kernel
    # with split K, and the tensor-core kernel (which needs no scratch)
    (1, 64, 8192, _abi.PER_GROUP, 128),
    (16, 4096, 8192, _abi.PER_GROUP, 128),
    (1, 3072, 3072, _abi.PER_GROUP, 128),
    (2, 3072, 3072, _abi.PER_GROUP, 128),
    (3, 300, 3072, _abi.PER_CHANNEL, 0),
    (16, 64, 2048, _abi.PER_GROUP, 32),
    (40, 200, 1024, _abi.PER_GROUP, 128),
]


def _gate(y, ref):
    d = (y.double() - ref.double()).abs().max().item()
    m = ref.double().abs().max().item()
    return d / m if m > 0 else d


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"M{c[0]}-{c[1]}x{c[2]}-g{c[3]}:{c[4]}")
def test_noalloc_matches_linear_twice(case):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_ternary_weight_b200.build import build
    build()
    import sparse_ternary_weight_b200 as sw
    M, N, K, gran, group = case
    g = torch.Generator(device="cuda")
    g.manual_seed(1234 + N + K)
    W = torch.randn((N, K), generator=g, device="cuda") * 0.02
    X = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    P = sw.quantize_pack(W, gran, group)
    ref = sw.linear(X, P, torch.float32)
    L = _abi.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), device="cuda")
        st = L.sherry_linear_noalloc(X.data_ptr(), M, N, K, P.idx.data_ptr(), P.sgn.data_ptr(),
                                     P.scales.data_ptr(), P.granularity, P.group, Y.data_ptr(), _abi.F32, stream)
        assert st == _abi.OK, L.sherry_status_string(st)
        torch.cuda.synchronize()
        assert _gate(Y, ref) <= 1e-3
        assert torch.equal(Y, ref)   # same kernels and schedule: the same bits


def test_noalloc_rejects_bad_arguments():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = _abi.lib()
    # invalid shapes are reported exactly as by sherry_linear, before any launch
    assert L.sherry_linear_noalloc(0x10000, 1, 8, 48, 0x10000, 0x10000, 0x10000, _abi.PER_GROUP, 32, 0x10000,
                                   _abi.F32, None) == _abi.ERR_SHAPE
