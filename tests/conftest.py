import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.oracle(omp=False)


@pytest.fixture(scope="session")
def orc_omp():
    import oracle
    return oracle.oracle(omp=True)


@pytest.fixture(autouse=True)
def _device_status_guard(request):
    """After every GPU test: no bounded device wait may have timed out during it,
    and every cached linear workspace has its split-K ticket region back at zero
    (each call that completes must leave it so).  A nonzero status makes the
    binding drop its cached workspaces; dirty tickets are reported and the
    buffer dropped, so one failure does not spread to the next test."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import sys as _sys
    if "sparse_ternary_weight_b200" not in _sys.modules:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import sparse_ternary_weight_b200 as sw
    from sparse_ternary_weight_b200 import _abi
    if _abi._lib is None:
        return
    st = sw.device_status()
    assert st == 0, f"a bounded device wait timed out during {request.node.name} (status {st})"
    ticket_bytes = 256 * 1024
    for key, buf in list(sw._ws_cache.items()):
        if key[1] != "linear":
            continue
        dirty = int(buf[:ticket_bytes].view(torch.int32).ne(0).sum())
        if dirty:
            sw._ws_cache.pop(key, None)
        assert dirty == 0, f"{request.node.name} left {dirty} nonzero ticket words in the {key} workspace"
