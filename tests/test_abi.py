"""The C-ABI library loads and exports every symbol include/sherry.h declares;
host-side argument checks return their documented status without launching
anything (these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_ternary_weight_b200 import _abi
from sparse_ternary_weight_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(sherry_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def L():
    build()
    return _abi.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sherry_quantize_pack", "sherry_linear", "sherry_unpack", "sherry_linear_batched",
                     "sherry_num_scales", "sherry_workspace_bytes", "sherry_status_string"):
        assert required in names


def test_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.SO_PATH], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if line.strip()}
    missing = declared_functions() - exported
    assert not missing, missing
    for name in declared_functions():
        assert hasattr(L, name)
    # the binding declares exactly the header's functions
    assert set(_abi.SIGNATURES) == declared_functions()


def test_size_queries(L):
    assert L.sherry_idx_bytes(3072, 3072) == 3072 * 3072 // 8
    assert L.sherry_sgn_bytes(3072, 3072) == 3072 * 3072 // 32
    # 1.25 bit / weight for the two planes
    assert (L.sherry_idx_bytes(64, 256) + L.sherry_sgn_bytes(64, 256)) * 8 == 64 * 256 * 1.25
    assert L.sherry_num_scales(64, 256, _abi.PER_GROUP, 128) == 128
    assert L.sherry_num_scales(64, 256, _abi.PER_CHANNEL, 0) == 64
    assert L.sherry_num_scales(64, 256, _abi.PER_TENSOR, 0) == 1
    assert L.sherry_num_scales(64, 256, _abi.PER_GROUP, 96) == -1
    assert L.sherry_num_scales(64, 48, _abi.PER_CHANNEL, 0) == -1
    assert L.sherry_idx_bytes(64, 48) == 0
    assert L.sherry_workspace_bytes(_abi.OP_QUANTIZE_PACK, 0, 64, 256, _abi.PER_GROUP, 128) == 0
    assert L.sherry_workspace_bytes(_abi.OP_QUANTIZE_PACK, 0, 64, 256, _abi.PER_TENSOR, 0) > 0
    assert L.sherry_version() > 0
    for s in range(11):
        assert L.sherry_status_string(s)


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def test_quantize_pack_validation(L):
    q = L.sherry_quantize_pack
    args = lambda **kw: [kw.get("W", FAKE), kw.get("dt", _abi.F32), kw.get("N", 4), kw.get("K", 64),
                         kw.get("g", _abi.PER_GROUP), kw.get("group", 32), kw.get("idx", FAKE),
                         kw.get("sgn", FAKE), kw.get("sc", FAKE), None, 0, None]
    assert q(*args(K=48)) == _abi.ERR_SHAPE
    assert q(*args(K=0)) == _abi.ERR_SHAPE
    assert q(*args(K=_abi.MAX_K + 32)) == _abi.ERR_SHAPE
    assert q(*args(N=-1)) == _abi.ERR_SHAPE
    assert q(*args(group=0)) == _abi.ERR_GROUP
    assert q(*args(group=16)) == _abi.ERR_GROUP
    assert q(*args(group=128)) == _abi.ERR_GROUP
    assert q(*args(g=3)) == _abi.ERR_GRANULARITY
    assert q(*args(dt=9)) == _abi.ERR_DTYPE
    assert q(*args(W=None)) == _abi.ERR_NULL
    assert q(*args(sc=None)) == _abi.ERR_NULL
    assert q(*args(W=FAKE + 4)) == _abi.ERR_ALIGN
    assert q(*args(idx=FAKE + 8)) == _abi.ERR_ALIGN
    # per-tensor needs a workspace
    assert q(*args(g=_abi.PER_TENSOR)) == _abi.ERR_WORKSPACE
    # empty per-group / per-channel tensors are a no-op
    assert q(*args(N=0, W=None, idx=None, sgn=None)) == _abi.OK


def test_linear_validation(L):
    f = L.sherry_linear
    args = lambda **kw: [kw.get("X", FAKE), kw.get("M", 1), kw.get("N", 8), kw.get("K", 64), kw.get("idx", FAKE),
                         kw.get("sgn", FAKE), kw.get("sc", FAKE), kw.get("g", _abi.PER_GROUP),
                         kw.get("group", 32), kw.get("Y", FAKE), kw.get("yd", _abi.F32), None, 0, None]
    assert f(*args(M=-1)) == _abi.ERR_SHAPE
    assert f(*args(K=40)) == _abi.ERR_SHAPE
    assert f(*args(group=48)) == _abi.ERR_GROUP
    assert f(*args(g=9)) == _abi.ERR_GRANULARITY
    assert f(*args(yd=4)) == _abi.ERR_DTYPE
    assert f(*args(X=None)) == _abi.ERR_NULL
    assert f(*args(idx=None)) == _abi.ERR_NULL
    assert f(*args(Y=FAKE + 2)) == _abi.ERR_ALIGN
    assert f(*args(X=FAKE + 8)) == _abi.ERR_ALIGN
    # nothing to do
    assert f(*args(M=0)) == _abi.OK
    assert f(*args(N=0, idx=None, sgn=None, sc=None)) == _abi.OK


def test_batched_validation(L):
    d = (_abi.LinearDesc * 2)()
    for i in range(2):
        d[i] = _abi.LinearDesc(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, _abi.PER_GROUP, 32)
    assert L.sherry_linear_batched(d, 2, -1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE
    assert L.sherry_linear_batched(d, _abi.MAX_BATCH + 1, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE
    d[1].K = 40
    assert L.sherry_linear_batched(d, 2, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE
    d[1].K = 64
    d[1].Y = FAKE + 4
    assert L.sherry_linear_batched(d, 2, 1, _abi.F32, None, 0, None) == _abi.ERR_ALIGN
    assert L.sherry_linear_batched(d, 0, 1, _abi.F32, None, 0, None) == _abi.OK
    assert L.sherry_linear_batched(d, 2, 0, _abi.F32, None, 0, None) == _abi.ERR_ALIGN


def test_unpack_validation(L):
    u = L.sherry_unpack
    assert u(FAKE, FAKE, FAKE, 4, 50, _abi.PER_CHANNEL, 0, FAKE, None) == _abi.ERR_SHAPE
    assert u(None, FAKE, FAKE, 4, 64, _abi.PER_CHANNEL, 0, FAKE, None) == _abi.ERR_NULL
    assert u(FAKE, FAKE, FAKE, 4, 64, _abi.PER_CHANNEL, 0, None, None) == _abi.ERR_NULL
    assert u(FAKE, FAKE, FAKE, 4, 64, _abi.PER_CHANNEL, 0, FAKE + 2, None) == _abi.ERR_ALIGN
    assert u(None, None, None, 0, 64, _abi.PER_CHANNEL, 0, None, None) == _abi.OK


def test_product_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "SO_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _abi.lib()


def test_product_rejects_cpu_tensors():
    import torch
    import sparse_ternary_weight_b200 as sw
    with pytest.raises(ValueError, match="CUDA"):
        sw.quantize_pack(torch.zeros(4, 64))


def test_unpack_batched_validation(L):
    d = (_abi.UnpackDesc * 2)()
    for i in range(2):
        d[i] = _abi.UnpackDesc(FAKE, FAKE, FAKE, 8, 64, _abi.PER_GROUP, 32, FAKE)
    assert L.sherry_unpack_batched(None, 1, None) == _abi.ERR_NULL
    assert L.sherry_unpack_batched(d, -1, None) == _abi.ERR_SHAPE
    assert L.sherry_unpack_batched(d, _abi.MAX_BATCH + 1, None) == _abi.ERR_SHAPE
    assert L.sherry_unpack_batched(d, 0, None) == _abi.OK
    d[1].K = 40
    assert L.sherry_unpack_batched(d, 2, None) == _abi.ERR_SHAPE
    d[1].K = 64
    d[1].group = 48
    assert L.sherry_unpack_batched(d, 2, None) == _abi.ERR_GROUP
    d[1].group = 32
    d[1].W_out = None
    assert L.sherry_unpack_batched(d, 2, None) == _abi.ERR_NULL
    d[1].W_out = FAKE + 8
    assert L.sherry_unpack_batched(d, 2, None) == _abi.ERR_ALIGN


def test_header_constants_match_binding():
    """Every numeric #define of include/sherry.h equals its mirror in the ctypes binding."""
    import os
    import re
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sherry.h")).read()
    defines = {}
    for name, expr in re.findall(r"^#define SHERRY_(\w+)\s+([^/\n]+)", text, flags=re.M):
        expr = expr.strip().replace("(size_t)", "")
        if re.fullmatch(r"[\d\s()<]+", expr):
            defines[name] = eval(expr)  # integers and shifts only
    assert {"OK", "MAX_K", "MAX_BATCH", "NOALLOC_SCRATCH_BYTES", "PER_GROUP", "BF16", "OP_UNPACK"} <= set(defines)
    for name, value in defines.items():
        assert getattr(_abi, name) == value, name


def test_fake_quant_and_batched_quantize_validation(L):
    fq = L.sherry_fake_quant
    args = lambda **kw: [kw.get("W", FAKE), kw.get("dt", _abi.F32), kw.get("N", 4), kw.get("K", 64),
                         kw.get("g", _abi.PER_GROUP), kw.get("group", 32), kw.get("Wq", FAKE),
                         kw.get("qdt", _abi.F32), kw.get("idx", FAKE), kw.get("sgn", FAKE), kw.get("sc", FAKE),
                         kw.get("ws", None), kw.get("wsb", 0), None]
    assert fq(*args(K=48)) == _abi.ERR_SHAPE
    assert fq(*args(g=7)) == _abi.ERR_GRANULARITY
    assert fq(*args(group=48)) == _abi.ERR_GROUP
    assert fq(*args(dt=3)) == _abi.ERR_DTYPE
    assert fq(*args(qdt=3)) == _abi.ERR_DTYPE
    assert fq(*args(Wq=None)) == _abi.ERR_NULL
    assert fq(*args(idx=None)) == _abi.ERR_NULL
    assert fq(*args(Wq=FAKE + 4)) == _abi.ERR_ALIGN
    assert fq(*args(g=_abi.PER_TENSOR, group=0)) == _abi.ERR_WORKSPACE  # per-tensor needs its partial sums
    # batched: every desc is validated before anything runs
    D = _abi.QuantizeDesc
    good = D(FAKE, FAKE, FAKE, FAKE, None, 4, 64, _abi.F32, _abi.PER_GROUP, 32, _abi.F32)
    bad = D(FAKE, FAKE, FAKE, FAKE, None, 4, 48, _abi.F32, _abi.PER_GROUP, 32, _abi.F32)
    arr = (D * 2)(good, bad)
    assert L.sherry_quantize_pack_batched(arr, 2, None, 0, None) == _abi.ERR_SHAPE
    assert L.sherry_quantize_pack_batched(arr, -1, None, 0, None) == _abi.ERR_SHAPE
    assert L.sherry_quantize_pack_batched(None, 1, None, 0, None) == _abi.ERR_NULL
    assert L.sherry_quantize_pack_batched_workspace_bytes(arr, 2) == 0
    t = D(FAKE, FAKE, FAKE, FAKE, None, 4, 3072, _abi.F32, _abi.PER_TENSOR, 0, _abi.F32)
    arr2 = (D * 2)(good, t)
    # per-tensor: one partial sum per 1024-weight subtree of each row, 256-byte aligned
    assert L.sherry_quantize_pack_batched_workspace_bytes(arr2, 2) == 256
    assert L.sherry_quantize_pack_batched(arr2, 2, None, 0, None) == _abi.ERR_WORKSPACE


def test_wait_budget_setter(L):
    prev = L.sherry_set_wait_budget(1000)
    assert L.sherry_set_wait_budget(0) == 1000
    assert L.sherry_set_wait_budget(prev) > 1000  # the default (about 2 s of clock cycles)


def test_linear_chain_validation(L):
    D = _abi.LinearDesc
    good = D(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 256, _abi.PER_GROUP, 128)
    arr = (D * 2)(good, good)
    pb = lambda *v: (ctypes.c_int * len(v))(*v)
    ch = L.sherry_linear_chain
    assert ch(arr, 2, None, 1, 1, _abi.F32, None, 0, None) == _abi.ERR_NULL
    assert ch(arr, 2, pb(0, 1), 1, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE      # last bound != count
    assert ch(arr, 2, pb(1, 2), 1, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE      # first bound != 0
    assert ch(arr, 2, pb(0, 2, 1, 2), 3, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE  # decreasing
    assert ch(arr, 2, pb(0, 1, 2), 0, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE   # no phase
    assert ch(arr, 2, pb(0, 1, 2), 2, 1, 7, None, 0, None) == _abi.ERR_DTYPE
    bad = (D * 2)(good, D(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 48, _abi.PER_GROUP, 128))
    assert ch(bad, 2, pb(0, 1, 2), 2, 1, _abi.F32, None, 0, None) == _abi.ERR_SHAPE
    assert L.sherry_linear_chain_workspace_bytes(bad, 2, pb(0, 1, 2), 2, 1) == 0
    # M = 0: nothing to do
    assert ch(arr, 2, pb(0, 1, 2), 2, 0, _abi.F32, None, 0, None) == _abi.OK


def test_timeout_count_starts_at_zero(L):
    # host-side count of nonzero device statuses; no device work, so it runs without a GPU
    assert L.sherry_timeout_count() == 0


def test_tequila_scratch_stays_out_of_the_ticket_region(L):
    # M = 300 runs a kernel without split-K tickets, so the linear needs no workspace;
    # the bf16 path's fp32 scratch still starts after the 256 KiB ticket region
    M, N, K = 300, 200, 512
    f32 = L.sherry_linear_tequila_workspace_bytes(M, N, K, _abi.PER_GROUP, 64, _abi.F32)
    bf16 = L.sherry_linear_tequila_workspace_bytes(M, N, K, _abi.PER_GROUP, 64, _abi.BF16)
    assert bf16 >= 256 * 1024 + M * N * 4
    assert bf16 - f32 >= M * N * 4
