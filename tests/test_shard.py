"""Tensor-parallel partitions of packed weights: world size 2 over gloo on CPU.

Each rank takes its N-split or K-split of one packed weight (host slicing of
the planes, sparse_ternary_weight_b200.shard), computes its part of Y with the
oracle (fp64, CPU), and the collective (all-gather of N shards, all-reduce of
K partials) must give the unsplit oracle result: exactly for the N-split, within
fp64 rounding for the K-split.  The partition logic is the product's; the
arithmetic here is the oracle's, since these ranks have no GPU."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _packed(orc, N, K, gran, group, seed):
    import torch
    import sparse_ternary_weight_b200 as sw
    from sparse_ternary_weight_b200 import synth
    W = synth.weights_student_t(N, K, seed)
    idx, sgn, sc = orc.quantize_pack(W, gran, group)
    return sw.PackedWeight(torch.from_numpy(idx.view(np.int32)), torch.from_numpy(sgn), torch.from_numpy(sc.copy()),
                           N, K, gran, group)


def _host(P):
    return P.idx.numpy().view(np.uint32), P.sgn.numpy(), P.scales.numpy()


def _rank_main(rank, ws, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from sparse_ternary_weight_b200 import shard, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        orc = oracle.oracle()
        out = []
        for gran, group in ((oracle.PER_GROUP, 128), (oracle.PER_CHANNEL, 128), (oracle.PER_TENSOR, 128)):
            N, K, M = 512, 1024, 3
            P = _packed(orc, N, K, gran, group, 35000 + gran)
            Xb = synth.activations_bf16(M, K, 35500)
            full = orc.linear(Xb, *_host(P), N, K, gran, group)
            # N-split: each rank's rows, gathered along N
            Pr, r0, r1 = shard.shard_rows(P, ws, rank)
            y = torch.from_numpy(orc.linear(Xb, *_host(Pr), Pr.N, K, gran, group))
            yn = shard.gather_rows(y, ws).numpy()
            # K-split: each rank's K range (whole groups), partial sums reduced
            Pk, k0, k1 = shard.shard_k(P, ws, rank)
            yk = torch.from_numpy(orc.linear(np.ascontiguousarray(Xb[:, k0:k1]), *_host(Pk), N, k1 - k0, gran, group))
            shard.reduce_k(yk)
            out.append((gran, bool(np.array_equal(yn, full)),
                        float(np.abs(yk.numpy() - full).max() / np.abs(full).max()), (r0, r1, k0, k1)))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_bounds_cover_the_range():
    from sparse_ternary_weight_b200 import shard
    for n, world, align in ((3072, 2, 1), (5120, 3, 512), (8192, 4, 128), (100, 8, 32)):
        parts = [shard.bounds(n, world, r, align) for r in range(world)]
        assert parts[0][0] == 0 and parts[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
        assert all(lo % align == 0 for lo, _ in parts)


def test_tensor_parallel_gloo_two_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        for gran, n_exact, k_err, b in res[rank]:
            assert n_exact, (rank, gran)
            assert k_err < 1e-12, (rank, gran, k_err)
    # the two ranks' ranges tile N and K
    assert res[0][0][3][1] == res[1][0][3][0] and res[0][0][3][3] == res[1][0][3][2]
