"""N-sharded layer on CPU: the row partition and the all-gather's column order.

Rows of T are independent, so the sharded layer is the unsharded one with
its output columns computed on different ranks: gathering the ranks' column
slices must give exactly the oracle's full Y.  The ranks are real processes
over gloo; each computes its slice with the oracle (this test checks the
partition and the gather, not the kernels)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from ternary_weight_03_b200 import sharded


@pytest.mark.parametrize("N", [1, 7, 8, 9, 100, 1024, 1031])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_row_ranges_partition_n(N, world):
    seen = []
    prev_e = 0
    for r in range(world):
        b, e = sharded.row_range(N, world, r)
        assert b == prev_e and b <= e
        if r < world - 1 and e < N:
            assert (e - b) % 8 == 0
        assert e - b <= sharded.slice_width(N, world)
        seen += list(range(b, e))
        prev_e = e
    assert seen == list(range(N))


def test_bad_arguments():
    with pytest.raises(ValueError):
        sharded.row_range(10, 2, 2)
    with pytest.raises(ValueError):
        sharded.slice_width(0, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, K, M, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import oracle
    import synth
    from ternary_weight_03_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        o = oracle.get()
        T = synth.trits(61, N, K)
        X = synth.activations(62, M, K)
        a = synth.alpha_for(63)
        b, e = sh.row_range(N, world, rank)
        # a rank's packed rows are the packing of its row slice
        for fmt in (2, 16):
            assert np.array_equal(o.pack(fmt, T)[b:e], o.pack(fmt, T[b:e]))
        y_local = torch.from_numpy(o.linear(T[b:e], X, a)) if e > b else torch.zeros((M, 0),
                                                                                       dtype=torch.float64)
        Y = sh.gather_columns(y_local, N)
        q.put((rank, Y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N", [(2, 1000), (2, 9), (3, 100), (3, 17)])
def test_gather_gives_the_full_layer(world, N):
    import oracle
    import synth
    K, M = 300, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, K, M, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = oracle.get().linear(synth.trits(61, N, K), synth.activations(62, M, K), synth.alpha_for(63))
    for r in range(world):
        assert got[r].shape == (M, N)
        assert np.array_equal(got[r], ref), f"rank {r}"


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 8, 64])
def test_sharded_linear_one_rank_gpu(M):
    """On one GPU (a one-rank NCCL group) the sharded layer runs the library's
    kernel on all rows and the gather is the identity: same bits as tl.linear."""
    import torch
    import torch.distributed as dist
    import synth
    import ternary_weight_03_b200 as tl
    from ternary_weight_03_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    N, K = 1000, 3000
    T = synth.trits(71, N, K)
    X = torch.from_numpy(synth.activations(72, M, K)).cuda()
    a = synth.alpha_for(73)
    P = torch.from_numpy(tl.pack(2, T)).cuda()
    ref = tl.linear(2, P, a, X, K).clone()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        layer = sharded.ShardedLinear(2, P, a, N, K)
        Y = layer.forward(X)
        torch.cuda.synchronize()
        assert Y.shape == (M, N)
        assert torch.equal(Y.view(torch.int16), ref.contiguous().view(torch.int16))
    finally:
        dist.destroy_process_group()
