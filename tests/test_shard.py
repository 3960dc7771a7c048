"""Column-parallel sharding of the matmuls over ranks (decode_gemv_qmm_b200.shard), on CPU.

Two gloo ranks each take their row slice of every weight matrix (a plain byte
slice of the block layout), compute it with the oracle and all-gather the
slices; the result must equal the unsharded oracle bit for bit, because every
output is computed by exactly one rank with the same per-row arithmetic. The
fused Q4_0 gate/up shards the same way (gate and up rows share the slice).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synthetic as syn


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_row_ranges_cover_and_balance():
    from decode_gemv_qmm_b200 import shard

    for N in (1, 7, 896, 1153, 151936):
        for world in (1, 2, 3, 8):
            rr = [shard.row_range(N, r, world) for r in range(world)]
            assert rr[0][0] == 0 and rr[-1][1] == N
            assert all(rr[i][1] == rr[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in rr]
            assert max(sizes) - min(sizes) <= 1 and max(sizes) == shard.max_rows(N, world)


def test_weight_shard_is_the_rows_bytes():
    from decode_gemv_qmm_b200 import shard

    g = syn.rng(3)
    n, k = 37, 96
    wb, q, d = syn.q8_0_weights(g, n, k)
    for world in (2, 3):
        parts = [shard.weight_shard(wb, n, k, r, world) for r in range(world)]
        assert np.array_equal(np.concatenate(parts), wb.reshape(-1))
        r0, r1 = shard.row_range(n, world - 1, world)
        assert np.array_equal(parts[-1].reshape(r1 - r0, -1), syn.pack_q8_0(q[r0:r1], d[r0:r1]))
    w4, _, _ = syn.q4_0_weights(g, n, k)
    p = shard.weight_shard(w4, n, k, 1, 2, wtype=syn.Q4_0)
    assert p.size == (n - n // 2) * (k // 32) * 18


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import oracle
    from decode_gemv_qmm_b200 import shard

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for m, n, k in ((1, 1152, 896), (3, 1153, 256), (1, 5, 64)):
            g = syn.rng(100 + n)
            W, _, _ = syn.q8_0_weights(g, n, k)
            x = syn.act_f32(g, m, k)
            Wl = shard.weight_shard(W, n, k, rank, world)

            def local(w, xx, nl):
                return torch.from_numpy(oracle.gemv(syn.Q8_0, np.ascontiguousarray(w), xx.numpy(), nl)[0])

            y = shard.sharded_gemv(Wl, torch.from_numpy(x), n, rank, world, local=local)
            res[(m, n, k)] = y.numpy()
        # fused gate/up: gate and up rows in the same slice, silu(g) * u local
        m, n, k = 2, 301, 128
        g = syn.rng(7)
        Wg, Wu = syn.q4_0_weights(g, n, k)[0], syn.q4_0_weights(g, n, k)[0]
        x = syn.act_f32(g, m, k)
        Wgl = shard.weight_shard(Wg, n, k, rank, world, wtype=syn.Q4_0)
        Wul = shard.weight_shard(Wu, n, k, rank, world, wtype=syn.Q4_0)
        r0, r1 = shard.row_range(n, rank, world)
        yl = oracle.swiglu(syn.Q4_0, np.ascontiguousarray(Wgl), np.ascontiguousarray(Wul), x, r1 - r0)["out"]
        res["gateup"] = shard.gather_rows(torch.from_numpy(yl), n, rank, world).numpy()
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_equals_unsharded_bitwise(world):
    import oracle

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for (m, n, k) in ((1, 1152, 896), (3, 1153, 256), (1, 5, 64)):
        g = syn.rng(100 + n)
        W, _, _ = syn.q8_0_weights(g, n, k)
        x = syn.act_f32(g, m, k)
        ref = oracle.gemv(syn.Q8_0, W, x, n)[0]
        for r in range(world):
            got = out[r][(m, n, k)]
            assert got.shape == ref.shape
            assert np.array_equal(got.view(np.uint64), ref.view(np.uint64)), (r, m, n, k)
    m, n, k = 2, 301, 128
    g = syn.rng(7)
    Wg, Wu = syn.q4_0_weights(g, n, k)[0], syn.q4_0_weights(g, n, k)[0]
    x = syn.act_f32(g, m, k)
    ref = oracle.swiglu(syn.Q4_0, Wg, Wu, x, n)["out"]
    for r in range(world):
        assert np.array_equal(out[r]["gateup"].view(np.uint64), ref.view(np.uint64))
