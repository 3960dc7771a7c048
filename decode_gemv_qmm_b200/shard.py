"""Column-parallel (output-feature) sharding of the block-quantized matmuls over ranks.

One process per GPU. Rank r of G owns rows [r0, r1) = [r N / G, (r + 1) N / G) of
every weight matrix. Rows of the ggml block layout are contiguous (N rows of K/32
blocks), so a shard is one contiguous byte slice of W and needs no repacking; the
rank computes y[:, r0:r1] with the library's kernels on its own slice, and one
all-gather (NCCL over NVLink / NVSwitch; gloo on CPU in the tests) assembles y.
Every output is computed by exactly one rank. With a local function whose
per-row arithmetic does not depend on N (the oracle) the gathered y equals the
unsharded result bit for bit; with the GPU kernels each slice is within the
library's tolerance (a slice may take another kernel form than the whole
matrix would).

The fused gate/up SwiGLU shards the same way (gate and up rows share the slice,
so silu(g) * u stays local). A row-parallel split of K (the down projection)
would need an all-reduce instead; it is not provided.

These helpers only move bytes and call a local compute function; all arithmetic
is the library's (or, in tests, whatever `local` function is passed in).
"""
from __future__ import annotations

import torch

BLOCK = 32
BLOCK_BYTES = {0: 34, 1: 18}  # QMM_Q8_0, QMM_Q4_0


def row_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """Rows [r0, r1) of an N-row matrix owned by `rank` of `world` (contiguous, sizes differ by <= 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    return rank * N // world, (rank + 1) * N // world


def max_rows(N: int, world: int) -> int:
    """The largest shard of an N-row matrix over `world` ranks."""
    return -(-N // world)


def weight_shard(W, N: int, K: int, rank: int, world: int, wtype: int = 0):
    """The byte slice of the block-quantized matrix W (N rows of K/32 blocks,
    flat bytes or [N, row_bytes]) holding the rows `rank` owns; same type as W
    (a view, not a copy)."""
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    row_bytes = (K // BLOCK) * BLOCK_BYTES[wtype]
    r0, r1 = row_range(N, rank, world)
    flat = W.reshape(-1)
    if flat.shape[0] != N * row_bytes:
        raise ValueError(f"W has {flat.shape[0]} bytes, expected {N * row_bytes}")
    return flat[r0 * row_bytes:r1 * row_bytes]


def gather_rows(y_local: torch.Tensor, N: int, rank: int, world: int, group=None) -> torch.Tensor:
    """All-gather the column slices y_local = y[:, r0:r1] (M x (r1 - r0)) of every
    rank into y (M x N). Shards are padded to the largest one for the collective."""
    import torch.distributed as dist

    M = y_local.shape[0]
    r0, r1 = row_range(N, rank, world)
    if y_local.shape != (M, r1 - r0):
        raise ValueError(f"local slice has shape {tuple(y_local.shape)}, expected {(M, r1 - r0)}")
    if world == 1:
        return y_local
    mr = max_rows(N, world)
    send = torch.zeros((M, mr), dtype=y_local.dtype, device=y_local.device)
    send[:, :r1 - r0] = y_local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send.contiguous(), group=group)
    cols = []
    for r in range(world):
        a, b = row_range(N, r, world)
        cols.append(parts[r][:, :b - a])
    return torch.cat(cols, dim=1)


def sharded_gemv(W_local, X: torch.Tensor, N: int, rank: int, world: int, *, local=None, group=None,
                 flags: int = 0, stream=None) -> torch.Tensor:
    """y = X . dequant(W)^T with W's rows sharded over the ranks: this rank's rows
    by `local(W_local, X, n_local)` (default: the library's qmm_q8_gemv on the
    current CUDA device), then one all-gather of the slices."""
    r0, r1 = row_range(N, rank, world)
    if local is None:
        import decode_gemv_qmm_b200 as qmm

        def local(w, x, n):
            return qmm.qmm_q8_gemv(w, x, n, flags=flags, stream=stream)

    y_local = local(W_local, X, r1 - r0)
    return gather_rows(y_local, N, rank, world, group=group)
