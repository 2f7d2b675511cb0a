"""Column-parallel (N-split) projections over several GPUs, one process per GPU.

Every projection's weight rows are independent output features, so rank r of g owns
a contiguous block of whole 128-row tiles of every weight matrix and computes those
output columns for all canvas rows; the quantized activation is replicated (each rank
quantizes its own copy of the input).  One all-gather of the f32 column blocks gives
every rank the full output.  Where the next projection's input is produced from
column-sharded outputs (SwiGLU of gate and up, in front of down), each rank quantizes
its own K-slice and the int8 codes, scales and scaled sums are gathered instead: the
activation layout is super-block-major, so a slice of whole super-blocks is a
contiguous range of each buffer and the gather is a plain concatenation.

All data movement here is torch.distributed (NCCL on GPUs, gloo on CPU); every GEMM
is a dllm_qgemm call on the rank's own shard.  No operand of any kernel lives on
another GPU.
"""
from __future__ import annotations

import math

TILE_ROWS = 128
SB = 256


def shard_tiles(n_tiles: int, world: int, rank: int) -> tuple[int, int, int]:
    """(first tile, end tile, padded tile count) of rank's block: ceil(n_tiles/world)
    tiles per rank, the last ranks possibly short or empty."""
    if world < 1 or not 0 <= rank < world or n_tiles < 0:
        raise ValueError("bad shard request")
    per = math.ceil(n_tiles / world) if n_tiles else 0
    t0 = min(rank * per, n_tiles)
    t1 = min(t0 + per, n_tiles)
    return t0, t1, per


def shard_rows(N: int, world: int, rank: int) -> tuple[int, int, int]:
    """(first row, end row, padded width) of rank's rows of an N-row weight matrix
    (N a multiple of 128): whole tiles, padded width = the largest shard."""
    if N % TILE_ROWS:
        raise ValueError("N must be a multiple of 128")
    t0, t1, per = shard_tiles(N // TILE_ROWS, world, rank)
    return t0 * TILE_ROWS, t1 * TILE_ROWS, per * TILE_ROWS


def shard_k(K: int, world: int, rank: int) -> tuple[int, int]:
    """Rank's K-slice for a K-sharded activation: equal slices of whole super-blocks."""
    if K % (SB * world):
        raise ValueError("K must split into equal slices of whole 256-element super-blocks")
    ks = K // world
    return rank * ks, (rank + 1) * ks


def gather_columns(local, out, N: int, world: int, group=None, scratch=None):
    """All-gather rank blocks of output columns: `local` is this rank's [M][Wp] block
    (Wp = padded width from shard_rows; columns past the rank's real width are don't
    care), `out` receives the full [M][N].  `scratch`, if given, is a [world*M][Wp]
    buffer of local's dtype (reused across calls)."""
    import torch
    import torch.distributed as dist
    M, Wp = local.shape
    if scratch is None:
        scratch = torch.empty((world * M, Wp), dtype=local.dtype, device=local.device)
    if world == 1:
        scratch.copy_(local)
    else:
        dist.all_gather_into_tensor(scratch, local.contiguous(), group=group)
    full = scratch.view(world, M, Wp).permute(1, 0, 2).reshape(M, world * Wp)
    out.copy_(full[:, :N])
    return out


def gather_act_k(local_bufs, full_bufs, world: int, group=None):
    """All-gather K-slices of a quantized activation: local_bufs = (q, scale, sums) of
    this rank's slice (dllm.alloc_act(M, K/world)), full_bufs = those of the whole K
    (dllm.alloc_act(M, K)); the rank order is the K order."""
    import torch.distributed as dist
    for lb, fb in zip(local_bufs, full_bufs):
        if fb.numel() != world * lb.numel():
            raise ValueError("full buffer is not world x the slice")
        if world == 1:
            fb.copy_(lb)
        else:
            dist.all_gather_into_tensor(fb, lb, group=group)
    return full_bufs


class ColumnParallelQGemm:
    """This rank's rows of one projection: repacked once, then out = x W^T for the
    full N through a local GEMM and gather_columns."""

    def __init__(self, gguf_rows, qtype: int, N: int, K: int, world: int, rank: int, device, group=None):
        """gguf_rows: this rank's GGUF blocks, rows shard_rows(N, world, rank) of the
        matrix, as a flat uint8 device tensor."""
        import torch
        from . import dllm
        self.qtype, self.N, self.K, self.world, self.rank, self.group = qtype, N, K, world, rank, group
        self.n0, self.n1, self.Wp = shard_rows(N, world, rank)
        self.rows = self.n1 - self.n0
        self.w = None
        if self.rows:
            self.w = torch.empty(dllm.dllm_repacked_bytes(qtype, self.rows, K), dtype=torch.uint8, device=device)
            repack = dllm.dllm_repack_q4k if qtype == dllm.DLLM_Q4_K else dllm.dllm_repack_q6k
            repack(gguf_rows, self.rows, K, self.w)

    def workspace_bytes(self, M: int) -> int:
        from . import dllm
        return dllm.dllm_qgemm_workspace_bytes(self.qtype, self.rows, self.K, M) if self.rows else 0

    def local(self, act, M: int, local_out, workspace=None, workspace_bytes: int = 0):
        """This rank's columns into local_out [M][Wp] (the padding columns untouched)."""
        from . import dllm
        if self.rows:
            dllm.dllm_qgemm(self.w, self.qtype, self.rows, self.K, *act, M, None, 0, local_out, self.Wp,
                            workspace, workspace_bytes)
        return local_out

    def __call__(self, act, M: int, out, local_out, scratch=None, workspace=None, workspace_bytes: int = 0):
        self.local(act, M, local_out, workspace, workspace_bytes)
        return gather_columns(local_out, out, self.N, self.world, self.group, scratch)
