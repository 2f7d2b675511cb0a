"""Column-parallel (N-split) host logic on CPU: shard arithmetic, and two gloo ranks that
each compute their own weight rows (with the oracle standing in for the GPU GEMM) and
all-gather the columns, compared with the oracle's unsplit result; the K-sliced
quantized activation gathered the same way equals the quantization of the whole K."""
import datetime
import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch.multiprocessing as mp

from quantized_int8_gemm_q4_b200 import nsplit

ROOT = Path(__file__).resolve().parent.parent


@pytest.mark.parametrize("N", [128, 384, 4096, 12288, 126464])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_rows_cover_whole_tiles_in_rank_order(N, world):
    got = [nsplit.shard_rows(N, world, r) for r in range(world)]
    widths = {wp for _, _, wp in got}
    assert len(widths) == 1
    wp = widths.pop()
    assert got[0][0] == 0 and got[-1][1] == N
    for (a0, a1, _), (b0, b1, _) in zip(got, got[1:]):
        assert a1 == b0                      # contiguous, in rank order, disjoint
    for n0, n1, _ in got:
        assert n0 % 128 == 0 and n1 % 128 == 0 and 0 <= n1 - n0 <= wp
    assert wp == 128 * -(-(N // 128) // world)  # every shard but the last ones is full


def test_shard_rows_and_k_reject_bad_shapes():
    with pytest.raises(ValueError):
        nsplit.shard_rows(100, 2, 0)
    with pytest.raises(ValueError):
        nsplit.shard_rows(256, 2, 2)
    with pytest.raises(ValueError):
        nsplit.shard_k(12288, 5, 0)          # 48 super-blocks do not split 5 ways
    assert [nsplit.shard_k(12288, 8, r) for r in (0, 7)] == [(0, 1536), (10752, 12288)]


def _tile_sb_major(a, Mp, per_sb):
    """[M][K/256 * per_sb] -> super-block-major [K/256][Mp][per_sb] (rows padded with 0)."""
    M = a.shape[0]
    nsb = a.shape[1] // per_sb
    p = np.zeros((Mp, nsb * per_sb), a.dtype)
    p[:M] = a
    return np.ascontiguousarray(p.reshape(Mp, nsb, per_sb).transpose(1, 0, 2))


def _worker(rank, world, port, qout):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch
    import torch.distributed as dist

    import oracle
    from quantized_int8_gemm_q4_b200 import nsplit as ns
    from quantized_int8_gemm_q4_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # columns: N = 3 tiles over 2 ranks (2 + 1 tiles: the second shard is padded)
        for qt, N, K, M in ((synth.Q4_K, 384, 512, 20), (synth.Q6_K, 256, 768, 9)):
            w = synth.weights(qt, N, K, 31, qt)
            x = synth.activations(M, K, 31, qt)
            q, s, _ = oracle.quantize_act(x)
            n0, n1, wp = ns.shard_rows(N, world, rank)
            local = torch.full((M, wp), float("nan"))
            if n1 > n0:
                out, _, _ = oracle.qgemm(qt, w, N, K, q, s, n0=n0, n1=n1, nthreads=1)
                local[:, :n1 - n0] = torch.from_numpy(out)
            full = torch.empty((M, N))
            ns.gather_columns(local, full, N, world)
            ref, _, _ = oracle.qgemm(qt, w, N, K, q, s, nthreads=1)
            res[f"cols{qt}"] = bool(np.array_equal(full.numpy(), ref))
        # K-sliced activation: quantize this rank's slice, gather, compare with the whole
        M, K = 13, 1536
        x = synth.activations(M, K, 32)
        k0, k1 = ns.shard_k(K, world, rank)
        ql, sl, al = oracle.quantize_act(x[:, k0:k1])
        qf, sf, af = oracle.quantize_act(x)
        Mp = 16
        loc = (torch.from_numpy(_tile_sb_major(ql, Mp, 256)).reshape(-1),
               torch.from_numpy(_tile_sb_major(sl, Mp, 1)).reshape(-1),
               torch.from_numpy(_tile_sb_major(al, Mp, 8)).reshape(-1))
        full = tuple(torch.empty(world * t.numel(), dtype=t.dtype) for t in loc)
        ns.gather_act_k(loc, full, world)
        ref = (_tile_sb_major(qf, Mp, 256).reshape(-1), _tile_sb_major(sf, Mp, 1).reshape(-1),
               _tile_sb_major(af, Mp, 8).reshape(-1))
        res["act"] = all(np.array_equal(f.numpy(), r) for f, r in zip(full, ref))
        qout.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_gather_columns_and_k_slices_equal_the_unsplit_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res in got:
        assert res == {"cols12": True, "cols14": True, "act": True}, (rank, res)


def test_single_rank_gather_is_a_copy():
    import torch
    local = torch.arange(12, dtype=torch.float32).view(3, 4)
    out = torch.empty((3, 3))
    nsplit.gather_columns(local, out, 3, 1)
    assert torch.equal(out, local[:, :3])
