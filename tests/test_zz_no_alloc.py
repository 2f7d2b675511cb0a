"""dllm_qgemm_noalloc: the GEMM with its scratch in the library's fixed device array
instead of a caller workspace.  Each case calls it twice in a row through the C-ABI
and compares both results with dllm_qgemm on a caller-owned workspace and with the
oracle (in full, or on sampled column ranges for the full-size shapes), within the
parity tolerance |a - b| <= max(1e-5 |b|, 1e-6 T), T the oracle's sum of |terms|.  The file is named to be collected last, so the
cases also run after every other GPU test has used the library in the same process.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth
from tests import gpu_util as gu

Q4, Q6 = dllm.DLLM_Q4_K, dllm.DLLM_Q6_K


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()


def test_scratch_limit_constant_and_status_string():
    assert dllm.DLLM_NOALLOC_SCRATCH_BYTES == 32 << 20
    assert "scratch" in dllm.status_string(dllm.DLLM_ERR_SCRATCH_LIMIT)


@pytest.mark.parametrize("args", [
    dict(N=100), dict(K=300), dict(M=0), dict(ldo=64), dict(n_rows=33, rows=1),
])
def test_bad_arguments_rejected_before_the_device(args):
    """Argument errors come back from the host checks, so they need no GPU."""
    L = dllm.load()
    a = dict(N=128, K=256, M=16, ldo=128, n_rows=0, rows=None)
    a.update(args)
    fake = 1 << 20  # 16-byte aligned, never dereferenced: the checks fail first
    rows = fake if a["rows"] else None
    rc = L.dllm_qgemm_noalloc(fake, Q4, a["N"], a["K"], fake, fake, fake, a["M"], rows, a["n_rows"], fake,
                              a["ldo"], None)
    assert rc == dllm.DLLM_ERR_ARG


def _existing(wd, qtype, N, K, act, rows_t, n_rows, n_out):
    wsb = dllm.dllm_qgemm_workspace_bytes(qtype, N, K, act.M, n_rows)
    ws = dllm.alloc_workspace(wsb)
    out = torch.full((n_out, N), float("nan"), device="cuda")
    dllm.dllm_qgemm(wd, qtype, N, K, act.q, act.scale, act.sums, act.M, rows_t, n_rows, out, N, ws, wsb)
    return out.cpu().numpy()


def _noalloc_twice(wd, qtype, N, K, act, rows_t, n_rows, n_out):
    res = []
    for _ in range(2):
        out = torch.full((n_out, N), float("nan"), device="cuda")
        dllm.dllm_qgemm_noalloc(wd, qtype, N, K, act.q, act.scale, act.sums, act.M, rows_t, n_rows, out, N)
        res.append(out.cpu().numpy())
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    return res


def _close(got, ref, T):
    ok, worst = gu.tol_ok(got, ref.astype(np.float64), T)
    assert ok, f"worst error / bound = {worst}"


# split-K shapes (few tiles, K split over CTAs), a shape with no scratch at all, and
# row lists (gathered into the scratch) with a ragged count and duplicates
CASES = [
    (Q4, 48, 256, 4096, None),
    (Q6, 17, 384, 4096, None),
    (Q4, 40, 16384, 1024, None),
    (Q4, 130, 256, 2048, [5, 0, 129, 5, 77, 64, 3]),
    (Q6, 64, 128, 3072, [63, 1, 2]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("qtype,M,N,K,rows", CASES)
def test_noalloc_matches_workspace_entry(qtype, M, N, K, rows):
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    seed = 90 + M
    w, x = gu.make_case(qtype, M, N, K, seed)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    n_rows = 0 if rows is None else len(rows)
    rows_t = None if rows is None else torch.tensor(np.asarray(rows, np.int32), device="cuda")
    n_out = M if rows is None else n_rows
    ref = _existing(wd, qtype, N, K, act, rows_t, n_rows, n_out)
    oq, os_, _ = act.host()
    o_rows = None if rows is None else np.asarray(rows, np.int32)
    _, ref64, T = oracle.qgemm(qtype, w, N, K, oq, os_, rows=o_rows)
    for got in _noalloc_twice(wd, qtype, N, K, act, rows_t, n_rows, n_out):
        _close(got, ref, T)
        _close(got, ref64, T)


def _sampled_oracle(out, w, qtype, N, K, oq, os_, rows, width, seed):
    """Column ranges (first, last, random) of `out` against the oracle, with its T."""
    rng = np.random.default_rng(seed)
    for n0 in sorted({0, N - width, int(rng.integers(0, N - width))}):
        _, ref64, T = oracle.qgemm(qtype, w, N, K, oq, os_, rows=rows, n0=n0, n1=n0 + width)
        _close(out[:, n0:n0 + width], ref64, T)


@pytest.mark.gpu
def test_noalloc_output_projection_full_vocab():
    """LLaDA-8B output projection (126464 x 4096, Q6_K) on 32 requested rows of a
    128-row canvas: the gathered rows live in the fixed scratch.  Both calls are
    checked against the existing entry point in full and against the oracle on sampled
    column ranges."""
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    qtype, N, K, M = Q6, 126464, 4096, 128
    wg = synth.device_weights(qtype, N, K, 93)
    wd = dllm.repack(qtype, wg, N, K)
    w_host = wg.cpu().numpy().reshape(N, K // 256, 210)
    del wg
    x = synth.device_activations(M, K, 93)
    act = gu.Act(x.cpu().numpy())
    rows = synth.block_rows(M, 32, 93)
    rows_t = torch.tensor(np.asarray(rows, np.int32), device="cuda")
    ref = _existing(wd, qtype, N, K, act, rows_t, 32, 32)
    oq, os_, _ = act.host()
    for got in _noalloc_twice(wd, qtype, N, K, act, rows_t, 32, 32):
        assert np.array_equal(got, ref)  # same plan and arithmetic: the same bits
        _sampled_oracle(got, w_host, qtype, N, K, oq, os_, rows, 128, 93)


@pytest.mark.gpu
def test_noalloc_tail_split_plan():
    """A weight whose 192 tiles leave 44 over after one round on 148 SMs: the tail
    split (44 tiles cut into 148 K-pieces) keeps its arrival counters and K-piece
    partials in the fixed scratch, which the entry point clears before each call."""
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    qtype, M, N, K = Q4, 128, 24576, 4096
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = dllm.dllm_debug_plan(N // 128, K, M, 0, sms)
    if sms == 148:
        assert plan["tail_k"] > 0, plan
    assert plan["bytes"] <= dllm.DLLM_NOALLOC_SCRATCH_BYTES
    w, x = gu.make_case(qtype, M, N, K, 94)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    ref = _existing(wd, qtype, N, K, act, None, 0, M)
    oq, os_, _ = act.host()
    for got in _noalloc_twice(wd, qtype, N, K, act, None, 0, M):
        assert np.array_equal(got, ref)
        _sampled_oracle(got, w, qtype, N, K, oq, os_, None, 64, 94)


@pytest.mark.gpu
def test_noalloc_rejects_calls_beyond_the_scratch():
    """1024 rows of a 4096 x 4096 projection split K four ways over 8 row tiles:
    64 MiB of partial sums, beyond the fixed array.  Nothing is launched."""
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    M, N, K = 1024, 4096, 4096
    assert dllm.dllm_qgemm_workspace_bytes(Q4, N, K, M) > dllm.DLLM_NOALLOC_SCRATCH_BYTES
    wd = torch.zeros(dllm.dllm_repacked_bytes(Q4, N, K), dtype=torch.uint8, device="cuda")
    q, s, u = dllm.alloc_act(M, K)
    out = torch.full((M, N), float("nan"), device="cuda")
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_qgemm_noalloc(wd, Q4, N, K, q, s, u, M, None, 0, out, N)
    assert e.value.code == dllm.DLLM_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.isnan(out).all().item()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
