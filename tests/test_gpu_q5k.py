"""Q5_K through the C-ABI: the repack into the split form, byte for byte, and the GEMM
against the oracle's Q5_K GEMM (which decodes the 176-byte blocks directly), within
|gpu - oracle| <= max(1e-5 |oracle|, 1e-6 T)."""
import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth
from tests import gpu_util as gu
from tests.q5k_split import split_q5k

pytestmark = pytest.mark.gpu

Q4, Q5 = dllm.DLLM_Q4_K, dllm.DLLM_Q5_K


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()
    yield
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


@pytest.mark.parametrize("N,K", [(128, 256), (256, 1024), (384, 4096)])
def test_repack_q5k_is_the_split_in_the_q4k_tile_layout(N, K):
    w = synth.q5k_weights(N, K, 70, N, K)
    dev = dllm.repack(Q5, w, N, K)
    assert dev.numel() == dllm.dllm_repacked_bytes(Q5, N, K)
    assert np.array_equal(dev.cpu().numpy(), gu.repack_reference(Q4, split_q5k(w)))


@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (17, 256, 512), (64, 384, 1024), (160, 256, 4096),
                                   (130, 128, 12288)])
def test_qgemm_q5k_matches_oracle(M, N, K):
    w = synth.q5k_weights(N, K, 71, M, N, K)
    x = synth.activations(M, K, 71, M, N, K)
    wd = dllm.repack(Q5, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q5, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q5, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst


def test_qgemm_q5k_requested_rows_and_noalloc():
    M, N, K = 160, 256, 2048
    w = synth.q5k_weights(N, K, 72)
    x = synth.activations(M, K, 72)
    wd = dllm.repack(Q5, w, N, K)
    act = gu.Act(x)
    rows = synth.block_rows(M, 32, 72)
    got = gu.gemm(wd, Q5, N, K, act, rows=rows).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q5, w, N, K, oq, os_, rows=rows)
    assert gu.tol_ok(got, ref, T)[0]
    out = torch.full((M, N), float("nan"), device="cuda")
    dllm.dllm_qgemm_noalloc(wd, Q5, N, K, act.q, act.scale, act.sums, M, None, 0, out, N)
    _, ref_full, T_full = oracle.qgemm(Q5, w, N, K, oq, os_)
    assert gu.tol_ok(out.cpu().numpy(), ref_full, T_full)[0]


def test_qkv_q5k_three_segments():
    M, Nq, Nkv, K = 40, 256, 128, 1024
    x = synth.activations(M, K, 73)
    wts = [synth.q5k_weights(n, K, 73, i) for i, n in enumerate((Nq, Nkv, Nkv))]
    wd = [dllm.repack(Q5, wt, wt.shape[0], K) for wt in wts]
    act = gu.Act(x)
    oq_, os_, _ = oracle.quantize_act(x)
    outs = [torch.empty((M, n), device="cuda") for n in (Nq, Nkv, Nkv)]
    wsb = dllm.dllm_qgemm_workspace_bytes(Q5, Nq + 2 * Nkv, K, M)
    work = dllm.alloc_workspace(max(wsb, 256))
    dllm.dllm_qkv_qgemm(wd[0], wd[1], wd[2], Q5, Nq, Nkv, K, act.q, act.scale, act.sums, M, outs[0], Nq,
                        outs[1], outs[2], Nkv, work, wsb)
    for o, wt in zip(outs, wts):
        _, ref, T = oracle.qgemm(Q5, wt, wt.shape[0], K, oq_, os_)
        assert gu.tol_ok(o.cpu().numpy(), ref, T)[0]


def test_q5k_debug_integer_view_is_rejected():
    M, N, K = 16, 128, 256
    w = synth.q5k_weights(N, K, 74)
    wd = dllm.repack(Q5, w, N, K)
    act = gu.Act(synth.activations(M, K, 74))
    S = torch.empty((M, N, K // 256), dtype=torch.int32, device="cuda")
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_debug_sb_ints(wd, Q5, N, K, act.q, act.scale, act.sums, M, S)
    assert e.value.code == dllm.DLLM_ERR_ARG
