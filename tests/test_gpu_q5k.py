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


def test_qgemm_q5k_extreme_blocks():
    """The split at its limits (block [d, dmin, 12 scale bytes, 32 qh, 128 qs]): every
    5-bit code 31 (all low nibbles 15, every fifth bit set) with sc = m = 63; the same
    under the largest d the split can hold (4094: 16 d = 65504, the f16 maximum) and the
    largest dmin; all codes 0, so only -dmin * m is left; against activations that
    quantize to +-127 and an all-zero row."""
    M, N, K = 48, 256, 1024
    w = synth.q5k_weights(N, K, 73).copy()
    b = w.reshape(N, K // 256, 176)
    one = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    big_d = np.frombuffer(np.float16(4094.0).tobytes(), np.uint8)
    big = np.frombuffer(np.float16(65504.0).tobytes(), np.uint8)
    b[:128, :, 4:16] = 0xFF                               # sc_j = m_j = 63 for every j
    b[:128, :, 16:176] = 0xFF                             # qh and qs: every q = 31
    b[:64, :, 0:2] = one
    b[:64, :, 2:4] = one
    b[64:128, :, 0:2] = big_d
    b[64:128, :, 2:4] = big
    b[128:192, :, 16:176] = 0                             # q = 0: the min term alone
    x = synth.activations(M, K, 73)
    x[0] = 3.0
    x[1] = -3.0
    x[2] = 0.0
    wd = dllm.repack(Q5, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q5, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    assert (oq[0] == 127).all() and (oq[1] == -127).all()
    _, ref, T = oracle.qgemm(Q5, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst
    assert not out[2].any()
    # closed form of row 0 on the first rows: (63 * 31 - 63) per weight, K weights, da = 3/127
    np.testing.assert_allclose(out[0, :64], (63 * 31 - 63) * 127 * K * (3.0 / 127), rtol=1e-6)


def test_repack_q5k_scale_out_of_range_is_reported():
    """|d| >= 4096 cannot be split (16 d overflows f16): the repack reports
    DLLM_ERR_SCALE_RANGE in the device error word and nothing faults; the largest
    splittable d (4094) is accepted."""
    N, K = 128, 512
    w = synth.q5k_weights(N, K, 74).copy()
    b = w.reshape(N, K // 256, 176)
    b[5, 1, 0:2] = np.frombuffer(np.float16(4094.0).tobytes(), np.uint8)
    dllm.repack(Q5, w, N, K)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    b[7, 0, 0:2] = np.frombuffer(np.float16(4096.0).tobytes(), np.uint8)
    dllm.repack(Q5, w, N, K)
    assert dllm.dllm_get_device_status() == dllm.DLLM_ERR_SCALE_RANGE
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK  # read and cleared


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
