"""Failure detection on the device without faulting it: every barrier wait in the GEMM
kernel is bounded, and a wait that runs out ends the kernel with DLLM_ERR_TIMEOUT in the
device error word instead of hanging.  The test makes one run out (a producer that
issues no copy, so nothing ever fills the rings), checks the reported status, and then
checks that the context still computes correct results."""
import time

import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()
    yield
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def test_bounded_wait_reports_timeout_and_context_survives():
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    t0 = time.monotonic()
    dllm.dllm_debug_bounded_wait()
    status = dllm.dllm_get_device_status()  # synchronizes the stream
    elapsed = time.monotonic() - t0
    assert status == dllm.DLLM_ERR_TIMEOUT, dllm.status_string(status)
    assert 1.5 < elapsed < 60.0, elapsed  # the kernel's limit is 2 s
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK  # reading the word cleared it

    # the same context still runs a split-K GEMM correctly
    M, N, K = 48, 256, 4096
    w, x = gu.make_case(dllm.DLLM_Q4_K, M, N, K, 77)
    wd = dllm.repack(dllm.DLLM_Q4_K, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, dllm.DLLM_Q4_K, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(dllm.DLLM_Q4_K, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst
    assert np.isfinite(out).all()


@pytest.mark.parametrize("two_tiles", [False, True])
def test_attention_bounded_waits_report_timeout_and_context_survives(two_tiles):
    """The attention kernels' waits are bounded too: with producers that issue no copy,
    every role gives up after about 2 s, the status reads DLLM_ERR_TIMEOUT, and the same
    context then computes attention correctly with that kernel."""
    from quantized_int8_gemm_q4_b200 import synth
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    t0 = time.monotonic()
    dllm.dllm_debug_attention_stall(two_tiles)
    status = dllm.dllm_get_device_status()
    elapsed = time.monotonic() - t0
    assert status == dllm.DLLM_ERR_TIMEOUT, dllm.status_string(status)
    assert 1.5 < elapsed < 60.0, elapsed
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK

    Lq, Lk, H, Hkv = (300, 200, 64, 8) if two_tiles else (130, 200, 4, 2)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert dllm.dllm_debug_attention_tiles(Lq, H, sms) == (2 if two_tiles else 1)
    q, k, v = synth.attention_inputs(Lq, Lk, H, Hkv, 128, 8)
    o = torch.empty((Lq, H, 128), device="cuda")
    dllm.dllm_attention(*(torch.from_numpy(a).cuda() for a in (q, k, v)), Lq, Lk, H, Hkv, 128, o)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    f32 = [a.astype(np.float32) for a in (q, k, v)]
    ref = oracle.attention(*f32)
    A = oracle.attention(f32[0], f32[1], np.abs(f32[2]))
    assert np.all(np.abs(o.cpu().numpy() - ref) <= 2.0 ** -9 * A + 2.0 ** -24 * Lk * np.abs(f32[2]).max())
