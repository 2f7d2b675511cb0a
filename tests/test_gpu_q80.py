"""Q8_0 through the C-ABI: the repack into the codes and scales planes, byte for byte,
and the GEMM against the oracle's Q8_0 GEMM (which decodes the 34-byte blocks directly),
within |gpu - oracle| <= max(1e-5 |oracle|, 1e-6 T), T the oracle's sum of |terms|."""
import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

Q8 = dllm.DLLM_Q8_0


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()
    yield
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def planes_reference(w: np.ndarray, N: int, K: int) -> np.ndarray:
    """The documented repacked layout, from the GGUF bytes: int8 codes [N][K], then the
    f16 block scales as [N/128][K/256][128][8]."""
    blocks = w.reshape(N, K // 32, 34)
    codes = blocks[:, :, 2:].reshape(N, K)
    d = blocks[:, :, :2].reshape(N // 128, 128, K // 256, 8, 2).transpose(0, 2, 1, 3, 4)
    return np.concatenate([codes.reshape(-1), np.ascontiguousarray(d).reshape(-1)])


@pytest.mark.parametrize("N,K", [(128, 256), (256, 1024), (384, 4096)])
def test_repack_q80_is_the_codes_and_scales_planes(N, K):
    w = synth.weights(synth.Q8_0, N, K, 80, N, K)
    dev = dllm.repack(Q8, w, N, K)
    assert dev.numel() == dllm.dllm_repacked_bytes(Q8, N, K) == N * K // 256 * 272
    assert np.array_equal(dev.cpu().numpy(), planes_reference(w, N, K))


@pytest.mark.parametrize("M,N,K", [
    (1, 128, 256),      # one token: a token group of 16 with 15 padded rows
    (16, 128, 256),     # one group of 16
    (17, 256, 512),     # a group of 32 with 15 unused tokens
    (33, 384, 768),     # two groups (32 + 16)
    (64, 128, 1024),
    (160, 256, 4096),   # the LLaDA-8B canvas of config 1, K = hidden
    (130, 128, 12288),  # the down projection's K
])
def test_qgemm_q80_matches_oracle(M, N, K):
    w = synth.weights(synth.Q8_0, N, K, 81, M, N, K)
    x = synth.activations(M, K, 81, M, N, K)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst


def test_qgemm_q80_full_projection_sampled_columns():
    """A 4096 x 4096 projection on a 128-token canvas (every SM busy, several units per
    CTA at other sizes): column ranges against the oracle."""
    M, N, K = 128, 4096, 4096
    w = synth.weights(synth.Q8_0, N, K, 82)
    x = synth.activations(M, K, 82)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    for n0 in (0, 1920, N - 128):
        _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_, n0=n0, n1=n0 + 128)
        ok, worst = gu.tol_ok(out[:, n0:n0 + 128], ref, T)
        assert ok, (n0, worst)


@pytest.mark.parametrize("M,cols", [
    (512, (0, 2048, 3968)),   # 16 token groups x 32 tiles = 512 units: 3 or 4 per CTA
    (176, (0, 3072, 3968)),   # 5 groups of 32 + one of 16 = 192 units: CTAs 0-43 take a
                              # second unit, some of them a 16-token unit after a 32-token one
])
def test_qgemm_q80_several_units_per_cta(M, cols):
    """More units than SMs: each CTA runs the persistent loop over several units (tensor
    memory, the barrier phases and the stage ring carried from one unit to the next)."""
    N, K = 4096, 4096
    w = synth.weights(synth.Q8_0, N, K, 86, M)
    x = synth.activations(M, K, 86, M)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    for n0 in cols:
        _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_, n0=n0, n1=n0 + 128)
        ok, worst = gu.tol_ok(out[:, n0:n0 + 128], ref, T)
        assert ok, (n0, worst)


def test_qgemm_q80_wide_ldo_and_row_list_leave_other_columns():
    """ldo > N: the columns past N keep what the caller put there, with and without a
    row list."""
    M, N, K, ldo = 40, 256, 512, 384
    w = synth.weights(synth.Q8_0, N, K, 87)
    x = synth.activations(M, K, 87)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    oq, os_, _ = oracle.quantize_act(x)
    for rows in (None, [39, 0, 17, 17, 5]):
        out = gu.gemm(wd, Q8, N, K, act, rows=rows, ldo=ldo).cpu().numpy()
        assert np.isnan(out[:, N:]).all()
        _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_, rows=rows)
        assert gu.tol_ok(out[:, :N], ref, T)[0]


@pytest.mark.parametrize("n_rows", [1, 7, 32])
def test_qgemm_q80_requested_rows_and_noalloc(n_rows):
    M, N, K = 160, 256, 2048
    w = synth.weights(synth.Q8_0, N, K, 83, n_rows)
    x = synth.activations(M, K, 83)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    rows = synth.block_rows(M, n_rows, 83)
    got = gu.gemm(wd, Q8, N, K, act, rows=rows).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_, rows=rows)
    assert gu.tol_ok(got, ref, T)[0]
    full = torch.full((M, N), float("nan"), device="cuda")
    dllm.dllm_qgemm_noalloc(wd, Q8, N, K, act.q, act.scale, act.sums, M, None, 0, full, N)
    _, ref_full, T_full = oracle.qgemm(Q8, w, N, K, oq, os_)
    assert gu.tol_ok(full.cpu().numpy(), ref_full, T_full)[0]
    # the requested rows equal the same rows of the full output, bit for bit
    assert np.array_equal(got, full.cpu().numpy()[rows])


def test_qkv_q80_three_segments():
    M, Nq, Nkv, K = 40, 256, 128, 1024
    x = synth.activations(M, K, 84)
    wts = [synth.weights(synth.Q8_0, n, K, 84, i) for i, n in enumerate((Nq, Nkv, Nkv))]
    wd = [dllm.repack(Q8, wt, wt.shape[0], K) for wt in wts]
    act = gu.Act(x)
    oq_, os_, _ = oracle.quantize_act(x)
    outs = [torch.empty((M, n), device="cuda") for n in (Nq, Nkv, Nkv)]
    wsb = dllm.dllm_qgemm_workspace_bytes(Q8, Nq + 2 * Nkv, K, M)
    work = dllm.alloc_workspace(max(wsb, 256))
    dllm.dllm_qkv_qgemm(wd[0], wd[1], wd[2], Q8, Nq, Nkv, K, act.q, act.scale, act.sums, M, outs[0], Nq,
                        outs[1], outs[2], Nkv, work, max(wsb, 256))
    for o, wt in zip(outs, wts):
        _, ref, T = oracle.qgemm(Q8, wt, wt.shape[0], K, oq_, os_)
        assert gu.tol_ok(o.cpu().numpy(), ref, T)[0]


def test_q80_extreme_codes_and_scales():
    """The exact conversion at its limits: every code -128 (the int8 minimum) against
    activations that quantize to +-127, the largest block dot (32 * 128 * 127 = 520,192,
    inside the 2^22 the preset trick allows); every code 127 under the largest f16 scale
    (65504); blocks whose scale is 0; all-zero activation rows."""
    M, N, K = 48, 256, 1024
    w = synth.weights(synth.Q8_0, N, K, 88).copy()
    b = w.reshape(N, K // 32, 34)
    b[:64, :, 2:] = 0x80                                  # q = -128
    b[:64, :, 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    b[64:128, :, 2:] = 127
    b[64:128, :, 0:2] = np.frombuffer(np.float16(65504.0).tobytes(), np.uint8)
    b[128:192, :, 0:2] = 0                                # d = 0: no contribution
    x = synth.activations(M, K, 88)
    x[0] = 3.0                                            # quantizes to +127 everywhere
    x[1] = -3.0                                           # -127
    x[2] = 0.0                                            # all-zero row: scale 0
    x[3, ::2] = 5.0
    x[3, 1::2] = -5.0
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    assert (oq[0] == 127).all() and (oq[1] == -127).all()
    _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst
    assert not out[2].any() and not out[:, 128:192].any()
    # the extreme rows in closed form: 32 blocks of 32 codes, d = 1, da = 3/127
    np.testing.assert_allclose(out[0, :64], -128 * 127 * K * (3.0 / 127), rtol=1e-6)


def test_q80_vocabulary_width_sampled():
    """The 126464-row output projection in Q8_0 on 32 requested rows: 988 weight tiles,
    several per CTA, sampled column ranges against the oracle."""
    M, N, K = 160, 126464, 4096
    w = synth.weights(synth.Q8_0, N, K, 89)
    x = synth.activations(M, K, 89)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(x)
    rows = synth.block_rows(M, 32, 89)
    out = gu.gemm(wd, Q8, N, K, act, rows=rows).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    for n0 in (0, 63232, N - 128):
        _, ref, T = oracle.qgemm(Q8, w, N, K, oq, os_, rows=rows, n0=n0, n1=n0 + 128)
        ok, worst = gu.tol_ok(out[:, n0:n0 + 128], ref, T)
        assert ok, (n0, worst)


def test_q80_deterministic_and_integer_views_rejected():
    M, N, K = 48, 128, 512
    w = synth.weights(synth.Q8_0, N, K, 85)
    wd = dllm.repack(Q8, w, N, K)
    act = gu.Act(synth.activations(M, K, 85))
    a = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    b = gu.gemm(wd, Q8, N, K, act).cpu().numpy()
    assert np.array_equal(a, b)
    S = torch.empty((M, N, K // 256), dtype=torch.int32, device="cuda")
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_debug_sb_ints(wd, Q8, N, K, act.q, act.scale, act.sums, M, S)
    assert e.value.code == dllm.DLLM_ERR_ARG
