"""Fused quantizers (RMSNorm -> quantize, SwiGLU -> quantize) vs the CPU oracle,
element by element, through the C-ABI.

The oracle forms the normalised or gated value in fp64 and rounds it to f32 once; so
does the kernel, but it sums the squares of RMSNorm in another order and calls CUDA's
exp instead of the C library's.  Both differences are far below an f32 rounding step.
Each test therefore brackets the oracle's fp64 value (scaling the sum of squares,
or the fp64 SwiGLU value, by 1 -+ delta) and compares:
  - bit for bit (codes, scales, scaled sub-block sums) every 256-block whose f32
    values are the same at both ends of the bracket, i.e. unique;
  - in any other block (about 1% of RMSNorm blocks at K = 4096, as the bracket is
    conservative), that the codes and scale are exactly the quantization of one
    admissible choice of f32 inputs, each element at one end of its bracket.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

Q4, Q6 = dllm.DLLM_Q4_K, dllm.DLLM_Q6_K


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()
    yield
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def _host(q, s, u, M, K):
    return gu.untile_q(q, M, K), gu.untile_scale(s, M, K), gu.untile_sums(u, M, K)


def _quantize_block(v, amax):
    """The activation quantizer's reading for one block with a given amax, in numpy f32."""
    if amax == 0:
        return np.zeros(v.shape, np.int8), np.float32(0)
    iscale = np.float32(127) / amax
    return np.clip(np.rint(v * iscale), -127, 127).astype(np.int8), amax / np.float32(127)


def _valid_block(qg, sg, lo, hi):
    """True if (codes qg, scale sg) quantize some block whose element i is lo[i] or
    hi[i] (adjacent f32 values, |lo| <= |hi|).  The block's amax is max|lo| or max|hi|."""
    for amax in {np.float32(np.abs(lo).max()), np.float32(np.abs(hi).max())}:
        c_lo, sc = _quantize_block(lo, amax)
        c_hi, _ = _quantize_block(hi, amax)
        if sc.view(np.uint32) == np.float32(sg).view(np.uint32) and np.all((qg == c_lo) | (qg == c_hi)):
            return True
    return False


def _compare(got, y, y_lo, y_hi, d, M, K):
    """got = (q, scale, (hi, lo)) from the GPU; y the oracle's f32 value and y_lo / y_hi
    the two ends of its bracket (|y_lo| <= |y| <= |y_hi|), d its relative half-width.
    A block whose ends agree
    must match the oracle bit for bit; any other block must be a valid quantization of
    one admissible choice.  The scaled sums must match the GPU's own codes and scales
    exactly.  Returns the number of ambiguous blocks."""
    q, s, (hi, lo) = got
    oq, os_, _ = oracle.quantize_act(y)
    nsb = K // 256
    uniq = (y_lo.view(np.uint32) == y_hi.view(np.uint32)).reshape(M, nsb, 256).all(-1)
    ub = np.repeat(uniq, 256, axis=1)
    assert np.array_equal(q[ub], oq[ub])
    assert np.array_equal(s[uniq].view(np.uint32), os_[uniq].view(np.uint32))
    for m, b in zip(*np.nonzero(~uniq)):
        cols = slice(256 * b, 256 * b + 256)
        assert _valid_block(q[m, cols], s[m, b], y_lo[m, cols], y_hi[m, cols]), (m, b)
    t = q.reshape(M, K // 32, 32).astype(np.int32).sum(-1)
    v = np.repeat(s, 8, axis=1) * t.astype(np.float32)
    assert np.array_equal((hi + lo).view(np.uint32), v.view(np.uint32))
    assert np.all(hi.view(np.uint32) & 0x1FFF == 0)
    # An element is ambiguous when its value lies within d (relative) of an f32 rounding
    # boundary: probability about 2 d / 2^-23.  Far more ambiguous blocks than that
    # would mean a broken bracket, and a vacuous test.
    n_amb = int((~uniq).sum())
    expect = uniq.size * min(1.0, 256 * 2 * d * 2.0 ** 23)
    assert n_amb <= 2 + 4 * expect, (n_amb, expect)
    return n_amb


def _rms_rows(M, K, seed):
    x = synth.activations(M, K, seed, M, K)
    rng = np.random.default_rng(seed * 31 + M)
    x *= rng.uniform(1e-3, 1e3, (M, 1)).astype(np.float32)
    if M > 4:
        x[1] = 0.0                      # all-zero row: y = 0, scale 0
        x[2] = -2.5                     # constant row
        x[3] = 0.0
        x[3, K // 2] = 7.0              # one non-zero element
        x[4, :256] *= 1e4               # one block dominates the row's norm
    return x


def _gamma(K, seed):
    return np.random.default_rng(seed).uniform(0.25, 2.0, K).astype(np.float32)


def _run_rms(x, gamma, eps, ldx=None):
    M, K = x.shape
    ldx = K if ldx is None else ldx
    xb = np.zeros((M, ldx), np.float32)
    xb[:, :K] = x
    if ldx > K:
        xb[:, K:] = np.nan              # never read
    xd = torch.from_numpy(xb).cuda()
    gd = torch.from_numpy(gamma).cuda()
    q, s, u = dllm.alloc_act(M, K)
    q.fill_(0x55)
    s.fill_(float("nan"))
    dllm.dllm_rmsnorm_quantize(xd, M, K, ldx, gd, eps, None, 0, q, s, u)
    return q, s, u


def _rms_bracket(x, gamma, eps):
    K = x.shape[1]
    d = 4.0 * K * 2.0 ** -53 + 2.0 ** -50
    return (oracle.rmsnorm(x, gamma, eps), oracle.rmsnorm(x, gamma, eps, ss_scale=1 + d),
            oracle.rmsnorm(x, gamma, eps, ss_scale=1 - d), d)


@pytest.mark.parametrize("M,K", [(1, 256), (5, 512), (16, 256), (17, 768), (64, 3584), (128, 4096), (257, 1024),
                                 (3, 8448), (2, 16384),
                                 # more than 12 rows per SM (148 SMs): the form with up to four
                                 # super-blocks per warp (uneven at 3584, re-read past 16 at 8448)
                                 (1800, 4096), (1790, 3584), (1781, 8448), (1800, 256)])
def test_rmsnorm_quantize(M, K):
    x = _rms_rows(M, K, 41)
    gamma = _gamma(K, K)
    eps = 1e-5
    q, s, u = _run_rms(x, gamma, eps)
    _compare(_host(q, s, u, M, K), *_rms_bracket(x, gamma, eps), M, K)
    Mp = (M + 15) // 16 * 16
    if Mp > M:  # padding rows are zero
        full = q.cpu().numpy().reshape(K // 256, Mp // 8, 16, 8, 16).transpose(1, 3, 0, 2, 4).reshape(Mp, K)
        assert not full[M:].any()
        assert not s.cpu().numpy().reshape(K // 256, Mp)[:, M:].any()


@pytest.mark.parametrize("eps,M", [(1e-6, 24), (1.0, 24), (1e4, 24), (1e-5, 1800)])
def test_rmsnorm_quantize_eps_and_stride(eps, M):
    """eps across its range and a row stride ldx > K (at 1800 rows, in the form with four
    super-blocks per warp)."""
    K, ldx = 2048, 2304
    x = _rms_rows(M, K, 42)
    gamma = _gamma(K, 7)
    q, s, u = _run_rms(x, gamma, eps, ldx=ldx)
    _compare(_host(q, s, u, M, K), *_rms_bracket(x, gamma, eps), M, K)


def test_rmsnorm_quantize_deterministic():
    M, K = 48, 4096
    x = _rms_rows(M, K, 43)
    gamma = _gamma(K, 8)
    a = [t.cpu().numpy().copy() for t in _run_rms(x, gamma, 1e-5)]
    b = [t.cpu().numpy().copy() for t in _run_rms(x, gamma, 1e-5)]
    for p, r in zip(a, b):
        assert np.array_equal(p, r)


def _swiglu_inputs(M, K, seed):
    rng = np.random.default_rng(seed)
    g = (rng.standard_normal((M, K)) * rng.uniform(0.1, 20, (M, 1))).astype(np.float32)
    u = (rng.standard_normal((M, K)) * rng.uniform(0.1, 20, (M, 1))).astype(np.float32)
    if M > 3:
        g[1] = 0.0                      # SiLU(0) = 0: an all-zero row
        g[2, :256] = -800.0             # exp(-g) overflows: h = -0
        g[3, :256] = 60.0               # h = g * u exactly
    return g, u


def _swiglu_bracket(g, u):
    d = 1e-14
    return oracle.swiglu(g, u), oracle.swiglu(g, u, h_scale=1 - d), oracle.swiglu(g, u, h_scale=1 + d), d


@pytest.mark.parametrize("M,K", [(1, 256), (7, 512), (16, 2304), (33, 3584), (128, 12288), (200, 1024)])
def test_swiglu_quantize(M, K):
    g, u = _swiglu_inputs(M, K, M + K)
    gd, ud = torch.from_numpy(g).cuda(), torch.from_numpy(u).cuda()
    q, s, a = dllm.alloc_act(M, K)
    dllm.dllm_swiglu_quantize(gd, ud, M, K, K, q, s, a)
    _compare(_host(q, s, a, M, K), *_swiglu_bracket(g, u), M, K)


def test_swiglu_quantize_interleaved_columns():
    """gate and up as the two column ranges of one [M][2K] buffer."""
    M, K = 40, 1536
    g, u = _swiglu_inputs(M, K, 5)
    buf = torch.from_numpy(np.concatenate([g, u], axis=1)).cuda()
    q, s, a = dllm.alloc_act(M, K)
    dllm.dllm_swiglu_quantize(buf, buf[:, K:], M, K, 2 * K, q, s, a)
    _compare(_host(q, s, a, M, K), *_swiglu_bracket(g, u), M, K)


# ------------------------------------------------------------------ chains through the GEMMs

def test_chain_rmsnorm_qkv_and_gateup_swiglu_down():
    """RMSNorm -> quantize -> gate/up (one launch) -> SwiGLU -> quantize -> down, each
    stage checked against the oracle run on the GPU's own input to that stage."""
    M, h, f = 48, 1024, 2816
    x = _rms_rows(M, h, 44)
    gamma = _gamma(h, 9)
    wg = synth.weights(Q4, f, h, 51)
    wu = synth.weights(Q4, f, h, 52)
    wdn = synth.weights(Q6, h, f, 53)
    dg, du, dd = dllm.repack(Q4, wg, f, h), dllm.repack(Q4, wu, f, h), dllm.repack(Q6, wdn, h, f)
    xd = torch.from_numpy(x).cuda()
    gd = torch.from_numpy(gamma).cuda()
    qh, sh, uh = dllm.alloc_act(M, h)
    qf, sf, uf = dllm.alloc_act(M, f)
    o_gu = torch.empty((M, 2 * f), device="cuda")
    o_d = torch.empty((M, h), device="cuda")
    ws_b = max(dllm.dllm_qgemm_workspace_bytes(Q4, 2 * f, h, M), dllm.dllm_qgemm_workspace_bytes(Q6, h, f, M))
    ws = dllm.alloc_workspace(max(ws_b, 256))
    # the whole chain back to back on one stream (programmatic dependent launches)
    dllm.dllm_rmsnorm_quantize(xd, M, h, h, gd, 1e-5, None, 0, qh, sh, uh)
    dllm.dllm_qkv_qgemm(dg, du, None, Q4, f, f, h, qh, sh, uh, M, o_gu, 2 * f, o_gu[:, f:], None, 2 * f, ws, ws_b)
    dllm.dllm_swiglu_quantize(o_gu, o_gu[:, f:], M, f, 2 * f, qf, sf, uf)
    dllm.dllm_qgemm(dd, Q6, h, f, qf, sf, uf, M, None, 0, o_d, h, ws, ws_b)
    torch.cuda.synchronize()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK

    _compare(_host(qh, sh, uh, M, h), *_rms_bracket(x, gamma, 1e-5), M, h)
    oq, os_, _ = oracle.quantize_act(oracle.rmsnorm(x, gamma, 1e-5))
    gu_host = o_gu.cpu().numpy()
    for w, cols in ((wg, slice(0, f)), (wu, slice(f, 2 * f))):
        _, ref, T = oracle.qgemm(Q4, w, f, h, oq, os_)
        ok, worst = gu.tol_ok(gu_host[:, cols], ref, T)
        assert ok, worst
    g_in, u_in = np.ascontiguousarray(gu_host[:, :f]), np.ascontiguousarray(gu_host[:, f:])
    _compare(_host(qf, sf, uf, M, f), *_swiglu_bracket(g_in, u_in), M, f)
    fq, fs, _ = oracle.swiglu_quantize(g_in, u_in)
    _, ref, T = oracle.qgemm(Q6, wdn, h, f, fq, fs)
    ok, worst = gu.tol_ok(o_d.cpu().numpy(), ref, T)
    assert ok, worst


def _run_rms_rows(x, gamma, eps, rows):
    M, K = x.shape
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    gd = torch.from_numpy(gamma).cuda()
    r = torch.from_numpy(np.asarray(rows, np.int32)).cuda()
    n = len(rows)
    q, s, u = dllm.alloc_act(n, K)
    q.fill_(0x55)
    s.fill_(float("nan"))
    dllm.dllm_rmsnorm_quantize(xd, M, K, K, gd, eps, r, n, q, s, u)
    return q, s, u


@pytest.mark.parametrize("M", [160, 1800])
def test_rmsnorm_quantize_rows(M):
    """A row list: output row i is canvas row rows[i] (any order, duplicates), equal bit for
    bit to that row of the full-canvas result (at 1800 rows the full canvas runs the form
    with four super-blocks per warp, the 37-row list the one with one per warp)."""
    K = 4096
    x = _rms_rows(M, K, 47)
    gamma = _gamma(K, 11)
    rows = np.concatenate([synth.block_rows(M, 32, 48), [0, M - 1, 5, 5, 37]]).astype(np.int32)
    n = len(rows)
    q, s, u = _run_rms_rows(x, gamma, 1e-5, rows)
    xr = np.ascontiguousarray(x[rows])
    got = _host(q, s, u, n, K)
    _compare(got, *_rms_bracket(xr, gamma, 1e-5), n, K)
    full = _host(*_run_rms(x, gamma, 1e-5), M, K)
    assert np.array_equal(got[0], full[0][rows])
    assert np.array_equal(got[1].view(np.uint32), full[1][rows].view(np.uint32))
    Mp = (n + 15) // 16 * 16
    qa = q.cpu().numpy().reshape(K // 256, Mp // 8, 16, 8, 16).transpose(1, 3, 0, 2, 4).reshape(Mp, K)
    assert not qa[n:].any()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def test_rmsnorm_quantize_row_out_of_range():
    """An entry outside [0, M) zero-fills its output row and reports DLLM_ERR_ROW_RANGE;
    the other rows are unaffected."""
    M, K = 64, 1024
    x = _rms_rows(M, K, 49)
    gamma = _gamma(K, 12)
    rows = np.array([3, M, 10, -1, 63], np.int32)
    q, s, u = _run_rms_rows(x, gamma, 1e-5, rows)
    assert dllm.dllm_get_device_status() == dllm.DLLM_ERR_ROW_RANGE
    gq, gs, (hi, lo) = _host(q, s, u, len(rows), K)
    for i in (1, 3):
        assert not gq[i].any() and not gs[i].any() and not hi[i].any() and not lo[i].any()
    ok = np.array([0, 2, 4])
    xr = np.ascontiguousarray(x[rows[ok]])
    sub = (gq[ok], gs[ok], (hi[ok], lo[ok]))
    _compare(sub, *_rms_bracket(xr, gamma, 1e-5), len(ok), K)


def test_final_rmsnorm_output_rows():
    """Final RMSNorm -> quantize on the 32 requested rows only (a compact activation),
    then the output projection on that activation, with no row list."""
    M, h, V = 96, 1024, 2048
    x = _rms_rows(M, h, 45)
    gamma = _gamma(h, 10)
    w = synth.weights(Q6, V, h, 54)
    wd = dllm.repack(Q6, w, V, h)
    rows = synth.block_rows(M, 32, 46)
    q, s, u = _run_rms_rows(x, gamma, 1e-6, rows)
    out = torch.empty((32, V), device="cuda")
    wsb = dllm.dllm_qgemm_workspace_bytes(Q6, V, h, 32)
    ws = dllm.alloc_workspace(max(wsb, 256))
    dllm.dllm_qgemm(wd, Q6, V, h, q, s, u, 32, None, 0, out, V, ws, wsb)
    xr = np.ascontiguousarray(x[rows])
    _compare(_host(q, s, u, 32, h), *_rms_bracket(xr, gamma, 1e-6), 32, h)
    oq, os_, _ = oracle.rmsnorm_quantize(xr, gamma, 1e-6)
    _, ref, T = oracle.qgemm(Q6, w, V, h, oq, os_)
    ok, worst = gu.tol_ok(out.cpu().numpy(), ref, T)
    assert ok, worst
    # the same logits as normalising the whole canvas and gathering rows in the GEMM
    qa, sa, ua = _run_rms(x, gamma, 1e-6)
    r = torch.from_numpy(rows).cuda()
    out2 = torch.empty((32, V), device="cuda")
    wsb2 = dllm.dllm_qgemm_workspace_bytes(Q6, V, h, M, 32)
    ws2 = dllm.alloc_workspace(max(wsb2, 256))
    dllm.dllm_qgemm(wd, Q6, V, h, qa, sa, ua, M, r, 32, out2, V, ws2, wsb2)
    assert torch.equal(out, out2)
