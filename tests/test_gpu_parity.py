"""CUDA path vs the CPU oracle, element by element, through the C-ABI.

Bit-exact: activation quantization (int8, scales, per-32 sums), the weight repack,
the per-sub-block int32 dots, and the per-super-block integers the tensor-core path
forms.  Floating point: |gpu - oracle| <= max(1e-5 |oracle|, 1e-6 T), T the sum of
absolute terms (the tolerance the method's target states).
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


# ------------------------------------------------------------------ quantize

def _special_rows(M, K):
    x = synth.activations(M, K, 21, M, K)
    rng = np.random.default_rng(M * 7 + K)
    x *= rng.uniform(1e-4, 1e4, (M, 1)).astype(np.float32)
    if M > 3:
        x[1] = 0.0                                   # all-zero row
        x[2, :256] = -2.5                            # constant block
        x[3, :8] = [127, 0.5, 1.5, 2.5, -0.5, -1.5, 63.5, -127]  # ties with iscale = 1
        x[3, 8:256] = 0
    return x


@pytest.mark.parametrize("M,K", [(1, 256), (15, 512), (16, 256), (17, 768), (64, 4096), (160, 4096), (257, 1024)])
def test_quantize_bitexact(M, K):
    x = _special_rows(M, K)
    act = gu.Act(x)
    q, s, (hi, lo) = act.host()
    oq, os_, oa = oracle.quantize_act(x)
    assert np.array_equal(q, oq)
    assert np.array_equal(s.view(np.uint32), os_.view(np.uint32))
    # scaled per-32 sums: hi + lo == f32(scale * sum) exactly, hi exact in tf32
    v = np.repeat(os_, 8, axis=1) * oa.astype(np.float32)
    assert np.array_equal((hi + lo).view(np.uint32), v.view(np.uint32))
    assert np.all(hi.view(np.uint32) & 0x1FFF == 0)
    Mp = (M + 15) // 16 * 16
    if Mp > M:  # padded rows are zero
        full = act.q.cpu().numpy().reshape(K // 256, Mp // 8, 16, 8, 16).transpose(1, 3, 0, 2, 4).reshape(Mp, K)
        assert not full[M:].any()


def test_quantize_strided_input():
    M, K, ldx = 20, 512, 1024
    xb = synth.activations(M, ldx, 22)
    x = torch.from_numpy(xb).cuda()
    q, s, u = dllm.alloc_act(M, K)
    dllm.dllm_quantize_act(x, M, K, ldx, q, s, u)
    oq, os_, _ = oracle.quantize_act(np.ascontiguousarray(xb[:, :K]))
    assert np.array_equal(gu.untile_q(q, M, K), oq)
    assert np.array_equal(gu.untile_scale(s, M, K), os_)


# ------------------------------------------------------------------ repack and integer paths

@pytest.mark.parametrize("qtype", [Q4, Q6])
def test_repack_bitexact(qtype):
    N, K = 256, 768
    w = synth.weights(qtype, N, K, 31)
    dev = dllm.repack(qtype, w, N, K)
    assert np.array_equal(dev.cpu().numpy(), gu.repack_reference(qtype, w))


@pytest.mark.parametrize("qtype", [Q4, Q6])
@pytest.mark.parametrize("M,N,K", [(3, 128, 256), (17, 256, 512)])
def test_subblock_dots_bitexact(qtype, M, N, K):
    w, x = gu.make_case(qtype, M, N, K, 32)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    nsub = K // 32 if qtype == Q4 else K // 16
    dots = torch.zeros((M, N, nsub), dtype=torch.int32, device="cuda")
    dllm.dllm_debug_subblock_dots(wd, qtype, N, K, act.q, M, dots)
    oq, _, _ = oracle.quantize_act(x)
    od, _, _ = oracle.sb_ints(qtype, w, N, K, oq)
    assert np.array_equal(dots.cpu().numpy(), od)


@pytest.mark.parametrize("qtype", [Q4, Q6])
@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (17, 256, 768), (64, 128, 512), (160, 384, 256)])
def test_tensor_core_integers_bitexact(qtype, M, N, K):
    w, x = gu.make_case(qtype, M, N, K, 33)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    S = torch.zeros((M, N, K // 256), dtype=torch.int32, device="cuda")
    dllm.dllm_debug_sb_ints(wd, qtype, N, K, act.q, act.scale, act.sums, M, S)
    oq, _, _ = oracle.quantize_act(x)
    _, oS, _ = oracle.sb_ints(qtype, w, N, K, oq)
    assert np.array_equal(S.cpu().numpy().astype(np.int64), oS)


def test_tensor_core_integers_extreme_values():
    # largest magnitudes the planes and sums can take: every quant at its maximum,
    # every 6-bit scale and min 63, every activation +-127
    M, N, K = 16, 128, 512
    w = synth.q4k_weights(N, K, 34).copy()
    w[..., 4:144] = 0xFF
    x = np.full((M, K), 3.0, np.float32)
    x[::2] *= -1
    wd = dllm.repack(Q4, w, N, K)
    act = gu.Act(x)
    S = torch.zeros((M, N, K // 256), dtype=torch.int32, device="cuda")
    dllm.dllm_debug_sb_ints(wd, Q4, N, K, act.q, act.scale, act.sums, M, S)
    oq, os_, _ = oracle.quantize_act(x)
    _, oS, _ = oracle.sb_ints(Q4, w, N, K, oq)
    assert np.abs(oS).max() == 945 * 127 * 256
    assert np.array_equal(S.cpu().numpy().astype(np.int64), oS)
    # the min term is largest here too (every m = 63, every |sum32| = 32 * 127)
    out = gu.gemm(wd, Q4, N, K, act).cpu().numpy()
    _, ref, T = oracle.qgemm(Q4, w, N, K, oq, os_)
    assert gu.tol_ok(out, ref, T)[0]
    # Q6_K: q = 0 with scale -128 gives (q-32)*sc = 4096, the largest product
    w6 = synth.q6k_weights(N, K, 34).copy()
    w6[..., 0:192] = 0
    w6[..., 192:208] = np.uint8(0x80)
    wd6 = dllm.repack(Q6, w6, N, K)
    S6 = torch.zeros((M, N, K // 256), dtype=torch.int32, device="cuda")
    dllm.dllm_debug_sb_ints(wd6, Q6, N, K, act.q, act.scale, act.sums, M, S6)
    _, oS6, _ = oracle.sb_ints(Q6, w6, N, K, oq)
    assert np.array_equal(S6.cpu().numpy().astype(np.int64), oS6)


# ------------------------------------------------------------------ f32 GEMM

SHAPES = [(1, 128, 256), (15, 128, 512), (16, 256, 256), (17, 384, 768), (64, 256, 512), (160, 128, 512),
          (257, 256, 256),
          # K long enough that tiles are split over several CTAs (chunk partials + fix-up)
          (17, 256, 2048), (160, 128, 4096), (1, 384, 4096), (300, 256, 3072)]


@pytest.mark.parametrize("qtype", [Q4, Q6])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_qgemm_parity(qtype, M, N, K):
    w, x = gu.make_case(qtype, M, N, K, 40)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, qtype, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst


def test_config0_exact_case():
    """Q4_K, M=64, K=512, N=256, seed 0 (the smallest named workload)."""
    M, N, K = 64, 256, 512
    w = synth.q4k_weights(N, K, 0)
    x = synth.activations(M, K, 0)
    wd = dllm.repack(Q4, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q4, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q4, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst
    dots = torch.zeros((M, N, K // 32), dtype=torch.int32, device="cuda")
    dllm.dllm_debug_subblock_dots(wd, Q4, N, K, act.q, M, dots)
    od, _, _ = oracle.sb_ints(Q4, w, N, K, oq)
    assert np.array_equal(dots.cpu().numpy(), od)


@pytest.mark.parametrize("qtype", [Q4, Q6])
def test_qgemm_ldo_and_determinism(qtype):
    M, N, K, ldo = 40, 256, 512, 300
    w, x = gu.make_case(qtype, M, N, K, 41)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    a = gu.gemm(wd, qtype, N, K, act, ldo=ldo)
    b = gu.gemm(wd, qtype, N, K, act, ldo=ldo)
    assert torch.equal(a[:, :N], b[:, :N])
    assert torch.isnan(a[:, N:]).all()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_)
    assert gu.tol_ok(a[:, :N].cpu().numpy(), ref, T)[0]


# ------------------------------------------------------------------ rows (logits only on requested rows)

@pytest.mark.parametrize("qtype", [Q6, Q4])
@pytest.mark.parametrize("n_rows", [1, 2, 4, 8, 16, 32])
def test_rows_equal_full_slice(qtype, n_rows):
    M, N, K = 160, 256, 512
    w, x = gu.make_case(qtype, M, N, K, 50)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    full = gu.gemm(wd, qtype, N, K, act)
    rows = synth.block_rows(M, n_rows, 50, n_rows)
    got = gu.gemm(wd, qtype, N, K, act, rows=rows)
    assert torch.equal(got, full[torch.from_numpy(rows).long().cuda()])
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_, rows=rows)
    assert gu.tol_ok(got.cpu().numpy(), ref, T)[0]


def test_rows_duplicates_and_order():
    M, N, K = 64, 128, 256
    w, x = gu.make_case(Q6, M, N, K, 51)
    wd = dllm.repack(Q6, w, N, K)
    act = gu.Act(x)
    full = gu.gemm(wd, Q6, N, K, act)
    rows = np.array([63, 0, 0, 17, 63], np.int32)
    got = gu.gemm(wd, Q6, N, K, act, rows=rows)
    assert torch.equal(got, full[torch.from_numpy(rows).long().cuda()])


def test_rows_out_of_range_sets_status():
    M, N, K = 48, 128, 256
    w, x = gu.make_case(Q4, M, N, K, 52)
    wd = dllm.repack(Q4, w, N, K)
    act = gu.Act(x)
    full = gu.gemm(wd, Q4, N, K, act)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    rows = np.array([5, 48, -1, 7], np.int32)
    got = gu.gemm(wd, Q4, N, K, act, rows=rows)
    assert dllm.dllm_get_device_status() == dllm.DLLM_ERR_ROW_RANGE
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK  # cleared
    assert torch.equal(got[0], full[5]) and torch.equal(got[3], full[7])
    assert (got[1] == 0).all() and (got[2] == 0).all()


# ------------------------------------------------------------------ Q/K/V in one launch

@pytest.mark.parametrize("qtype", [Q4, Q6])
@pytest.mark.parametrize("with_v", [True, False])
def test_qkv_matches_oracle_and_separate(qtype, with_v):
    """One launch over two or three weight matrices sharing one quantized activation.
    The fused launch may split K differently from separate launches (the split
    depends on the launch's total N), so it is compared with the oracle and with the
    separate launches within the tolerance, and with itself bit for bit."""
    M, Nq, Nkv, K = 40, 256, 128, 512
    x = synth.activations(M, K, 60)
    wts = [synth.weights(qtype, n, K, 60, i) for i, n in enumerate((Nq, Nkv, Nkv))]
    wd = [dllm.repack(qtype, w, w.shape[0], K) for w in wts]
    act = gu.Act(x)
    oq_, os_, _ = oracle.quantize_act(x)

    def fused():
        oq = torch.empty((M, Nq), device="cuda")
        ok = torch.empty((M, Nkv), device="cuda")
        ov = torch.empty((M, Nkv), device="cuda") if with_v else None
        wsb = dllm.dllm_qgemm_workspace_bytes(qtype, Nq + (2 if with_v else 1) * Nkv, K, M)
        work = dllm.alloc_workspace(wsb)
        dllm.dllm_qkv_qgemm(wd[0], wd[1], wd[2] if with_v else None, qtype, Nq, Nkv, K, act.q, act.scale,
                            act.sums, M, oq, Nq, ok, ov, Nkv, work, wsb)
        return [oq, ok] + ([ov] if with_v else [])

    outs, again = fused(), fused()
    for i, o in enumerate(outs):
        assert torch.equal(o, again[i])
        _, ref, T = oracle.qgemm(qtype, wts[i], wts[i].shape[0], K, oq_, os_)
        assert gu.tol_ok(o.cpu().numpy(), ref, T)[0]
        sep = gu.gemm(wd[i], qtype, wts[i].shape[0], K, act).cpu().numpy()
        assert gu.tol_ok(sep, ref, T)[0]


# ------------------------------------------------------------------ full-size shapes, sampled outputs

def _sampled_parity(qtype, M, N, K, seed, rows=None, n_samples=3, width=64):
    w = synth.weights(qtype, N, K, seed)
    x = synth.activations(M, K, seed)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, qtype, N, K, act, rows=rows).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    rng = np.random.default_rng(seed)
    starts = sorted(set([0, N - width] + list(rng.integers(0, N - width, n_samples))))
    for n0 in starts:
        _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_, rows=rows, n0=int(n0), n1=int(n0) + width)
        ok, worst = gu.tol_ok(out[:, n0:n0 + width], ref, T)
        assert ok, (n0, worst)
    return out


def test_full_qkv_shape_sampled():
    # LLaDA-8B-shaped attention projections on a 160-token canvas: Q|K|V as one N = 12288 launch
    _sampled_parity(Q4, 160, 12288, 4096, 1)


def test_config1_qkv_three_segments_and_o_sampled():
    """The attention-projection workload exactly as named: a 160-token canvas
    (32 prompt + 128 masked), one quantized activation shared by Q, K and V through
    dllm_qkv_qgemm with three 4096 x 4096 Q4_K segments, then O (4096 x 4096, Q4_K) on a
    second quantized activation; sampled output columns of every projection against the
    oracle."""
    M, K, N = 160, 4096, 4096
    xa, xo = synth.activations(M, K, 1, 0), synth.activations(M, K, 1, 1)
    wq, wk, wv, wo = (synth.weights(Q4, N, K, 1, i) for i in range(4))
    dq, dk, dv, do = (dllm.repack(Q4, w, N, K) for w in (wq, wk, wv, wo))
    act, act_o = gu.Act(xa), gu.Act(xo)
    outs = [torch.full((M, N), float("nan"), device="cuda") for _ in range(3)]
    wsb = dllm.dllm_qgemm_workspace_bytes(Q4, 3 * N, K, M)
    work = dllm.alloc_workspace(max(wsb, 256))
    dllm.dllm_qkv_qgemm(dq, dk, dv, Q4, N, N, K, act.q, act.scale, act.sums, M, outs[0], N, outs[1], outs[2], N,
                        work, wsb)
    o_out = gu.gemm(do, Q4, N, K, act_o).cpu().numpy()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    qa, sa, _ = oracle.quantize_act(xa)
    qo, so, _ = oracle.quantize_act(xo)
    rng = np.random.default_rng(11)
    cases = [(w, o.cpu().numpy(), qa, sa) for w, o in zip((wq, wk, wv), outs)] + [(wo, o_out, qo, so)]
    for w, out, q_, s_ in cases:
        for n0 in sorted({0, N - 64, int(rng.integers(0, N - 64))}):
            _, ref, T = oracle.qgemm(Q4, w, N, K, q_, s_, n0=n0, n1=n0 + 64)
            ok, worst = gu.tol_ok(out[:, n0:n0 + 64], ref, T)
            assert ok, (n0, worst)


@pytest.mark.parametrize("K", [4096, 3584])
@pytest.mark.parametrize("dd", ["random", "min_dominant"])
def test_min_term_worst_case_long_k(K, dd):
    """The Q4_K min term at its largest over a whole LLaDA-8B / Dream-7B K range: every
    6-bit scale and min 63, every quant 15, and each canvas row constant (+-3.0, so every
    code is +-127 and every per-32 sum is 32 * 127 with one sign per row).  The min-term
    accumulator then grows monotonically over K/32 sub-block steps (128 at K = 4096, 112
    at K = 3584), against a d-term of the opposite sign.  min_dominant sets d = 1e-3 and
    dmin = 1e-2 in every block, so that the two terms nearly cancel and the tolerance is
    set by 1e-6 * sum|terms|."""
    M, N = 16, 256
    w = synth.q4k_weights(N, K, 35).copy()
    w[..., 4:144] = 0xFF
    if dd == "min_dominant":
        w[..., 0:2] = np.frombuffer(np.float16(1e-3).tobytes(), np.uint8)
        w[..., 2:4] = np.frombuffer(np.float16(1e-2).tobytes(), np.uint8)
    x = np.full((M, K), 3.0, np.float32)
    x[::2] *= -1
    wd = dllm.repack(Q4, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, Q4, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(Q4, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst


def test_full_ffn_shapes_sampled():
    _sampled_parity(Q4, 256, 12288, 4096, 2, width=32)
    _sampled_parity(Q6, 160, 4096, 12288, 2, width=32)


def test_full_output_projection_rows_sampled():
    M = 160
    rows = synth.block_rows(M, 32, 3)
    _sampled_parity(Q6, M, 126464, 4096, 3, rows=rows, n_samples=4, width=128)


@pytest.mark.parametrize("M", [512, 1024])
def test_full_ffn_canvas_sweep_sampled(M):
    """LLaDA-8B FFN at the larger canvases of the sweep: gate/up (Q4_K) and down (Q6_K)
    with several 128-row token super-tiles per weight tile."""
    _sampled_parity(Q4, M, 12288, 4096, 5, n_samples=2, width=32)
    _sampled_parity(Q6, M, 4096, 12288, 6, n_samples=2, width=32)


def test_dream_qkv_fused_sampled():
    """Dream-7B attention projections in one launch: Q N=3584 and K, V N=512 (28 Q heads,
    4 KV heads) over K=3584 (14 super-blocks, so K-chunks of unequal length)."""
    M, K, Nq, Nkv = 160, 3584, 3584, 512
    x = synth.activations(M, K, 7)
    act = gu.Act(x)
    oq_, os_, _ = oracle.quantize_act(x)
    ws_ = [synth.weights(Q4, n, K, 7, i) for i, n in enumerate((Nq, Nkv, Nkv))]
    wd = [dllm.repack(Q4, w, w.shape[0], K) for w in ws_]
    outs = [torch.empty((M, Nq), device="cuda"), torch.empty((M, Nkv), device="cuda"),
            torch.empty((M, Nkv), device="cuda")]
    wsb = dllm.dllm_qgemm_workspace_bytes(Q4, Nq + 2 * Nkv, K, M)
    work = dllm.alloc_workspace(wsb)
    dllm.dllm_qkv_qgemm(wd[0], wd[1], wd[2], Q4, Nq, Nkv, K, act.q, act.scale, act.sums, M, outs[0], Nq, outs[1],
                        outs[2], Nkv, work, wsb)
    rng = np.random.default_rng(7)
    for w, o in zip(ws_, outs):
        got = o.cpu().numpy()
        N = w.shape[0]
        for n0 in sorted(set([0, N - 64] + list(rng.integers(0, N - 64, 2)))):
            _, ref, T = oracle.qgemm(Q4, w, N, K, oq_, os_, n0=int(n0), n1=int(n0) + 64)
            ok, worst = gu.tol_ok(got[:, n0:n0 + 64], ref, T)
            assert ok, (N, n0, worst)


def test_dream_down_and_output_sampled():
    """Dream-7B down projection (Q6_K, K=18944: 74 super-blocks) and output projection
    (Q6_K, vocab 152064, K=3584) on 32 requested rows of a 160-row canvas."""
    _sampled_parity(Q6, 160, 3584, 18944, 8, n_samples=2, width=32)
    rows = synth.block_rows(160, 32, 9)
    _sampled_parity(Q6, 160, 152064, 3584, 9, rows=rows, n_samples=3, width=128)


# ------------------------------------------------------------------ split-K workspace contract

def test_workspace_shared_across_calls_and_shapes():
    """One zero-filled workspace reused by GEMMs whose tiles split K differently: every
    call stays correct and leaves each arrival counter at a multiple of 16."""
    M, K = 48, 4096
    x = synth.activations(M, K, 70)
    act = gu.Act(x)
    oq, os_, _ = oracle.quantize_act(x)
    cases = []
    # few tiles split K four ways; 128 tiles fill the SMs without splitting
    for i, (qtype, N) in enumerate([(Q4, 128), (Q6, 384), (Q4, 16384), (Q6, 128)]):
        w = synth.weights(qtype, N, K, 70, i)
        _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_)
        cases.append((qtype, N, dllm.repack(qtype, w, N, K), ref, T))
    wsb = max(dllm.dllm_qgemm_workspace_bytes(qt, N, K, M) for qt, N, *_ in cases)
    ws = dllm.alloc_workspace(wsb)
    first = {}
    for rep in range(3):
        for qtype, N, wd, ref, T in cases:
            out = torch.empty((M, N), device="cuda")
            dllm.dllm_qgemm(wd, qtype, N, K, act.q, act.scale, act.sums, M, None, 0, out, N, ws, wsb)
            got = out.cpu().numpy()
            assert gu.tol_ok(got, ref, T)[0]
            if rep == 0:
                first[N, qtype] = got
            else:
                assert np.array_equal(first[N, qtype], got)
    torch.cuda.synchronize()
    ctr = ws[:4 * 3].cpu().numpy().view(np.uint32)  # tiles of the split calls: one counter each
    assert np.all(ctr % 16 == 0) and np.all(ctr > 0)


def test_workspace_shared_by_tail_split_and_uniform_split():
    """The step's own mix on one workspace: a 4096-row projection whose 32 tiles split K
    four ways (O, down) between launches of a 192-tile gate/up whose 44 leftover tiles
    are cut into K-pieces (tail split, arrival counters up to tile 191).  The partial
    sums of the small calls must never land on the counters of the large one: every
    repetition gives the same bits, within the oracle's bound."""
    M, K, F = 128, 4096, 12288
    x = synth.activations(M, K, 71)
    act = gu.Act(x)
    oq, os_, _ = oracle.quantize_act(x)
    wo = synth.weights(Q4, K, K, 71, 0)
    wg, wu = synth.weights(Q4, F, K, 71, 1), synth.weights(Q4, F, K, 71, 2)
    do, dg, du = dllm.repack(Q4, wo, K, K), dllm.repack(Q4, wg, F, K), dllm.repack(Q4, wu, F, K)
    wsb = max(dllm.dllm_qgemm_workspace_bytes(Q4, K, K, M), dllm.dllm_qgemm_workspace_bytes(Q4, 2 * F, K, M))
    ws = dllm.alloc_workspace(wsb)
    og, ou, oo = (torch.empty((M, n), device="cuda") for n in (F, F, K))
    first = None
    for rep in range(4):
        dllm.dllm_qgemm(do, Q4, K, K, act.q, act.scale, act.sums, M, None, 0, oo, K, ws, wsb)
        dllm.dllm_qkv_qgemm(dg, du, None, Q4, F, F, K, act.q, act.scale, act.sums, M, og, F, ou, None, F, ws, wsb)
        got = [t.cpu().numpy() for t in (oo, og, ou)]
        if first is None:
            first = got
            for w, o, n in ((wo, got[0], K), (wg, got[1], F), (wu, got[2], F)):
                for n0 in (0, n - 256, n // 2):
                    _, ref, T = oracle.qgemm(Q4, w, n, K, oq, os_, n0=n0, n1=n0 + 256)
                    assert gu.tol_ok(o[:, n0:n0 + 256], ref, T)[0], n0
        else:
            for a, b in zip(first, got):
                assert np.array_equal(a, b)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def test_workspace_too_small_is_rejected():
    M, N, K = 32, 256, 2048
    w, x = gu.make_case(Q4, M, N, K, 71)
    wd = dllm.repack(Q4, w, N, K)
    act = gu.Act(x)
    wsb = dllm.dllm_qgemm_workspace_bytes(Q4, N, K, M)
    assert wsb > 0  # two tiles on many SMs: K is split
    out = torch.empty((M, N), device="cuda")
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_qgemm(wd, Q4, N, K, act.q, act.scale, act.sums, M, None, 0, out, N, None, 0)
    assert e.value.code == dllm.DLLM_ERR_WORKSPACE
    small = dllm.alloc_workspace(wsb - 256)
    with pytest.raises(dllm.DllmError):
        dllm.dllm_qgemm(wd, Q4, N, K, act.q, act.scale, act.sums, M, None, 0, out, N, small, wsb - 256)


# ------------------------------------------------------------------ tail split
# 192 tiles of 128 rows on B200's 148 SMs: one round of whole tiles, then the 44 tiles
# left are cut into 148 K-pieces (3 or 4 per tile), one more unit per SM, summed by the
# last arriving piece in piece order.

TAIL_N = 192 * 128


@pytest.mark.parametrize("qtype,M", [(Q4, 16), (Q4, 160), (Q6, 48)])
def test_tail_split_parity(qtype, M):
    N, K = TAIL_N, 4096
    w, x = gu.make_case(qtype, M, N, K, 42)
    wd = dllm.repack(qtype, w, N, K)
    act = gu.Act(x)
    out = gu.gemm(wd, qtype, N, K, act).cpu().numpy()
    oq, os_, _ = oracle.quantize_act(x)
    _, ref, T = oracle.qgemm(qtype, w, N, K, oq, os_)
    ok, worst = gu.tol_ok(out, ref, T)
    assert ok, worst


def test_tail_split_independent_of_M_and_rows():
    """The K pieces depend on the weight shape only: the same rows at another canvas
    height, or gathered by a row list, give the same bits."""
    N, K, M = TAIL_N, 4096, 160
    w, x = gu.make_case(Q4, M, N, K, 43)
    wd = dllm.repack(Q4, w, N, K)
    full = gu.gemm(wd, Q4, N, K, gu.Act(x))
    part = gu.gemm(wd, Q4, N, K, gu.Act(x[:16].copy()))
    assert torch.equal(part, full[:16])
    rows = synth.block_rows(M, 32, 44)
    act = gu.Act(x)
    got = gu.gemm(wd, Q4, N, K, act, rows=rows)
    assert torch.equal(got, full[torch.from_numpy(rows).long().cuda()])
    again = gu.gemm(wd, Q4, N, K, act)
    assert torch.equal(again, full)


def test_tail_split_gate_up_in_one_launch():
    """gate and up (2 x 12288 rows) in one launch, as the step runs them."""
    M, F, K = 32, 12288, 4096
    wg = synth.weights(Q4, F, K, 45)
    wu = synth.weights(Q4, F, K, 46)
    x = synth.activations(M, K, 45)
    dg, du = dllm.repack(Q4, wg, F, K), dllm.repack(Q4, wu, F, K)
    act = gu.Act(x)
    og = torch.empty((M, F), device="cuda")
    ou = torch.empty((M, F), device="cuda")
    wsb = dllm.dllm_qgemm_workspace_bytes(Q4, 2 * F, K, M)
    ws = dllm.alloc_workspace(max(wsb, 256))
    dllm.dllm_qkv_qgemm(dg, du, None, Q4, F, F, K, act.q, act.scale, act.sums, M, og, F, ou, None, F, ws, wsb)
    oq, os_, _ = oracle.quantize_act(x)
    for w, o in ((wg, og), (wu, ou)):
        _, ref, T = oracle.qgemm(Q4, w, F, K, oq, os_)
        ok, worst = gu.tol_ok(o.cpu().numpy(), ref, T)
        assert ok, worst
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
