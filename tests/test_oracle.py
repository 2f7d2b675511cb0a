"""Pins of the CPU oracle against things other than itself.

What pins each oracle function (so a dropped term, a wrong sign or index, or a
transposed operand fails at least one test):

  f16_to_f64     every one of the 65536 bit patterns vs numpy's float16 conversion
  q4k_decode     hand-derived block (golden/q4k_handmade.txt); gguf package decode
                 of random and edge blocks (the external reference the pages trust)
  q6k_decode     hand-derived block (golden/q6k_handmade.txt); gguf package decode
  quantize_act   hand-derived ties and scales (golden/quantize_handmade.txt);
                 properties: max|q| = 127 per non-zero block, |x - q*scale| <= scale/2,
                 sums = sums of q; numpy float32 re-evaluation of the same reading
  qgemm          brute force: fp64 dequantize (gguf-pinned) then matmul on tiny shapes;
                 invariants: zero activations, zero nibbles, q = 32, linear in d,
                 single non-zero activation, super-block permutation, row gathering
  sb_ints        bit-exact int64 brute force from the decoded integers (numpy), and
                 consistency with qgemm's fp64 combine
"""
import numpy as np
import pytest

import oracle
from quantized_int8_gemm_q4_b200 import synth
from tests.conftest import read_golden

gguf = pytest.importorskip("gguf")
from gguf import GGMLQuantizationType as GT  # noqa: E402
from gguf import quants as gq  # noqa: E402


def f32_ulp(x):
    x = np.abs(np.asarray(x, np.float64)).astype(np.float32)
    return np.spacing(x).astype(np.float64)


# ---------------------------------------------------------------- f16

def test_f16_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32)
    ref = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits[::1]])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


# ---------------------------------------------------------------- decoders

def test_q4k_handmade_block():
    g = read_golden("q4k_handmade.txt")
    blk = np.zeros(144, np.uint8)
    blk[0:2] = np.frombuffer(int(g["d_bits"], 16).to_bytes(2, "little"), np.uint8)
    blk[2:4] = np.frombuffer(int(g["dmin_bits"], 16).to_bytes(2, "little"), np.uint8)
    blk[4:16] = [int(t, 16) for t in g["scale_bytes"].split()]
    for c in range(4):
        for l in range(32):
            blk[16 + 32 * c + l] = (l % 16) | (((c + l) % 16) << 4)
    d, dmin, sc, mn, q = oracle.q4k_decode(blk)
    assert (d, dmin) == (1.0, 0.5)
    assert list(sc) == [int(t) for t in g["sc"].split()]
    assert list(mn) == [int(t) for t in g["m"].split()]
    deq = oracle.dequant(oracle.Q4_K, blk, 1, 256)[0]
    ext = gq.dequantize(blk.reshape(1, 144), GT.Q4_K)[0]
    for k, v in g["values"].items():
        assert deq[k] == v, k
        assert ext[k] == v, k


def test_q6k_handmade_block():
    g = read_golden("q6k_handmade.txt")
    blk = np.zeros(210, np.uint8)
    for p in range(128):
        blk[p] = (p % 16) | (((p // 16) % 16) << 4)
    for p in range(64):
        blk[128 + p] = p
    blk[192:208] = (np.arange(16) - 8).astype(np.int8).view(np.uint8)
    blk[208:210] = np.frombuffer(int(g["d_bits"], 16).to_bytes(2, "little"), np.uint8)
    d, sc, q = oracle.q6k_decode(blk)
    assert d == 0.25 and list(sc) == list(range(-8, 8))
    deq = oracle.dequant(oracle.Q6_K, blk, 1, 256)[0]
    ext = gq.dequantize(blk.reshape(1, 210), GT.Q6_K)[0]
    for k, v in g["values"].items():
        assert deq[k] == v, k
        assert ext[k] == v, k


def _edge_q4k_blocks():
    rng = np.random.default_rng(123)
    out = []
    for fill in (0x00, 0xFF, 0x0F, 0xF0, 0xC0, 0x3F):
        b = np.full(144, fill, np.uint8)
        b[0:4] = np.array([0.0078125, 0.001], np.float16).view(np.uint8)
        out.append(b)
    b = rng.integers(0, 256, 144).astype(np.uint8)
    b[0:4] = np.array([-3.5, 65504.0], np.float16).view(np.uint8)   # negative d, max f16
    out.append(b)
    b = rng.integers(0, 256, 144).astype(np.uint8)
    b[0:4] = np.array([2 ** -24, 2 ** -20], np.float16).view(np.uint8)  # subnormals
    out.append(b)
    return np.stack(out)


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
def test_decode_matches_gguf_package(qtype):
    N, K = 24, 1024
    w = synth.weights(qtype, N, K, 7)
    blocks = w.reshape(-1, oracle.BLOCK_BYTES[qtype])
    if qtype == oracle.Q4_K:
        blocks = np.concatenate([blocks, _edge_q4k_blocks()])
    else:
        extra = np.random.default_rng(5).integers(0, 256, (6, 210)).astype(np.uint8)  # any int8 scale
        extra[:, 208:210] = np.array([0.01, -2.0, 1e-4, 65504.0, 2 ** -24, 1.0],
                                     np.float16).view(np.uint8).reshape(6, 2)
        blocks = np.concatenate([blocks, extra])
    nb = blocks.shape[0]
    ours = oracle.dequant(qtype, blocks, nb, 256)
    ext = gq.dequantize(blocks, GT.Q4_K if qtype == oracle.Q4_K else GT.Q6_K).astype(np.float64)
    fin = np.isfinite(ext)
    assert fin.mean() > 0.95
    # gguf evaluates in f32: one or two roundings of the exact value
    assert np.all(np.abs(ours[fin] - ext[fin]) <= 2 * f32_ulp(ours[fin]) + 1e-45)


def test_q4k_decode_is_not_symmetric_in_nibbles():
    # low nibble -> sub-block 2c, high nibble -> 2c+1; a swap would fail here
    blk = np.zeros(144, np.uint8)
    blk[0:2] = np.array([1.0], np.float16).view(np.uint8)
    blk[4:8] = [1, 2, 0, 0]       # sc0 = 1, sc1 = 2
    blk[16] = 0x31                # low 1 -> k=0, high 3 -> k=32
    deq = oracle.dequant(oracle.Q4_K, blk, 1, 256)[0]
    assert deq[0] == 1.0 and deq[32] == 6.0 and np.count_nonzero(deq) == 2


# ---------------------------------------------------------------- quantize

def test_quantize_handmade():
    g = read_golden("quantize_handmade.txt")
    x = np.zeros((1, 768), np.float32)
    ax = [float(t) for t in g["A_x"].split()]
    bx = [float(t) for t in g["B_x"].split()]
    x[0, :len(ax)] = ax
    x[0, 256:256 + len(bx)] = bx
    q, s, a = oracle.quantize_act(x)
    assert list(q[0, :len(ax)]) == [int(t) for t in g["A_q"].split()]
    assert list(q[0, 256:256 + len(bx)]) == [int(t) for t in g["B_q"].split()]
    assert np.all(q[0, len(ax):256] == 0) and np.all(q[0, 256 + len(bx):] == 0)
    assert s[0, 0] == np.float32(1.0)
    assert s[0, 1] == np.float32(4) / np.float32(127)
    assert s[0, 2] == 0.0
    assert a[0, 0] == int(g["A_sum0"]) and a[0, 8] == int(g["B_sum0"])
    assert np.all(a[0, 16:] == 0)


def test_quantize_properties():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((37, 2048)).astype(np.float32) * rng.uniform(1e-3, 1e3, (37, 1)).astype(np.float32)
    x[5, 256:512] = 0.0
    x[6, :256] = 7.0                       # constant block: every q = 127
    q, s, a = oracle.quantize_act(x)
    qb = q.reshape(37, 8, 256).astype(np.int32)
    xb = x.reshape(37, 8, 256).astype(np.float64)
    nz = np.abs(xb).max(-1) > 0
    assert np.all(np.abs(qb).max(-1)[nz] == 127)
    assert np.all(qb[~nz] == 0) and np.all(s[~nz] == 0)
    assert np.all(qb[6, 0] == 127)
    err = np.abs(xb - qb * s[..., None].astype(np.float64))
    assert np.all(err <= s[..., None] * (0.5 + 1e-5))
    assert np.array_equal(a, q.reshape(37, 64, 32).astype(np.int32).sum(-1))
    # the same reading re-evaluated with numpy float32 arithmetic
    amax = np.abs(x.reshape(37, 8, 256)).max(-1)
    with np.errstate(divide="ignore"):
        iscale = np.where(amax > 0, np.float32(127) / amax, np.float32(0)).astype(np.float32)
    qq = np.clip(np.rint(x.reshape(37, 8, 256) * iscale[..., None]), -127, 127)
    assert np.array_equal(qq.astype(np.int8).reshape(37, 2048), q)
    assert np.array_equal(np.where(amax > 0, amax / np.float32(127), 0).astype(np.float32), s)


# ---------------------------------------------------------------- GEMM

def _brute(qtype, w, N, K, q, s):
    """fp64 dequantize (gguf-pinned decoder) then fp64 matmul."""
    W = oracle.dequant(qtype, w, N, K)
    A = q.astype(np.float64) * np.repeat(s.astype(np.float64), 256, axis=1)
    return A @ W.T


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 4, 256), (4, 3, 512), (2, 5, 768)])
def test_qgemm_vs_bruteforce(qtype, M, N, K):
    w = synth.weights(qtype, N, K, 11, M, N, K)
    x = synth.activations(M, K, 11, M, N, K)
    q, s, _ = oracle.quantize_act(x)
    out, out64, T = oracle.qgemm(qtype, w, N, K, q, s)
    ref = _brute(qtype, w, N, K, q, s)
    assert np.all(np.abs(out64 - ref) <= 1e-12 * T)
    assert np.array_equal(out, out64.astype(np.float32))
    # the external decoder gives the same result to f32 decode precision
    ext = gq.dequantize(w.reshape(-1, oracle.BLOCK_BYTES[qtype]),
                        GT.Q4_K if qtype == oracle.Q4_K else GT.Q6_K).reshape(N, K).astype(np.float64)
    A = q.astype(np.float64) * np.repeat(s.astype(np.float64), 256, axis=1)
    assert np.all(np.abs(out64 - A @ ext.T) <= 1e-6 * T)


def test_qgemm_zero_activations():
    w = synth.q4k_weights(8, 512, 1)
    q = np.zeros((3, 512), np.int8)
    s = np.ones((3, 2), np.float32)
    out, out64, T = oracle.qgemm(oracle.Q4_K, w, 8, 512, q, s)
    assert np.all(out == 0) and np.all(T == 0)


def test_qgemm_zero_nibbles_leave_min_term():
    N, K, M = 6, 512, 4
    w = synth.q4k_weights(N, K, 2).copy()
    w[..., 16:] = 0                                   # every q = 0
    x = synth.activations(M, K, 2)
    q, s, a32 = oracle.quantize_act(x)
    out, out64, T = oracle.qgemm(oracle.Q4_K, w, N, K, q, s)
    exp = np.zeros((M, N))
    for n in range(N):
        for sb in range(K // 256):
            _, dmin, _, mn, _ = oracle.q4k_decode(w[n, sb])
            exp[:, n] -= s[:, sb].astype(np.float64) * dmin * (a32[:, 8 * sb:8 * sb + 8] @ mn.astype(np.float64))
    assert np.all(np.abs(out64 - exp) <= 1e-13 * T)
    assert np.any(out64 != 0)


def test_qgemm_q6k_q32_is_zero():
    N, K, M = 4, 512, 3
    w = synth.q6k_weights(N, K, 3).copy()
    # q = 32 everywhere: low nibbles 0, high 2 bits = 2 -> each high-bit byte 0b10101010
    w[..., 0:128] = 0
    w[..., 128:192] = 0xAA
    q, s, _ = oracle.quantize_act(synth.activations(M, K, 3))
    out, out64, T = oracle.qgemm(oracle.Q6_K, w, N, K, q, s)
    assert np.all(out64 == 0)


def test_qgemm_linear_in_d():
    N, K, M = 5, 768, 4
    w = synth.q4k_weights(N, K, 4).copy()
    w[..., 2:4] = 0                                   # dmin = 0
    q, s, _ = oracle.quantize_act(synth.activations(M, K, 4))
    _, o1, _ = oracle.qgemm(oracle.Q4_K, w, N, K, q, s)
    d = w[..., 0:2].copy().view(np.float16)
    w2 = w.copy()
    w2[..., 0:2] = (d * np.float16(2)).view(np.uint8)  # exact in f16
    _, o2, _ = oracle.qgemm(oracle.Q4_K, w2, N, K, q, s)
    assert np.array_equal(o2, 2 * o1)
    w3 = w.copy()
    w3[..., 0:2] = (-d).view(np.uint8)
    _, o3, _ = oracle.qgemm(oracle.Q4_K, w3, N, K, q, s)
    assert np.array_equal(o3, -o1)


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
def test_qgemm_single_activation(qtype):
    N, K = 7, 512
    w = synth.weights(qtype, N, K, 5)
    W = oracle.dequant(qtype, w, N, K)
    for k in (0, 31, 32, 255, 256, 300, 511):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 3.0
        q, s, _ = oracle.quantize_act(x)
        assert q[0, k] == 127
        _, o, _ = oracle.qgemm(qtype, w, N, K, q, s)
        # a single non-zero activation picks column k of the weight matrix
        assert np.all(np.abs(o[0] - float(s[0, k // 256]) * 127 * W[:, k]) <= 1e-12 * np.abs(W[:, k]).max())


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
def test_superblock_permutation_invariance(qtype):
    N, K, M = 4, 1024, 3
    w = synth.weights(qtype, N, K, 6)
    q, s, _ = oracle.quantize_act(synth.activations(M, K, 6))
    perm = np.array([2, 0, 3, 1])
    wp = w[:, perm]
    qp = q.reshape(M, 4, 256)[:, perm].reshape(M, K)
    sp = s[:, perm]
    _, S, Sm = oracle.sb_ints(qtype, w, N, K, q)
    _, Sp, Smp = oracle.sb_ints(qtype, wp, N, K, qp)
    assert np.array_equal(S[..., perm], Sp) and np.array_equal(Sm[..., perm], Smp)
    _, o, T = oracle.qgemm(qtype, w, N, K, q, s)
    _, op, _ = oracle.qgemm(qtype, wp, N, K, qp, sp)
    assert np.all(np.abs(o - op) <= 1e-13 * T)


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
def test_rows_equal_sliced_full(qtype):
    N, K, M = 9, 512, 40
    w = synth.weights(qtype, N, K, 8)
    q, s, _ = oracle.quantize_act(synth.activations(M, K, 8))
    full, _, _ = oracle.qgemm(qtype, w, N, K, q, s)
    rows = np.array([33, 7, 7, 39, 0], np.int32)
    r, _, _ = oracle.qgemm(qtype, w, N, K, q, s, rows=rows)
    assert np.array_equal(r, full[rows])
    with pytest.raises(ValueError):
        oracle.qgemm(qtype, w, N, K, q, s, rows=np.array([40], np.int32))


@pytest.mark.parametrize("qtype", [oracle.Q4_K, oracle.Q6_K])
def test_sb_ints_bruteforce(qtype):
    N, K, M = 3, 512, 2
    w = synth.weights(qtype, N, K, 9)
    q, s, a32 = oracle.quantize_act(synth.activations(M, K, 9))
    dots, S, Smin = oracle.sb_ints(qtype, w, N, K, q)
    qa = q.astype(np.int64)
    for n in range(N):
        for sb in range(K // 256):
            if qtype == oracle.Q4_K:
                _, _, sc, mn, qq = oracle.q4k_decode(w[n, sb])
                sub, qi = 32, qq.astype(np.int64)
            else:
                _, sc, qq = oracle.q6k_decode(w[n, sb])
                sub, qi = 16, qq.astype(np.int64) - 32
            a = qa[:, 256 * sb:256 * sb + 256]
            d = (a.reshape(M, -1, sub) * qi.reshape(-1, sub)).sum(-1)
            nsub = 256 // sub
            assert np.array_equal(dots[:, n, nsub * sb:nsub * sb + nsub], d)
            assert np.array_equal(S[:, n, sb], d @ sc.astype(np.int64))
            if qtype == oracle.Q4_K:
                assert np.array_equal(Smin[:, n, sb], a32[:, 8 * sb:8 * sb + 8].astype(np.int64) @ mn.astype(np.int64))
            else:
                assert np.all(Smin[:, n, sb] == 0)
