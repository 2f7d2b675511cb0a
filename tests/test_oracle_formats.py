"""Pins of the oracle's Q5_K and Q8_0 decoders and of its GEMM on those formats,
against things other than the oracle itself.

  q5k_decode  hand-derived block (golden/q5k_q80_handmade.txt) that fixes the qh bit
              order and the nibble order; gguf package dequantization of random and
              edge blocks; structure: with qh = 0 the block equals the Q4_K block of
              the same remaining bytes, and setting every fifth bit adds 16 d sc_j
  q80_decode  hand-derived block; gguf package dequantization; linear in d
  qgemm       fp64 dequantize (gguf-pinned) then matmul, by brute force on tiny shapes;
              the integers (dots, S, Smin) against numpy brute force from the decoded
              quants
These two formats are the oracle side of the next weight formats; the CUDA library
does not implement them yet.
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
    return np.spacing(np.abs(np.asarray(x, np.float64)).astype(np.float32)).astype(np.float64)


def _q5k_handmade():
    g4 = read_golden("q4k_handmade.txt")
    blk = np.zeros(176, np.uint8)
    blk[0:2] = np.frombuffer(int(g4["d_bits"], 16).to_bytes(2, "little"), np.uint8)
    blk[2:4] = np.frombuffer(int(g4["dmin_bits"], 16).to_bytes(2, "little"), np.uint8)
    blk[4:16] = [int(t, 16) for t in g4["scale_bytes"].split()]
    blk[16:48] = np.arange(32)
    for c in range(4):
        for l in range(32):
            blk[48 + 32 * c + l] = (l % 16) | (((c + l) % 16) << 4)
    return blk


def test_q5k_handmade_block():
    g = read_golden("q5k_q80_handmade.txt")
    g4 = read_golden("q4k_handmade.txt")
    blk = _q5k_handmade()
    d, dmin, sc, mn, q = oracle.q5k_decode(blk)
    assert (d, dmin) == (1.0, 0.5)
    assert list(sc) == [int(t) for t in g4["sc"].split()]
    assert list(mn) == [int(t) for t in g4["m"].split()]
    assert q.max() <= 31
    deq = oracle.dequant(oracle.Q5_K, blk, 1, 256)[0]
    ext = gq.dequantize(blk.reshape(1, 176), GT.Q5_K)[0]
    values = {int(k.split()[1]): float(v) for k, v in g.items() if k.startswith("q5k_value ")}
    assert len(values) == 14
    for k, v in values.items():
        assert deq[k] == v, k
        assert ext[k] == v, k


def test_q80_handmade_block():
    g = read_golden("q5k_q80_handmade.txt")
    blk = np.zeros(34, np.uint8)
    blk[0:2] = np.frombuffer(int(g["q80_d_bits"], 16).to_bytes(2, "little"), np.uint8)
    qs = [int(t) for t in g["q80_q"].split()]
    blk[2:34] = np.array(qs + [3] * (32 - len(qs)), np.int8).view(np.uint8)
    d, q = oracle.q80_decode(blk)
    assert d == 0.5 and list(q[:5]) == qs
    row = np.tile(blk, 8)  # a 256-weight span is eight blocks
    deq = oracle.dequant(oracle.Q8_0, row, 1, 256)[0]
    want = [float(t) for t in g["q80_values"].split()]
    assert list(deq[:5]) == want and np.all(deq[5:32] == float(g["q80_rest"]))
    assert np.array_equal(deq[32:64], deq[:32])
    ext = gq.dequantize(row.reshape(8, 34), GT.Q8_0).reshape(-1)
    assert np.array_equal(ext.astype(np.float64), deq)


def _edge_f16():
    return np.array([0.01, -2.0, 1e-4, 65504.0, 2 ** -24, 1.0, 0.0, -0.0], np.float16).view(np.uint8).reshape(-1, 2)


@pytest.mark.parametrize("qtype", [oracle.Q5_K, oracle.Q8_0])
def test_decode_matches_gguf_package(qtype):
    N, K = 16, 1024
    w = synth.weights(qtype, N, K, 17)
    rng = np.random.default_rng(18)
    if qtype == oracle.Q5_K:
        blocks = w.reshape(-1, 176)
        extra = rng.integers(0, 256, (8, 176)).astype(np.uint8)
        extra[:, 0:2] = _edge_f16()
        extra[:, 2:4] = _edge_f16()[::-1]
        blocks = np.concatenate([blocks, extra])
        ext = gq.dequantize(blocks, GT.Q5_K).reshape(blocks.shape[0], 256)
        ours = oracle.dequant(qtype, blocks, blocks.shape[0], 256)
    else:
        blocks = w.reshape(-1, 34)
        extra = rng.integers(0, 256, (8, 34)).astype(np.uint8)  # any int8, -128 included
        extra[:, 0:2] = _edge_f16()
        blocks = np.concatenate([blocks, extra])
        ext = gq.dequantize(blocks, GT.Q8_0).reshape(-1, 256)
        ours = oracle.dequant(qtype, blocks.reshape(-1), blocks.shape[0] // 8, 256)
    ext = ext.astype(np.float64)
    fin = np.isfinite(ext)
    assert fin.mean() > 0.9
    # gguf evaluates in f32: one or two roundings of the exact value
    assert np.all(np.abs(ours[fin] - ext[fin]) <= 2 * f32_ulp(ours[fin]) + 1e-45)


def test_q5k_structure():
    rng = np.random.default_rng(19)
    b5 = rng.integers(0, 256, (6, 176)).astype(np.uint8)
    b5[:, 0:4] = np.array([0.25, 0.125], np.float16).view(np.uint8)
    b5[:, 16:48] = 0
    b4 = np.concatenate([b5[:, 0:16], b5[:, 48:176]], axis=1)  # the Q4_K block of the same bytes
    d5 = oracle.dequant(oracle.Q5_K, b5, 6, 256)
    d4 = oracle.dequant(oracle.Q4_K, b4, 6, 256)
    assert np.array_equal(d5, d4)
    b5[:, 16:48] = 0xFF  # every fifth bit set: + 16 d sc_j
    d5f = oracle.dequant(oracle.Q5_K, b5, 6, 256)
    for i in range(6):
        _, _, sc, _, _ = oracle.q5k_decode(b5[i])
        assert np.array_equal(d5f[i] - d4[i], 16 * 0.25 * np.repeat(sc.astype(np.float64), 32))


def test_q80_linear_in_d():
    w = synth.weights(oracle.Q8_0, 4, 512, 20).reshape(-1, 34).copy()
    base = oracle.dequant(oracle.Q8_0, w.reshape(-1), 4, 512)
    d = w[:, 0:2].copy().view(np.float16)
    w[:, 0:2] = (d * np.float16(2)).view(np.uint8)
    assert np.array_equal(oracle.dequant(oracle.Q8_0, w.reshape(-1), 4, 512), 2 * base)


def _brute(qtype, w, N, K, q, s):
    W = oracle.dequant(qtype, w, N, K)
    A = q.astype(np.float64) * np.repeat(s.astype(np.float64), 256, axis=1)
    return A @ W.T


@pytest.mark.parametrize("qtype", [oracle.Q5_K, oracle.Q8_0])
@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 4, 256), (4, 3, 512), (2, 5, 768)])
def test_qgemm_vs_bruteforce(qtype, M, N, K):
    w = synth.weights(qtype, N, K, 21, M, N, K)
    q, s, _ = oracle.quantize_act(synth.activations(M, K, 21, M, N, K))
    out, out64, T = oracle.qgemm(qtype, w, N, K, q, s)
    ref = _brute(qtype, w, N, K, q, s)
    assert np.all(np.abs(out64 - ref) <= 1e-12 * T + 1e-300)
    assert np.array_equal(out, out64.astype(np.float32))
    rows = np.array([M - 1, 0], np.int32)
    r, _, _ = oracle.qgemm(qtype, w, N, K, q, s, rows=rows)
    assert np.array_equal(r, out[rows])


@pytest.mark.parametrize("qtype", [oracle.Q5_K, oracle.Q8_0])
def test_sb_ints_bruteforce(qtype):
    N, K, M = 3, 512, 2
    w = synth.weights(qtype, N, K, 22)
    q, s, a32 = oracle.quantize_act(synth.activations(M, K, 22))
    dots, S, Smin = oracle.sb_ints(qtype, w, N, K, q)
    qa = q.astype(np.int64)
    for n in range(N):
        for sb in range(K // 256):
            a = qa[:, 256 * sb:256 * sb + 256]
            if qtype == oracle.Q5_K:
                _, _, sc, mn, qq = oracle.q5k_decode(w[n, sb])
                dd = (a.reshape(M, 8, 32) * qq.astype(np.int64).reshape(8, 32)).sum(-1)
                assert np.array_equal(S[:, n, sb], dd @ sc.astype(np.int64))
                assert np.array_equal(Smin[:, n, sb], a32[:, 8 * sb:8 * sb + 8].astype(np.int64) @ mn.astype(np.int64))
            else:
                qq = np.concatenate([oracle.q80_decode(w[n, sb, 34 * b:34 * b + 34])[1] for b in range(8)])
                dd = (a.reshape(M, 8, 32) * qq.astype(np.int64).reshape(8, 32)).sum(-1)
                assert np.array_equal(S[:, n, sb], dd.sum(-1))
                assert np.all(Smin[:, n, sb] == 0)
            assert np.array_equal(dots[:, n, 8 * sb:8 * sb + 8], dd)
